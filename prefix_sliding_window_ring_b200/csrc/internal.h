// Host-side declarations shared by the library's translation units.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace ps {

constexpr int kMaxBatchPerLaunch = 128;  // batch entries passed by value per launch

struct BatchIds {
  int32_t seq[kMaxBatchPerLaunch];
  int32_t P[kMaxBatchPerLaunch];     // host bookkeeping of each entry's ring state
  int32_t head[kMaxBatchPerLaunch];
  int32_t count[kMaxBatchPerLaunch];
  int32_t owner[kMaxBatchPerLaunch];  // sequence whose slab holds the prefix rows
  int64_t t[kMaxBatchPerLaunch];
};

// tmap.cu: a 3-D bf16 tensor map with 128-byte swizzle; dims innermost first,
// byte strides of dims 1 and 2, box sizes b0..b2, L2 promotion of its loads
// (0 none, 1 128 bytes, 2 256 bytes).  False if encoding failed.
bool encode_map3d_bf16(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                       uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2,
                       int l2_promotion = 2);
// The same for a map of `rank` dimensions (strides[i]: bytes between
// consecutive indices of dimension i + 1).
bool encode_map_bf16(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                     const uint64_t* strides, const uint32_t* box, int l2_promotion = 2);

// ring.cu
constexpr int kMaxPageSets = 256;  // page-table entries per update launch
// page_table[idx[i]] = phys[i] for i < n (paged caches), in launches of kMaxPageSets.
cudaError_t launch_page_set(const CacheDev& c, const int32_t* idx, const int32_t* phys, int n,
                            cudaStream_t st);
cudaError_t launch_meta_set(const CacheDev& c, int seq, const DevMeta& m, cudaStream_t st);
cudaError_t launch_prefix_store(const CacheDev& c, int esize, int seq, const void* k,
                                const void* v, int P_s, cudaStream_t st);
cudaError_t launch_ring_append(const CacheDev& c, int esize, const BatchIds& ids, int B,
                               const void* k, const void* v, int n, cudaStream_t st);
cudaError_t launch_ring_import(const CacheDev& c, int esize, int seq, const DevMeta& m_new,
                               const void* k, const void* v, int n, cudaStream_t st);
cudaError_t launch_ring_export(const CacheDev& c, int esize, int seq, void* k, void* v,
                               int64_t* pos, int32_t* count_out, cudaStream_t st);
cudaError_t launch_debug_wait_timeout(const CacheDev& c, long long limit_cycles, cudaStream_t st);
cudaError_t launch_debug_visible(const CacheDev& c, int seq, int64_t t, int64_t* pos_out,
                                 int32_t* n_out, cudaStream_t st);

// decode.cu
struct DecodeWs {
  float* part_ml;   // per (pair, CTA) piece: (max, sum) per query head, base-2 domain
  float* part_o;    // per piece: unnormalised accumulators [G][d]
};
// Workspace of one decode call (launches of more than kMaxBatchPerLaunch
// entries run in turn and reuse it).
DecodeWs decode_ws_layout(void* ws, int B, int Hkv, int G, int d, int sm_count, size_t* bytes);
size_t decode_workspace_bytes(int B, int Hq, int Hkv, int d, int sm_count);
// ids.P / ids.head / ids.count: each entry's ring state as the host bookkeeping
// has it.  The kernel checks them against the device record.
// k_new / v_new: NULL for a plain decode; for a decode step, the appended rows
// [B][Hkv][d] at positions ids.t (ids then holds the state after the append),
// which the launch reads for the attention, writes to their ring slots, and
// after which it commits the new bookkeeping.
// Tensor maps of a bf16 cache's K/V for the tensor-core decode kernel: prefix
// slabs and ring pages, each with a box of 64 rows ([0]) and of 8 rows ([1])
// of one 64-column block, and (whole, when encodable) a box of 64 rows of
// both column blocks of a 128-column row, which fills a whole tile with one
// copy.
struct DecodeMaps {
  // Atom maps: 5D views (64 columns, 8 rows, 64-column block, atom of the
  // slab, slab) of the prefix slabs and of the ring slabs, 128-byte swizzle.
  // A box of A atoms lands as A groups of [column block][8 rows] -- the
  // decode kernel's tile layout -- so one copy brings A atoms of every column
  // block.  Boxes of 8 atoms (a 64-row tile) and 1 atom; ring slabs also one
  // page (page_rows / 8 atoms; paged caches with 8 < page_rows < 64).
  CUtensorMap kpa[2], vpa[2];  // prefix slabs (prefix_atoms)
  CUtensorMap kra[3], vra[3];  // ring slabs (ring_atoms)
  // 3D maps with one 8-row box of one 64-column block: copies that do not
  // start on an atom of their slab, and ring slabs that are not whole atoms
  CUtensorMap kpre8, vpre8, kring8, vring8;
  int prefix_atoms;  // 1 if the prefix atom maps exist (every prefix atom inside the buffer)
  int ring_atoms;  // 1 if the ring atom maps exist (page_rows a multiple of 8)
  int page_box;    // 1 if the one-page ring atom maps exist
};
bool make_decode_maps(const CacheDev& c, DecodeMaps* m);
// maps: the cache's decode maps (bf16 caches; NULL for float32).
cudaError_t launch_decode(const CacheDev& c, int dtype, int G, const BatchIds& ids, int B, int Hq,
                          const void* q, const void* k_new, const void* v_new, void* out,
                          float scale, const DecodeWs& ws, int sm_count, const DecodeMaps* maps,
                          cudaStream_t st);

// Small chunk blocks on the tensor-core decode kernel (bf16, head_dim 64 or
// 128): entry e is a group of nq (1..8) consecutive queries of one sequence's
// block, the first at position t0 + i0 (i0-th of the block); its q / out rows
// start at packed row qrow and its block's key rows at packed row brow of
// k_blk / v_blk.  cols (1, 2, 4 or 8) = the kernel's columns, >= nq * Hq/Hkv.
// Default largest block of the small path (ps_set_chunk_small_max).
constexpr int kChunkSmallMaxDefault = 64;
struct SmallChunkEntry {
  int seq, P, head, count, owner;  // the ring state before the block
  int64_t t0;
  int32_t i0, nq, qrow, brow;
};
// (group, kv head) pairs of the small-block path that are resident at once
// in clusters of two CTAs (one wave); 0 if the occupancy query fails.
int chunk_small_pair_capacity(int d);
cudaError_t launch_chunk_small_batch(const CacheDev& c, int cols, int gq,
                                     const SmallChunkEntry* e, int B, int Hq, const void* q,
                                     const void* k_blk, const void* v_blk, int64_t blk_rows,
                                     void* out, float scale, int sm_count, const DecodeMaps& maps,
                                     cudaStream_t st);

// chunk_tc.cu (tcgen05 chunk kernel: bf16, head_dim 128)
bool chunk_tc_supported(const CacheDev& c, int dtype, int d, int G);
// One sequence's block in a batched chunk or prompt launch: n >= 1 queries at
// t0..t0+n-1, rows packed end to end in q / k_blk / v_blk / out in entry order.
struct ChunkEntry {
  int seq;
  int n;
  int64_t t0;
  int64_t next_pos;  // the sequence's ring state from the host's bookkeeping
  int P, head, count, owner;
};
constexpr int kMaxChunkBatch = 64;  // entries per launch
// prompt != 0: queries inside the prefix attend causally to the prefix rows
// [0, t] (k_blk / v_blk unused); otherwise chunks at t0 == next_pos.
cudaError_t launch_chunk_tc(const CacheDev& c, int G, const ChunkEntry* e, int nb, int Hq,
                            const void* q, const void* k_blk, const void* v_blk, void* out,
                            float scale, int prompt, int sm_count, cudaStream_t st);

// attend.cu (CUDA-core chunk kernel)
cudaError_t launch_chunk_cc(const CacheDev& c, int dtype, int G, int seq, int64_t t0, int n,
                            int Hq, const void* q, const void* k_blk, const void* v_blk,
                            void* out, float scale, int prompt, cudaStream_t st);

// api.cu: error message of the calling thread, and cache accessors.
int set_error(int code, const char* fmt, ...);

}  // namespace ps

struct ps_cache;
namespace ps {
// Every host-side check of ps_attend_decode except the workspace's (the
// message is set on failure); *G receives Hq / Hkv.
int check_decode_call(ps_cache* c, const void* q, const int* seq_ids, const int64_t* t, int B,
                      int Hq, const void* out, int* G);
int cache_hkv(const ps_cache* c);
int cache_head_dim(const ps_cache* c);
int cache_sm_count(const ps_cache* c);
}  // namespace ps
