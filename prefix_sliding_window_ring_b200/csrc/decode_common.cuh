// Pieces shared by the two decode streaming kernels (the CUDA-core one in
// decode.cu, the tensor-core one in decode_mma.cu): launch arguments, the
// flattened tile ranges of the split, tile flags and the pair merge.
//
// Split.  Each (batch entry, kv head) pair's visible rows are cut into tiles
// (how many depends on the kernel's tile shape); the tiles of all pairs are
// laid end to end, entry-major then kv head, and CTA c of nctas streams the
// tiles [T c / nctas, T (c + 1) / nctas).  For every (CTA range, pair) piece
// a CTA emits one partial (max, sum, accumulator) triple; k_decode_merge
// combines each pair's partials into the output.
#pragma once
#include <math.h>
#include <string.h>

#include "attn_common.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

namespace ps {
namespace dec {

using namespace attn;

constexpr long long kWaitLimitCycles = 1ll << 30;  // about half a second
constexpr int kPieceBatch = 8;  // partials read together by the pair merge
constexpr int kMergeThreads = 128;
constexpr float kRaiseLog2 = 8.0f;  // running-max hysteresis, log2 units
constexpr int kMinTilesPerCta = 2;
constexpr int kDecMaxCtasPerSm = 2;  // CTAs per SM of either streaming kernel, at most

struct DecodeArgs {
  CacheDev c;
  const void* q;
  const void* knew;  // decode step: appended rows [B][Hkv][D] (NULL for a plain decode)
  const void* vnew;
  void* out;
  float qscale;
  int Hq, B, nctas;
  int csize;           // tensor-core kernel: CTAs per pair in a cluster (0: flattened split)
  int32_t total;       // tiles of all pairs of the launch
  float* part_ml;      // [nctas + B*Hkv][G][2]: per (CTA range, pair) piece (max, sum), base 2
  float* part_o;       // [nctas + B*Hkv][G][D]: per piece unnormalised accumulators
  int32_t seq[kMaxBatchPerLaunch];
  int32_t P[kMaxBatchPerLaunch];      // prefix length of entry b
  int32_t head[kMaxBatchPerLaunch];   // physical ring slot of entry b's oldest window row
  int32_t count[kMaxBatchPerLaunch];  // ring rows of entry b
  int32_t owner[kMaxBatchPerLaunch];  // sequence whose slab holds entry b's prefix rows
  int64_t t[kMaxBatchPerLaunch];
  int32_t tcum[kMaxBatchPerLaunch + 1];  // tcum[b] = Hkv * (tiles per head of entries before b)
};

// Chunk mode of the tensor-core kernel (small chunk blocks; cluster mode):
// entry b of the launch's DecodeArgs is a group of nq[b] consecutive queries
// of a block, the first at position t[b], the i0[b]-th of its block (the ring
// state is the one before the block); the block's rows start at row brow[b]
// of the launch's block buffers, the group's q / out rows at row qrow[b].  The
// kernel's G columns hold the group's queries x gq heads (query k, head h in
// column k gq + h).  A separate kernel instantiation, so the decode kernels
// carry none of it.
struct ChunkArgs {
  int gq, lgq;  // query heads per kv head, and its log2
  int32_t qrow[kMaxBatchPerLaunch];
  int32_t nq[kMaxBatchPerLaunch];
  int32_t i0[kMaxBatchPerLaunch];
  int32_t brow[kMaxBatchPerLaunch];
};
// Kernel parameters above 4 KB need CUDA 12.1 and sm_70 or later (limit 32764 bytes).
static_assert(sizeof(DecodeArgs) <= 32764, "decode arguments fit the kernel parameter space");

// Tiles of the launch.  Pair (b, g) is cut into tph(b) = ceil(rows_b / TR)
// tiles of TR consecutive logical rows (the last one ragged); the tiles of all
// pairs are laid end to end (entry-major, then kv head) and CTA c streams the
// tiles [T c / NC, T (c + 1) / NC).  So every CTA streams the same number of
// tiles, and only a pair's last tile is ever short.
struct PairTiles {
  int b, g;
  int32_t tph;    // tiles of the pair
  int32_t first;  // flattened index of the pair's first tile
};
__device__ __forceinline__ PairTiles pair_of_tile(const DecodeArgs& a, int32_t x) {
  int lo = 0, hi = a.B - 1;
  while (lo < hi) {  // last entry with tcum[b] <= x
    const int mid = (lo + hi + 1) >> 1;
    if (a.tcum[mid] <= x) lo = mid; else hi = mid - 1;
  }
  PairTiles pt;
  pt.b = lo;
  pt.tph = (a.tcum[lo + 1] - a.tcum[lo]) / a.c.Hkv;
  pt.g = (x - a.tcum[lo]) / pt.tph;
  pt.first = a.tcum[lo] + pt.g * pt.tph;
  return pt;
}

// First flattened tile of CTA c's range, and the CTA whose range holds tile x.
// First flattened tile of CTA c's range, and the CTA whose range holds tile x.
__device__ __forceinline__ int32_t range_start(int64_t c, int64_t T, int64_t NC) {
  return (int32_t)(T * c / NC);
}
__device__ __forceinline__ int32_t cta_of_tile(int64_t x, int64_t T, int64_t NC) {
  return (int32_t)(((x + 1) * NC - 1) / T);
}

enum : int32_t {
  TD_FIRST = 1,  // first tile of a piece (brings the piece's q rows)
  TD_LAST = 2,   // last tile of a piece
  TD_END = 4,    // no more tiles
  TD_NEW = 8,    // the tile's last row is the appended token (decode step)
  TD_QMASK = 16, // chunk mode: per-row query masks in the descriptor
};

// Pair merge: one thread per four consecutive output elements of one pair.
// It runs as a programmatic dependent launch after k_decode: its CTAs may be
// scheduled while k_decode drains, and griddepcontrol.wait returns once every
// k_decode CTA has finished and its partials are visible.  The pieces of a
// pair sit in the slots of the consecutive CTA ranges [first, last] that hold
// its rows; their (max, sum, accumulator) triples combine by the usual online
// rescaling (base-2 exponents, the max subtracted before exponentiating).
template <typename T, int D, int G>
__global__ void __launch_bounds__(kMergeThreads) k_decode_merge(const __grid_constant__ DecodeArgs a) {
  ptx::pdl_launch_dependents();  // the next call's streaming grid may be scheduled
  ptx::pdl_wait_primary();
  constexpr int Q = G * D / 4;  // float4 groups per pair
  const int Hkv = a.c.Hkv;
  const int64_t gi = (int64_t)blockIdx.x * kMergeThreads + threadIdx.x;
  if (a.knew != nullptr && gi < a.B) {  // decode step: commit each entry's new bookkeeping
    DevMeta m;
    memset(&m, 0, sizeof(m));
    m.next_pos = a.t[gi] + 1;
    m.P = a.P[gi];
    m.head = a.head[gi];
    m.count = a.count[gi];
    m.owner = a.owner[gi];
    a.c.meta[a.seq[gi]] = m;
  }
  if (gi >= (int64_t)a.B * Hkv * Q) return;
  const int pair = (int)(gi / Q), qi = (int)(gi % Q);
  const int h = qi * 4 / D, e0 = qi * 4 % D;
  const int b = pair / Hkv, g = pair % Hkv;
  const int64_t R = a.total, NC = a.nctas;
  const int32_t tph = (a.tcum[b + 1] - a.tcum[b]) / Hkv;
  const int32_t pfirst = a.tcum[b] + g * tph;
  const int64_t first = cta_of_tile(pfirst, R, NC), last = cta_of_tile(pfirst + tph - 1, R, NC);
  float M = -INFINITY, L = 0.f;
  float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int64_t c0 = first; c0 <= last; c0 += kPieceBatch) {
    float2 ml[kPieceBatch];
    float4 o[kPieceBatch];
#pragma unroll
    for (int j = 0; j < kPieceBatch; ++j) {
      const int64_t sl = c0 + j + pair;
      const bool in = c0 + j <= last;
      ml[j] = in ? __ldcg((const float2*)(a.part_ml + ((size_t)sl * G + h) * 2))
                 : make_float2(-INFINITY, 0.f);
      o[j] = in ? __ldcg((const float4*)(a.part_o + ((size_t)sl * G + h) * D + e0))
                : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float bm = M;
#pragma unroll
    for (int j = 0; j < kPieceBatch; ++j) bm = fmaxf(bm, ml[j].x);
    if (bm == -INFINITY) continue;
    const float sc = exp2f(M - bm);  // M = -inf gives 0
    L *= sc;
    A.x *= sc; A.y *= sc; A.z *= sc; A.w *= sc;
#pragma unroll
    for (int j = 0; j < kPieceBatch; ++j) {
      const float w = (ml[j].x == -INFINITY) ? 0.f : exp2f(ml[j].x - bm);
      L += ml[j].y * w;
      A.x += o[j].x * w; A.y += o[j].y * w; A.z += o[j].z * w; A.w += o[j].w * w;
    }
    M = bm;
  }
  T* orow = (T*)a.out + ((size_t)b * a.Hq + (size_t)g * G + h) * D + e0;
  store_out<T>(orow + 0, A.x / L);
  store_out<T>(orow + 1, A.y / L);
  store_out<T>(orow + 2, A.z / L);
  store_out<T>(orow + 3, A.w / L);
}

// The pair merge as a programmatic dependent launch of the streaming grid.
template <typename T, int D, int G>
cudaError_t launch_merge(const DecodeArgs& a, cudaStream_t st) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  const int64_t groups = (int64_t)a.B * a.c.Hkv * (G * D / 4);
  cfg.gridDim = dim3((unsigned)((groups + kMergeThreads - 1) / kMergeThreads));
  cfg.blockDim = dim3(kMergeThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_decode_merge<T, D, G>, a);
}

}  // namespace dec

// decode_mma.cu: the tensor-core streaming kernel (bfloat16) and its merge.
cudaError_t launch_decode_mma(const dec::DecodeArgs& a, int G, const DecodeMaps& maps,
                              int sm_count, cudaStream_t st);
// The same kernel in chunk mode (8 columns, cluster mode): block rows from
// k_blk / v_blk ([blk_rows][Hkv][d], 16-byte aligned).
cudaError_t launch_chunk_small(const dec::DecodeArgs& a, const dec::ChunkArgs& ch,
                               const DecodeMaps& maps, const void* k_blk, const void* v_blk,
                               int64_t blk_rows, int sm_count, cudaStream_t st);

}  // namespace ps
