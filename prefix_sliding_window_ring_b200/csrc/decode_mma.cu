// Decode attention for bfloat16 caches (head_dim 64 or 128) with the per-row
// products on the tensor cores, and the decode step that appends the token in
// the same pass.
//
// Why tensor cores for a bandwidth-bound kernel.  Per visible K/V row a
// decode query does 2 G d multiply-adds for its G query heads.  Done on the
// CUDA cores (one lane per 16 bytes of a row, shuffle reductions for the
// scores) that costs about 50 warp instructions per row, which caps an SM at
// about the copy bandwidth and leaves no slack to absorb the pipeline's start
// and end.  As warp-level MMAs the same work is about 4 warp instructions per
// row, so HBM is the only bound.  The products themselves are negligible
// (G <= 8 heads padded to the MMA's 8 columns).
//
// Work division (as in the CUDA-core kernel): each (batch entry, kv head)
// pair's visible rows are cut into tiles of kTR rows, the tiles of all pairs
// are laid end to end and CTA c streams the tiles [T c / NC, T (c + 1) / NC);
// every (CTA range, pair) piece emits one partial, merged by k_decode_merge.
// The tile layout (decode_pack.cuh) places every row at the offset within its
// 8-row atom that its row or slot has modulo 8, so that whole atoms can be
// loaded by tensor-map copies; no atom holds rows of two pieces.
//
// Streaming.  Two producers (one lane of each of warps kMW and kMW + 1) take
// alternate tiles: per tile a producer issues tensor-map copies
// (cp.async.bulk.tensor, 128-byte swizzle, no multicast) of the 8-row atoms
// holding each piece's K and V rows into a kStages-deep ring of shared-memory
// stages -- one copy per 64-row tile, per small page or per atom, all column
// blocks at once through 5D maps of the prefix and ring slabs (8-row boxes of
// one column block where a copy cannot start on an atom of its slab) -- and
// the pair's q rows with the first tile of a piece and the appended token of a
// decode step by plain bulk copies.  Rows a copy brings before or after its
// piece are masked.
// No evicted row is a valid row of any tile ("Prefix Sliding" digest, section
// 06: the prefix and the window are walked separately).
//
// Consumers (kMW warps).  Warp w takes the 16-row groups w, w + kMW, ... of
// every tile and keeps its own online-softmax state for its rows:
//   S^T (16 rows x 8 heads) = K (16 x d) Q^T (d x 8)   m16n8k16 bf16 MMAs,
//       K fragments by ldmatrix from the swizzled tile, Q^T (heads beyond G
//       zero) in registers;
//   per head a running max raised lazily (only when a score passes it by more
//       than 2^8, so the accumulators are rescaled on few groups; a warp vote
//       decides, the rare raise takes a shuffle maximum over the 16 rows);
//   weights p = 2^(s - max) rounded to bfloat16 and transposed in registers
//       (movmatrix) into the B fragment of
//   O^T (d x 8) += V^T (d x 16 rows) P^T (16 rows x 8)   with V^T fragments
//       by transposing ldmatrix.
// Rows of a group that are not valid get score -inf and their V rows in
// shared memory are zeroed first, so nothing outside the visible set reaches
// the accumulators.  At the end of a piece the warps' states are merged
// through shared memory into the piece's partial.
//
// Every wait is bounded; a time-out stops the CTA, sets ERR_TIMEOUT and lets
// the copies already issued land before the CTA exits.
#include <math.h>
#include <string.h>

#include <atomic>

#include "decode_common.cuh"
#include "decode_pack.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

#ifndef PS_DMMA_TR
#define PS_DMMA_TR 64
#endif
#ifndef PS_DMMA_STAGES
#define PS_DMMA_STAGES 3
#endif
#ifndef PS_DMMA_CTAS_PER_SM
#define PS_DMMA_CTAS_PER_SM 2
#endif
#ifndef PS_DMMA_L2_PROMOTION
#define PS_DMMA_L2_PROMOTION 2
#endif

namespace ps {

namespace {

using namespace dec;

constexpr int kMW = 4;                      // consumer warps
constexpr int kProd = 2;                    // producer warps (one lane each), alternate tiles
constexpr int kThreadsM = (kMW + kProd) * 32;
constexpr int kTR = PS_DMMA_TR;             // rows per tile
constexpr int kStagesM = PS_DMMA_STAGES;
constexpr int kGroups = kTR / 16;           // 16-row MMA groups per tile
constexpr int kBox = 64;                    // rows of the large tensor-map box
constexpr int kMaxCluster = 8;              // CTAs per pair in cluster mode, at most
constexpr int kTblMax = 256;                // page-table entries staged in shared memory
static_assert(kTR == 64, "tile rows: 64 (the valid-row mask is one 64-bit word)");
constexpr float kMaxFloor = -1e30f;         // running max of a column before its first row
static_assert(PS_DMMA_CTAS_PER_SM <= kDecMaxCtasPerSm, "workspace slots cover every CTA");

struct MmaDecodeArgs {
  DecodeMaps maps;  // first: tensor maps must be 64-byte aligned
  DecodeArgs a;
};
struct MmaChunkArgs {
  DecodeMaps maps;
  // the launch's block rows k_blk / v_blk [rows][Hkv][D], boxes of 8 rows of
  // one 64-column block of one kv head
  CUtensorMap kblk, vblk;
  DecodeArgs a;
  ChunkArgs ch;
};
static_assert(sizeof(MmaDecodeArgs) <= 32764, "decode arguments fit the kernel parameter space");
static_assert(sizeof(MmaChunkArgs) <= 32764, "chunk arguments fit the kernel parameter space");
template <bool CHUNK> struct MmaArgsOf { using type = MmaDecodeArgs; };
template <> struct MmaArgsOf<true> { using type = MmaChunkArgs; };
template <bool CHUNK> using MmaArgs = typename MmaArgsOf<CHUNK>::type;

struct TileDescM {
  uint32_t mask[kTR / 32];  // valid rows: bit r % 32 of word r / 32
  int32_t pair, flags;
  int32_t slot;             // partial-result slot of the piece: CTA range + pair
  int32_t new_row;          // TD_NEW: tile row of the appended token
  uint8_t qv[kTR];          // TD_QMASK: bit k of row r set if the group's query k sees it
};

// ------------------------------------------------------------- warp MMA --
__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void ldsm4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
// d += a b, m16n8k16, bf16 inputs, f32 accumulators (row-major A, column-major B)
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Online-softmax state of one consumer lane: lane (g, t) holds, for the
// columns 2t and 2t+1 (query heads; in chunk mode query x head), the running
// max m (log2 units; +inf for a padding column, which then gets weight 0; a
// valid column starts at the finite floor kMaxFloor, so that a column whose
// rows so far were all masked gets weight ex2(-inf - floor) = 0, not NaN), its
// partial sum l over the rows it has seen, and O^T rows d = 16 mt + g and
// 16 mt + g + 8 of both columns.
template <int D, int G>
struct MmaState {
  static constexpr int KS = D / 16;  // k-steps of S^T, m-tiles of O^T
  uint32_t qf[KS][2];                // Q^T fragments
  float o[KS][4];
  float m[2], l[2];

  // ncols: valid columns (<= G); the others are padding
  __device__ __forceinline__ void init(const uint8_t* qs, int ncols) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      // columns g >= ncols are padding: zero columns of Q^T (their q rows are not loaded)
      const uint8_t* row = qs + (size_t)(g < ncols ? g : 0) * D * 2 + (size_t)(16 * ks + 2 * t) * 2;
      const uint32_t lo = *(const uint32_t*)row, hi = *(const uint32_t*)(row + 16);
      qf[ks][0] = g < ncols ? lo : 0u;
      qf[ks][1] = g < ncols ? hi : 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) o[ks][e] = 0.f;
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      m[hh] = 2 * t + hh < ncols ? kMaxFloor : INFINITY;
      l[hh] = 0.f;
    }
  }
};

// CHUNK: chunk mode (a pair is a group of a block's queries and one kv head;
// its columns are the group's queries x gq heads; always with CL).
// CL: cluster mode.  Pair p is streamed by the csize CTAs of cluster p, CTA
// rank r taking an equal share of its padded rows (dec_cluster_share).  Each
// CTA then pushes its merged state into its peers' shared memory
// (asynchronous remote stores that count their bytes on the receiver's
// barrier: its (max, sum) per column to all, its accumulator values of output
// slice r to rank r), waits for theirs and combines its own slice of the
// pair's output from local shared memory -- no partials in global memory, no
// second grid, no CTA reading another's memory.  The sequence's record is
// checked (and a decode step's new state committed) by rank 0 of kv head 0
// once its copies are issued.  Otherwise the flattened split with
// k_decode_merge.
template <int D, int G, bool CL, bool CHUNK>
__global__ void __launch_bounds__(kThreadsM, PS_DMMA_CTAS_PER_SM)
    k_decode_mma(const __grid_constant__ MmaArgs<CHUNK> ma) {
  static_assert(CL || !CHUNK, "chunk mode runs in cluster mode");
  constexpr int HALVES = D / 64;                       // 128-byte column blocks of a row
  // Tile layout in shared memory: 8-row atoms one after the other, each
  // holding its rows of every 64-column block ([atom][block][8 rows][128
  // bytes], 128-byte swizzle inside each 1 KiB block), so one atom-map copy
  // brings whole atoms of all column blocks.
  constexpr uint32_t kAtomBytes = HALVES * 1024;       // one 8-row atom, all column blocks
  constexpr uint32_t kTileBytes = (kTR / 8) * kAtomBytes;  // K (or V) of one tile
  constexpr int KS = D / 16;
  const DecodeArgs& a = ma.a;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* const kbuf = (uint8_t*)(((uintptr_t)dsm_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* const vbuf = kbuf + kStagesM * kTileBytes;
  uint8_t* const qbuf = vbuf + kStagesM * kTileBytes;  // [kStagesM][G][D] bf16
  __shared__ __align__(8) uint64_t full[kStagesM], empty[kStagesM];
  __shared__ __align__(8) uint64_t sync_a, sync_b, sync_m;
  __shared__ __align__(8) uint64_t pub_bar;  // cluster: the peers' states have arrived
  __shared__ TileDescM desc[kStagesM];
  __shared__ int abort_flag;
  // The warps' merge buffer.  In cluster mode a CTA streams one piece, so
  // once every warp has consumed its last tile the K stages hold nothing more
  // and the buffer lives there (two CTAs per SM fit at any G); the flattened
  // split streams the next piece meanwhile and keeps a buffer of its own.
  using Merge = MergeSmem<G, D, kMW>;
  static_assert(sizeof(Merge) <= (size_t)kStagesM * kTileBytes, "merge buffer fits the K stages");
  __shared__ __align__(16) uint8_t sm_own[CL ? 16 : sizeof(Merge)];
  Merge& sm = *reinterpret_cast<Merge*>(CL ? kbuf : sm_own);
  __shared__ float pub_ml[G][2];  // cluster: this CTA's merged (max, sum) per column
  // cluster: the states the peers push here -- each rank's (max, sum) per
  // column, and its accumulator values of the output slice this CTA combines
  // (slice r of the G*D outputs belongs to rank r)
  __shared__ float rcv_ml[kMaxCluster][G][2];
  __shared__ __align__(16) float rcv_o[G * D];
  // paged cache: the page-table row of the piece's sequence (read by the producer only)
  __shared__ __align__(16) int32_t tbl[kProd][kTblMax + 4];  // one per producer
  __shared__ __align__(8) uint64_t tbl_bar[kProd];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Hkv = a.c.Hkv;
  const int64_t R = a.total, NC = a.nctas;
  // Columns of pair (b, g): a decode pair's G query heads; a chunk pair's
  // nq queries x gq heads.  q and out rows: [rows][Hq][D].
  constexpr int kLgG = G == 8 ? 3 : G == 4 ? 2 : G == 2 ? 1 : 0;
  auto lgq = [&]() -> int {
    if constexpr (CHUNK) return ma.ch.lgq; else return kLgG;
  };
  auto nq_of = [&](int b) -> int {
    if constexpr (CHUNK) return ma.ch.nq[b]; else return 1;
  };
  auto qrow_of = [&](int b) -> int {
    if constexpr (CHUNK) return ma.ch.qrow[b]; else return b;
  };
  // ring state the entry's queries see (a chunk group: the state before its block)
  auto next_pos_of = [&](int b) -> int64_t {
    if constexpr (CHUNK) return a.t[b] - ma.ch.i0[b]; else return a.t[b] + 1;
  };
  auto qo_off = [&](int b, int g, int c) -> size_t {
    const int gq = 1 << lgq();
    return ((size_t)(qrow_of(b) + (c >> lgq())) * a.Hq + (size_t)g * gq + (c & (gq - 1))) *
           (size_t)D;
  };
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStagesM; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], kMW);
    }
    ptx::mbar_init(&sync_a, kMW);
    ptx::mbar_init(&sync_b, kMW);
    ptx::mbar_init(&sync_m, kMW);
    ptx::mbar_init(&pub_bar, 1);
    for (int p = 0; p < kProd; ++p) ptx::mbar_init(&tbl_bar[p], 1);
    abort_flag = 0;
    ptx::fence_mbar_init();
    // cluster: the peers' states arrive as asynchronous stores that count
    // their bytes on pub_bar -- from each of the csize - 1 peers its slice of
    // G * D / csize values and its (max, sum) per column
    if (CL)
      ptx::mbar_arrive_expect_tx(
          &pub_bar, (uint32_t)((a.csize - 1) * (G * D / a.csize + 2 * G) * sizeof(float)));
  }
  if (warp == kMW && lane == 0) {
    // fetch the tensor maps' descriptors while the previous grid drains
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      if (ma.maps.prefix_atoms) {
        ptx::prefetch_tmap(&ma.maps.kpa[k]);
        ptx::prefetch_tmap(&ma.maps.vpa[k]);
      }
      if (ma.maps.ring_atoms) {
        ptx::prefetch_tmap(&ma.maps.kra[k]);
        ptx::prefetch_tmap(&ma.maps.vra[k]);
      }
    }
    if (ma.maps.page_box) {
      ptx::prefetch_tmap(&ma.maps.kra[2]);
      ptx::prefetch_tmap(&ma.maps.vra[2]);
    }
    ptx::prefetch_tmap(&ma.maps.kring8);
    ptx::prefetch_tmap(&ma.maps.vring8);
    if constexpr (CHUNK) {
      ptx::prefetch_tmap(&ma.kblk);
      ptx::prefetch_tmap(&ma.vblk);
    }
  }
  __syncthreads();
  // Cluster mode: every CTA of the cluster must have initialised its barriers
  // before any remote arrive (the consumers' epilogue).  All threads arrive
  // here; the consumers wait at once, the producer only after setting up its
  // first piece, which so overlaps the barrier.
  if (CL) ptx::cluster_arrive();
  // Programmatic dependent launch: the next grid may be scheduled.  Only the
  // producer waits for the previous grid (griddepcontrol.wait), just before its
  // first copy: everything the consumers read or write in global memory comes
  // after a tile that the producer issued after that wait, and the setup of
  // the first piece overlaps the previous grid's tail.
  ptx::pdl_launch_dependents();

  if (warp >= kMW) {
    if (lane != 0) return;
    // ----------------------------------------------------------- producers --
    // Producer pw issues the tiles i with i % kProd == pw; both walk every
    // piece and tile so that each knows every tile's stage and phase.
    const int pw = warp - kMW;
    const bool step = a.knew != nullptr;
    const int32_t page = a.c.page_table ? a.c.page_rows : 0;
    int i = 0;  // tiles handed out so far
    bool alive = true;
    bool waited = false;  // griddepcontrol.wait done
    int tbl_n = 0;        // page-table rows staged so far (the barrier's phase)
    auto wait_primary = [&]() {
      if (!waited) {
        if (CL) ptx::cluster_wait_one();
        ptx::pdl_wait_primary();
        waited = true;
      }
    };
    // One piece of pair (b, g): its tiles [j0, j1) (flattened split, tph
    // tiles in all), or with rank >= 0 the cluster share of CTA `rank`.
    // check: compare the device record with the launch's state (flattened
    // split: every piece; cluster mode: rank 0 of kv head 0, which also
    // commits a decode step's new state -- no other CTA of the launch reads
    // or writes the record, so it is done once the copies are issued, off the
    // output's path).
    auto piece = [&](int b, int g, int32_t tph, int32_t j0, int32_t j1, int rank, bool check) {
      const int s = a.seq[b];
      DevMeta m;
      m.next_pos = next_pos_of(b);
      m.P = a.P[b];
      m.head = a.head[b];
      m.count = a.count[b];
      m.owner = a.owner[b];
      const DecRuns runs = [&]() {
        if constexpr (CHUNK)
          return dec_runs_chunk(m, a.c.W, m.next_pos, ma.ch.i0[b], ma.ch.nq[b], page);
        else
          return dec_runs(m, a.c.W, a.t[b], page, step);
      }();
      bool bad = (!CHUNK && runs.rows != m.P + m.count) ||
                 (rank < 0 && dec_tiles(runs, kTR) != tph);
      const int pair = b * Hkv + g;
      // the pair's q rows: one bulk copy per query of the entry, its heads of
      // kv head g each (a decode entry: one copy of G heads)
      const uint32_t qbytes = (uint32_t)((nq_of(b) << lgq()) * D * 2);
      auto load_q = [&](int st) {
        for (int k = 0; k < nq_of(b); ++k)
          ptx::bulk_g2s(qbuf + ((size_t)st * G + ((size_t)k << lgq())) * D * 2,
                        (const uint16_t*)a.q + qo_off(b, g, k << lgq()),
                        (uint32_t)((1 << lgq()) * D * 2), &full[st]);
      };
      const int zpre = m.owner * Hkv + g;
      // padded rows [xs, xe) of this piece, in tiles of kTR rows (the last may be short)
      int32_t xs, xe;
      if (rank >= 0) {
        dec_cluster_share(runs, rank, a.csize, &xs, &xe);
      } else {
        xs = j0 * kTR;
        xe = min(j1 * kTR, runs.padded);
      }
      const int32_t nt = xe > xs ? (xe - xs + kTR - 1) / kTR : 0;
      // Paged cache: stage the sequence's page-table row in shared memory with
      // one bulk copy, so that a page's physical number is a shared-memory read
      // instead of a dependent global load on this thread.
      const int32_t* tab = nullptr;  // shared copy, or NULL: read the global table
      if (page && nt > 0 && a.c.npg <= kTblMax && alive) {
        wait_primary();  // the table may just have been written by the previous grid
        const uintptr_t src = (uintptr_t)(a.c.page_table + (int64_t)s * a.c.npg);
        const uintptr_t src16 = src & ~(uintptr_t)15;
        const int lead = (int)((src - src16) / 4);
        const uint32_t bytes = (uint32_t)(((src - src16) + (size_t)a.c.npg * 4 + 15) & ~(size_t)15);
        if (tbl_n > 0) fence_proxy_async_smem();  // earlier reads before the copy overwrites
        ptx::mbar_arrive_expect_tx(&tbl_bar[pw], bytes);
        ptx::bulk_g2s(tbl[pw], (const void*)src16, bytes, &tbl_bar[pw]);
        if (ptx::mbar_wait_bounded(&tbl_bar[pw], tbl_n & 1, &abort_flag, kWaitLimitCycles)) {
          tab = tbl[pw] + lead;
        } else {
          alive = false;
        }
        ++tbl_n;
      }
      auto phys_of = [&](int32_t slot) -> int {
        return tab ? tab[pg_div(slot, page, runs.plg)] : ring_page(a.c, s, slot);
      };
      // the atom maps of a prefix (pre) or ring copy
      auto amap = [&](bool pre, bool isv, int k) -> const CUtensorMap* {
        return pre ? (isv ? &ma.maps.vpa[k] : &ma.maps.kpa[k])
                   : (isv ? &ma.maps.vra[k] : &ma.maps.kra[k]);
      };
      for (int32_t k = 0; k < nt && alive; ++k) {
        if (i % kProd != pw) {  // the other producer's tile
          ++i;
          continue;
        }
        const int32_t x0 = xs + k * kTR, x1 = min(x0 + kTR, xe);
        const int st = i % kStagesM;
        if (i >= kStagesM && !ptx::mbar_wait_bounded(&empty[st], ((i / kStagesM) - 1) & 1,
                                                      &abort_flag, kWaitLimitCycles)) {
          alive = false;
          break;
        }
        wait_primary();
        uint8_t* const kd = kbuf + (size_t)st * kTileBytes;
        uint8_t* const vd = vbuf + (size_t)st * kTileBytes;
        const int32_t flags0 = (k == 0 ? TD_FIRST : 0) | (k == nt - 1 ? TD_LAST : 0);
        int32_t wsrc, wrow;
        const bool qdep = CHUNK && dec_tile_qdep(runs, x0, x1);
        if (!qdep && dec_range_whole(runs, kTR, x0, x1, &wsrc, &wrow)) {
          // the common case: the tile is kTR rows of one run, copied whole
          desc[st].mask[0] = 0xffffffffu;
          desc[st].mask[1] = 0xffffffffu;
          desc[st].pair = pair;
          desc[st].flags = flags0;
          desc[st].slot = (int32_t)blockIdx.x + pair;
          desc[st].new_row = -1;
          ptx::mbar_arrive_expect_tx(&full[st],
                                     2u * kTR * D * 2u + ((flags0 & TD_FIRST) ? qbytes : 0u));
          if (flags0 & TD_FIRST) load_q(st);
          const bool pre = wsrc == RUN_PREFIX;
          const int32_t y = pre ? wrow : (page ? pg_mod(wrow, page, runs.plg) : wrow);
          const int32_t z = pre ? zpre : phys_of(wrow) * Hkv + g;
          if (pre ? ma.maps.prefix_atoms : ma.maps.ring_atoms) {  // one copy per operand: 8 atoms
            ptx::tma_load_5d(kd, amap(pre, false, 0), 0, 0, 0, y >> 3, z, &full[st]);
            ptx::tma_load_5d(vd, amap(pre, true, 0), 0, 0, 0, y >> 3, z, &full[st]);
          } else {  // an atom of a column block per copy
            for (int t = 0; t < kTR / 8; ++t) {
#pragma unroll
              for (int h = 0; h < HALVES; ++h) {
                ptx::tma_load_3d(kd + t * kAtomBytes + h * 1024, pre ? &ma.maps.kpre8 : &ma.maps.kring8,
                                 h * 64, y + 8 * t, z, &full[st]);
                ptx::tma_load_3d(vd + t * kAtomBytes + h * 1024, pre ? &ma.maps.vpre8 : &ma.maps.vring8,
                                 h * 64, y + 8 * t, z, &full[st]);
              }
            }
          }
          ++i;
          continue;
        }
        uint64_t mask = 0;  // valid tile rows
        int32_t flags = flags0 | (qdep ? TD_QMASK : 0);
        int32_t new_row = -1;
        // One pass: each copy is issued as the tile's pieces are walked and
        // its bytes counted; the barrier's arrival with the byte count comes
        // last (an mbarrier's tx-count may run below zero until then, and the
        // phase cannot complete before the arrival).
        uint32_t bytes = 0;
        if (flags & TD_FIRST) {
          load_q(st);
          bytes += qbytes;
        }
        dec_range_pieces(runs, x0, x1, [&](int32_t src, int32_t row, int32_t sr, int32_t n) {
          mask |= (n >= 64 ? ~0ull : ((1ull << n) - 1ull)) << sr;
          if (src == RUN_NEW) {  // the appended token, straight from the caller's rows
            flags |= TD_NEW;
            new_row = sr;
            const uint16_t* kn = (const uint16_t*)a.knew + (size_t)pair * D;
            const uint16_t* vn = (const uint16_t*)a.vnew + (size_t)pair * D;
#pragma unroll
            for (int h = 0; h < HALVES; ++h) {  // row sr % 8 == 0: the swizzle is the identity
              ptx::bulk_g2s(kd + (sr >> 3) * kAtomBytes + h * 1024, kn + h * 64, 128u, &full[st]);
              ptx::bulk_g2s(vd + (sr >> 3) * kAtomBytes + h * 1024, vn + h * 64, 128u, &full[st]);
            }
            bytes += 2u * D * 2u;
            return;
          }
          if constexpr (CHUNK) {
            if (src == RUN_BLK) {
              // the block's rows from the caller's buffers, whole atoms from
              // the one holding the piece's first row
              const int32_t lead = sr & (kPadRows - 1);
              int32_t y = ma.ch.brow[b] + row - lead;
              for (int32_t x = sr - lead; x < sr + n; x += kPadRows, y += kPadRows) {
#pragma unroll
                for (int h = 0; h < HALVES; ++h) {
                  ptx::tma_load_3d(kd + (x >> 3) * kAtomBytes + h * 1024, &ma.kblk, h * 64, g, y,
                                   &full[st]);
                  ptx::tma_load_3d(vd + (x >> 3) * kAtomBytes + h * 1024, &ma.vblk, h * 64, g, y,
                                   &full[st]);
                }
                bytes += 2u * kPadRows * D * 2u;
              }
              return;
            }
          }
          const bool pre = src == RUN_PREFIX;
          int32_t y, z;
          if (pre) {
            y = row;
            z = zpre;
          } else {  // a ring piece lies within one page
            y = page ? pg_mod(row, page, runs.plg) : row;
            z = phys_of(row) * Hkv + g;
          }
          // copy whole atoms, from the one that holds the piece's first row
          // (its row or slot minus the offset within the atom: same page)
          const int32_t lead = sr & (kPadRows - 1);
          sr -= lead;
          y -= lead;
          n += lead;
          // Atom-map copies when the copy starts on an atom of its slab (prefix
          // rows always; ring rows of whole-atom slabs, except the newest row
          // of a plain decode, which starts an atom of the tile whatever its
          // slot); otherwise 8-row boxes of each column block.
          if ((pre ? ma.maps.prefix_atoms : ma.maps.ring_atoms) && (y & (kPadRows - 1)) == 0) {
            if (!pre && ma.maps.page_box && lead == 0 && n == page) {
              // a whole small page: one copy per operand
              ptx::tma_load_5d(kd + (sr >> 3) * kAtomBytes, &ma.maps.kra[2], 0, 0, 0, y >> 3, z,
                               &full[st]);
              ptx::tma_load_5d(vd + (sr >> 3) * kAtomBytes, &ma.maps.vra[2], 0, 0, 0, y >> 3, z,
                               &full[st]);
              bytes += 2u * (uint32_t)page * D * 2u;
              return;
            }
            while (n > 0) {  // 8 atoms or 1 atom per copy
              const bool big = n >= kBox;
              const int32_t rows = big ? kBox : kPadRows;
              ptx::tma_load_5d(kd + (sr >> 3) * kAtomBytes, amap(pre, false, big ? 0 : 1), 0, 0, 0,
                               y >> 3, z, &full[st]);
              ptx::tma_load_5d(vd + (sr >> 3) * kAtomBytes, amap(pre, true, big ? 0 : 1), 0, 0, 0,
                               y >> 3, z, &full[st]);
              bytes += 2u * (uint32_t)rows * D * 2u;
              sr += rows;
              y += rows;
              n -= rows;
            }
            return;
          }
          while (n > 0) {  // an atom of a column block per copy
#pragma unroll
            for (int h = 0; h < HALVES; ++h) {
              ptx::tma_load_3d(kd + (sr >> 3) * kAtomBytes + h * 1024,
                               pre ? &ma.maps.kpre8 : &ma.maps.kring8, h * 64, y, z, &full[st]);
              ptx::tma_load_3d(vd + (sr >> 3) * kAtomBytes + h * 1024,
                               pre ? &ma.maps.vpre8 : &ma.maps.vring8, h * 64, y, z, &full[st]);
            }
            bytes += 2u * kPadRows * D * 2u;
            sr += kPadRows;
            y += kPadRows;
            n -= kPadRows;
          }
        });
        desc[st].mask[0] = (uint32_t)mask;
        desc[st].mask[1] = (uint32_t)(mask >> 32);
        desc[st].pair = pair;
        desc[st].flags = flags;
        desc[st].slot = (int32_t)blockIdx.x + pair;
        desc[st].new_row = new_row;
        if (CHUNK && qdep) {
          // chunk mode: which of the group's queries see each row (prefix rows:
          // all; rows outside the pieces are masked anyway)
          uint32_t* qw = (uint32_t*)desc[st].qv;
          for (int w = 0; w < kTR / 4; ++w) qw[w] = 0xffffffffu;
          dec_range_pieces(runs, x0, x1, [&](int32_t src, int32_t row, int32_t sr, int32_t n) {
            if (src == RUN_PREFIX) return;
            for (int32_t r = 0; r < n; ++r)
              desc[st].qv[sr + r] = (uint8_t)dec_row_queries(runs, src, row + r);
          });
        }
        ptx::mbar_arrive_expect_tx(&full[st], bytes);
        ++i;
      }
      if (check && pw == 0) {
        const DevMeta md = a.c.meta[s];
        DevMeta me = md;  // the device record before this launch (a step advances it by one)
        if (step) {
          const int64_t W = a.c.W, cn = (int64_t)md.count + 1;
          me.next_pos = md.next_pos + 1;
          me.count = (int32_t)(cn < W ? cn : W);
          me.head = (int32_t)((md.head + (cn > W ? 1 : 0)) % W);
        }
        if (me.next_pos != m.next_pos || me.P != m.P || me.head != m.head ||
            me.count != m.count || me.owner != m.owner)
          bad = true;
        if (CL && step) {
          DevMeta mn;
          memset(&mn, 0, sizeof(mn));
          mn.next_pos = m.next_pos;
          mn.P = m.P;
          mn.head = m.head;
          mn.count = m.count;
          mn.owner = m.owner;
          a.c.meta[s] = mn;
        }
      }
      if (pw == 0 && bad) atomicOr(a.c.err, ERR_BATCH);
      if (pw == 0 && !runs.ring_ok) atomicOr(a.c.err, ERR_RING);
    };
    if (CL) {
      const int pair = blockIdx.x / a.csize, rank = (int)ptx::cluster_ctarank();
      const int b = pair / Hkv, g = pair % Hkv;
      piece(b, g, 0, 0, 0, rank, rank == 0 && g == 0);
    } else {
      const int32_t x1 = range_start(blockIdx.x + 1, R, NC);
      for (int32_t x = range_start(blockIdx.x, R, NC); x < x1 && alive;) {
        const PairTiles pt = pair_of_tile(a, x);
        const int32_t j0 = x - pt.first, j1 = min(pt.tph, x1 - pt.first);
        x = pt.first + j1;
        piece(pt.b, pt.g, pt.tph, j0, j1, -1, true);
      }
    }
    if (alive && i % kProd == pw) {  // end marker (its producer): a descriptor with no bytes
      wait_primary();
      const int st = i % kStagesM;
      if (i < kStagesM || ptx::mbar_wait_bounded(&empty[st], ((i / kStagesM) - 1) & 1,
                                                  &abort_flag, kWaitLimitCycles)) {
        TileDescM end;
        for (int w = 0; w < kTR / 32; ++w) end.mask[w] = 0u;
        end.pair = 0; end.flags = TD_END; end.slot = 0; end.new_row = -1;
        desc[st] = end;
        ptx::mbar_arrive(&full[st]);
        ++i;
      }
    }
    if (abort_flag) {  // let the copies already issued land before the CTA exits
      int quiet = 0;
      for (int k = max(0, i - kStagesM); k < i; ++k)
        if (k % kProd == pw)
          ptx::mbar_wait_bounded(&full[k % kStagesM], (k / kStagesM) & 1, &quiet, kWaitLimitCycles);
    }
    return;
  }

  // -------------------------------------------------------------- consumers --
  if (CL) ptx::cluster_wait();
  auto csync = [&](uint64_t* bar, int phase) -> bool {
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(bar);
    return __all_sync(0xffffffffu,
                      ptx::mbar_wait_bounded(bar, phase & 1, &abort_flag, kWaitLimitCycles));
  };
  const unsigned FULL = 0xffffffffu;
  const int g = lane >> 2, tq = lane & 3;
  const int sw = lane & 7;  // 128-byte swizzle: 16-byte chunk c of row r sits at c ^ (r & 7)
  // ldmatrix source rows of this lane: K as the A operand (matrices: rows 0-7 /
  // 8-15 of k 0-7, then of k 8-15), V transposed (rows 0-7 of d 0-7 / 8-15,
  // then rows 8-15)
  const int krow = (lane & 7) + ((lane >> 3) & 1) * 8, kchk = lane >> 4;
  const int vrow = (lane & 7) + ((lane >> 4) & 1) * 8, vchk = (lane >> 3) & 1;
  const float qs = a.qscale;
  MmaState<D, G> st;
  int np = 0;
  // cluster mode: this CTA's rank, the cluster size and the outputs per slice
  // (slice r of the G * D outputs belongs to rank r)
  const int rank = CL ? (int)ptx::cluster_ctarank() : 0, C = CL ? a.csize : 1;
  const int SL = G * D / C;
  // cluster mode: hand four merged values of outputs idx..idx+3 (one row,
  // one slice: D and SL are multiples of 4) to the slice's owner -- kept here
  // for this CTA's slice, else an asynchronous store that counts its bytes on
  // the owner's pub_bar -- and, from the thread holding a row's first values,
  // the row's (max, sum) to every peer.  No fence, no separate arrival.
  auto publish = [&](int idx, const float (&v)[4], float mx, float l) {
    const int r = idx / SL, h = idx / D, e = idx % D;
    if (r == rank) {
#pragma unroll
      for (int q = 0; q < 4; ++q) sm.o[0][h][e + q] = v[q];
    } else {
      ptx::st_async_v4_f32(ptx::map_to_rank(&rcv_o[rank * SL + (idx - r * SL)], r), v[0], v[1],
                           v[2], v[3], ptx::map_to_rank(&pub_bar, r));
    }
    if (e == 0) {
      pub_ml[h][0] = mx;
      pub_ml[h][1] = l;
      for (int r2 = 0; r2 < C; ++r2) {
        if (r2 == rank) continue;
        const uint32_t bar = ptx::map_to_rank(&pub_bar, r2);
        ptx::st_async_f32(ptx::map_to_rank(&rcv_ml[rank][h][0], r2), mx, bar);
        ptx::st_async_f32(ptx::map_to_rank(&rcv_ml[rank][h][1], r2), l, bar);
      }
    }
  };
  bool stopped = false;
  for (int i = 0;; ++i) {
    const int stg = i % kStagesM;
    const bool ok = ptx::mbar_wait_bounded(&full[stg], (i / kStagesM) & 1, &abort_flag,
                                           kWaitLimitCycles);
    if (!__all_sync(FULL, ok)) { stopped = true; break; }
    const TileDescM d = desc[stg];
    if (d.flags & TD_END) break;
    if (d.flags & TD_FIRST)
      st.init(qbuf + (size_t)stg * G * D * 2, CHUNK ? nq_of(d.pair / Hkv) << lgq() : G);
    uint8_t* const kt = kbuf + (size_t)stg * kTileBytes;
    uint8_t* const vt = vbuf + (size_t)stg * kTileBytes;
    const uint32_t kt_s = ptx::smem_u32(kt), vt_s = ptx::smem_u32(vt);
    bool wrote = false;
#pragma unroll 1
    for (int grp = warp; grp < kGroups; grp += kMW) {
      // (the mask word is read from shared memory: indexing a local copy by
      // the loop variable would put the copy in local memory)
      const uint32_t vm = (desc[stg].mask[grp >> 1] >> ((grp & 1) * 16)) & 0xffffu;
      if (vm == 0) continue;
      const int R0 = grp * 16;
      if (vm != 0xffffu) {
        // rows outside the visible set: their V rows must not reach O
        for (int idx = lane; idx < 16 * HALVES * 8; idx += 32) {
          const int r = idx / (HALVES * 8), h = (idx / 8) % HALVES, ch = idx % 8;
          if (!((vm >> r) & 1u))
            *(uint4*)(vt + ((R0 + r) >> 3) * kAtomBytes + h * 1024 + ((R0 + r) & 7) * 128 + ch * 16) =
                make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
        wrote = true;
      }
      // S^T = K Q^T
      float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int h = ks >> 2, chunk = (ks & 3) * 2 + kchk;
        uint32_t af[4];
        ldsm4(kt_s + ((R0 + krow) >> 3) * kAtomBytes + h * 1024 + ((R0 + krow) & 7) * 128 +
                  ((chunk ^ sw) << 4),
              af);
        mma16816(c, af, st.qf[ks][0], st.qf[ks][1]);
      }
      const bool r0 = (vm >> g) & 1u, r1 = (vm >> (g + 8)) & 1u;
      bool v00 = r0, v01 = r0, v10 = r1, v11 = r1;
      if (CHUNK && (d.flags & TD_QMASK)) {  // column 2tq + hh holds query (2tq + hh) >> lgq
        const uint32_t qa = desc[stg].qv[R0 + g], qb = desc[stg].qv[R0 + g + 8];
        const int k0 = (2 * tq) >> lgq(), k1 = (2 * tq + 1) >> lgq();
        v00 = v00 && ((qa >> k0) & 1u);
        v01 = v01 && ((qa >> k1) & 1u);
        v10 = v10 && ((qb >> k0) & 1u);
        v11 = v11 && ((qb >> k1) & 1u);
      }
      const float s0 = v00 ? c[0] * qs : -INFINITY, s1 = v01 ? c[1] * qs : -INFINITY;
      const float s2 = v10 ? c[2] * qs : -INFINITY, s3 = v11 ? c[3] * qs : -INFINITY;
      const bool need = s0 > st.m[0] + kRaiseLog2 || s2 > st.m[0] + kRaiseLog2 ||
                        s1 > st.m[1] + kRaiseLog2 || s3 > st.m[1] + kRaiseLog2;
      if (__any_sync(FULL, need)) {
        // rare: raise the running max of a head to the group's max
        float gm[2] = {fmaxf(s0, s2), fmaxf(s1, s3)};
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          gm[hh] = fmaxf(gm[hh], __shfl_xor_sync(FULL, gm[hh], 4));
          gm[hh] = fmaxf(gm[hh], __shfl_xor_sync(FULL, gm[hh], 8));
          gm[hh] = fmaxf(gm[hh], __shfl_xor_sync(FULL, gm[hh], 16));
          if (gm[hh] > st.m[hh] + kRaiseLog2) {
            const float alpha = ex2(st.m[hh] - gm[hh]);  // 0 when the max was -inf
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
              st.o[mt][hh] *= alpha;
              st.o[mt][hh + 2] *= alpha;
            }
            st.l[hh] *= alpha;
            st.m[hh] = gm[hh];
          }
        }
      }
      // every valid column's max is finite here (at least the floor); a
      // padding column's is +inf
      const float p0 = ex2(s0 - st.m[0]), p1 = ex2(s1 - st.m[1]);
      const float p2 = ex2(s2 - st.m[0]), p3 = ex2(s3 - st.m[1]);
      st.l[0] += p0 + p2;
      st.l[1] += p1 + p3;
      const uint32_t b0 = movm_t(pack_bf16(p0, p1)), b1 = movm_t(pack_bf16(p2, p3));
      // O^T += V^T P^T
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        const int h = mt >> 2, chunk = (mt & 3) * 2 + vchk;
        uint32_t af[4];
        ldsm4_t(vt_s + ((R0 + vrow) >> 3) * kAtomBytes + h * 1024 + ((R0 + vrow) & 7) * 128 +
                    ((chunk ^ sw) << 4),
                af);
        mma16816(st.o[mt], af, b0, b1);
      }
    }
    if ((d.flags & TD_NEW) && warp == (d.new_row >> 4) % kMW) {
      // decode step: store the appended token in its ring slot (the evicted
      // row's, never visible to this step's queries); tile row new_row is a
      // multiple of 8, where the swizzle is the identity
      const int b = d.pair / Hkv, gg = d.pair % Hkv, s = a.seq[b];
      const int32_t slot = (int32_t)(((int64_t)a.head[b] + a.count[b] - 1) % a.c.W);
      const int phys = ring_page(a.c, s, slot);
      const size_t row = (size_t)ring_row(a.c, phys, gg, slot) * D;
      constexpr int V16 = D * 2 / 16;  // 16-byte pieces per row
      for (int x = lane; x < 2 * V16; x += 32) {
        const bool isv = x >= V16;
        const int xi = isv ? x - V16 : x;
        const uint4 val =
            *(const uint4*)((isv ? vt : kt) + (d.new_row >> 3) * kAtomBytes + (xi / 8) * 1024 +
                            (xi % 8) * 16);
        ((uint4*)((uint16_t*)(isv ? a.c.V : a.c.K) + row))[xi] = val;
      }
      if (lane == 0 && gg == 0) a.c.pos[pos_index(a.c, phys, slot)] = a.t[b];
    }
    if (wrote) fence_proxy_async_smem();  // generic writes before the stage's next copies
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(&empty[stg]);
    if (!(d.flags & TD_LAST)) continue;

    // ---- end of a (CTA range, pair) piece: merge the warps' states ----
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      st.l[hh] += __shfl_xor_sync(FULL, st.l[hh], 4);
      st.l[hh] += __shfl_xor_sync(FULL, st.l[hh], 8);
      st.l[hh] += __shfl_xor_sync(FULL, st.l[hh], 16);
    }
    // cluster mode: the merge buffer is the K stages; every warp must be done
    // reading its last tile first
    if (CL && !csync(&sync_m, np)) { stopped = true; break; }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int h = 2 * tq + hh;
      if (h < G) {
        if (g == 0) {
          sm.m[warp][h] = st.m[hh];
          sm.l[warp][h] = st.l[hh];
        }
#pragma unroll
        for (int mt = 0; mt < KS; ++mt) {
          sm.o[warp][h][16 * mt + g] = st.o[mt][hh];
          sm.o[warp][h][16 * mt + g + 8] = st.o[mt][hh + 2];
        }
      }
    }
    if (!csync(&sync_a, np)) { stopped = true; break; }
    const int64_t slot = d.slot;
    float* pml = a.part_ml + (size_t)slot * G * 2;
    float* po = a.part_o + (size_t)slot * G * D;
    if constexpr (CL) {
      // four values per thread, published as soon as merged; this CTA's slice
      // is kept in place (each thread rewrites only its own values)
      for (int idx = 4 * threadIdx.x; idx < G * D; idx += 4 * kMW * 32) {
        const int h = idx / D, e = idx % D;
        float mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < kMW; ++w) mx = fmaxf(mx, sm.m[w][h]);
        float l = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int w = 0; w < kMW; ++w) {
          const float wt = (mx == -INFINITY) ? 0.f : exp2f(sm.m[w][h] - mx);
          l += sm.l[w][h] * wt;
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[q] += sm.o[w][h][e + q] * wt;
        }
        publish(idx, acc, mx, l);
      }
    } else {
      for (int idx = threadIdx.x; idx < G * D; idx += kMW * 32) {
        const int h = idx / D, e = idx % D;
        float mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < kMW; ++w) mx = fmaxf(mx, sm.m[w][h]);
        float l = 0.f, acc = 0.f;
#pragma unroll
        for (int w = 0; w < kMW; ++w) {
          const float wt = (mx == -INFINITY) ? 0.f : exp2f(sm.m[w][h] - mx);
          l += sm.l[w][h] * wt;
          acc += sm.o[w][h][e] * wt;
        }
        po[idx] = acc;
        if (e == 0) {
          pml[h * 2] = mx;
          pml[h * 2 + 1] = l;
        }
      }
    }
    // the merged state in shared memory before it is read (next piece's
    // merge; cluster mode: this CTA's slice and (max, sum) in the combine)
    if (!csync(&sync_b, np)) { stopped = true; break; }
    ++np;
  }

  if (CL && !stopped && !abort_flag) {
    // ---- cluster: combine the pair's csize states into its output ----
    if (np == 0) {  // no tiles in this CTA's share: publish an empty state
      const float zero[4] = {0.f, 0.f, 0.f, 0.f};
      for (int idx = 4 * threadIdx.x; idx < G * D; idx += 4 * kMW * 32)
        publish(idx, zero, -INFINITY, 0.f);
      if (!csync(&sync_b, 0)) stopped = true;
    }
    if (!stopped) {
      // the peers' states are here once all their bytes have landed
      const bool ok = ptx::mbar_wait_cluster_bounded(&pub_bar, 0, &abort_flag, kWaitLimitCycles);
      if (__all_sync(FULL, ok)) {
        const int pair = blockIdx.x / C, b = pair / Hkv, gg = pair % Hkv;
        const int ncols = nq_of(b) << lgq();  // valid columns of the pair
        // this CTA's slice of the outputs: each rank's weight 2^(m_r - M) / L
        // per column (L = sum_r l_r 2^(m_r - M)), found by every output thread
        // of the column for itself
        for (int k = threadIdx.x; k < SL; k += kMW * 32) {
          const int idx = rank * SL + k, h = idx / D, e = idx % D;
          if (h < ncols) {
            float mr[kMaxCluster], lr[kMaxCluster];
            float M = -INFINITY;
#pragma unroll
            for (int r = 0; r < kMaxCluster; ++r) {
              if (r < C) {
                mr[r] = r == rank ? pub_ml[h][0] : rcv_ml[r][h][0];
                lr[r] = r == rank ? pub_ml[h][1] : rcv_ml[r][h][1];
                M = fmaxf(M, mr[r]);
              }
            }
            float L = 0.f;
#pragma unroll
            for (int r = 0; r < kMaxCluster; ++r) {
              if (r < C) {
                mr[r] = (mr[r] == -INFINITY) ? 0.f : exp2f(mr[r] - M);
                L += lr[r] * mr[r];
              }
            }
            const float inv = 1.f / L;
            float A = 0.f;
#pragma unroll
            for (int r = 0; r < kMaxCluster; ++r)
              if (r < C) A += (r == rank ? sm.o[0][h][e] : rcv_o[r * SL + k]) * (mr[r] * inv);
            store_out<uint16_t>((uint16_t*)a.out + qo_off(b, gg, h) + e, A);
          }
        }
      }
    }
  }
  if (threadIdx.x == 0 && abort_flag) atomicOr(a.c.err, ERR_TIMEOUT);
}

// Resident CTAs per SM of one instantiation (at most PS_DMMA_CTAS_PER_SM).
template <int D, int G, bool CL, bool CHUNK>
int ctas_per_sm(size_t dyn) {
  static std::atomic<int> cached{0};
  int n = cached.load();
  if (n == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_decode_mma<D, G, CL, CHUNK>,
                                                      kThreadsM, dyn) != cudaSuccess ||
        n < 1)
      n = 1;
    if (n > PS_DMMA_CTAS_PER_SM) n = PS_DMMA_CTAS_PER_SM;
    cached.store(n);
  }
  return n;
}

template <int D, int G, bool CL, bool CHUNK>
cudaError_t configure(size_t dyn) {
  static std::atomic<uint64_t> configured{0};  // one bit per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(k_decode_mma<D, G, CL, CHUNK>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
    if (e != cudaSuccess) return e;
    // all of the unified L1/shared memory as shared, so that two CTAs fit per SM
    e = cudaFuncSetAttribute(k_decode_mma<D, G, CL, CHUNK>,
                             cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  return cudaSuccess;
}

// Clusters of c CTAs of one instantiation that are resident at once (the
// occupancy API's count: clusters must fit inside a GPC, so it is below
// 2 * SMs / c for c = 4 and 8).  Cached per cluster size; 0 on failure.
template <int D, int G, bool CHUNK>
int cluster_capacity(int c, size_t dyn) {
  static std::atomic<int> cached[4] = {{-1}, {-1}, {-1}, {-1}};
  const int k = c == 8 ? 3 : c == 4 ? 2 : c == 2 ? 1 : 0;
  int n = cached[k].load();
  if (n < 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(c * 64));
    cfg.blockDim = dim3(kThreadsM);
    cfg.dynamicSmemBytes = dyn;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)c;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, k_decode_mma<D, G, true, CHUNK>, &cfg) != cudaSuccess)
      n = 0;
    cached[k].store(n);
  }
  return n;
}

// Clusters of c CTAs that one launch of `pairs` clusters may use: all
// resident at once, and for c = 8 no more than three quarters of the
// capacity (measured: 32 clusters of 8, nearly the 33 that fit, ran slower
// than the same pairs in 64 clusters of 4).
template <int D, int G, bool CHUNK>
bool clusters_fit(int64_t pairs, int c, size_t dyn) {
  const int64_t cap = cluster_capacity<D, G, CHUNK>(c, dyn);
  return c == 8 ? 4 * pairs <= 3 * cap : pairs <= cap;
}

template <int D, int G, bool CHUNK>
constexpr size_t dyn_smem() {
  return 1024 + (size_t)kStagesM * (2 * (D / 64) * kTR * 128 + G * D * 2);
}

template <int D, int G, bool CHUNK>
cudaError_t launch_mma(MmaArgs<CHUNK>& ma, int sm_count, cudaStream_t st) {
  DecodeArgs& a = ma.a;
  const int32_t page = a.c.page_table ? a.c.page_rows : 0;
  const bool step = a.knew != nullptr;
  a.tcum[0] = 0;
  int32_t tmin = INT32_MAX, tmax = 0;
  for (int b = 0; b < a.B; ++b) {
    DevMeta m;
    memset(&m, 0, sizeof(m));
    m.P = a.P[b];
    m.head = a.head[b];
    m.count = a.count[b];
    m.owner = a.owner[b];
    DecRuns r;
    if constexpr (CHUNK) {
      m.next_pos = a.t[b] - ma.ch.i0[b];
      r = dec_runs_chunk(m, a.c.W, m.next_pos, ma.ch.i0[b], ma.ch.nq[b], page);
    } else {
      m.next_pos = a.t[b] + 1;
      r = dec_runs(m, a.c.W, a.t[b], page, step);
    }
    const int32_t tph = dec_tiles(r, kTR);
    a.tcum[b + 1] = a.tcum[b] + a.c.Hkv * tph;
    tmin = tph < tmin ? tph : tmin;
    tmax = tph > tmax ? tph : tmax;
  }
  a.total = a.tcum[a.B];
  constexpr size_t dyn = dyn_smem<D, G, CHUNK>();
  const int64_t pairs = (int64_t)a.B * a.c.Hkv;
  cudaError_t e;
  if ((e = configure<D, G, true, CHUNK>(dyn)) != cudaSuccess) return e;
  int csize = 0;
  if constexpr (CHUNK) {
    // no workspace: always clusters, of the largest size that fits (else
    // pairs of CTAs, in waves)
    csize = 2;
    for (int c = kMaxCluster; c >= 2; c /= 2)
      if (clusters_fit<D, G, true>(pairs, c, dyn)) { csize = c; break; }
  } else {
    if ((e = configure<D, G, false, false>(dyn)) != cudaSuccess) return e;
#ifndef PS_DMMA_NO_CLUSTER
    // Cluster mode when there are few pairs of about equal length: csize CTAs
    // per pair with csize the largest of 8, 4, 2 that fits (clusters_fit),
    // provided that fills at least half of the resident slots and gives each
    // CTA a few tiles.  Otherwise the flattened split.
    const int64_t slots = (int64_t)sm_count * ctas_per_sm<D, G, true, false>(dyn);
    for (int c = kMaxCluster; c >= 2; c /= 2) {
      if (clusters_fit<D, G, false>(pairs, c, dyn)) {
        if (2 * pairs * c >= slots && tmin >= 2 * c && 4 * tmax <= 5 * tmin) csize = c;
        break;
      }
    }
#endif
  }
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t dcfg = {};
  dcfg.blockDim = dim3(kThreadsM);
  dcfg.dynamicSmemBytes = dyn;
  dcfg.stream = st;
  dcfg.attrs = attr;
  if (csize > 0) {
    a.csize = csize;
    a.nctas = (int)(pairs * csize);
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)csize;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    dcfg.numAttrs = 2;
    dcfg.gridDim = dim3((unsigned)a.nctas);
    return cudaLaunchKernelEx(&dcfg, k_decode_mma<D, G, true, CHUNK>, ma);
  }
  if constexpr (!CHUNK) {
    a.csize = 0;
    int64_t nc = ((int64_t)a.total + kMinTilesPerCta - 1) / kMinTilesPerCta;
    const int64_t maxc = (int64_t)sm_count * ctas_per_sm<D, G, false, false>(dyn);
    if (nc > maxc) nc = maxc;
    if (nc < 1) nc = 1;
    a.nctas = (int)nc;
    dcfg.numAttrs = 1;
    dcfg.gridDim = dim3((unsigned)a.nctas);
    e = cudaLaunchKernelEx(&dcfg, k_decode_mma<D, G, false, false>, ma);
    if (e != cudaSuccess) return e;
    return launch_merge<uint16_t, D, G>(a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool make_decode_maps(const CacheDev& c, DecodeMaps* m) {
  const uint64_t row = (uint64_t)c.d * 2;
  const uint64_t prows = c.pstride > 0 ? (uint64_t)c.pstride : 1;
  const char* kring = (const char*)c.K + (size_t)c.rbase * row;
  const char* vring = (const char*)c.V + (size_t)c.rbase * row;
  const uint64_t nslab = (uint64_t)c.S * c.Hkv, nring = (uint64_t)c.nphys * c.Hkv;
  const uint64_t rstride = (uint64_t)c.rstride * row;
  const int pr = PS_DMMA_L2_PROMOTION;
  bool ok = encode_map3d_bf16(&m->kpre8, c.K, c.d, prows, nslab, row, prows * row, 64, kPadRows,
                              1, pr) &&
            encode_map3d_bf16(&m->vpre8, c.V, c.d, prows, nslab, row, prows * row, 64, kPadRows,
                              1, pr) &&
            encode_map3d_bf16(&m->kring8, kring, c.d, (uint64_t)c.page_rows, nring, row, rstride,
                              64, kPadRows, 1, pr) &&
            encode_map3d_bf16(&m->vring8, vring, c.d, (uint64_t)c.page_rows, nring, row, rstride,
                              64, kPadRows, 1, pr);
  const uint32_t halves = (uint32_t)(c.d / 64);
  const uint64_t astr[4] = {row, 128, (uint64_t)kPadRows * row, 0};
  // Prefix slabs: atoms covering rows [0, P_max) rounded up to a whole atom.
  // A copy of the last atom reads up to 7 rows past P_max: the slab's own
  // ring rows (unpaged), the next slab or the ring pages (paged).  Used only
  // when even the last slab's last atom ends inside the buffer (V, the last
  // region, has as many rows as K); otherwise prefix copies take the 3D maps.
  m->prefix_atoms = 0;
  const uint64_t pat = (uint64_t)(c.P_max > 0 ? (c.P_max + kPadRows - 1) / kPadRows : 1);
  const uint64_t pre_rows = nslab * (uint64_t)c.pstride;
  const uint64_t ring_end = (uint64_t)c.rbase + (nring - 1) * (uint64_t)c.rstride + c.page_rows;
  const uint64_t buf_rows = pre_rows > ring_end ? pre_rows : ring_end;
  if (ok && (nslab - 1) * prows + pat * kPadRows <= buf_rows) {
    const uint64_t dims[5] = {64, (uint64_t)kPadRows, halves, pat, nslab};
    const uint64_t str[4] = {astr[0], astr[1], astr[2], prows * row};
    bool pok = true;
    for (int k = 0; k < 2 && pok; ++k) {
      const uint32_t box[5] = {64, (uint32_t)kPadRows, halves, k == 0 ? 8u : 1u, 1};
      pok = encode_map_bf16(&m->kpa[k], c.K, 5, dims, str, box, pr) &&
            encode_map_bf16(&m->vpa[k], c.V, 5, dims, str, box, pr);
    }
    m->prefix_atoms = pok ? 1 : 0;
  }
  // Ring slabs: only when a slab (a page, or the whole ring) is whole atoms,
  // so that no copy leaves it.
  m->ring_atoms = 0;
  m->page_box = 0;
  if (ok && c.page_rows % kPadRows == 0) {
    const uint64_t dims[5] = {64, (uint64_t)kPadRows, halves,
                              (uint64_t)(c.page_rows / kPadRows), nring};
    const uint64_t str[4] = {astr[0], astr[1], astr[2], rstride};
    bool rok = true;
    for (int k = 0; k < 2 && rok; ++k) {
      const uint32_t box[5] = {64, (uint32_t)kPadRows, halves, k == 0 ? 8u : 1u, 1};
      rok = encode_map_bf16(&m->kra[k], kring, 5, dims, str, box, pr) &&
            encode_map_bf16(&m->vra[k], vring, 5, dims, str, box, pr);
    }
    m->ring_atoms = rok ? 1 : 0;
    if (rok && c.page_table && c.page_rows > kPadRows && c.page_rows < kBox) {
      const uint32_t box[5] = {64, (uint32_t)kPadRows, halves,
                               (uint32_t)(c.page_rows / kPadRows), 1};
      m->page_box = encode_map_bf16(&m->kra[2], kring, 5, dims, str, box, pr) &&
                    encode_map_bf16(&m->vra[2], vring, 5, dims, str, box, pr);
    }
  }
  return ok;
}

int chunk_small_pair_capacity(int d) {
  if (d == 128) {
    constexpr size_t dyn = dyn_smem<128, 8, true>();
    if (configure<128, 8, true, true>(dyn) != cudaSuccess) return 0;
    return cluster_capacity<128, 8, true>(2, dyn);
  }
  if (d == 64) {
    constexpr size_t dyn = dyn_smem<64, 8, true>();
    if (configure<64, 8, true, true>(dyn) != cudaSuccess) return 0;
    return cluster_capacity<64, 8, true>(2, dyn);
  }
  return 0;
}

cudaError_t launch_chunk_small(const DecodeArgs& a, const ChunkArgs& ch, const DecodeMaps& maps,
                               const void* k_blk, const void* v_blk, int64_t blk_rows,
                               int sm_count, cudaStream_t st) {
  MmaChunkArgs ma;
  memset(&ma, 0, sizeof(ma));
  ma.maps = maps;
  ma.a = a;
  ma.ch = ch;
  const int D = a.c.d;
  const uint64_t row = (uint64_t)D * 2;
  // block rows [rows][Hkv][D]: dimensions (column, kv head, row), boxes of 8
  // rows of one 64-column block of one head (the ring tiles' atom layout)
  if (!encode_map3d_bf16(&ma.kblk, k_blk, (uint64_t)D, (uint64_t)a.c.Hkv, (uint64_t)blk_rows, row,
                         row * a.c.Hkv, 64, 1, kPadRows, PS_DMMA_L2_PROMOTION) ||
      !encode_map3d_bf16(&ma.vblk, v_blk, (uint64_t)D, (uint64_t)a.c.Hkv, (uint64_t)blk_rows, row,
                         row * a.c.Hkv, 64, 1, kPadRows, PS_DMMA_L2_PROMOTION))
    return cudaErrorInvalidValue;
  if (D == 128) return launch_mma<128, 8, true>(ma, sm_count, st);
  if (D == 64) return launch_mma<64, 8, true>(ma, sm_count, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode_mma(const DecodeArgs& a, int G, const DecodeMaps& maps, int sm_count,
                              cudaStream_t st) {
  MmaDecodeArgs ma;
  memset(&ma, 0, sizeof(ma));
  ma.maps = maps;
  ma.a = a;
  const int D = a.c.d;
#define PS_DMMA_CASE(DD, GG) \
  if (D == DD && G == GG) return launch_mma<DD, GG, false>(ma, sm_count, st);
  PS_DMMA_CASE(128, 1) PS_DMMA_CASE(128, 2) PS_DMMA_CASE(128, 4) PS_DMMA_CASE(128, 8)
  PS_DMMA_CASE(64, 1) PS_DMMA_CASE(64, 2) PS_DMMA_CASE(64, 4) PS_DMMA_CASE(64, 8)
#undef PS_DMMA_CASE
  return cudaErrorInvalidValue;
}

}  // namespace ps
