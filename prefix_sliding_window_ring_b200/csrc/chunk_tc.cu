// Chunked prefill/extend and prompt prefill on the tcgen05 tensor cores
// (bf16, head_dim 128).
//
// A block of n queries at positions t0..t0+n-1 attends to the pinned prefix,
// the ring entries of each query's window and the block itself, causally
// ("Prefix Sliding" digest, sections 03 and 06); prompt queries (t < P)
// attend to the prefix rows [0, t].  Prefix rows are read from the slab of the
// sequence that owns them (itself, or the sequence whose prefix it shares).
// One launch serves a batch of sequences, each with its own block, packed end
// to end.  One CTA takes a 128-row query tile of one entry: 128/G consecutive
// positions of each of the G query heads that share one key/value head, so
// every key tile feeds all G heads at once.  The grid covers the query tiles
// of all entries, so the GPU fills up across sequences.
//
// Key tiles (128 rows) are walked range by range -- prefix rows, the ring
// window as at most two contiguous slot runs split at the physical wrap, then
// the block rows -- so no evicted row is ever loaded; only tiles on a window
// or causal edge are masked element by element.
//
// Roles (12 warps):
//   warp 0   TMA producer: Q once, then the K tiles into a 2-stage ring
//            (tensor-map tiled loads with 128-byte swizzle, no multicast);
//   warp 3   TMA producer of the V tiles (its own 2-stage ring);
//   warp 1   MMA issuer: S_j = Q K_j^T into one of two TMEM buffers, then
//            O += P_j V_j with P_j read from TMEM (kind::f16, f32 accumulate);
//   warp 2   owns the TMEM allocation (S in two 128-column buffers, O);
//   warps 4-11 softmax: each query row is shared by two threads (same TMEM
//            lane, one half of the columns each), which exchange row maxima
//            and sums through shared memory.  They load S_j from TMEM, mask,
//            keep a running max (raised lazily, rescaling O in TMEM only when
//            it grows by more than 2^8), write P_j (bf16) back over S_j and
//            finally normalise O into the output.  One column pair in eight
//            takes its exponentials on the FMA pipe (exp2_fma2).
// Every wait is bounded: a time-out sets ERR_TIMEOUT, every role stops, the
// MMA issuer waits for its issued work and the TMEM is freed.
#include <math.h>
#include <string.h>

#include <atomic>

#include "chunk_sched.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

namespace ps {

namespace {

constexpr int kBM = 128;          // query rows per CTA
constexpr int kHD = 128;          // head dim
constexpr int kThreadsTC = 384;  // 4 service warps + 8 softmax warps
constexpr int kSoftWarps = 8;    // two per TMEM lane quadrant, one per half of the columns
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;
constexpr float kRaiseThreshold = 8.0f;  // log2 units: rescale O only past 2^8
constexpr long long kWaitLimit = 1ll << 31;  // about a second
constexpr uint32_t kTileBytes = kBN * kHD * 2;  // one K or V tile: 32 KiB

__host__ __device__ __forceinline__ uint32_t col_s(int st) { return st ? 128u : 0u; }

struct ChunkArgs {
  CUtensorMap qmap;   // q [N][Hq][128] (entries packed): box (64, 1, PT)
  CUtensorMap kpre;   // cache K prefix rows [S*Hkv][pstride][128]: box (64, 128, 1)
  CUtensorMap vpre;
  CUtensorMap kring;  // cache K ring pages [nphys*Hkv][page_rows][128]: box (64, 128, 1)
  CUtensorMap vring;
  CUtensorMap kring_p;  // pages smaller than a key tile: box (64, page_rows, 1)
  CUtensorMap vring_p;
  CUtensorMap kblk;   // k_blk [N][Hkv][128] (entries packed): box (64, 1, 128)
  CUtensorMap vblk;
  CacheDev c;
  void* out;   // [N][Hq][128]
  int Hq, G, PT;
  int prompt;  // queries inside the prefix: causal over the prefix rows only
  int nb;      // entries
  float sc;    // softmax scale * log2(e)
  int32_t seq[kMaxChunkBatch];
  int32_t n[kMaxChunkBatch];
  int64_t t0[kMaxChunkBatch];
  int64_t tok0[kMaxChunkBatch];     // first packed row of the entry
  int32_t qtc[kMaxChunkBatch + 1];  // query tiles of the entries before b
  // each entry's ring state from the host's bookkeeping (no dependent load
  // before the first copy; the device record is checked against it)
  int64_t next_pos[kMaxChunkBatch];
  int32_t P[kMaxChunkBatch];
  int32_t head[kMaxChunkBatch];
  int32_t count[kMaxChunkBatch];
  int32_t owner[kMaxChunkBatch];
};
// Kernel parameters above 4 KB need CUDA 12.1 and sm_70 or later (limit 32764 bytes).
static_assert(sizeof(ChunkArgs) <= 32764, "chunk arguments fit the kernel parameter space");

struct __align__(1024) TcSmem {
  uint8_t q[2][kBM * 128];       // two 64-column blocks of 128-byte rows
  uint8_t k[2][2][kBN * 128];    // [stage][column block]
  uint8_t v[2][2][kBN * 128];
};

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, int* abort_flag) {
  return ptx::mbar_wait_bounded(bar, parity, abort_flag, kWaitLimit);
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^y for two values on the FMA pipe, so that part of a tile's exponentials
// leaves the special-function unit.  Cody and Waite's reduction: 2^y =
// 2^floor(y) * 2^f with f = y - floor(y) in [0, 1), and 2^f from a cubic
// 1 + c1 f + c2 f^2 + c3 f^3 whose coefficients were fitted here by
// least squares on relative error over [0, 1) (largest relative error
// 2.7e-4, well below the rounding of the bf16 P it feeds).  floor(y) comes
// from adding 1.5 * 2^23 rounded down, which leaves it in the low bits of the
// sum; shifting those bits by 23 adds it to the exponent field of the cubic's
// value.  y is clamped at -127: there f = 0, the cubic is exactly 1, and the
// exponent field drops to zero, so y <= -127 (a masked -inf included) gives
// +0 exactly; the scaled scores never exceed 2^8 (the lazy maximum).
constexpr float kExpC1 = 0.6951161f, kExpC2 = 0.22877206f, kExpC3 = 0.0755871f;
__device__ __forceinline__ float2 exp2_fma2(float2 y) {
  constexpr float kMagic = 12582912.f;  // 1.5 * 2^23
  y.x = fmaxf(y.x, -127.f);
  y.y = fmaxf(y.y, -127.f);
  const float2 t = __fadd2_rd(y, make_float2(kMagic, kMagic));  // 1.5 * 2^23 + floor(y)
  const float2 fl = __fadd2_rn(t, make_float2(-kMagic, -kMagic));  // floor(y), exact
  const float2 f = __ffma2_rn(fl, make_float2(-1.f, -1.f), y);     // y - floor(y), exact
  float2 q = __ffma2_rn(make_float2(kExpC3, kExpC3), f, make_float2(kExpC2, kExpC2));
  q = __ffma2_rn(q, f, make_float2(kExpC1, kExpC1));
  q = __ffma2_rn(q, f, make_float2(1.f, 1.f));
  return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23)));
}
#ifndef PS_CHUNK_EXP_FMA_EVERY
#define PS_CHUNK_EXP_FMA_EVERY 8
#endif
// one column pair in kExpFmaEvery takes its exponentials on the FMA pipe (0: none)
constexpr int kExpFmaEvery = PS_CHUNK_EXP_FMA_EVERY;

// max of three (max.f32 with three sources, sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// SP: a paged cache whose pages are smaller than a key tile (8 to 64 rows)
template <bool SP>
__global__ void __launch_bounds__(kThreadsTC, 1) k_chunk_tc(const __grid_constant__ ChunkArgs a) {
  extern __shared__ uint8_t dsm_raw[];
  TcSmem& sm = *reinterpret_cast<TcSmem*>(
      (uint8_t*)(((uintptr_t)dsm_raw + 1023) & ~(uintptr_t)1023));
  __shared__ __align__(8) uint64_t q_full, k_full[2], k_empty[2], v_full[2], v_empty[2];
  __shared__ __align__(8) uint64_t s_full[2], p_full[2], o_full, mma_done;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ float xchg[2][2][kBM];  // [parity][column half][row]: partial maxima / sums

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.y;
  const int PT = a.PT;
  // this CTA's entry and query tile
  int eb = 0;
  {
    int hi = a.nb - 1;
    while (eb < hi) {  // last entry with qtc[b] <= blockIdx.x
      const int mid = (eb + hi + 1) >> 1;
      if (a.qtc[mid] <= (int)blockIdx.x) eb = mid; else hi = mid - 1;
    }
  }
  const int seq = a.seq[eb], n = a.n[eb];
  const int64_t t0 = a.t0[eb], tok0 = a.tok0[eb];
  // an entry's query tiles run last first: later queries see more keys (causal
  // prompts, windows not yet full), so the longest CTAs start first and the
  // launch ends on short ones
  const int i0 = (a.qtc[eb + 1] - 1 - (int)blockIdx.x) * PT;
  DevMeta m;
  m.next_pos = a.next_pos[eb];
  m.P = a.P[eb];
  m.head = a.head[eb];
  m.count = a.count[eb];
  m.owner = a.owner[eb];
  const int64_t plo = t0 + i0;
  const int64_t phi = t0 + min(i0 + PT, n) - 1;
  const int spage = a.c.page_table ? a.c.page_rows : 0;  // ring page size of the schedule
  const KSched ks = make_sched(m, a.c.W, spage, t0, plo, phi, a.prompt != 0);
  const int T = ks.ntiles;

  if (threadIdx.x == 0) {
    ptx::mbar_init(&q_full, 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&k_full[i], 1);
      ptx::mbar_init(&k_empty[i], 1);
      ptx::mbar_init(&v_full[i], 1);
      ptx::mbar_init(&v_empty[i], 1);
      ptx::mbar_init(&s_full[i], 1);
      ptx::mbar_init(&p_full[i], kSoftWarps);
    }
    ptx::mbar_init(&o_full, 1);
    ptx::mbar_init(&mma_done, 1);
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 2) {
    ptx::tmem_alloc(&tmem_slot, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 0 || warp == 3) {
    // ----------------------------------------------------------- producers --
    // Lane 0 waits for free stages and issues the copies.  With pages smaller
    // than a tile (SP) a ring tile is kBN / spage whole pages, one box each,
    // which the lanes map and copy one page apiece (their page-table reads
    // run side by side); a page past the ring's end or not yet mapped gets
    // slab -1, which the copy fills with zeros, and its rows are masked.
    // Warp 0 copies the K tiles and warp 3 the V tiles, each into its own
    // 2-stage ring, so that a K tile never waits behind a V tile's free
    // stage (and a tile's page copies are issued by two warps at once).
    const int prefix_z = m.owner * a.c.Hkv + g;  // prefix rows live in the owner's slab
    int issued_k = 0, issued_v = 0;
    if (lane == 0 && warp == 0) {
      ptx::mbar_arrive_expect_tx(&q_full, 2 * kBM * 128);
      for (int hh = 0; hh < a.G; ++hh)
        for (int b = 0; b < 2; ++b)
          ptx::tma_load_3d(&sm.q[b][hh * PT * 128], &a.qmap, b * 64, g * a.G + hh,
                           (int32_t)(tok0 + i0), &q_full);
      if (i0 == 0 && g == 0) {  // once per entry: the device record must agree
        const DevMeta md = a.c.meta[seq];
        const bool bad = md.next_pos != m.next_pos || md.P != m.P || md.head != m.head ||
                         md.count != m.count || md.owner != m.owner ||
                         (a.prompt ? t0 + n > m.P : m.next_pos != t0);
        if (bad) atomicOr(a.c.err, ERR_BATCH);
      }
    }
    const bool isv = warp == 3;  // this warp's operand
    const CUtensorMap* mpre = isv ? &a.vpre : &a.kpre;
    const CUtensorMap* mblk = isv ? &a.vblk : &a.kblk;
    uint64_t* full = isv ? v_full : k_full;
    uint64_t* empty = isv ? v_empty : k_empty;
    uint8_t* const buf = isv ? &sm.v[0][0][0] : &sm.k[0][0][0];
    constexpr int kColBlk = kBN * 128;  // bytes of one 64-column block of a tile
    int issued = 0;
    if constexpr (!SP) {
      const CUtensorMap* mring = isv ? &a.vring : &a.kring;
      if (lane == 0) {
        for (int j = 0; j < T && !abort_flag; ++j) {
          const int st = j & 1;
          const KTile kt = tile_of(ks, j);
          if (j >= 2 && !wait_bar(&empty[st], ((j >> 1) - 1) & 1, &abort_flag)) break;
          // a ring tile lies within one page: (slot within the page, page's slab)
          const int32_t kslot = (int32_t)kt.row;  // ring slot (ring tiles)
          const int ring_z = kt.src == 0 ? ring_page(a.c, seq, kslot) * a.c.Hkv + g : 0;
          const int32_t ring_y = kt.src == 0 ? kslot % a.c.page_rows : 0;
          const int32_t blk_row = (int32_t)(tok0 + kt.row);  // block tiles: packed row
          ptx::mbar_arrive_expect_tx(&full[st], kTileBytes);
          for (int b = 0; b < 2; ++b) {
            uint8_t* dst = buf + (st * 2 + b) * kColBlk;
            if (kt.src == 2)
              ptx::tma_load_3d(dst, mpre, b * 64, (int32_t)kt.row, prefix_z, &full[st]);
            else if (kt.src == 0)
              ptx::tma_load_3d(dst, mring, b * 64, ring_y, ring_z, &full[st]);
            else
              ptx::tma_load_3d(dst, mblk, b * 64, g, blk_row, &full[st]);
          }
          issued = j + 1;
        }
      }
    } else {
      const CUtensorMap* mring_p = isv ? &a.vring_p : &a.kring_p;
      const bool plane = lane * spage < kBN;  // this lane copies a page of a tile
      for (int j = 0; j < T; ++j) {
        const int st = j & 1;
        const KTile kt = tile_of(ks, j);
        const bool ptile = kt.src == 0;  // a ring tile: whole pages
        const int32_t kslot = (int32_t)kt.row;  // its first slot, a page edge
        int pz = -1;  // this lane's page of a small-page tile: its slab
        if (ptile && plane && kslot + lane * spage < a.c.W) {
          const int ph = ring_page(a.c, seq, kslot + lane * spage);
          pz = ph >= 0 ? ph * a.c.Hkv + g : -1;
        }
        const int32_t blk_row = (int32_t)(tok0 + kt.row);  // block tiles: packed row
        // lane 0 waits; the warp follows its decision
        int go = 1;
        if (lane == 0)
          go = !abort_flag && (j < 2 || wait_bar(&empty[st], ((j >> 1) - 1) & 1, &abort_flag));
        if (!__shfl_sync(0xffffffffu, go, 0)) break;
        if (lane == 0) {
          ptx::mbar_arrive_expect_tx(&full[st], kTileBytes);
          if (!ptile)  // prefix or block rows: one box per column block
            for (int b = 0; b < 2; ++b) {
              uint8_t* dst = buf + (st * 2 + b) * kColBlk;
              if (kt.src == 2)
                ptx::tma_load_3d(dst, mpre, b * 64, (int32_t)kt.row, prefix_z, &full[st]);
              else
                ptx::tma_load_3d(dst, mblk, b * 64, g, blk_row, &full[st]);
            }
        }
        if (ptile && plane) {
          uint8_t* dst = buf + st * 2 * kColBlk + lane * spage * 128;
          ptx::tma_load_3d(dst, mring_p, 0, 0, pz, &full[st]);
          ptx::tma_load_3d(dst + kColBlk, mring_p, 64, 0, pz, &full[st]);
        }
        issued = j + 1;
      }
    }
    if (isv) issued_v = issued; else issued_k = issued;
    if (lane == 0 && abort_flag) {  // let the copies already issued land before the CTA exits
      int quiet = 0;
      ptx::mbar_wait_bounded(&q_full, 0, &quiet, kWaitLimit);
      for (int j = issued_k > 2 ? issued_k - 2 : 0; j < issued_k; ++j)
        ptx::mbar_wait_bounded(&k_full[j & 1], (j >> 1) & 1, &quiet, kWaitLimit);
      for (int j = issued_v > 2 ? issued_v - 2 : 0; j < issued_v; ++j)
        ptx::mbar_wait_bounded(&v_full[j & 1], (j >> 1) & 1, &quiet, kWaitLimit);
    }
    __syncwarp();  // the whole warp meets the final block barrier together
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      constexpr uint32_t idesc_s = ptx::idesc_bf16_f32(kBM, kBN, 0, 0);
      constexpr uint32_t idesc_o = ptx::idesc_bf16_f32(kBM, kHD, 0, 1);
      bool ok = wait_bar(&q_full, 0, &abort_flag);
      int pv_next = 0;  // next P V product to issue
      auto issue_pv = [&](int jj) -> bool {
        const int st = jj & 1;
        if (!wait_bar(&p_full[st], (jj >> 1) & 1, &abort_flag)) return false;
        if (!wait_bar(&v_full[st], (jj >> 1) & 1, &abort_flag)) return false;
        ptx::tc_fence_after();
        for (int k = 0; k < kBN / 16; ++k) {
          // B = V tile, MN-major: 64-column blocks 16 KiB apart, 8-row groups 1 KiB apart
          const uint64_t bdesc = ptx::sdesc_sw128(sm.v[st][0] + k * 16 * 128, 16384, 1024);
          ptx::mma_ts(tmem + kColO, tmem + col_s(st) + k * 8, bdesc, idesc_o,
                      (jj > 0 || k > 0) ? 1u : 0u);
        }
        ptx::mma_commit(&v_empty[st]);
        ptx::mma_commit(&o_full);
        return true;
      };
      for (int j = 0; j < T && ok; ++j) {
        const int st = j & 1;
        if (!wait_bar(&k_full[st], (j >> 1) & 1, &abort_flag)) { ok = false; break; }
        ptx::tc_fence_after();
        for (int k = 0; k < kHD / 16; ++k) {
          const int b = k >> 2, kk = k & 3;
          const uint64_t adesc = ptx::sdesc_sw128(sm.q[b] + kk * 32, 16, 1024);
          const uint64_t bdesc = ptx::sdesc_sw128(sm.k[st][b] + kk * 32, 16, 1024);
          ptx::mma_ss(tmem + col_s(st), adesc, bdesc, idesc_s, k > 0 ? 1u : 0u);
        }
        ptx::mma_commit(&s_full[st]);
        ptx::mma_commit(&k_empty[st]);
        if (j >= 1) {
          if (!issue_pv(j - 1)) { ok = false; break; }
          pv_next = j;
        }
      }
      if (ok && T > 0) issue_pv(pv_next);
      ptx::mma_commit(&mma_done);
      int quiet = 0;
      ptx::mbar_wait_bounded(&mma_done, 0, &quiet, kWaitLimit);
    }
    __syncwarp();  // the whole warp meets the final block barrier together
  } else if (warp >= 4) {
    // ------------------------------------------------------------- softmax --
    const int quad = warp & 3;            // TMEM lane quadrant this warp may access
    const int half = (warp - 4) >> 2;     // which 64 columns of S / O it owns
    const int r = quad * 32 + lane;       // query row of this thread
    const int hh = r / PT, i = i0 + r % PT;
    const int64_t tq = t0 + i;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const int cbase = half * 64;          // first S/O column of this thread
    // A prompt query t sees [0, t]: the mask below with the prefix taken as [0, t].
    const int W = a.c.W, P = a.prompt ? (int)(tq + 1) : m.P;
    // lowest ring or block key of this query / of any query of the tile: the
    // window's start, or the schedule's rlo where that is higher (the first
    // ring tile over pages smaller than a tile starts at a page edge below it)
    const int64_t qlo = max(tq - W + 1, ks.rlo);
    const int64_t tlo = max(phi - W + 1, ks.rlo);
    const float sc = a.sc;
    const int pair_bar = 2 + quad;        // named barrier of the two warps of this quadrant
    auto pair_sync = [&]() { asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory"); };
    float m_run = -INFINITY, l_run = 0.f;  // m_run: reference max (log2 units); l_run: my half
    // After a failed wait (ok == false) a warp skips all work but still meets its
    // partner at every pair barrier, so neither can be left waiting there.
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      const int st = j & 1;
      if (ok) ok = __all_sync(0xffffffffu, wait_bar(&s_full[st], (j >> 1) & 1, &abort_flag));
      float x[64];
      float mloc = -INFINITY;
      if (ok) {
        ptx::tc_fence_after();
        uint32_t raw0[32], raw1[32];
        ptx::tmem_ld32(tmem + lane_base + col_s(st) + cbase, raw0);
        ptx::tmem_ld32(tmem + lane_base + col_s(st) + cbase + 32, raw1);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          x[c] = __uint_as_float(raw0[c]);
          x[32 + c] = __uint_as_float(raw1[c]);
        }
        const KTile kt = tile_of(ks, j);
        // element masks only for tiles on a window or causal edge
        const bool full = kt.valid == kBN &&
                          (kt.src == 2 && kt.pos0 + kBN <= P
                               ? true
                               : (kt.pos0 >= tlo && kt.pos0 + kBN - 1 <= plo));
        if (!full) {
          auto clampc = [](int64_t v) -> int { return v < -1 ? -1 : (v > kBN ? kBN : (int)v); };
          // c < pre_c: pinned prefix (prefix tiles only)
          const int pre_c = kt.src == 2 ? clampc(P - kt.pos0) - cbase : 0;
          const int lo_c = clampc(qlo - kt.pos0) - cbase;  // window start
          const int hi_c = clampc(tq - kt.pos0) - cbase;          // causal end
          const int vc = kt.valid - cbase;
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const bool vis = c < vc && (c < pre_c || (c >= lo_c && c <= hi_c));
            if (!vis) x[c] = -INFINITY;
          }
        }
        // row max of the raw scores (the scale is positive), as a tree of
        // three-input maxima
        float t8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) t8[u] = fmax3(x[u], x[8 + u], x[16 + u]);
#pragma unroll
        for (int u = 0; u < 8; ++u) t8[u] = fmax3(t8[u], x[24 + u], x[32 + u]);
#pragma unroll
        for (int u = 0; u < 8; ++u) t8[u] = fmax3(t8[u], x[40 + u], x[48 + u]);
#pragma unroll
        for (int u = 0; u < 8; ++u) t8[u] = fmaxf(t8[u], x[56 + u]);
        mloc = fmax3(fmax3(t8[0], t8[1], t8[2]), fmax3(t8[3], t8[4], t8[5]), fmaxf(t8[6], t8[7]));
      }
      xchg[st][half][r] = mloc;
      pair_sync();
      if (!ok) continue;
      const float mx = fmaxf(mloc, xchg[st][half ^ 1][r]) * sc;  // row max, log2 units
      // Raise the reference max lazily.  tcgen05.ld/st are warp-collective, so
      // the O rescale runs for the whole warp when any lane needs it.
      const bool raise = mx > m_run + kRaiseThreshold || (m_run == -INFINITY && mx > -INFINITY);
      const float m_new = raise ? mx : m_run;
      const bool need_o = raise && j > 0 && m_run > -INFINITY;
      if (__any_sync(0xffffffffu, need_o)) {
        const float alpha = need_o ? ex2(m_run - m_new) : 1.f;
        // O holds P_0..P_{j-1} times V: wait for the last product, then rescale my half
        ok = __all_sync(0xffffffffu, wait_bar(&o_full, (j - 1) & 1, &abort_flag));
        if (!ok) continue;
        ptx::tc_fence_after();
        uint32_t o0[32], o1[32];
        ptx::tmem_ld32(tmem + lane_base + kColO + cbase, o0);
        ptx::tmem_ld32(tmem + lane_base + kColO + cbase + 32, o1);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          o0[c] = __float_as_uint(__uint_as_float(o0[c]) * alpha);
          o1[c] = __float_as_uint(__uint_as_float(o1[c]) * alpha);
        }
        ptx::tmem_st32(tmem + lane_base + kColO + cbase, o0);
        ptx::tmem_st32(tmem + lane_base + kColO + cbase + 32, o1);
        ptx::tmem_wait_st();
        l_run *= alpha;
      }
      m_run = m_new;
      const float mu = m_run == -INFINITY ? 0.f : m_run;
      // two columns per packed f32x2 FMA / add (sm_100): scale and shift,
      // then the running sums; the exponentials one by one
      const float2 sc2 = make_float2(sc, sc), nmu2 = make_float2(-mu, -mu);
      float2 s4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                      make_float2(0.f, 0.f)};
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        const float2 y = __ffma2_rn(make_float2(x[c], x[c + 1]), sc2, nmu2);
        float p0, p1;
        if (kExpFmaEvery > 0 && (c >> 1) % (kExpFmaEvery > 0 ? kExpFmaEvery : 1) ==
                                    kExpFmaEvery - 1) {
          const float2 e = exp2_fma2(y);
          p0 = e.x;
          p1 = e.y;
        } else {
          p0 = ex2(y.x);
          p1 = ex2(y.y);
        }
        s4[(c >> 1) & 3] = __fadd2_rn(s4[(c >> 1) & 3], make_float2(p0, p1));
        pk[c >> 1] = pack_bf16(p0, p1);
      }
      const float2 s01 = __fadd2_rn(s4[0], s4[1]), s23 = __fadd2_rn(s4[2], s4[3]);
      const float2 sall = __fadd2_rn(s01, s23);
      l_run += sall.x + sall.y;
      // P occupies the first 64 columns of the S buffer; my 64 keys are 32 of them.
      // The partner read its scores from those columns before the pair barrier.
      ptx::tmem_st32(tmem + lane_base + col_s(st) + half * 32, pk);
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&p_full[st]);
    }
    if (ok && T > 0) {
      // mma_done is committed once, after the last product: a parity wait on
      // o_full here could take an older phase while two products are in flight.
      ok = wait_bar(&mma_done, 0, &abort_flag);
      ok = __all_sync(0xffffffffu, ok);
    }
    // row sum = both halves (the parity slot 0/1 of the last tile is not reused here)
    xchg[T & 1][half][r] = l_run;
    pair_sync();
    const float l_row = l_run + xchg[T & 1][half ^ 1][r];
    if (ok && T > 0) {
      ptx::tc_fence_after();
      const float inv = 1.f / l_row;
      uint16_t* orow = (uint16_t*)a.out + ((size_t)(tok0 + i) * a.Hq + (size_t)g * a.G + hh) * kHD;
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        uint32_t o[32];
        ptx::tmem_ld32(tmem + lane_base + kColO + cbase + c2 * 32, o);
        ptx::tmem_wait_ld();
        if (i < n) {
          uint32_t w[16];
#pragma unroll
          for (int c = 0; c < 16; ++c)
            w[c] = pack_bf16(__uint_as_float(o[2 * c]) * inv, __uint_as_float(o[2 * c + 1]) * inv);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            *(uint4*)(orow + cbase + c2 * 32 + v4 * 8) =
                make_uint4(w[4 * v4], w[4 * v4 + 1], w[4 * v4 + 2], w[4 * v4 + 3]);
        }
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && abort_flag) atomicOr(a.c.err, ERR_TIMEOUT);
  if (warp == 2) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool chunk_tc_supported(const CacheDev& c, int dtype, int d, int G) {
  // ring tiles of a paged cache: pages of 128-row multiples, or whole pages of
  // 8 to 64 rows that divide the tile
  const bool pages_ok = !c.page_table || c.page_rows % kBN == 0 ||
                        (kBN % c.page_rows == 0 && c.page_rows % 8 == 0);
  return pages_ok && dtype == 1 && d == kHD && (G == 1 || G == 2 || G == 4 || G == 8);
}

cudaError_t launch_chunk_tc(const CacheDev& c, int G, const ChunkEntry* e, int nb, int Hq,
                            const void* q, const void* k_blk, const void* v_blk, void* out,
                            float scale, int prompt, int sm_count, cudaStream_t st) {
  (void)sm_count;
  if (nb < 1 || nb > kMaxChunkBatch) return cudaErrorInvalidValue;
  ChunkArgs a;
  memset(&a, 0, sizeof(a));
  const uint64_t row = kHD * 2;  // bytes per head row
  const int PT = kBM / G;
  int64_t N = 0;  // packed rows of all entries
  a.qtc[0] = 0;
  for (int b = 0; b < nb; ++b) {
    if (e[b].n < 1) return cudaErrorInvalidValue;
    a.seq[b] = e[b].seq;
    a.n[b] = e[b].n;
    a.t0[b] = e[b].t0;
    a.tok0[b] = N;
    a.qtc[b + 1] = a.qtc[b] + (e[b].n + PT - 1) / PT;
    a.next_pos[b] = e[b].next_pos;
    a.P[b] = e[b].P;
    a.head[b] = e[b].head;
    a.count[b] = e[b].count;
    a.owner[b] = e[b].owner;
    N += e[b].n;
  }
  if (N > INT32_MAX) return cudaErrorInvalidValue;
  bool ok = encode_map3d_bf16(&a.qmap, q, kHD, Hq, N, row, (uint64_t)Hq * row, 64, 1, PT);
  // prefix rows: [S*Hkv][pstride] rows from the buffer start; ring pages:
  // [nphys*Hkv][page_rows] slabs rstride rows apart from row rbase
  const uint64_t prows = c.pstride > 0 ? (uint64_t)c.pstride : 1;
  const char* kring = (const char*)c.K + (size_t)c.rbase * row;
  const char* vring = (const char*)c.V + (size_t)c.rbase * row;
  ok = ok && encode_map3d_bf16(&a.kpre, c.K, kHD, prows, (uint64_t)c.S * c.Hkv, row, prows * row, 64, kBN, 1);
  ok = ok && encode_map3d_bf16(&a.vpre, c.V, kHD, prows, (uint64_t)c.S * c.Hkv, row, prows * row, 64, kBN, 1);
  ok = ok && encode_map3d_bf16(&a.kring, kring, kHD, (uint64_t)c.page_rows, (uint64_t)c.nphys * c.Hkv, row,
                   (uint64_t)c.rstride * row, 64, kBN, 1);
  ok = ok && encode_map3d_bf16(&a.vring, vring, kHD, (uint64_t)c.page_rows, (uint64_t)c.nphys * c.Hkv, row,
                   (uint64_t)c.rstride * row, 64, kBN, 1);
  if (c.page_table && small_pages(c.page_rows)) {  // whole-page boxes
    ok = ok && encode_map3d_bf16(&a.kring_p, kring, kHD, (uint64_t)c.page_rows,
                                 (uint64_t)c.nphys * c.Hkv, row, (uint64_t)c.rstride * row, 64,
                                 (uint32_t)c.page_rows, 1);
    ok = ok && encode_map3d_bf16(&a.vring_p, vring, kHD, (uint64_t)c.page_rows,
                                 (uint64_t)c.nphys * c.Hkv, row, (uint64_t)c.rstride * row, 64,
                                 (uint32_t)c.page_rows, 1);
  }
  // a prompt launch loads no block rows; its block maps describe the cache
  // K/V (never used) so that every map is well formed
  const uint64_t nblk = prompt ? prows : (uint64_t)N;
  ok = ok && encode_map3d_bf16(&a.kblk, prompt ? c.K : k_blk, kHD, c.Hkv, nblk, row, (uint64_t)c.Hkv * row, 64,
                   1, kBN);
  ok = ok && encode_map3d_bf16(&a.vblk, prompt ? c.V : v_blk, kHD, c.Hkv, nblk, row, (uint64_t)c.Hkv * row, 64,
                   1, kBN);
  if (!ok) return cudaErrorInvalidValue;
  a.c = c;
  a.out = out;
  a.Hq = Hq;
  a.G = G;
  a.PT = PT;
  a.prompt = prompt;
  a.nb = nb;
  a.sc = scale * 1.4426950408889634f;
  const size_t dyn = sizeof(TcSmem) + 1024;
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (!(configured.load() & (1ull << (dev & 63)))) {
    err = cudaFuncSetAttribute(k_chunk_tc<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)dyn);
    if (err == cudaSuccess)
      err = cudaFuncSetAttribute(k_chunk_tc<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)dyn);
    if (err != cudaSuccess) return err;
    configured.fetch_or(1ull << (dev & 63));
  }
  dim3 grid(a.qtc[nb], c.Hkv);
  if (c.page_table && small_pages(c.page_rows))
    k_chunk_tc<true><<<grid, kThreadsTC, dyn, st>>>(a);
  else
    k_chunk_tc<false><<<grid, kThreadsTC, dyn, st>>>(a);
  return cudaGetLastError();
}

}  // namespace ps
