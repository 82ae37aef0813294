// Decode attention (visible-range derivation, split streaming, split merge),
// and the decode step that appends the token in the same pass.
//
// Work division.  Each (batch entry, kv head) pair's visible rows -- the
// pinned prefix, then the ring window as at most two runs split at the
// physical wrap -- are cut into tiles of TR consecutive rows (only a pair's
// last tile is short; a tile may span the prefix/ring boundary or the wrap and
// is then assembled from several bulk copies).  The tiles of all pairs are
// laid end to end and CTA c of nctas (two per SM) streams tiles
// [T c / nctas, T (c + 1) / nctas), so every CTA streams the same number of
// tiles whatever the batch shape.  For every (CTA range, pair) piece a CTA
// emits one partial (max, sum, accumulator) triple; a small second grid
// merges each pair's partials into the output.  Both grids are programmatic
// dependent launches of the kernel before them.  No evicted row is ever
// fetched ("Prefix Sliding" digest, section 06: iterate the prefix blocks and
// the window blocks separately).
//
// Streaming.  Warp kCW is the producer: one lane issues bulk async copies
// (cp.async.bulk, no multicast) of K and V tiles of 14 KiB each into a
// kStages-deep shared-memory ring (much smaller copies leave HBM bandwidth
// unused), with a small descriptor per tile (pair, rows, first/last of piece,
// partial slot); the first tile of a piece also brings the pair's q rows.
// Each entry's ring state comes with the launch from the host's bookkeeping,
// so no copy waits on a metadata load; the device record is checked alongside.
// Prefix rows come from the slab of the sequence that owns them (a shared
// prefix); in a decode step the pair's last row, the appended token, comes
// from the caller's buffer and is stored to its ring slot by the consumer warp
// that holds it.  Each of the kCW consumer warps takes its own share of every
// tile and keeps its own online-softmax state; a stage is refilled once all of
// them have released it.
//
// Consumer arithmetic (per warp, LPR lanes per row, 8 scores per update):
// each lane forms partial dot products for 8 (row, query head) scores, a
// transpose-reduction leaves every lane with one complete score, the lane
// exponentiates only that score, and the 8 weights are gathered back for the
// weighted sum of the value rows.  Pairs of float32 values use the packed
// sm_100 FMA (each half is an ordinary IEEE fma).  A lane holds VEC elements
// of a row (16 bytes, or 8 for bfloat16 at G >= 8 so that q and the G
// accumulators stay in registers).  The running max of a head moves only when
// a score passes it by more than 2^8, so the accumulators are rescaled on few
// updates; the exact max is not needed, only one shared by the sum and the
// accumulator (the weights stay below 2^8).
//
// Every wait is bounded; a time-out stops the CTA, sets ERR_TIMEOUT and lets
// the copies already issued land before the CTA exits.
#include <type_traits>
#include <math.h>
#include <string.h>

#include <atomic>

#include "attn_common.cuh"
#include "decode_common.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

#ifndef PS_DEC_STAGES
#define PS_DEC_STAGES 3
#endif
#ifndef PS_DEC_WARP_BYTES
#define PS_DEC_WARP_BYTES 2048
#endif
#ifndef PS_DEC_CTAS_PER_SM
#define PS_DEC_CTAS_PER_SM 2
#endif

namespace ps {

namespace {

using namespace attn;
using namespace dec;

#ifndef PS_DEC_CONSUMER_WARPS
#define PS_DEC_CONSUMER_WARPS 7
#endif
// 7 consumer warps + 1 producer: 8 warps per CTA.  Warps are spread over the
// four SM sub-partitions, each with its own quarter of the register file, so
// two CTAs of 9 warps would put 5 warps on one sub-partition and only one CTA
// would fit; with 8 warps two CTAs of up to 128 registers fit.
constexpr int kCW = PS_DEC_CONSUMER_WARPS;   // consumer warps
constexpr int kThreadsDec = (kCW + 1) * 32;  // plus one producer warp
// Tile i sits in stage i % kStages.  Every consumer warp waits on every tile
// in order and releases it, so no warp can reach a stage two phases ahead of
// the one it needs (where the parity test would accept the older phase).
constexpr int kStages = PS_DEC_STAGES;

template <typename T, int D> struct DecTile {
  static constexpr int RW = PS_DEC_WARP_BYTES / (D * (int)sizeof(T));  // rows per warp per tile
  static constexpr int TR = RW * kCW;                                  // rows per tile (14 KiB)
};


// Elements of one row a lane holds: a 16-byte vector, or for bfloat16 with
// G >= 8 an 8-byte one -- q and the accumulator of all G heads live in
// registers, G * VEC * 2 floats, which must stay well inside the 128-register
// budget of a thread.
template <typename T, int G> struct LaneVec {
  static constexpr int N = (sizeof(T) == 2 && G >= 8) ? 4 : Vec<T>::N;
  using Raw = typename std::conditional<N * sizeof(T) == 16, uint4, uint2>::type;
};

// Pairs of a lane's vector as float2 (exact widening for bfloat16).
template <typename T> struct Vec2;
template <> struct Vec2<float> {
  __device__ __forceinline__ static void unpack(const uint4& x, float2* f) {
    f[0] = make_float2(__uint_as_float(x.x), __uint_as_float(x.y));
    f[1] = make_float2(__uint_as_float(x.z), __uint_as_float(x.w));
  }
};

// Online-softmax state of one lane (see the file comment).  Pairs of values
// are float2 so the packed sm_100 FMA/MUL (__ffma2_rn, __fmul2_rn: two IEEE
// operations each) apply directly.
template <typename T, int D, int G>
struct DecState {
  static constexpr int VEC = LaneVec<T, G>::N;
  using Raw = typename LaneVec<T, G>::Raw;
  static constexpr int V2 = VEC / 2;
  static constexpr int LPR = D / VEC;   // lanes per row
  static constexpr int RPI = 32 / LPR;  // rows per warp load instruction
  static constexpr int U = 8 / G;       // rows per row group per update
  static constexpr int STEP = RPI * U;  // rows per warp per update
  static constexpr int S1 = LPR / 2, S2 = LPR / 4, S3 = LPR / 8;
  static_assert(LPR >= 8, "the transpose-reduction needs at least 8 lanes per row");

  float2 q[G][V2];
  float2 o[G][V2];
  float m[G];
  float mo, lpart;  // running max and partial sum of this lane's own head
  int c, rs, base, kown;

  __device__ __forceinline__ static int lane_of(int k) {
    return ((k & 4) ? S1 : 0) | ((k & 2) ? S2 : 0) | ((k & 1) ? S3 : 0);
  }

  __device__ __forceinline__ void init(const T* __restrict__ qrow, float qscale) {
    const int lane = threadIdx.x & 31;
    c = lane % LPR;
    rs = lane / LPR;
    base = rs * LPR;
    kown = ((c & S1) ? 4 : 0) | ((c & S2) ? 2 : 0) | ((c & S3) ? 1 : 0);
    const float2 s2 = make_float2(qscale, qscale);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const Raw raw = *(const Raw*)(qrow + (size_t)h * D + c * VEC);
      Vec2<T>::unpack(raw, q[h]);
#pragma unroll
      for (int e = 0; e < V2; ++e) {
        q[h][e] = __fmul2_rn(q[h][e], s2);
        o[h][e] = make_float2(0.f, 0.f);
      }
      m[h] = -INFINITY;
    }
    mo = -INFINITY;
    lpart = 0.f;
  }

  __device__ __forceinline__ void update(const Raw (&kr)[U], const Raw (&vr)[U],
                                         const bool (&ok)[U]) {
    const unsigned FULL = 0xffffffffu;
    const int lane = threadIdx.x & 31;
    // partial dot products of the 8 (row u, head h) scores, index u*G + h
    float v[8];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float2 kf[V2];
      Vec2<T>::unpack(kr[u], kf);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float2 acc = __fmul2_rn(q[h][0], kf[0]);
#pragma unroll
        for (int e = 1; e < V2; ++e) acc = __ffma2_rn(q[h][e], kf[e], acc);
        v[u * G + h] = acc.x + acc.y;
      }
    }
    // transpose-reduction: 8 values -> 1 complete score per lane
    {
      const bool b1 = (lane & S1) != 0;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float send = b1 ? v[k] : v[k + 4];
        const float keep = b1 ? v[k + 4] : v[k];
        v[k] = keep + __shfl_xor_sync(FULL, send, S1);
      }
      const bool b2 = (lane & S2) != 0;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const float send = b2 ? v[k] : v[k + 2];
        const float keep = b2 ? v[k + 2] : v[k];
        v[k] = keep + __shfl_xor_sync(FULL, send, S2);
      }
      const bool b3 = (lane & S3) != 0;
      {
        const float send = b3 ? v[0] : v[1];
        const float keep = b3 ? v[1] : v[0];
        v[0] = keep + __shfl_xor_sync(FULL, send, S3);
      }
#pragma unroll
      for (int s = S3 / 2; s >= 1; s >>= 1) v[0] += __shfl_xor_sync(FULL, v[0], s);
    }
    bool okown = false;
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (kown / G == u) okown = ok[u];
    const float sc = okown ? v[0] : -INFINITY;
    // tile max of this lane's head (reduce over the lanes holding other rows)
    float tm = sc;
    if (G <= 4) tm = fmaxf(tm, __shfl_xor_sync(FULL, tm, S1));
    if (G <= 2) tm = fmaxf(tm, __shfl_xor_sync(FULL, tm, S2));
    if (G == 1) tm = fmaxf(tm, __shfl_xor_sync(FULL, tm, S3));
    // The running max moves only when a score passes it by more than 2^8
    // (weights stay below 2^8, far from float overflow), so the rescale of
    // the accumulators is skipped for nearly every row group.
    const float mo_new = tm > mo + kRaiseLog2 ? tm : mo;
    const float p = okown ? exp2f(sc - mo_new) : 0.f;
    if (mo_new != mo) lpart *= exp2f(mo - mo_new);
    lpart += p;
    mo = mo_new;
    // every head's new max, in every lane (the same rule as mo)
    float mold[G];
    bool raise = false;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float th = __shfl_sync(FULL, tm, base | lane_of(h));
      mold[h] = m[h];
      if (th > m[h] + kRaiseLog2) { m[h] = th; raise = true; }
    }
    float pk[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) pk[k] = __shfl_sync(FULL, p, base | lane_of(k));
    if (raise) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float alpha = exp2f(mold[h] - m[h]);  // 0 when mold is -inf, 1 when unchanged
        const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
        for (int e = 0; e < V2; ++e) o[h][e] = __fmul2_rn(o[h][e], a2);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float2 vf[V2];
      Vec2<T>::unpack(vr[u], vf);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float2 w2 = make_float2(pk[u * G + h], pk[u * G + h]);
#pragma unroll
        for (int e = 0; e < V2; ++e) o[h][e] = __ffma2_rn(w2, vf[e], o[h][e]);
      }
    }
  }

  // Rows [0, nrows) of a contiguous tile in shared memory (row stride D).
  __device__ __forceinline__ void tile(const T* ks, const T* vs, int nrows) {
    for (int r0 = 0; r0 < nrows; r0 += STEP) {
      Raw kr[U], vr[U];
      bool ok[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int r = r0 + u * RPI + rs;
        ok[u] = r < nrows;
        kr[u] = Raw{};
        vr[u] = kr[u];
        if (ok[u]) {
          kr[u] = *(const Raw*)(ks + (size_t)r * D + c * VEC);
          vr[u] = *(const Raw*)(vs + (size_t)r * D + c * VEC);
        }
      }
      update(kr, vr, ok);
    }
  }

  // Finish the row group's sums, merge the warp's row groups, publish in sm[warp].
  __device__ __forceinline__ void to_smem(MergeSmem<G, D, kCW>& sm, int warp) {
    const unsigned FULL = 0xffffffffu;
    float ls = lpart;
    if (G <= 4) ls += __shfl_xor_sync(FULL, ls, S1);
    if (G <= 2) ls += __shfl_xor_sync(FULL, ls, S2);
    if (G == 1) ls += __shfl_xor_sync(FULL, ls, S3);
    float l[G];
#pragma unroll
    for (int h = 0; h < G; ++h) l[h] = __shfl_sync(FULL, ls, base | lane_of(h));
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float m2 = __shfl_xor_sync(FULL, m[h], off);
        const float l2 = __shfl_xor_sync(FULL, l[h], off);
        float mm, ll, a1, a2;
        merge_ml(m[h], l[h], m2, l2, mm, ll, a1, a2);
#pragma unroll
        for (int e = 0; e < V2; ++e) {
          const float ox = __shfl_xor_sync(FULL, o[h][e].x, off);
          const float oy = __shfl_xor_sync(FULL, o[h][e].y, off);
          o[h][e] = make_float2(o[h][e].x * a1 + ox * a2, o[h][e].y * a1 + oy * a2);
        }
        m[h] = mm;
        l[h] = ll;
      }
    }
    if (rs == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        if (c == 0) { sm.m[warp][h] = m[h]; sm.l[warp][h] = l[h]; }
#pragma unroll
        for (int e = 0; e < V2; ++e) {
          sm.o[warp][h][c * VEC + 2 * e] = o[h][e].x;
          sm.o[warp][h][c * VEC + 2 * e + 1] = o[h][e].y;
        }
      }
    }
  }
};

// Calls f(src, slab_row, dst_row, nrows) for the contiguous runs of the
// logical rows [x0, x1) of one pair (src 0: prefix rows, 1: ring rows),
// dst_row counted from x0 (a tile may span the prefix and both ring runs).
// Sets *bad if the rows reach block rows (a decode query never has them).
template <typename F>
__device__ __forceinline__ void for_each_run(const SegSet& s, int32_t x0, int32_t x1, bool* bad,
                                             F&& f) {
  int32_t L = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (i < s.n) {
      const int32_t lo = max(L, x0), hi = min(L + s.len[i], x1);
      if (hi > lo) {
        if (s.src[i] == 2) *bad = true;
        else f(s.src[i], s.row0[i] + (lo - L), lo - x0, hi - lo);
      }
      L += s.len[i];
    }
  }
}


// One tile as the producer hands it to the consumers (through shared memory,
// published by the mbarrier arrive that also carries the tile's bytes).
struct TileDesc {
  int32_t pair, nrows, flags;
  int32_t slot;  // partial-result slot of the tile's piece: CTA range + pair
};


template <typename T, int D, int G>
__global__ void __maxnreg__(65536 / (kThreadsDec * PS_DEC_CTAS_PER_SM) / 8 * 8)
    k_decode(const __grid_constant__ DecodeArgs a) {
  constexpr int TR = DecTile<T, D>::TR;
  constexpr int RW = DecTile<T, D>::RW;
  extern __shared__ __align__(128) unsigned char dsm[];
  T* ktile = (T*)dsm;                           // [kStages][TR][D]
  T* vtile = ktile + (size_t)kStages * TR * D;  // [kStages][TR][D]
  T* qtile = vtile + (size_t)kStages * TR * D;  // [kStages][G][D]: q of a piece's first tile
  __shared__ __align__(8) uint64_t full[kStages], empty[kStages];
  __shared__ __align__(8) uint64_t sync_a, sync_b;
  __shared__ TileDesc desc[kStages];
  __shared__ int abort_flag;
  __shared__ MergeSmem<G, D, kCW> sm;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Hkv = a.c.Hkv;
  const int64_t R = a.total, NC = a.nctas;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], kCW);
    }
    ptx::mbar_init(&sync_a, kCW);
    ptx::mbar_init(&sync_b, kCW);
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  // Launched as a programmatic dependent of the previous kernel on the stream:
  // everything above overlapped its tail; no memory is touched before it has
  // completed.  Then the merge grid may be scheduled (it waits for this one).
  ptx::pdl_wait_primary();
  ptx::pdl_launch_dependents();

  if (warp == kCW) {
    if (lane != 0) return;
    // ------------------------------------------------------------ producer --
    int i = 0;  // tiles handed out so far
    bool alive = true;
    const int32_t x1 = range_start(blockIdx.x + 1, R, NC);
    for (int32_t x = range_start(blockIdx.x, R, NC); x < x1 && alive;) {
      // one piece: the tiles of one pair inside this CTA's range
      const PairTiles pt = pair_of_tile(a, x);
      const int32_t j0 = x - pt.first, j1 = min(pt.tph, x1 - pt.first);
      x = pt.first + j1;
      const int s = a.seq[pt.b];
      // The ring state comes with the launch (the host's bookkeeping), so the
      // copies start without a dependent global load; the device's own record
      // is loaded alongside and compared once the piece's copies are issued.
      const DevMeta md = a.c.meta[s];
      DevMeta m;
      m.next_pos = a.t[pt.b] + 1;
      m.P = a.P[pt.b];
      m.head = a.head[pt.b];
      m.count = a.count[pt.b];
      m.owner = a.owner[pt.b];
      const SegSet segs = build_segments(m, a.c.W, a.t[pt.b]);
      bool bad = segs.total != m.P + m.count || (segs.total + TR - 1) / TR != pt.tph;
      const bool step = a.knew != nullptr;  // the pair's last row comes from knew/vnew
      const int pair = pt.b * Hkv + pt.g;
      for (int32_t j = j0; j < j1 && alive; ++j) {
        const int32_t r0 = j * TR, r1 = min(segs.total, r0 + TR);
        const int st = i % kStages;
        if (i >= kStages && !ptx::mbar_wait_bounded(&empty[st], ((i / kStages) - 1) & 1,
                                                    &abort_flag, kWaitLimitCycles)) {
          alive = false;
          break;
        }
        TileDesc d;
        d.pair = pair;
        d.nrows = max(r1 - r0, 0);
        const bool with_new = step && r1 == segs.total;
        d.flags = (j == j0 ? TD_FIRST : 0) | (j == j1 - 1 ? TD_LAST : 0) | (with_new ? TD_NEW : 0);
        d.slot = (int32_t)blockIdx.x + pair;
        desc[st] = d;
        // The first tile of a piece also brings the piece's G query rows, so
        // no consumer waits on a global load of q when a piece starts.
        const uint32_t bytes = (uint32_t)d.nrows * D * sizeof(T);
        const uint32_t qbytes = (d.flags & TD_FIRST) ? (uint32_t)(G * D * sizeof(T)) : 0u;
        ptx::mbar_arrive_expect_tx(&full[st], 2 * bytes + qbytes);
        if (qbytes)
          ptx::bulk_g2s(qtile + (size_t)st * G * D,
                        (const T*)a.q + ((size_t)pt.b * a.Hq + (size_t)pt.g * G) * D, qbytes,
                        &full[st]);
        T* kd = ktile + (size_t)st * TR * D;
        T* vd = vtile + (size_t)st * TR * D;
        auto copy = [&](int64_t crow, int32_t cdst, int32_t cn) {
          const uint32_t nb = (uint32_t)cn * D * sizeof(T);
          ptx::bulk_g2s(kd + (size_t)cdst * D, (const T*)a.c.K + (size_t)crow * D, nb, &full[st]);
          ptx::bulk_g2s(vd + (size_t)cdst * D, (const T*)a.c.V + (size_t)crow * D, nb, &full[st]);
        };
        for_each_run(segs, r0, with_new ? r1 - 1 : r1, &bad,
                     [&](int src, int64_t row, int32_t dst, int32_t nr) {
          if (src == 0) {  // prefix rows, from the slab of the sequence that owns them
            copy(prefix_row(a.c, a.owner[pt.b], pt.g, row), dst, nr);
            return;
          }
          // ring slots [row, row + nr): one copy per page they touch (a run
          // never wraps, so an unpaged ring takes one copy)
          const int32_t sa = (int32_t)row, se = sa + nr;
          for (int32_t s0 = sa; s0 < se;) {
            const int32_t pe = a.c.page_table ? (s0 / a.c.page_rows + 1) * a.c.page_rows : se;
            const int32_t cn = min(se, pe) - s0;
            copy(ring_row(a.c, ring_page(a.c, s, s0), pt.g, s0), dst + (s0 - sa), cn);
            s0 += cn;
          }
        });
        if (with_new) {  // the appended token, straight from the caller's rows
          const size_t src = (size_t)pair * D;
          const size_t dst = (size_t)(r1 - 1 - r0) * D;
          ptx::bulk_g2s(kd + dst, (const T*)a.knew + src, D * sizeof(T), &full[st]);
          ptx::bulk_g2s(vd + dst, (const T*)a.vnew + src, D * sizeof(T), &full[st]);
        }
        ++i;
      }
      // The device record is the state before this launch: for a decode step
      // it must advance to m by the one appended token.
      DevMeta me = md;
      if (step) {
        const int64_t W = a.c.W, cn = (int64_t)md.count + 1;
        me.next_pos = md.next_pos + 1;
        me.count = (int32_t)(cn < W ? cn : W);
        me.head = (int32_t)((md.head + (cn > W ? 1 : 0)) % W);
      }
      if (bad || me.next_pos != m.next_pos || me.P != m.P || me.head != m.head ||
          me.count != m.count || me.owner != m.owner)
        atomicOr(a.c.err, ERR_BATCH);
      if (!segs.ring_ok) atomicOr(a.c.err, ERR_RING);
    }
    if (alive) {  // end marker: a descriptor with no bytes
      const int st = i % kStages;
      if (i < kStages || ptx::mbar_wait_bounded(&empty[st], ((i / kStages) - 1) & 1, &abort_flag,
                                                kWaitLimitCycles)) {
        TileDesc end;
        end.pair = 0; end.nrows = 0; end.flags = TD_END; end.slot = 0;
        desc[st] = end;
        ptx::mbar_arrive(&full[st]);
        ++i;
      }
    }
    if (abort_flag) {  // let the copies already issued land before the CTA exits
      int quiet = 0;
      for (int k = max(0, i - kStages); k < i; ++k)
        ptx::mbar_wait_bounded(&full[k % kStages], (k / kStages) & 1, &quiet, kWaitLimitCycles);
    }
    return;
  }

  // -------------------------------------------------------------- consumers --
  // The consumer warps synchronise with mbarriers (bounded waits, one phase
  // per piece) rather than a named barrier, so a warp that gives up can never
  // leave the others waiting for good.
  auto csync = [&](uint64_t* bar, int phase) -> bool {
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(bar);
    return __all_sync(0xffffffffu,
                      ptx::mbar_wait_bounded(bar, phase & 1, &abort_flag, kWaitLimitCycles));
  };
  DecState<T, D, G> st;
  int np = 0;  // pieces finished by this CTA
  for (int i = 0;; ++i) {
    const int stg = i % kStages;
    const bool ok = ptx::mbar_wait_bounded(&full[stg], (i / kStages) & 1, &abort_flag,
                                           kWaitLimitCycles);
    if (!__all_sync(0xffffffffu, ok)) break;
    const TileDesc d = desc[stg];
    if (d.flags & TD_END) break;
    if (d.flags & TD_FIRST) st.init(qtile + (size_t)stg * G * D, a.qscale);
    const int mine = min(RW, d.nrows - warp * RW);  // this warp's rows of the tile
    if (mine > 0)
      st.tile(ktile + ((size_t)stg * TR + warp * RW) * D,
              vtile + ((size_t)stg * TR + warp * RW) * D, mine);
    if ((d.flags & TD_NEW) && warp == (d.nrows - 1) / RW) {
      // decode step: this warp holds the appended token; store it in its ring
      // slot (the evicted row's, never visible to this step's queries)
      const int b = d.pair / Hkv, g = d.pair % Hkv, s = a.seq[b];
      const int32_t slot = (int32_t)(((int64_t)a.head[b] + a.count[b] - 1) % a.c.W);
      const int phys = ring_page(a.c, s, slot);
      const size_t row = (size_t)ring_row(a.c, phys, g, slot) * D;
      const size_t so = ((size_t)stg * TR + d.nrows - 1) * D;
      constexpr int V16 = D * (int)sizeof(T) / 16;  // 16-byte pieces per row
      for (int x = lane; x < 2 * V16; x += 32) {
        const bool isv = x >= V16;
        const int xi = isv ? x - V16 : x;
        const uint4 val = ((const uint4*)((isv ? vtile : ktile) + so))[xi];
        ((uint4*)((T*)(isv ? a.c.V : a.c.K) + row))[xi] = val;
      }
      if (lane == 0 && g == 0) a.c.pos[pos_index(a.c, phys, slot)] = a.t[b];
    }
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(&empty[stg]);
    if (!(d.flags & TD_LAST)) continue;

    // ---- end of a (CTA range, pair) piece: publish its partial ----
    st.to_smem(sm, warp);  // this warp's (max, sum, accumulator) into sm[warp]
    if (!csync(&sync_a, np)) break;
    const int64_t slot = d.slot;  // unique per (CTA range, pair)
    float* pml = a.part_ml + (size_t)slot * G * 2;
    float* po = a.part_o + (size_t)slot * G * D;
    for (int idx = threadIdx.x; idx < G * D; idx += kCW * 32) {
      const int h = idx / D, e = idx % D;
      float mx = -INFINITY;
#pragma unroll
      for (int w = 0; w < kCW; ++w) mx = fmaxf(mx, sm.m[w][h]);
      float l = 0.f, acc = 0.f;
#pragma unroll
      for (int w = 0; w < kCW; ++w) {
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
    // sm is free for the next piece once every warp has read it
    if (!csync(&sync_b, np)) break;
    ++np;
  }
  if (threadIdx.x == 0 && abort_flag) atomicOr(a.c.err, ERR_TIMEOUT);
}


static_assert(PS_DEC_CTAS_PER_SM <= kDecMaxCtasPerSm, "workspace slots cover every CTA");
int max_ctas(int sm_count) { return sm_count * PS_DEC_CTAS_PER_SM; }

template <typename T, int D, int G>
cudaError_t launch_kernel(DecodeArgs a, int sm_count, cudaStream_t st) {
  // tiles per head of each entry, laid end to end, and the CTA count
  constexpr int TR = DecTile<T, D>::TR;
  a.tcum[0] = 0;
  for (int b = 0; b < a.B; ++b) {
    const int rows = a.P[b] + a.count[b];
    a.tcum[b + 1] = a.tcum[b] + a.c.Hkv * ((rows + TR - 1) / TR);
  }
  a.total = a.tcum[a.B];
  int64_t nc = ((int64_t)a.total + kMinTilesPerCta - 1) / kMinTilesPerCta;
  if (nc > max_ctas(sm_count)) nc = max_ctas(sm_count);
  if (nc < 1) nc = 1;
  a.nctas = (int)nc;
  const int nctas = a.nctas;
  constexpr size_t dyn = (size_t)kStages * (2 * DecTile<T, D>::TR + G) * D * sizeof(T);
  static std::atomic<uint64_t> configured{0};  // one bit per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(k_decode<T, D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)dyn);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(k_decode<T, D, G>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  // Both grids are programmatic dependent launches of the kernel before them.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t dcfg = {};
  dcfg.gridDim = dim3((unsigned)nctas);
  dcfg.blockDim = dim3(kThreadsDec);
  dcfg.dynamicSmemBytes = dyn;
  dcfg.stream = st;
  dcfg.attrs = attr;
  dcfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&dcfg, k_decode<T, D, G>, a);
  if (e != cudaSuccess) return e;
  return launch_merge<T, D, G>(a, st);
}

template <typename T, int D>
cudaError_t dispatch_G(int G, const DecodeArgs& a, int sm_count, cudaStream_t st) {
  switch (G) {
    case 1: return launch_kernel<T, D, 1>(a, sm_count, st);
    case 2: return launch_kernel<T, D, 2>(a, sm_count, st);
    case 4: return launch_kernel<T, D, 4>(a, sm_count, st);
    case 8: return launch_kernel<T, D, 8>(a, sm_count, st);
    default: return cudaErrorInvalidValue;
  }
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

DecodeWs decode_ws_layout(void* ws, int B, int Hkv, int G, int d, int sm_count, size_t* bytes) {
  const int Bl = B < kMaxBatchPerLaunch ? B : kMaxBatchPerLaunch;  // launches run in turn
  const size_t pairs = (size_t)Bl * Hkv;
  // one slot per (CTA range, pair) piece: range + pair, unique because
  // both grow in tile order
  const size_t slots = (size_t)sm_count * kDecMaxCtasPerSm + pairs;
  const size_t ml = align256(slots * G * 2 * sizeof(float));
  const size_t o = align256(slots * G * d * sizeof(float));
  DecodeWs w;
  char* p = (char*)ws;
  w.part_ml = (float*)p;
  w.part_o = (float*)(p + ml);
  if (bytes) *bytes = ml + o;
  return w;
}

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int d, int sm_count) {
  size_t bytes = 0;
  decode_ws_layout(nullptr, B, Hkv, Hq / Hkv, d, sm_count, &bytes);
  return bytes;
}

cudaError_t launch_decode(const CacheDev& c, int dtype, int G, const BatchIds& ids, int B, int Hq,
                          const void* q, const void* k_new, const void* v_new, void* out,
                          float scale, const DecodeWs& ws, int sm_count, const DecodeMaps* maps,
                          cudaStream_t st) {
  DecodeArgs a;
  memset(&a, 0, sizeof(a));
  a.c = c;
  a.q = q;
  a.knew = k_new;
  a.vnew = v_new;
  a.out = out;
  a.qscale = scale * kLog2e;
  a.Hq = Hq;
  a.B = B;
  a.part_ml = ws.part_ml;
  a.part_o = ws.part_o;
  for (int b = 0; b < B; ++b) {
    a.seq[b] = ids.seq[b];
    a.P[b] = ids.P[b];
    a.head[b] = ids.head[b];
    a.count[b] = ids.count[b];
    a.owner[b] = ids.owner[b];
    a.t[b] = ids.t[b];
  }
  if (dtype == 0) {
    if (c.d == 64) return dispatch_G<float, 64>(G, a, sm_count, st);
    return dispatch_G<float, 128>(G, a, sm_count, st);
  }
  // bfloat16: the tensor-core streaming kernel
  if (!maps) return cudaErrorInvalidValue;
  return launch_decode_mma(a, G, *maps, sm_count, st);
}

cudaError_t launch_chunk_small_batch(const CacheDev& c, int cols, int gq,
                                     const SmallChunkEntry* e, int B, int Hq, const void* q,
                                     const void* k_blk, const void* v_blk, int64_t blk_rows,
                                     void* out, float scale, int sm_count, const DecodeMaps& maps,
                                     cudaStream_t st) {
  if (B < 1 || B > kMaxBatchPerLaunch || gq < 1 || cols != 8 || cols % gq)
    return cudaErrorInvalidValue;
  DecodeArgs a;
  memset(&a, 0, sizeof(a));
  a.c = c;
  a.q = q;
  a.out = out;
  a.qscale = scale * kLog2e;
  a.Hq = Hq;
  a.B = B;
  ChunkArgs ch;
  memset(&ch, 0, sizeof(ch));
  ch.gq = gq;
  ch.lgq = gq == 8 ? 3 : gq == 4 ? 2 : gq == 2 ? 1 : 0;
  for (int b = 0; b < B; ++b) {
    if (e[b].nq < 1 || e[b].nq * gq > cols) return cudaErrorInvalidValue;
    a.seq[b] = e[b].seq;
    a.P[b] = e[b].P;
    a.head[b] = e[b].head;
    a.count[b] = e[b].count;
    a.owner[b] = e[b].owner;
    a.t[b] = e[b].t0 + e[b].i0;
    ch.i0[b] = e[b].i0;
    ch.nq[b] = e[b].nq;
    ch.qrow[b] = e[b].qrow;
    ch.brow[b] = e[b].brow;
  }
  return launch_chunk_small(a, ch, maps, k_blk, v_blk, blk_rows, sm_count, st);
}

}  // namespace ps
