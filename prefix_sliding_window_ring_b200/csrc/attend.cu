// CUDA-core attention over the visible rows of a prefix-sliding cache.
//
// Decode (a3-a5): one CTA per (batch entry, kv head, split).  The CTA derives
// the visible row ranges from the sequence's bookkeeping (prefix rows, then
// the ring window as at most two contiguous slot runs split at the physical
// wrap), streams its share of them once for all G query heads of the GQA group,
// and keeps an online softmax in float32 (digest section 06: iterate the
// prefix range and the window range separately so the evicted middle is never
// loaded).  The last CTA of a (batch entry, kv head) to finish merges the
// splits' (max, sum, accumulator) triples -- an atomic ticket, no spinning.
//
// Chunk (a6, CUDA-core variant): one CTA per (query row, kv head); the query's
// rows are the prefix, the ring part of its window and the block rows up to
// itself.
//
// Arithmetic: logits are kept in the base-2 domain (q is pre-multiplied by
// scale * log2(e)), weights are exp2(z - running max), accumulation is fp32.
#include <math.h>
#include <string.h>

#include <atomic>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace ps {

namespace {

constexpr int kNW = 4;             // warps per CTA
constexpr int kThreadsAttn = kNW * 32;
constexpr int kMaxSplit = 64;
constexpr float kLog2e = 1.4426950408889634f;

template <typename T> struct Vec;
template <> struct Vec<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void unpack(const uint4& x, float* f) {
    f[0] = __uint_as_float(x.x); f[1] = __uint_as_float(x.y);
    f[2] = __uint_as_float(x.z); f[3] = __uint_as_float(x.w);
  }
  __device__ __forceinline__ static void store(float* dst, const float* f) {
    *(float4*)dst = make_float4(f[0], f[1], f[2], f[3]);
  }
};
template <> struct Vec<uint16_t> {  // bfloat16 bit patterns
  static constexpr int N = 8;
  __device__ __forceinline__ static void unpack(const uint4& x, float* f) {
    f[0] = bf16lo(x.x); f[1] = bf16hi(x.x); f[2] = bf16lo(x.y); f[3] = bf16hi(x.y);
    f[4] = bf16lo(x.z); f[5] = bf16hi(x.z); f[6] = bf16lo(x.w); f[7] = bf16hi(x.w);
  }
};

template <typename T> __device__ __forceinline__ void store_out(T* dst, float v);
template <> __device__ __forceinline__ void store_out<float>(float* dst, float v) { *dst = v; }
template <> __device__ __forceinline__ void store_out<uint16_t>(uint16_t* dst, float v) {
  *dst = f2bf(v);
}

// Merge two online-softmax states (base-2 domain).
__device__ __forceinline__ void merge_ml(float m1, float l1, float m2, float l2, float& m,
                                         float& l, float& a1, float& a2) {
  m = fmaxf(m1, m2);
  if (m == -INFINITY) { l = 0.f; a1 = 0.f; a2 = 0.f; return; }
  a1 = exp2f(m1 - m);
  a2 = exp2f(m2 - m);
  l = l1 * a1 + l2 * a2;
}

template <int G, int D> struct MergeSmem {
  float m[kNW][G];
  float l[kNW][G];
  float wt[kNW][G];
  float o[kNW][G][D];
};

// Online-softmax state of one lane for the G query heads of a GQA group.
// Rows are read LPR lanes per row, RPI rows per warp instruction, U row slots
// per update; every lane of a row group ends an update with the same scores.
template <typename T, int D, int G>
struct AttnState {
  static constexpr int VEC = Vec<T>::N;
  static constexpr int LPR = D / VEC;   // lanes per row
  static constexpr int RPI = 32 / LPR;  // rows per warp load instruction
  static constexpr int U = G >= 8 ? 1 : (G >= 4 ? 2 : 4);
  static constexpr int STEP = RPI * U;  // rows per update
  float q[G][VEC];
  float mrun[G], lrun[G], o[G][VEC];
  int c, rs;

  __device__ __forceinline__ void init(const T* __restrict__ qrow, float qscale) {
    const int lane = threadIdx.x & 31;
    c = lane % LPR;
    rs = lane / LPR;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      uint4 raw = *(const uint4*)(qrow + (size_t)h * D + c * VEC);
      Vec<T>::unpack(raw, q[h]);
#pragma unroll
      for (int e = 0; e < VEC; ++e) q[h][e] *= qscale;
      mrun[h] = -INFINITY;
      lrun[h] = 0.f;
#pragma unroll
      for (int e = 0; e < VEC; ++e) o[h][e] = 0.f;
    }
  }

  // Fold U rows (this lane's 16-byte slices kr/vr; ok = row exists) into the state.
  __device__ __forceinline__ void update(const uint4 (&kr)[U], const uint4 (&vr)[U],
                                         const bool (&ok)[U]) {
    const unsigned FULL = 0xffffffffu;
    float sc[U][G];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float kf[VEC];
      Vec<T>::unpack(kr[u], kf);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc = fmaf(q[h][e], kf[e], acc);
        sc[u][h] = acc;
      }
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) {
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int h = 0; h < G; ++h) sc[u][h] += __shfl_xor_sync(FULL, sc[u][h], off);
    }
    float p[U][G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float mx = mrun[h];
#pragma unroll
      for (int u = 0; u < U; ++u) if (ok[u]) mx = fmaxf(mx, sc[u][h]);
      float alpha = (mx == -INFINITY) ? 1.f : exp2f(mrun[h] - mx);
      lrun[h] *= alpha;
#pragma unroll
      for (int e = 0; e < VEC; ++e) o[h][e] *= alpha;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        p[u][h] = ok[u] ? exp2f(sc[u][h] - mx) : 0.f;
        lrun[h] += p[u][h];
      }
      mrun[h] = mx;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float vf[VEC];
      Vec<T>::unpack(vr[u], vf);
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < VEC; ++e) o[h][e] = fmaf(p[u][h], vf[e], o[h][e]);
    }
  }

  // Rows [0, nrows) of a contiguous tile (row stride D elements).
  __device__ __forceinline__ void tile(const T* ks, const T* vs, int nrows) {
    for (int r0 = 0; r0 < nrows; r0 += STEP) {
      uint4 kr[U], vr[U];
      bool ok[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        int r = r0 + u * RPI + rs;
        ok[u] = r < nrows;
        kr[u] = make_uint4(0, 0, 0, 0);
        vr[u] = kr[u];
        if (ok[u]) {
          kr[u] = *(const uint4*)(ks + (size_t)r * D + c * VEC);
          vr[u] = *(const uint4*)(vs + (size_t)r * D + c * VEC);
        }
      }
      update(kr, vr, ok);
    }
  }

  // Merge this warp's row groups, then publish the warp's state in sm[warp].
  __device__ __forceinline__ void to_smem(MergeSmem<G, D>& sm, int warp) {
    const unsigned FULL = 0xffffffffu;
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float m2 = __shfl_xor_sync(FULL, mrun[h], off);
        float l2 = __shfl_xor_sync(FULL, lrun[h], off);
        float mm, ll, a1, a2;
        merge_ml(mrun[h], lrun[h], m2, l2, mm, ll, a1, a2);
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          float o2 = __shfl_xor_sync(FULL, o[h][e], off);
          o[h][e] = o[h][e] * a1 + o2 * a2;
        }
        mrun[h] = mm;
        lrun[h] = ll;
      }
    }
    if (rs == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        if (c == 0) { sm.m[warp][h] = mrun[h]; sm.l[warp][h] = lrun[h]; }
#pragma unroll
        for (int e = 0; e < VEC; ++e) sm.o[warp][h][c * VEC + e] = o[h][e];
      }
    }
  }
};

// Merge the kNW warp states in sm into slot 0 (all threads of the CTA call this).
template <int G, int D>
__device__ __forceinline__ void merge_warps(MergeSmem<G, D>& sm) {
  __syncthreads();
  if (threadIdx.x < G) {
    const int h = threadIdx.x;
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < kNW; ++w) mx = fmaxf(mx, sm.m[w][h]);
    float l = 0.f;
#pragma unroll
    for (int w = 0; w < kNW; ++w) {
      float a = (mx == -INFINITY) ? 0.f : exp2f(sm.m[w][h] - mx);
      sm.wt[w][h] = a;
      l += sm.l[w][h] * a;
    }
    sm.m[0][h] = mx;
    sm.l[0][h] = l;
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
    int h = idx / D, e = idx % D;
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < kNW; ++w) acc += sm.o[w][h][e] * sm.wt[w][h];
    sm.o[0][h][e] = acc;
  }
  __syncthreads();
}

// Stream logical rows [j_begin, j_end) of `segs` straight from global memory
// (warp w takes row groups w, w+kNW, ...); leave the CTA state in sm slot 0.
template <typename T, int D, int G>
__device__ __forceinline__ void stream_rows(const SegSet& segs, const T* __restrict__ kslab,
                                            const T* __restrict__ vslab,
                                            const T* __restrict__ kblk,
                                            const T* __restrict__ vblk, int64_t blk_stride,
                                            const T* __restrict__ qrow, float qscale,
                                            int32_t j_begin, int32_t j_end,
                                            MergeSmem<G, D>& sm) {
  using S = AttnState<T, D, G>;
  S st;
  st.init(qrow, qscale);
  const int warp = threadIdx.x >> 5;
  for (int32_t g0 = j_begin + warp * S::STEP; g0 < j_end; g0 += kNW * S::STEP) {
    uint4 kr[S::U], vr[S::U];
    bool ok[S::U];
#pragma unroll
    for (int u = 0; u < S::U; ++u) {
      int32_t j = g0 + u * S::RPI + st.rs;
      ok[u] = j < j_end;
      kr[u] = make_uint4(0, 0, 0, 0);
      vr[u] = kr[u];
      if (ok[u]) {
        int si; int32_t off;
        seg_locate(segs, j, si, off);
        const T* kp; const T* vp;
        if (segs.src[si] == 2) {
          size_t r = (size_t)(segs.row0[si] + off) * blk_stride;
          kp = kblk + r; vp = vblk + r;
        } else {
          size_t r = (size_t)(segs.row0[si] + off) * D;
          kp = kslab + r; vp = vslab + r;
        }
        kr[u] = __ldcs((const uint4*)(kp + st.c * S::VEC));
        vr[u] = __ldcs((const uint4*)(vp + st.c * S::VEC));
      }
    }
    st.update(kr, vr, ok);
  }
  st.to_smem(sm, warp);
  merge_warps<G, D>(sm);
}

struct AttnArgs {
  CacheDev c;
  const void* q;
  void* out;
  const void* kb;
  const void* vb;
  float qscale;
  float* part_ml;    // [B][Hkv][nsplit][G][2]
  float* part_o;     // [B][Hkv][nsplit][G][D]
  int32_t* tick;     // [B][Hkv]
  int nsplit, chunk, Hq, b_off, seq;
  int64_t t0;
  BatchIds ids;
};

// ---------------------------------------------------------------- decode --
// Pipelined split-K decode.  Warp kNW is the producer: one lane issues bulk
// async copies (cp.async.bulk, no multicast) of contiguous K and V row tiles
// into a kStages-deep shared-memory ring, each tile lying inside one visible
// range (prefix rows, or one contiguous run of ring slots), so no evicted or
// foreign row is ever fetched.  Warps 0..kNW-1 consume tiles round-robin with
// the online softmax of AttnState.  Every wait is bounded: on a time-out the
// CTA stops, reports ERR_TIMEOUT and drains its own copies before exiting.

constexpr int kThreadsDec = (kNW + 1) * 32;
// Tile i sits in stage i % kStages and is consumed by warp i % kNW.  With
// kStages a multiple of kNW every stage belongs to one warp, which therefore
// waits on its stages strictly in phase order: a warp can never reach a stage
// two phases early, where the parity test would mistake the older completed
// phase for the one it needs.
constexpr int kStages = 8;
static_assert(kStages % kNW == 0, "each pipeline stage must belong to one consumer warp");
constexpr long long kWaitLimitCycles = 1ll << 30;  // about half a second

template <typename T, int D> struct DecTile {
  static constexpr int TR = 4096 / (D * (int)sizeof(T));  // rows per tile (4 KiB of K)
};

// Tiles of the logical range [jb, je): split at range boundaries and every TR rows.
struct TilePlan {
  int n;              // pieces
  int ntiles;
  int32_t len[4];
  int32_t tbase[4];
  int64_t row0[4];    // slab row of the first row of each piece
};

__device__ __forceinline__ TilePlan plan_tiles(const SegSet& s, int32_t jb, int32_t je, int TR,
                                               bool* bad) {
  TilePlan tp;
  tp.n = 0;
  tp.ntiles = 0;
  int32_t L = 0;
  for (int i = 0; i < s.n; ++i) {
    int32_t a = max(L, jb), b = min(L + s.len[i], je);
    if (b > a) {
      if (s.src[i] == 2) {
        *bad = true;
      } else {
        tp.len[tp.n] = b - a;
        tp.tbase[tp.n] = tp.ntiles;
        tp.row0[tp.n] = s.row0[i] + (a - L);
        tp.ntiles += (b - a + TR - 1) / TR;
        tp.n++;
      }
    }
    L += s.len[i];
  }
  return tp;
}

__device__ __forceinline__ void tile_at(const TilePlan& tp, int i, int TR, int64_t& row,
                                        int& nrows) {
  int k = 0;
#pragma unroll
  for (int q = 1; q < 4; ++q)
    if (q < tp.n && i >= tp.tbase[q]) k = q;
  int32_t off = (i - tp.tbase[k]) * TR;
  row = tp.row0[k] + off;
  nrows = min(TR, tp.len[k] - off);
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreadsDec) k_decode(AttnArgs a) {
  constexpr int TR = DecTile<T, D>::TR;
  extern __shared__ __align__(1024) unsigned char dsm[];
  T* ktile = (T*)dsm;                               // [kStages][TR][D]
  T* vtile = ktile + (size_t)kStages * TR * D;      // [kStages][TR][D]
  __shared__ __align__(8) uint64_t full[kStages], empty[kStages];
  __shared__ int abort_flag;
  __shared__ int is_last;
  __shared__ MergeSmem<G, D> sm;

  const int split = blockIdx.x, g = blockIdx.y, bl = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int s = a.ids.seq[bl];
  const DevMeta m = a.c.meta[s];
  const int64_t t = m.next_pos - 1;
  const SegSet segs = build_segments(m, a.c.W, a.c.P_max, t);
  const int32_t j_begin = split * a.chunk;
  const int32_t j_end = min(segs.total, j_begin + a.chunk);
  bool bad = false;
  const TilePlan tp = plan_tiles(segs, j_begin, j_end, TR, &bad);
  if (threadIdx.x == 0) {
    if (split == 0) {
      if (t != a.ids.t[bl]) atomicOr(a.c.err, ERR_BATCH);
      if (!segs.ring_ok) atomicOr(a.c.err, ERR_RING);
      if ((int64_t)a.nsplit * a.chunk < segs.total) atomicOr(a.c.err, ERR_COVERAGE);
    }
    if (bad) atomicOr(a.c.err, ERR_BATCH);
    for (int i = 0; i < kStages; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], 1);
    }
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();

  const size_t slab = ((size_t)s * a.c.Hkv + g) * (size_t)a.c.slab_rows * D;
  const T* kslab = (const T*)a.c.K + slab;
  const T* vslab = (const T*)a.c.V + slab;
  if (warp == kNW) {
    if (lane == 0) {  // producer
      int issued = 0;
      for (int i = 0; i < tp.ntiles; ++i) {
        const int st = i % kStages;
        if (i >= kStages &&
            !ptx::mbar_wait_bounded(&empty[st], ((i / kStages) - 1) & 1, &abort_flag,
                                    kWaitLimitCycles))
          break;
        int64_t row;
        int nr;
        tile_at(tp, i, TR, row, nr);
        const uint32_t bytes = (uint32_t)nr * D * sizeof(T);
        ptx::mbar_arrive_expect_tx(&full[st], 2 * bytes);
        ptx::bulk_g2s(ktile + (size_t)st * TR * D, kslab + (size_t)row * D, bytes, &full[st]);
        ptx::bulk_g2s(vtile + (size_t)st * TR * D, vslab + (size_t)row * D, bytes, &full[st]);
        issued = i + 1;
      }
      if (abort_flag) {  // let the copies already issued land before the CTA exits
        int quiet = 0;
        for (int i = max(0, issued - kStages); i < issued; ++i)
          ptx::mbar_wait_bounded(&full[i % kStages], (i / kStages) & 1, &quiet, kWaitLimitCycles);
      }
    }
  } else {  // consumers
    AttnState<T, D, G> st;
    st.init((const T*)a.q + ((size_t)bl * a.Hq + (size_t)g * G) * D, a.qscale);
    for (int i = warp; i < tp.ntiles; i += kNW) {
      const int stg = i % kStages;
      bool ok = ptx::mbar_wait_bounded(&full[stg], (i / kStages) & 1, &abort_flag,
                                       kWaitLimitCycles);
      if (!__all_sync(0xffffffffu, ok)) break;
      int64_t row;
      int nr;
      tile_at(tp, i, TR, row, nr);
      st.tile(ktile + (size_t)stg * TR * D, vtile + (size_t)stg * TR * D, nr);
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&empty[stg]);
    }
    st.to_smem(sm, warp);
  }
  merge_warps<G, D>(sm);
  if (threadIdx.x == 0 && abort_flag) atomicOr(a.c.err, ERR_TIMEOUT);

  const int bg = (a.b_off + bl) * a.c.Hkv + g;  // workspace slot of (batch entry, kv head)
  float* pml = a.part_ml + ((size_t)bg * a.nsplit + split) * G * 2;
  float* po = a.part_o + ((size_t)bg * a.nsplit + split) * G * D;
  for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) po[idx] = sm.o[0][idx / D][idx % D];
  if (threadIdx.x < G) {
    pml[threadIdx.x * 2] = sm.m[0][threadIdx.x];
    pml[threadIdx.x * 2 + 1] = sm.l[0][threadIdx.x];
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    int old = atomicAdd(&a.tick[bg], 1);
    is_last = (old == a.nsplit - 1);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  const float* bml = a.part_ml + (size_t)bg * a.nsplit * G * 2;
  const float* bo = a.part_o + (size_t)bg * a.nsplit * G * D;
  T* orow = (T*)a.out + ((size_t)bl * a.Hq + (size_t)g * G) * D;
  for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
    int h = idx / D, e = idx % D;
    float mx = -INFINITY;
    for (int j = 0; j < a.nsplit; ++j) mx = fmaxf(mx, __ldcg(bml + ((size_t)j * G + h) * 2));
    float l = 0.f, acc = 0.f;
    for (int j = 0; j < a.nsplit; ++j) {
      float mj = __ldcg(bml + ((size_t)j * G + h) * 2);
      if (mj == -INFINITY) continue;
      float w = exp2f(mj - mx);
      l += __ldcg(bml + ((size_t)j * G + h) * 2 + 1) * w;
      acc += __ldcg(bo + ((size_t)j * G + h) * D + e) * w;
    }
    store_out<T>(orow + (size_t)h * D + e, acc / l);
  }
  if (threadIdx.x == 0) a.tick[bg] = 0;
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreadsAttn) k_chunk_cc(AttnArgs a) {
  __shared__ MergeSmem<G, D> sm;
  const int i = blockIdx.x, g = blockIdx.y;
  const DevMeta m = a.c.meta[a.seq];
  const int64_t t = a.t0 + i;
  const SegSet segs = build_segments(m, a.c.W, a.c.P_max, t);
  if (threadIdx.x == 0 && i == 0 && g == 0) {
    if (m.next_pos != a.t0) atomicOr(a.c.err, ERR_BATCH);
    if (!segs.ring_ok) atomicOr(a.c.err, ERR_RING);
  }
  const size_t slab = ((size_t)a.seq * a.c.Hkv + g) * (size_t)a.c.slab_rows * D;
  const int64_t bstride = (int64_t)a.c.Hkv * D;
  const T* qrow = (const T*)a.q + ((size_t)i * a.Hq + (size_t)g * G) * D;
  stream_rows<T, D, G>(segs, (const T*)a.c.K + slab, (const T*)a.c.V + slab,
                       (const T*)a.kb + (size_t)g * D, (const T*)a.vb + (size_t)g * D, bstride,
                       qrow, a.qscale, 0, segs.total, sm);
  T* orow = (T*)a.out + ((size_t)i * a.Hq + (size_t)g * G) * D;
  for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
    int h = idx / D, e = idx % D;
    store_out<T>(orow + (size_t)h * D + e, sm.o[0][h][e] / sm.l[0][h]);
  }
}

template <typename T, int D, int G>
cudaError_t launch_decode_kernel(dim3 grid, const AttnArgs& a, cudaStream_t st) {
  constexpr size_t dyn = (size_t)2 * kStages * DecTile<T, D>::TR * D * sizeof(T);
  static std::atomic<uint64_t> configured{0};  // one bit per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(k_decode<T, D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)dyn);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  k_decode<T, D, G><<<grid, kThreadsDec, dyn, st>>>(a);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t dispatch_decode_G(int G, dim3 grid, const AttnArgs& a, cudaStream_t st) {
  switch (G) {
    case 1: return launch_decode_kernel<T, D, 1>(grid, a, st);
    case 2: return launch_decode_kernel<T, D, 2>(grid, a, st);
    case 4: return launch_decode_kernel<T, D, 4>(grid, a, st);
    case 8: return launch_decode_kernel<T, D, 8>(grid, a, st);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T, int D>
cudaError_t dispatch_chunk_G(int G, dim3 grid, const AttnArgs& a, cudaStream_t st) {
  switch (G) {
    case 1: k_chunk_cc<T, D, 1><<<grid, kThreadsAttn, 0, st>>>(a); break;
    case 2: k_chunk_cc<T, D, 2><<<grid, kThreadsAttn, 0, st>>>(a); break;
    case 4: k_chunk_cc<T, D, 4><<<grid, kThreadsAttn, 0, st>>>(a); break;
    case 8: k_chunk_cc<T, D, 8><<<grid, kThreadsAttn, 0, st>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// Upper bound on decode CTAs per launch (sizes the workspace): 4 waves.
int max_ctas_per_launch(int sm_count) { return sm_count * 12; }

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

DecodePlan plan_decode(int B, int Hkv, int n_max, int sm_count) {
  // Pick the split count that minimises (waves x rows per CTA): every CTA of
  // a wave streams at about the same rate, so a launch lasts about that long.
  const int slots = sm_count * 3;  // resident decode CTAs per SM
  const int pairs = B * Hkv;
  DecodePlan best{1, n_max};
  long long best_cost = -1;
  const long long max_ctas = pairs > max_ctas_per_launch(sm_count) ? pairs
                                                                     : max_ctas_per_launch(sm_count);
  for (int ns = 1; ns <= kMaxSplit; ++ns) {
    int per = (n_max + ns - 1) / ns;
    if (per < 128 && ns > 1) break;
    per = (per + 31) / 32 * 32;
    int ns_eff = (n_max + per - 1) / per;
    long long ctas = (long long)pairs * ns_eff;
    if (ctas > max_ctas) break;
    long long waves = (ctas + slots - 1) / slots;
    long long cost = waves * (per + 96);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best.nsplit = ns_eff;
      best.chunk = per;
    }
  }
  return best;
}

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int d, int sm_count) {
  int G = Hq / Hkv;
  size_t tick = align256((size_t)B * Hkv * sizeof(int32_t));
  size_t pairs = (size_t)B * Hkv;  // B*Hkv*nsplit never exceeds max(pairs, max CTAs)
  size_t slots = pairs > (size_t)max_ctas_per_launch(sm_count) ? pairs
                                                               : (size_t)max_ctas_per_launch(sm_count);
  size_t ml = align256(slots * G * 2 * sizeof(float));
  size_t o = align256(slots * G * d * sizeof(float));
  return tick + ml + o;
}

DecodeWs decode_ws_layout(void* ws, int B, int Hkv, int G, int d, int nsplit, size_t* bytes) {
  DecodeWs w;
  char* p = (char*)ws;
  size_t tick = align256((size_t)B * Hkv * sizeof(int32_t));
  size_t slots = (size_t)B * Hkv * nsplit;
  size_t ml = align256(slots * G * 2 * sizeof(float));
  size_t o = align256(slots * G * d * sizeof(float));
  w.tick = (int32_t*)p;
  w.part_ml = (float*)(p + tick);
  w.part_o = (float*)(p + tick + ml);
  if (bytes) *bytes = tick + ml + o;
  return w;
}

cudaError_t launch_decode(const CacheDev& c, int dtype, int G, const BatchIds& ids, int B,
                          int b_off, int Hq, const void* q, void* out, float scale,
                          const DecodeWs& ws, const DecodePlan& plan, cudaStream_t st) {
  AttnArgs a;
  a.c = c;
  a.q = q;
  a.out = out;
  a.kb = nullptr;
  a.vb = nullptr;
  a.qscale = scale * kLog2e;
  a.part_ml = ws.part_ml;
  a.part_o = ws.part_o;
  a.tick = ws.tick;
  a.nsplit = plan.nsplit;
  a.chunk = plan.chunk;
  a.Hq = Hq;
  a.b_off = b_off;
  a.seq = 0;
  a.t0 = 0;
  a.ids = ids;
  dim3 grid(plan.nsplit, c.Hkv, B);
  if (dtype == 0) {
    if (c.d == 64) return dispatch_decode_G<float, 64>(G, grid, a, st);
    return dispatch_decode_G<float, 128>(G, grid, a, st);
  }
  if (c.d == 64) return dispatch_decode_G<uint16_t, 64>(G, grid, a, st);
  return dispatch_decode_G<uint16_t, 128>(G, grid, a, st);
}

cudaError_t launch_chunk_cc(const CacheDev& c, int dtype, int G, int seq, int64_t t0, int n,
                            int Hq, const void* q, const void* k_blk, const void* v_blk,
                            void* out, float scale, cudaStream_t st) {
  AttnArgs a;
  memset(&a, 0, sizeof(a));
  a.c = c;
  a.q = q;
  a.out = out;
  a.kb = k_blk;
  a.vb = v_blk;
  a.qscale = scale * kLog2e;
  a.Hq = Hq;
  a.seq = seq;
  a.t0 = t0;
  dim3 grid(n, c.Hkv);
  if (dtype == 0) {
    if (c.d == 64) return dispatch_chunk_G<float, 64>(G, grid, a, st);
    return dispatch_chunk_G<float, 128>(G, grid, a, st);
  }
  if (c.d == 64) return dispatch_chunk_G<uint16_t, 64>(G, grid, a, st);
  return dispatch_chunk_G<uint16_t, 128>(G, grid, a, st);
}

}  // namespace ps
