// Chunked prefill/extend on CUDA cores (the configurations the tensor-core
// kernel does not take: float32, head_dim 64).
//
// One CTA per (query row, kv head).  The CTA derives the query's visible row
// ranges from the sequence's bookkeeping -- prefix rows, the ring part of its
// window as at most two contiguous slot runs split at the physical wrap, then
// the block rows up to the query itself -- and streams them once for all G
// query heads of the GQA group with an online softmax in float32.  Evicted
// rows are never addressed ("Prefix Sliding" digest, section 06).
#include <math.h>
#include <string.h>

#include "attn_common.cuh"
#include "internal.h"

namespace ps {

namespace {

using namespace attn;

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
// Prefix rows come from the slab of sequence `owner`, ring slots from the
// pages of sequence `seq`, block rows from kblk / vblk.
template <typename T, int D, int G>
__device__ __forceinline__ void stream_rows(const SegSet& segs, const CacheDev& c, int seq,
                                            int owner, int g, const T* __restrict__ kblk,
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
          const int32_t x = (int32_t)segs.row0[si] + off;  // prefix row or ring slot
          const size_t r = (size_t)(segs.src[si] == 0 ? prefix_row(c, owner, g, x)
                                                      : ring_row(c, ring_page(c, seq, x), g, x)) *
                           D;
          kp = (const T*)c.K + r; vp = (const T*)c.V + r;
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
  int Hq, seq;
  int prompt;  // queries inside the prefix: causal over the prefix rows only
  int64_t t0;
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreadsAttn) k_chunk_cc(AttnArgs a) {
  __shared__ MergeSmem<G, D> sm;
  const int i = blockIdx.x, g = blockIdx.y;
  const DevMeta m = a.c.meta[a.seq];
  const int64_t t = a.t0 + i;
  SegSet segs = build_segments(m, a.c.W, t);
  if (a.prompt) {  // t < P: the visible rows are the prefix rows [0, t]
    segs.n = 1;
    segs.len[0] = (int32_t)(t + 1);
    segs.row0[0] = 0;
    segs.src[0] = 0;
    segs.total = (int32_t)(t + 1);
    segs.ring_ok = 1;
  }
  if (threadIdx.x == 0 && i == 0 && g == 0) {
    if (a.prompt ? a.t0 + gridDim.x > m.P : m.next_pos != a.t0) atomicOr(a.c.err, ERR_BATCH);
    if (!segs.ring_ok) atomicOr(a.c.err, ERR_RING);
  }
  const int64_t bstride = (int64_t)a.c.Hkv * D;
  const T* qrow = (const T*)a.q + ((size_t)i * a.Hq + (size_t)g * G) * D;
  stream_rows<T, D, G>(segs, a.c, a.seq, m.owner, g, (const T*)a.kb + (size_t)g * D, (const T*)a.vb + (size_t)g * D, bstride,
                       qrow, a.qscale, 0, segs.total, sm);
  T* orow = (T*)a.out + ((size_t)i * a.Hq + (size_t)g * G) * D;
  for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
    int h = idx / D, e = idx % D;
    store_out<T>(orow + (size_t)h * D + e, sm.o[0][h][e] / sm.l[0][h]);
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


}  // namespace

cudaError_t launch_chunk_cc(const CacheDev& c, int dtype, int G, int seq, int64_t t0, int n,
                            int Hq, const void* q, const void* k_blk, const void* v_blk,
                            void* out, float scale, int prompt, cudaStream_t st) {
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
  a.prompt = prompt;
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
