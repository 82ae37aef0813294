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

#include "internal.h"

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

// Stream logical rows [j_begin, j_end) of `segs` for the G query heads of kv
// head g; leave the CTA's merged state in (sm.m[0], sm.l[0], sm.o[0]).
template <typename T, int D, int G>
__device__ __forceinline__ void stream_rows(const SegSet& segs, const T* __restrict__ kslab,
                                            const T* __restrict__ vslab,
                                            const T* __restrict__ kblk,
                                            const T* __restrict__ vblk, int64_t blk_stride,
                                            const T* __restrict__ qrow, float qscale,
                                            int32_t j_begin, int32_t j_end,
                                            MergeSmem<G, D>& sm) {
  constexpr int VEC = Vec<T>::N;
  constexpr int LPR = D / VEC;          // lanes per row
  constexpr int RPI = 32 / LPR;         // rows per warp per load instruction
  constexpr int U = G >= 8 ? 1 : (G >= 4 ? 2 : 4);
  constexpr int STEP = RPI * U;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c = lane % LPR, rs = lane / LPR;
  const unsigned FULL = 0xffffffffu;

  float q[G][VEC];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    uint4 raw = *(const uint4*)(qrow + (size_t)h * D + c * VEC);
    Vec<T>::unpack(raw, q[h]);
#pragma unroll
    for (int e = 0; e < VEC; ++e) q[h][e] *= qscale;
  }
  float mrun[G], lrun[G], o[G][VEC];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    mrun[h] = -INFINITY; lrun[h] = 0.f;
#pragma unroll
    for (int e = 0; e < VEC; ++e) o[h][e] = 0.f;
  }

  for (int32_t g0 = j_begin + warp * STEP; g0 < j_end; g0 += kNW * STEP) {
    uint4 kr[U], vr[U];
    bool ok[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      int32_t j = g0 + u * RPI + rs;
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
        kr[u] = __ldcs((const uint4*)(kp + c * VEC));
        vr[u] = __ldcs((const uint4*)(vp + c * VEC));
      }
    }
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

  // merge the RPI row sub-groups of this warp
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
      mrun[h] = mm; lrun[h] = ll;
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
  __syncthreads();
  // merge the warps into slot 0: first the per-head max/sum and warp weights
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

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreadsAttn) k_decode(AttnArgs a) {
  __shared__ MergeSmem<G, D> sm;
  __shared__ int is_last;
  const int split = blockIdx.x, g = blockIdx.y, bl = blockIdx.z;
  const int s = a.ids.seq[bl];
  const DevMeta m = a.c.meta[s];
  const int64_t t = m.next_pos - 1;
  const SegSet segs = build_segments(m, a.c.W, a.c.P_max, t);
  if (threadIdx.x == 0 && split == 0) {
    if (t != a.ids.t[bl]) atomicOr(a.c.err, ERR_BATCH);
    if (!segs.ring_ok) atomicOr(a.c.err, ERR_RING);
    if ((int64_t)a.nsplit * a.chunk < segs.total) atomicOr(a.c.err, ERR_COVERAGE);
  }
  const int32_t j_begin = split * a.chunk;
  const int32_t j_end = min(segs.total, j_begin + a.chunk);
  const size_t slab = ((size_t)s * a.c.Hkv + g) * (size_t)a.c.slab_rows * D;
  const T* qrow = (const T*)a.q + ((size_t)bl * a.Hq + (size_t)g * G) * D;
  stream_rows<T, D, G>(segs, (const T*)a.c.K + slab, (const T*)a.c.V + slab, nullptr, nullptr,
                       0, qrow, a.qscale, j_begin, j_end, sm);

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

template <typename T, int D>
cudaError_t dispatch_decode_G(int G, dim3 grid, const AttnArgs& a, cudaStream_t st) {
  switch (G) {
    case 1: k_decode<T, D, 1><<<grid, kThreadsAttn, 0, st>>>(a); break;
    case 2: k_decode<T, D, 2><<<grid, kThreadsAttn, 0, st>>>(a); break;
    case 4: k_decode<T, D, 4><<<grid, kThreadsAttn, 0, st>>>(a); break;
    case 8: k_decode<T, D, 8><<<grid, kThreadsAttn, 0, st>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
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

int target_ctas(int sm_count) { return sm_count * 8; }

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

DecodePlan plan_decode(int B, int Hkv, int n_max, int sm_count) {
  DecodePlan p;
  int pairs = B * Hkv;
  int ns = (target_ctas(sm_count) + pairs - 1) / pairs;
  if (ns < 1) ns = 1;
  if (ns > kMaxSplit) ns = kMaxSplit;
  int per = (n_max + ns - 1) / ns;
  if (per < 64) per = 64;
  per = (per + 31) / 32 * 32;
  p.chunk = per;
  p.nsplit = (n_max + per - 1) / per;
  if (p.nsplit < 1) p.nsplit = 1;
  return p;
}

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int d, int sm_count) {
  int G = Hq / Hkv;
  size_t tick = align256((size_t)B * Hkv * sizeof(int32_t));
  size_t slots = (size_t)B * Hkv + (size_t)target_ctas(sm_count);  // >= B*Hkv*nsplit
  if (slots > (size_t)B * Hkv * kMaxSplit) slots = (size_t)B * Hkv * kMaxSplit;
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
