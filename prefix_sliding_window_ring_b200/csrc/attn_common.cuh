// Shared pieces of the CUDA-core attention kernels: 16-byte vector unpacking,
// output rounding and the merge of two online-softmax states.
//
// Arithmetic: logits are kept in the base-2 domain (q is pre-multiplied by
// scale * log2(e)), weights are exp2(z - running max), accumulation is fp32.
#pragma once
#include <math.h>

#include "common.cuh"

namespace ps {
namespace attn {

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

// Per-warp online-softmax states staged for a CTA-level merge.
template <int G, int D, int NW = kNW> struct MergeSmem {
  float m[NW][G];
  float l[NW][G];
  float wt[NW][G];
  float o[NW][G][D];
};

}  // namespace attn
}  // namespace ps
