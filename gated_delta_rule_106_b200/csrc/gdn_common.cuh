// Shared device helpers for the gated delta-rule kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn.h"

namespace gdn {

constexpr int kHeadDim = 128;   // d_k = d_v = 128 (model card, 架构 table)
constexpr int kConvTaps = 4;    // causal conv kernel 4
constexpr int kChunk = 64;      // chunked prefill chunk length

__host__ __device__ inline int elem_bytes(gdn_dtype t) {
  return t == GDN_F32 ? 4 : 2;
}

// 8 consecutive elements <-> 8 floats. bf16: one 16-byte access; fp32: two.
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&f)[8]) {
  uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ void load8(const float* p, float (&f)[8]) {
  float4 a = *reinterpret_cast<const float4*>(p);
  float4 b = *reinterpret_cast<const float4*>(p + 4);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&f)[8]) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}
__device__ __forceinline__ void store8(float* p, const float (&f)[8]) {
  *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(f[4], f[5], f[6], f[7]);
}

// 8 consecutive elements kept as loaded (bf16: one 16-byte vector; fp32: two)
// until they are needed, so that many loads can be in flight per thread
template <class Tx> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
  uint4 u;
  __device__ __forceinline__ void zero() { u = make_uint4(0, 0, 0, 0); }
  __device__ __forceinline__ void load(const __nv_bfloat16* p) {
    u = __ldg(reinterpret_cast<const uint4*>(p));
  }
  __device__ __forceinline__ void to_f32(float (&f)[8]) const {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 t = __bfloat1622float2(h[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
};
template <> struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ void load(const float* p) {
    a = __ldg(reinterpret_cast<const float4*>(p));
    b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  }
  __device__ __forceinline__ void to_f32(float (&f)[8]) const {
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
};

__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f32(float x) { return x; }

template <class T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// SiLU with the hardware reciprocal-based quotient (within 2 ulp; 0 once the
// denominator passes 2^126, where a * sigmoid(a) is below the smallest normal)
__device__ __forceinline__ float silu(float a) { return __fdividef(a, 1.0f + __expf(-a)); }

// Sequence index n with cu[n] <= t < cu[n+1] (skips empty sequences);
// cu is clamped into [0, T] by the caller's contract. Returns N-1 when t is
// past the last start (never read out of range).
__device__ __forceinline__ int seq_of(const int32_t* cu, int N, int64_t t) {
  int lo = 0, hi = N - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if ((int64_t)__ldg(cu + mid) <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ int64_t clamp_t(int64_t v, int64_t T) {
  return v < 0 ? 0 : (v > T ? T : v);
}

// seq_of, starting from the guess that sequences are of equal length: when the
// guessed sequence brackets t (always, for equal lengths, e.g. one token per
// sequence) this is one round of two independent loads instead of a chain
__device__ __forceinline__ int seq_locate(const int32_t* cu, int N, int64_t T, int64_t t) {
  int n = T > 0 ? (int)((t * N) / T) : 0;
  n = n < 0 ? 0 : (n > N - 1 ? N - 1 : n);
  const int64_t a = __ldg(cu + n), b = __ldg(cu + n + 1);
  if (a <= t && (t < b || n == N - 1)) return n;
  return seq_of(cu, N, t);
}

}  // namespace gdn
