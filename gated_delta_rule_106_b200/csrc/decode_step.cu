// Stepwise decode of the gated delta rule (the "delta_rule_stepwise" decode
// path named in the "Agnes-3.0-Flash Preview" leaderboard commentary, section
// 二.1; fp32 recurrent state per the model card's 架构 table):
//   per (sequence n, value head h), per state row i (d_v index):
//     s_i <- g s_i + beta (v_i - g s_i.k) k      o_i = scale * s_i.q
// which is S <- g S (I - beta k k^T) + beta v k^T, o = scale S q, row by row.
//
// Bound by HBM: each 64 KiB fp32 head state is read once and written once.
// A CTA owns half a head (64 rows, 32 KiB). Eight lanes share one 512-byte
// row (4 float4 each, interleaved so one warp-wide load covers four whole
// rows), so the two dot products are 8-lane shuffle reductions. Every thread
// issues all of its state loads (evict-first) before anything else, so a CTA
// has 32 KiB in flight; four CTAs per SM keep ~128 KiB in flight per SM.
#include "gdn_common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kDecThreads = 256;
constexpr int kRowsPerCta = 64;

__device__ __forceinline__ float dot4(float4 a, float4 b) {
  return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}

template <class Tin, class Tg, class To>
__global__ void __launch_bounds__(kDecThreads, 4)
decode_step_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                   const Tin* __restrict__ v, int64_t qs, int64_t ks,
                   int64_t vs, const Tg* __restrict__ g,
                   const Tg* __restrict__ beta, float* __restrict__ state,
                   int H_k, int H_v, float scale, To* __restrict__ o) {
  const int64_t nh = blockIdx.x >> 1;
  const int half = blockIdx.x & 1;
  const int n = (int)(nh / H_v);
  const int h = (int)(nh % H_v);
  const int kh = h / (H_v / H_k);
  const int tid = threadIdx.x;
  const int row = tid >> 3;         // 0..31
  const int sub = tid & 7;          // float4 slots sub, sub+8, sub+16, sub+24

  float* S = state + (nh * kHeadDim + half * kRowsPerCta) * kHeadDim;
  float4 s[2][4];
#pragma unroll
  for (int p = 0; p < 2; ++p)
#pragma unroll
    for (int m = 0; m < 4; ++m)
      s[p][m] = __ldcs(reinterpret_cast<const float4*>(
          S + (p * 32 + row) * kHeadDim + (sub + 8 * m) * 4));

  __shared__ __align__(16) float k_s[kHeadDim];
  __shared__ __align__(16) float q_s[kHeadDim];
  __shared__ float o_s[kRowsPerCta];
  if (tid < kHeadDim) k_s[tid] = to_f32(k[n * ks + kh * kHeadDim + tid]);
  else q_s[tid - kHeadDim] = to_f32(q[n * qs + kh * kHeadDim + tid - kHeadDim]);
  const float gg = to_f32(g[nh]);
  const float bb = to_f32(beta[nh]);
  const Tin* vrow = v + n * vs + h * kHeadDim + half * kRowsPerCta;
  float vi[2];
#pragma unroll
  for (int p = 0; p < 2; ++p) vi[p] = to_f32(vrow[p * 32 + row]);
  __syncthreads();

  const float4* k4 = reinterpret_cast<const float4*>(k_s);
  const float4* q4 = reinterpret_cast<const float4*>(q_s);
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    float sk = 0.f;
#pragma unroll
    for (int m = 0; m < 4; ++m) sk += dot4(s[p][m], k4[sub + 8 * m]);
    sk += __shfl_xor_sync(0xffffffffu, sk, 1);
    sk += __shfl_xor_sync(0xffffffffu, sk, 2);
    sk += __shfl_xor_sync(0xffffffffu, sk, 4);
    const float c = bb * (vi[p] - gg * sk);
    float so = 0.f;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const float4 kk = k4[sub + 8 * m];
      float4 t = s[p][m];
      t.x = fmaf(gg, t.x, c * kk.x);
      t.y = fmaf(gg, t.y, c * kk.y);
      t.z = fmaf(gg, t.z, c * kk.z);
      t.w = fmaf(gg, t.w, c * kk.w);
      so += dot4(t, q4[sub + 8 * m]);
      __stcs(reinterpret_cast<float4*>(S + (p * 32 + row) * kHeadDim +
                                       (sub + 8 * m) * 4), t);
    }
    so += __shfl_xor_sync(0xffffffffu, so, 1);
    so += __shfl_xor_sync(0xffffffffu, so, 2);
    so += __shfl_xor_sync(0xffffffffu, so, 4);
    if (sub == 0) o_s[p * 32 + row] = scale * so;
  }
  __syncthreads();
  if (tid < kRowsPerCta)
    o[nh * kHeadDim + half * kRowsPerCta + tid] = from_f32<To>(o_s[tid]);
}

template <class Tin, class Tg, class To>
cudaError_t launch_typed(const RecurArgs& a) {
  const int64_t blocks = (int64_t)a.N * a.H_v * 2;
  decode_step_kernel<Tin, Tg, To><<<(unsigned)blocks, kDecThreads, 0, a.stream>>>(
      static_cast<const Tin*>(a.q), static_cast<const Tin*>(a.k),
      static_cast<const Tin*>(a.v), a.q_row_stride, a.k_row_stride,
      a.v_row_stride, static_cast<const Tg*>(a.g),
      static_cast<const Tg*>(a.beta), a.state_out, a.H_k, a.H_v, a.scale,
      static_cast<To*>(a.o));
  return cudaGetLastError();
}

template <class Tin, class Tg>
cudaError_t pick_o(const RecurArgs& a) {
  return a.o_dtype == GDN_F32 ? launch_typed<Tin, Tg, float>(a)
                              : launch_typed<Tin, Tg, __nv_bfloat16>(a);
}
template <class Tin>
cudaError_t pick_g(const RecurArgs& a) {
  return a.gate_dtype == GDN_F32 ? pick_o<Tin, float>(a)
                                 : pick_o<Tin, __nv_bfloat16>(a);
}

}  // namespace

cudaError_t launch_decode_step(const RecurArgs& a) {
  if (a.N == 0) return cudaSuccess;
  return a.qkv_dtype == GDN_F32 ? pick_g<float>(a) : pick_g<__nv_bfloat16>(a);
}

}  // namespace gdn
