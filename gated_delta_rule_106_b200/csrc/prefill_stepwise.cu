// Stepwise gated delta rule over packed sequences on the CUDA cores, fp32.
//
// This serves gdn_stepwise_prefill: the recurrence
//   S_t = g_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T, o_t = scale S_t q_t
// ("Agnes-3.0-Flash Preview" leaderboard commentary, section 二.1: the chunked
// prefill and stepwise decode paths compute the same recurrence; the model
// card's 架构 table fixes the fp32 state) is advanced token by token. A warp
// owns 32 rows of one (sequence, value head) state; each lane keeps its
// 128-float row in registers for the whole sequence, so the state touches HBM
// only at the start and the end. Token t+1's q/k/v/g/beta are fetched while
// token t is being applied.
#include "gdn_common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kRowsPerWarp = 32;

template <class Tin, class Tg, class To>
__global__ void __launch_bounds__(32)
prefill_stepwise_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                        const Tin* __restrict__ v, int64_t qs, int64_t ks,
                        int64_t vs, const Tg* __restrict__ g,
                        const Tg* __restrict__ beta, const float* state_in,
                        float* state_out, const int32_t* __restrict__ cu,
                        int64_t T, int H_k, int H_v, float scale,
                        To* __restrict__ o) {
  const int blocks_per_head = kHeadDim / kRowsPerWarp;
  const int64_t nh = blockIdx.x / blocks_per_head;
  const int rb = blockIdx.x % blocks_per_head;
  const int n = (int)(nh / H_v);
  const int h = (int)(nh % H_v);
  const int kh = h / (H_v / H_k);
  const int lane = threadIdx.x;
  const int i = rb * kRowsPerWarp + lane;           // state row (d_v index)

  float s[kHeadDim];
  if (state_in) {
    const float4* src = reinterpret_cast<const float4*>(
        state_in + (nh * kHeadDim + i) * kHeadDim);
#pragma unroll
    for (int j = 0; j < kHeadDim / 4; ++j) {
      float4 t = src[j];
      s[4 * j] = t.x; s[4 * j + 1] = t.y; s[4 * j + 2] = t.z; s[4 * j + 3] = t.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < kHeadDim; ++j) s[j] = 0.f;
  }

  int64_t t0 = clamp_t(__ldg(cu + n), T);
  int64_t t1 = clamp_t(__ldg(cu + n + 1), T);
  if (t1 < t0) t1 = t0;

  __shared__ __align__(16) float kq[2][2][kHeadDim];   // [buf][k|q][d]
  // prefetch registers: lane holds 4 k and 4 q values, its v_i, g, beta
  float pk[4], pq[4], pv = 0.f, pg = 0.f, pb = 0.f;
  auto fetch = [&](int64_t t) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      pk[e] = to_f32(k[t * ks + kh * kHeadDim + lane * 4 + e]);
      pq[e] = to_f32(q[t * qs + kh * kHeadDim + lane * 4 + e]);
    }
    pv = to_f32(v[t * vs + h * kHeadDim + i]);
    pg = to_f32(g[t * H_v + h]);
    pb = to_f32(beta[t * H_v + h]);
  };
  if (t0 < t1) fetch(t0);
  int buf = 0;
  for (int64_t t = t0; t < t1; ++t) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      kq[buf][0][lane * 4 + e] = pk[e];
      kq[buf][1][lane * 4 + e] = pq[e];
    }
    const float vt = pv, gt = pg, bt = pb;
    __syncwarp();
    if (t + 1 < t1) fetch(t + 1);
    const float4* k4 = reinterpret_cast<const float4*>(kq[buf][0]);
    const float4* q4 = reinterpret_cast<const float4*>(kq[buf][1]);
    float sk0 = 0.f, sk1 = 0.f;
#pragma unroll
    for (int j = 0; j < kHeadDim / 4; ++j) {
      const float4 kk = k4[j];
      sk0 = fmaf(s[4 * j], kk.x, sk0);
      sk1 = fmaf(s[4 * j + 1], kk.y, sk1);
      sk0 = fmaf(s[4 * j + 2], kk.z, sk0);
      sk1 = fmaf(s[4 * j + 3], kk.w, sk1);
    }
    const float c = bt * (vt - gt * (sk0 + sk1));
    float so0 = 0.f, so1 = 0.f;
#pragma unroll
    for (int j = 0; j < kHeadDim / 4; ++j) {
      const float4 kk = k4[j];
      const float4 qq = q4[j];
      s[4 * j] = fmaf(gt, s[4 * j], c * kk.x);
      s[4 * j + 1] = fmaf(gt, s[4 * j + 1], c * kk.y);
      s[4 * j + 2] = fmaf(gt, s[4 * j + 2], c * kk.z);
      s[4 * j + 3] = fmaf(gt, s[4 * j + 3], c * kk.w);
      so0 = fmaf(s[4 * j], qq.x, so0);
      so1 = fmaf(s[4 * j + 1], qq.y, so1);
      so0 = fmaf(s[4 * j + 2], qq.z, so0);
      so1 = fmaf(s[4 * j + 3], qq.w, so1);
    }
    o[(t * H_v + h) * kHeadDim + i] = from_f32<To>(scale * (so0 + so1));
    buf ^= 1;
  }

  if (state_out) {
    float4* dst = reinterpret_cast<float4*>(state_out + (nh * kHeadDim + i) * kHeadDim);
#pragma unroll
    for (int j = 0; j < kHeadDim / 4; ++j)
      dst[j] = make_float4(s[4 * j], s[4 * j + 1], s[4 * j + 2], s[4 * j + 3]);
  }
}

template <class Tin, class Tg, class To>
cudaError_t launch_typed(const RecurArgs& a) {
  const int64_t blocks = (int64_t)a.N * a.H_v * (kHeadDim / kRowsPerWarp);
  prefill_stepwise_kernel<Tin, Tg, To><<<(unsigned)blocks, 32, 0, a.stream>>>(
      static_cast<const Tin*>(a.q), static_cast<const Tin*>(a.k),
      static_cast<const Tin*>(a.v), a.q_row_stride, a.k_row_stride,
      a.v_row_stride, static_cast<const Tg*>(a.g),
      static_cast<const Tg*>(a.beta), a.state_in, a.state_out, a.cu_seqlens,
      a.T_total, a.H_k, a.H_v, a.scale, static_cast<To*>(a.o));
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

cudaError_t launch_prefill_stepwise(const RecurArgs& a) {
  if (a.N == 0) return cudaSuccess;
  return a.qkv_dtype == GDN_F32 ? pick_g<float>(a) : pick_g<__nv_bfloat16>(a);
}

}  // namespace gdn
