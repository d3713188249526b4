// Fused causal depthwise conv (kernel 4) + SiLU + per-head L2 normalisation.
//
// The kernel-4 causal conv sits in front of the delta rule ("Agnes-3.0-Flash
// Preview" leaderboard commentary, section 二.1; model card 架构 table). The
// q and k channels are L2-normalised per 128-channel head before they enter
// the recurrence.
//
// HBM-bound: each token row is read once (plus a 3-row halo per tile, served
// from L2) and written once. A thread owns 8 consecutive channels (one 16-byte
// bf16 vector) for a run of kRowsPerTile tokens and keeps the last three
// pre-conv rows in registers as a sliding window; 16 threads cover one
// 128-channel head, so the L2 norm is a 16-lane shuffle reduction. A warp
// reads/writes 512 contiguous bytes of a row per access.
#include "gdn_common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kConvThreads = 128;
constexpr int kRowsPerTile = 16;

template <class Tw>
__device__ __forceinline__ void load_taps(const Tw* w, int c, float (&wt)[4][8]) {
  // w is [C, 4]: the 8 channels' taps are 32 consecutive values.
  float f[8];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    load8(w + (int64_t)c * 4 + q * 8, f);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      int flat = q * 8 + e;          // = (channel - c) * 4 + tap
      wt[flat & 3][flat >> 2] = f[e];
    }
  }
}

template <class Tx>
__device__ __forceinline__ void load_hist(const Tx* cs_in, int n, int C, int r,
                                          int c, float (&h)[8]) {
  if (cs_in) {
    load8(cs_in + ((int64_t)n * 3 + r) * C + c, h);
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) h[e] = 0.f;
  }
}

template <class Tx, class Tw, class Ty>
__global__ void __launch_bounds__(kConvThreads)
conv_silu_kernel(const Tx* __restrict__ x, int64_t xs, const Tw* __restrict__ w,
                 const Tw* __restrict__ bias, int C, int l2c, float eps,
                 const int32_t* __restrict__ cu, int N, int64_t T,
                 const Tx* __restrict__ cs_in, Ty* __restrict__ y, int64_t ys) {
  const int c = (blockIdx.x * kConvThreads + threadIdx.x) * 8;
  const bool active = c < C;
  const int64_t t0 = (int64_t)blockIdx.y * kRowsPerTile;
  const int64_t t1 = t0 + kRowsPerTile < T ? t0 + kRowsPerTile : T;

  float wt[4][8], b[8], h[3][8];   // h[j] = pre-conv row t-3+j
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    b[e] = 0.f;
#pragma unroll
    for (int j = 0; j < 3; ++j) h[j][e] = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) wt[j][e] = 0.f;
  }
  if (active) {
    load_taps(w, c, wt);
    if (bias) load8(bias + c, b);
  }

  int n = seq_of(cu, N, t0);
  int64_t s_start = clamp_t(__ldg(cu + n), T);
  int64_t s_end = clamp_t(__ldg(cu + n + 1), T);
  if (active) {
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const int64_t p = t0 - 3 + j;
      if (p >= s_start) load8(x + p * xs + c, h[j]);
      else load_hist(cs_in, n, C, (int)(3 + (p - s_start)), c, h[j]);
    }
  }

  for (int64_t t = t0; t < t1; ++t) {
    if (t >= s_end) {
      // enter the sequence that starts at t (skipping empty ones)
      while (n < N - 1 && t >= s_end) {
        ++n;
        s_start = clamp_t(__ldg(cu + n), T);
        s_end = clamp_t(__ldg(cu + n + 1), T);
      }
      if (active) {
#pragma unroll
        for (int j = 0; j < 3; ++j) load_hist(cs_in, n, C, j, c, h[j]);
      }
    }
    float cur[8], out[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) cur[e] = 0.f;
    if (active) load8(x + t * xs + c, cur);
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float a = b[e];
      a = fmaf(wt[0][e], h[0][e], a);
      a = fmaf(wt[1][e], h[1][e], a);
      a = fmaf(wt[2][e], h[2][e], a);
      a = fmaf(wt[3][e], cur[e], a);
      out[e] = silu(a);
      ss = fmaf(out[e], out[e], ss);
    }
    // 16 lanes = one 128-channel head
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if (c < l2c) {
      const float inv = 1.0f / sqrtf(ss + eps);
#pragma unroll
      for (int e = 0; e < 8; ++e) out[e] *= inv;
    }
    if (active) store8(y + t * ys + c, out);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      h[0][e] = h[1][e];
      h[1][e] = h[2][e];
      h[2][e] = cur[e];
    }
  }
}

// conv_state_out[n, r] = pre-conv row len_n - 3 + r of sequence n, shifted in
// from conv_state_in when the sequence is shorter than 3. One thread per
// (sequence, 16-byte column chunk) reads its three rows before writing any,
// so conv_state_out may alias conv_state_in.
__global__ void conv_state_kernel(const char* __restrict__ x, int64_t xs_bytes,
                                  int row_bytes, const int32_t* __restrict__ cu,
                                  int N, int64_t T, const char* cs_in,
                                  char* cs_out) {
  const int chunks = row_bytes / 16;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)N * chunks) return;
  const int n = (int)(idx / chunks);
  const int off = (int)(idx % chunks) * 16;
  const int64_t s = clamp_t(__ldg(cu + n), T);
  int64_t e = clamp_t(__ldg(cu + n + 1), T);
  if (e < s) e = s;
  const int64_t len = e - s;
  uint4 v[3];
#pragma unroll
  for (int r = 0; r < 3; ++r) {
    int64_t p = len - 3 + r;
    if (p >= 0) {
      v[r] = *reinterpret_cast<const uint4*>(x + (s + p) * xs_bytes + off);
    } else if (cs_in) {
      v[r] = *reinterpret_cast<const uint4*>(
          cs_in + ((int64_t)n * 3 + (3 + p)) * row_bytes + off);
    } else {
      v[r] = make_uint4(0, 0, 0, 0);
    }
  }
#pragma unroll
  for (int r = 0; r < 3; ++r)
    *reinterpret_cast<uint4*>(cs_out + ((int64_t)n * 3 + r) * row_bytes + off) = v[r];
}

template <class Tx, class Tw, class Ty>
cudaError_t launch_typed(const ConvArgs& a) {
  if (a.T_total > 0) {
    dim3 grid((unsigned)((a.channels / 8 + kConvThreads - 1) / kConvThreads),
              (unsigned)((a.T_total + kRowsPerTile - 1) / kRowsPerTile));
    conv_silu_kernel<Tx, Tw, Ty><<<grid, kConvThreads, 0, a.stream>>>(
        static_cast<const Tx*>(a.x), a.x_row_stride,
        static_cast<const Tw*>(a.w), static_cast<const Tw*>(a.bias), a.channels,
        a.l2norm_channels, a.l2_eps, a.cu_seqlens, a.N, a.T_total,
        static_cast<const Tx*>(a.conv_state_in), static_cast<Ty*>(a.y),
        a.y_row_stride);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (a.conv_state_out) {
    const int eb = sizeof(Tx);
    const int row_bytes = a.channels * eb;
    const int64_t threads = (int64_t)a.N * (row_bytes / 16);
    if (threads > 0) {
      conv_state_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, a.stream>>>(
          static_cast<const char*>(a.x), a.x_row_stride * eb, row_bytes,
          a.cu_seqlens, a.N, a.T_total,
          static_cast<const char*>(a.conv_state_in),
          static_cast<char*>(a.conv_state_out));
      return cudaGetLastError();
    }
  }
  return cudaSuccess;
}

template <class Tx, class Tw>
cudaError_t launch_y(const ConvArgs& a) {
  return a.y_dtype == GDN_F32 ? launch_typed<Tx, Tw, float>(a)
                              : launch_typed<Tx, Tw, __nv_bfloat16>(a);
}

template <class Tx>
cudaError_t launch_w(const ConvArgs& a) {
  return a.w_dtype == GDN_F32 ? launch_y<Tx, float>(a)
                              : launch_y<Tx, __nv_bfloat16>(a);
}

}  // namespace

cudaError_t launch_conv1d_silu(const ConvArgs& a) {
  return a.x_dtype == GDN_F32 ? launch_w<float>(a) : launch_w<__nv_bfloat16>(a);
}

}  // namespace gdn
