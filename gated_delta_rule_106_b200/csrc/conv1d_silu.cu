// Fused causal depthwise conv (kernel 4) + SiLU + per-head L2 normalisation.
//
// The kernel-4 causal conv sits in front of the delta rule ("Agnes-3.0-Flash
// Preview" leaderboard commentary, section 二.1; model card 架构 table). The
// q and k channels are L2-normalised per 128-channel head before they enter
// the recurrence.
//
// HBM-bound: each token row is read from HBM once and written once. A thread
// owns 4 consecutive channels (one 8-byte bf16 vector) of a tile of tokens and
// issues every load its outputs need before it computes, so that many loads
// are in flight; 4 channels (not 8) keep the register count low enough for
// 7 CTAs per SM. A tile whose tokens and their three predecessors all lie in
// one sequence (the common case in prefill) loads that window of rows once; a
// tile that meets a sequence start takes each token's predecessors from x inside
// its sequence and from the conv cache (or zeros) before its start. All threads
// of a block work on the same tokens, so the sequence bookkeeping is uniform; a
// warp covers one 128-channel head, so the L2 norm is a warp shuffle reduction.
#include "gdn_common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kConvThreads = 128;
constexpr int kV = 4;                    // channels per thread
constexpr int kHeadLanes = kHeadDim / kV; // lanes per 128-channel head
// tokens per tile (window path), and per batch of the per-token-source path;
// either way the loaded vectors of a thread stay in registers. Calls whose
// sequences average at most kShortLen tokens (decode) use tiles of 2 tokens:
// more CTAs, one short batch each.
template <class Tx> __host__ __device__ constexpr int conv_tile() { return sizeof(Tx) == 2 ? 8 : 4; }
template <class Tx> __host__ __device__ constexpr int conv_batch() { return sizeof(Tx) == 2 ? 4 : 2; }
constexpr int kShortLen = 4;

// kV consecutive elements kept as loaded
template <class Tx> struct RawV {
  static constexpr int kBytes = kV * (int)sizeof(Tx);
  static constexpr int kWords = kBytes / 4;
  uint32_t u[kWords];
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int i = 0; i < kWords; ++i) u[i] = 0u;
  }
  __device__ __forceinline__ void load(const Tx* p) {
    if constexpr (kBytes == 8) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
      u[0] = v.x; u[1] = v.y;
    } else {
#pragma unroll
      for (int i = 0; i < kBytes / 16; ++i) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(p) + i);
        u[4 * i] = v.x; u[4 * i + 1] = v.y; u[4 * i + 2] = v.z; u[4 * i + 3] = v.w;
      }
    }
  }
  __device__ __forceinline__ void store(Tx* p) const {
    if constexpr (kBytes == 8) {
      *reinterpret_cast<uint2*>(p) = make_uint2(u[0], u[1]);
    } else {
#pragma unroll
      for (int i = 0; i < kBytes / 16; ++i)
        reinterpret_cast<uint4*>(p)[i] = make_uint4(u[4 * i], u[4 * i + 1], u[4 * i + 2], u[4 * i + 3]);
    }
  }
  __device__ __forceinline__ void to_f32(float (&f)[kV]) const {
    if constexpr (sizeof(Tx) == 2) {
#pragma unroll
      for (int i = 0; i < kWords; ++i) {
        const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[i]));
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
      }
    } else {
#pragma unroll
      for (int i = 0; i < kV; ++i) f[i] = __uint_as_float(u[i]);
    }
  }
};
template <class T>
__device__ __forceinline__ void loadV(const T* p, float (&f)[kV]) {
  RawV<T> r;
  r.load(p);
  r.to_f32(f);
}
template <class Ty>
__device__ __forceinline__ void storeV(Ty* p, const float (&f)[kV]) {
  if constexpr (sizeof(Ty) == 2) {
    uint32_t u[kV / 2];
#pragma unroll
    for (int i = 0; i < kV / 2; ++i) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
      u[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    if constexpr (kV == 4) *reinterpret_cast<uint2*>(p) = make_uint2(u[0], u[1]);
    else *reinterpret_cast<uint4*>(p) = make_uint4(u[0], u[1], u[2], u[3]);
  } else {
#pragma unroll
    for (int i = 0; i < kV / 4; ++i)
      reinterpret_cast<float4*>(p)[i] = make_float4(f[4 * i], f[4 * i + 1], f[4 * i + 2], f[4 * i + 3]);
  }
}

template <class Tw>
__device__ __forceinline__ void load_taps_bias(const Tw* w, const Tw* bias, int c, bool active,
                                               float (&wt)[4][kV], float (&b)[kV]) {
#pragma unroll
  for (int e = 0; e < kV; ++e) {
    b[e] = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) wt[j][e] = 0.f;
  }
  if (active) {
    // w is [C, 4]: the kV channels' taps are 4 kV consecutive values
    float f[kV];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      loadV(w + (int64_t)c * 4 + q * kV, f);
#pragma unroll
      for (int e = 0; e < kV; ++e) {
        const int flat = q * kV + e;          // = (channel - c) * 4 + tap
        wt[flat & 3][flat >> 2] = f[e];
      }
    }
    if (bias) loadV(bias + c, b);
  }
}

// one output token from its four pre-conv inputs (oldest first, as floats):
// taps, SiLU, and the per-head L2 norm for the leading l2c channels
template <class Ty>
__device__ __forceinline__ void conv_token(const float (&f0)[kV], const float (&f1)[kV],
                                           const float (&f2)[kV], const float (&f3)[kV],
                                           const float (&wt)[4][kV], const float (&b)[kV],
                                           int c, int l2c, bool any_l2, float eps, bool store,
                                           Ty* dst) {
  float out[kV], ss = 0.f;
#pragma unroll
  for (int e = 0; e < kV; ++e) {
    const float a = fmaf(wt[3][e], f3[e], fmaf(wt[2][e], f2[e], fmaf(wt[1][e], f1[e], fmaf(wt[0][e], f0[e], b[e]))));
    out[e] = silu(a);
    ss = fmaf(out[e], out[e], ss);
  }
  if (any_l2) {   // block-uniform: some channel of the block is L2-normalised
#pragma unroll
    for (int off = kHeadLanes / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  }
  if (c < l2c) {
    const float inv = rsqrtf(ss + eps);
#pragma unroll
    for (int e = 0; e < kV; ++e) out[e] *= inv;
  }
  if (store) storeV(dst, out);
}

template <class Tx, class Tw, class Ty, int R, int RB>
__global__ void __launch_bounds__(kConvThreads)
conv_silu_kernel(const Tx* __restrict__ x, int64_t xs, const Tw* __restrict__ w,
                 const Tw* __restrict__ bias, int C, int l2c, float eps,
                 const int32_t* __restrict__ cu, int N, int64_t T,
                 const Tx* __restrict__ cs_in, int64_t css, Tx* cs_out, Ty* __restrict__ y,
                 int64_t ys) {
  const int c = (blockIdx.x * kConvThreads + threadIdx.x) * kV;
  const bool active = c < C;
  const bool any_l2 = (int)blockIdx.x * kConvThreads * kV < l2c;
  const int64_t t0 = (int64_t)blockIdx.y * R;

  // short-sequence tiles guess the sequence from equal lengths (one round of loads
  // for one token per sequence); long ones search
  int n = R == 2 ? seq_locate(cu, N, T, t0) : seq_of(cu, N, t0);
  int64_t s_start = clamp_t(__ldg(cu + n), T);
  int64_t s_end = clamp_t(__ldg(cu + n + 1), T);

  float wt[4][kV], b[kV];
  if (t0 - 3 >= s_start && t0 + R <= s_end) {
    // window path: rows t0-3 .. t0+R-1, each loaded once
    RawV<Tx> win[R + 3];
#pragma unroll
    for (int j = 0; j < R + 3; ++j) {
      win[j].zero();
      if (active) win[j].load(x + (t0 - 3 + j) * xs + c);
    }
    load_taps_bias(w, bias, c, active, wt, b);
    // each row converted once; the last three stay as floats
    float h0[kV], h1[kV], h2[kV], h3[kV];
    win[0].to_f32(h0);
    win[1].to_f32(h1);
    win[2].to_f32(h2);
    Ty* dst = y + t0 * ys + c;
#pragma unroll
    for (int i = 0; i < R; ++i, dst += ys) {
      win[i + 3].to_f32(h3);
      conv_token<Ty>(h0, h1, h2, h3, wt, b, c, l2c, any_l2, eps, active, dst);
#pragma unroll
      for (int e = 0; e < kV; ++e) {
        h0[e] = h1[e];
        h1[e] = h2[e];
        h2[e] = h3[e];
      }
    }
    return;
  }

  load_taps_bias(w, bias, c, active, wt, b);
  // per-token sources, RB tokens at a time: src[i][k] = pre-conv input of token
  // t at lag 3-k (k = 3: the token itself)
#pragma unroll 1
  for (int i0 = 0; i0 < R; i0 += RB) {
    RawV<Tx> src[RB][4];
    int nn[RB];
    int64_t s_lo[RB], s_hi[RB];
#pragma unroll
    for (int i = 0; i < RB; ++i) {
      const int64_t t = t0 + i0 + i;
      while (n < N - 1 && t >= s_end) {   // enter the sequence holding t (skip empty ones)
        ++n;
        s_start = clamp_t(__ldg(cu + n), T);
        s_end = clamp_t(__ldg(cu + n + 1), T);
      }
      // a token past the last sequence is treated as the start of one
      const int64_t st = t >= s_end ? t : s_start;
      nn[i] = n;
      s_lo[i] = s_start;
      s_hi[i] = s_end;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int64_t pr = t - 3 + k;
        src[i][k].zero();
        if (active && t < T) {
          if (pr >= st) src[i][k].load(x + pr * xs + c);
          else if (cs_in) src[i][k].load(cs_in + ((int64_t)n * 3 + (3 + (pr - st))) * css + c);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < RB; ++i) {
      const int64_t t = t0 + i0 + i;
      float f0[kV], f1[kV], f2[kV], f3[kV];
      src[i][0].to_f32(f0);
      src[i][1].to_f32(f1);
      src[i][2].to_f32(f2);
      src[i][3].to_f32(f3);
      conv_token<Ty>(f0, f1, f2, f3, wt, b, c, l2c, any_l2, eps, active && t < T, y + t * ys + c);
      // a sequence that lies whole in this batch (this thread alone read its cache
      // rows) gets its new cache here: its last three pre-conv rows, oldest first
      if constexpr (R == 2) {   // only the short-sequence tiles are given cs_out
        if (cs_out && active && t < T && t == s_hi[i] - 1 && s_lo[i] >= t0 + i0) {
#pragma unroll
          for (int r = 0; r < 3; ++r) src[i][r + 1].store(cs_out + ((int64_t)nn[i] * 3 + r) * css + c);
        }
      }
    }
  }
}

// conv_state_out[n, r] = pre-conv row len_n - 3 + r of sequence n, shifted in
// from conv_state_in when the sequence is shorter than 3. One thread per
// (sequence, 16-byte column chunk) reads its three rows before writing any,
// so conv_state_out may alias conv_state_in.
// Sequences that lie whole in one fused_rb-token batch of the conv kernel had
// their cache written there (fused_rb = 0: none did).
__global__ void conv_state_kernel(const char* __restrict__ x, int64_t xs_bytes,
                                  int row_bytes, const int32_t* __restrict__ cu,
                                  int N, int64_t T, const char* cs_in,
                                  char* cs_out, int fused_rb) {
  const int chunks = row_bytes / 16;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)N * chunks) return;
  const int n = (int)(idx / chunks);
  const int off = (int)(idx % chunks) * 16;
  const int64_t s = clamp_t(__ldg(cu + n), T);
  int64_t e = clamp_t(__ldg(cu + n + 1), T);
  if (e < s) e = s;
  if (fused_rb > 0 && e > s && s / fused_rb == (e - 1) / fused_rb) return;
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
  int fused_rb = 0;
  if (a.T_total > 0) {
    const bool short_seqs = (int64_t)a.N * kShortLen >= a.T_total;
    const int R = short_seqs ? 2 : conv_tile<Tx>();
    dim3 grid((unsigned)((a.channels / kV + kConvThreads - 1) / kConvThreads),
              (unsigned)((a.T_total + R - 1) / R));
    auto kern = short_seqs ? conv_silu_kernel<Tx, Tw, Ty, 2, 2>
                           : conv_silu_kernel<Tx, Tw, Ty, conv_tile<Tx>(), conv_batch<Tx>()>;
    // the short-sequence tiles write the new cache of the sequences they hold whole
    fused_rb = short_seqs && a.conv_state_out ? 2 : 0;
    kern<<<grid, kConvThreads, 0, a.stream>>>(
        static_cast<const Tx*>(a.x), a.x_row_stride,
        static_cast<const Tw*>(a.w), static_cast<const Tw*>(a.bias), a.channels,
        a.l2norm_channels, a.l2_eps, a.cu_seqlens, a.N, a.T_total,
        static_cast<const Tx*>(a.conv_state_in),
        a.cs_row_stride ? a.cs_row_stride : (int64_t)a.channels,
        fused_rb ? static_cast<Tx*>(a.conv_state_out) : nullptr, static_cast<Ty*>(a.y),
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
          static_cast<char*>(a.conv_state_out), fused_rb);
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

cudaError_t launch_conv_state_roll(const void* x, int64_t x_row_stride, gdn_dtype x_dtype,
                                   int channels, const int32_t* cu, int N, int64_t T,
                                   const void* cs_in, void* cs_out, cudaStream_t stream) {
  const int eb = elem_bytes(x_dtype);
  const int row_bytes = channels * eb;
  const int64_t threads = (int64_t)N * (row_bytes / 16);
  if (threads == 0) return cudaSuccess;
  conv_state_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, stream>>>(
      static_cast<const char*>(x), x_row_stride * eb, row_bytes, cu, N, T,
      static_cast<const char*>(cs_in), static_cast<char*>(cs_out), 0);
  return cudaGetLastError();
}

cudaError_t launch_conv1d_silu(const ConvArgs& a) {
  return a.x_dtype == GDN_F32 ? launch_w<float>(a) : launch_w<__nv_bfloat16>(a);
}

}  // namespace gdn
