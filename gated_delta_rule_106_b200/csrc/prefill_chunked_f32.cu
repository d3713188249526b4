// Chunked (C = 64) gated delta rule for fp32 inputs, on the CUDA cores in fp32.
//
// The chunked prefill path ("delta_rule_chunked", chunk = 64: "Agnes-3.0-
// Flash Preview" leaderboard commentary, section 二.1; fp32 recurrent state:
// model card, 架构 table) for inputs given in fp32, where the tolerance (1e-4
// of the output rms and of the state norm) leaves no room for 16-bit tensor-
// core operands. Per 64-token chunk of L tokens, with G_t = sum_{s<=t} log g_s
// and S0 the state entering the chunk:
//   A_ts = beta_t e^{G_t-G_s} k_t.k_s (s < t);   T = (I + A)^{-1}
//   W = T diag(beta e^G) K;   U = T diag(beta) V;   M_ts = e^{G_t-G_s} q_t.k_s (s <= t)
//   Delta = U - W S0^T;   O = scale (diag(e^G) Q S0^T + M Delta)
//   S_L = e^{G_L} S0 + Delta^T diag(e^{G_L-G}) K
// which is the stepwise recurrence S_t = g_t S_{t-1}(I - beta_t k_t k_t^T) +
// beta_t v_t k_t^T, o_t = scale S_t q_t, regrouped by chunk (the WY / UT form).
//
// One CTA per (sequence, value head), 512 threads. The fp32 state stays in
// registers for the whole sequence: thread (row i = tid / 4, quarter c = tid % 4)
// holds S[i][4(c + 4m) .. 4(c + 4m) + 3] for m = 0..7, so row dot products are
// float4 reads of a shared row (broadcast to the eight rows of a warp) and a
// four-lane shuffle sum. The chunk's K, Q, V, W, A, T, M live in shared memory.
// The decay exponents are differences of prefix sums kept in fp64, so long
// chunks with strong decay lose no digits to cancellation.
#include "gdn_common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kF32Threads = 512;
constexpr int kLdk = 132;     // row stride (floats) of the [64][128] tiles
constexpr int kLdt = 65;      // row stride (floats) of the [64][64] tiles

struct F32Smem {
  float K[kChunk * kLdk];
  float Q[kChunk * kLdk];
  float V[kChunk * kLdk];     // V, then U = T diag(beta) V, then Delta [t][i]
  float W[kChunk * kLdk];     // W = T diag(beta e^G) K, then the staged outputs
  float A[kChunk * kLdt];
  float T[kChunk * kLdt];
  float M[kChunk * kLdt];
  float X[kChunk * kLdt];     // merge scratch of the blocked inverse
  double G[kChunk];
  float beta[kChunk], gam[kChunk], tail[kChunk];
  float gL;
};

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float dot4(float4 a, float4 b) {
  return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}

// 4 consecutive elements as floats (bf16: 8 bytes, fp32: 16 bytes)
__device__ __forceinline__ float4 load4(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}

// One merge level of the blocked inverse of the 64x64 unit lower-triangular
// I + A (diagonal b x b blocks already inverted in T): for each pair of blocks,
// X = A21 T11, then T21 = -T22 X.
template <int b>
__device__ __forceinline__ void merge_level(F32Smem& sh, int tid) {
  constexpr int pairs = kChunk / (2 * b), outs = pairs * b * b;
  for (int idx = tid; idx < outs; idx += kF32Threads) {
    const int p = idx / (b * b), r = (idx / b) % b, c = idx % b, o = 2 * b * p;
    float acc = 0.f;
    for (int m = c; m < b; ++m) acc = fmaf(sh.A[(o + b + r) * kLdt + o + m], sh.T[(o + m) * kLdt + o + c], acc);
    sh.X[(o + b + r) * kLdt + o + c] = acc;
  }
  __syncthreads();
  for (int idx = tid; idx < outs; idx += kF32Threads) {
    const int p = idx / (b * b), r = (idx / b) % b, c = idx % b, o = 2 * b * p;
    float acc = 0.f;
    for (int m = 0; m <= r; ++m) acc = fmaf(sh.T[(o + b + r) * kLdt + o + b + m], sh.X[(o + b + m) * kLdt + o + c], acc);
    sh.T[(o + b + r) * kLdt + o + c] = -acc;
  }
  __syncthreads();
}

template <class Tin, class Tg, class To>
__global__ void __launch_bounds__(kF32Threads, 1)
chunked_f32_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                   int64_t qs, int64_t ks, int64_t vs, const Tg* __restrict__ g,
                   const Tg* __restrict__ beta, const float* state_in, float* state_out,
                   const int32_t* __restrict__ cu, int64_t T, int H_k, int H_v, float scale,
                   To* __restrict__ o) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  F32Smem& sh = *reinterpret_cast<F32Smem*>(smem_raw);
  const int64_t nh = blockIdx.x;
  const int n = (int)(nh / H_v), h = (int)(nh % H_v), kh = h / (H_v / H_k);
  const int tid = threadIdx.x, lane = tid & 31;
  const int i = tid >> 2, cq = tid & 3;   // state row, column quarter

  float S[32];
  if (state_in) {
    const float* src = state_in + (nh * kHeadDim + i) * kHeadDim;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const float4 t = ld4(src + 4 * (cq + 4 * m));
      S[4 * m] = t.x; S[4 * m + 1] = t.y; S[4 * m + 2] = t.z; S[4 * m + 3] = t.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) S[j] = 0.f;
  }

  const int64_t s0 = clamp_t(__ldg(cu + n), T);
  int64_t s1 = clamp_t(__ldg(cu + n + 1), T);
  if (s1 < s0) s1 = s0;
  const int nch = (int)((s1 - s0 + kChunk - 1) / kChunk);

  for (int c = 0; c < nch; ++c) {
    const int64_t t0 = s0 + (int64_t)c * kChunk;
    const int L = (int)((s1 - t0) < kChunk ? (s1 - t0) : kChunk);

    // ---- tiles: K, Q (key head kh), V (value head h); rows past L are zero ----
    for (int idx = tid; idx < kChunk * 32; idx += kF32Threads) {
      const int r = idx >> 5, c4 = idx & 31;
      float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), qv = kv, vv = kv;
      if (r < L) {
        const int64_t t = t0 + r;
        kv = load4(k + t * ks + kh * kHeadDim + 4 * c4);
        qv = load4(q + t * qs + kh * kHeadDim + 4 * c4);
        vv = load4(v + t * vs + h * kHeadDim + 4 * c4);
      }
      *reinterpret_cast<float4*>(sh.K + r * kLdk + 4 * c4) = kv;
      *reinterpret_cast<float4*>(sh.Q + r * kLdk + 4 * c4) = qv;
      *reinterpret_cast<float4*>(sh.V + r * kLdk + 4 * c4) = vv;
    }
    // ---- gates: G_t (fp64 prefix sum of log g), beta, e^G, e^{G_L - G} ----
    if (tid < 32) {
      double lg[2];
      float be[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int t = 2 * lane + j;
        lg[j] = 0.0;
        be[j] = 0.f;
        if (t < L) {
          const int64_t idx = (t0 + t) * H_v + h;
          lg[j] = log((double)fmaxf(to_f32(g[idx]), 1.17549435e-38f));
          be[j] = to_f32(beta[idx]);
        }
      }
      double incl = lg[0] + lg[1];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      const double excl = incl - (lg[0] + lg[1]);
      const double GL = __shfl_sync(0xffffffffu, incl, 31);
      const double Gt[2] = {excl + lg[0], excl + lg[0] + lg[1]};
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int t = 2 * lane + j;
        sh.G[t] = Gt[j];
        sh.beta[t] = be[j];
        sh.gam[t] = expf((float)Gt[j]);
        sh.tail[t] = expf((float)(GL - Gt[j]));
      }
      if (lane == 0) sh.gL = expf((float)GL);
    }
    __syncthreads();

    // ---- A (strictly lower) and M (lower, diagonal included): a thread makes a
    //      4 x 4 block of one of them, rows t = tg + 16a, columns s = sg + 16b ----
    {
      const int which = tid >> 8, tg = (tid >> 4) & 15, sg = tid & 15;
      const float* X = which ? sh.Q : sh.K;
      float acc[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b2 = 0; b2 < 4; ++b2) acc[a][b2] = 0.f;
#pragma unroll 4
      for (int d4 = 0; d4 < 32; ++d4) {
        float4 xa[4], kb[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) xa[a] = ld4(X + (tg + 16 * a) * kLdk + 4 * d4);
#pragma unroll
        for (int b2 = 0; b2 < 4; ++b2) kb[b2] = ld4(sh.K + (sg + 16 * b2) * kLdk + 4 * d4);
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b2 = 0; b2 < 4; ++b2) acc[a][b2] += dot4(xa[a], kb[b2]);
      }
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const int t = tg + 16 * a;
        const double Gt = sh.G[t];
        const float bt = sh.beta[t];
#pragma unroll
        for (int b2 = 0; b2 < 4; ++b2) {
          const int s = sg + 16 * b2;
          const float dec = expf((float)(Gt - sh.G[s]));
          if (which == 0) sh.A[t * kLdt + s] = s < t ? bt * dec * acc[a][b2] : 0.f;
          else sh.M[t * kLdt + s] = s <= t ? dec * acc[a][b2] : 0.f;
        }
      }
    }
    // T starts as zeros (its upper triangle stays zero)
    for (int idx = tid; idx < kChunk * kLdt; idx += kF32Threads) sh.T[idx] = 0.f;
    __syncthreads();

    // ---- T = (I + A)^{-1}: 16 x 16 diagonal blocks by forward substitution
    //      (one column per thread), then merges 16 -> 32 -> 64 ----
    if (tid < 64) {
      const int B = tid >> 4, j = tid & 15, o0 = 16 * B;
      float x[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float acc = (r == j) ? 1.f : 0.f;
#pragma unroll
        for (int m = 0; m < r; ++m) acc = fmaf(-sh.A[(o0 + r) * kLdt + o0 + m], x[m], acc);
        x[r] = acc;
      }
#pragma unroll
      for (int r = 0; r < 16; ++r) sh.T[(o0 + r) * kLdt + o0 + j] = x[r];
    }
    __syncthreads();
    merge_level<16>(sh, tid);
    merge_level<32>(sh, tid);

    // ---- W = T diag(beta e^G) K and U = T diag(beta) V: rows t = tw + 16a,
    //      the float4 column chunk d4 ----
    {
      const int tw = tid >> 5, d4 = tid & 31;
      float4 wa[4], ua[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) wa[a] = ua[a] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
      for (int s = 0; s < kChunk; ++s) {
        const float4 kv = ld4(sh.K + s * kLdk + 4 * d4);
        const float4 vv = ld4(sh.V + s * kLdk + 4 * d4);
        const float bs = sh.beta[s], bgs = bs * sh.gam[s];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          const float tv = sh.T[(tw + 16 * a) * kLdt + s];
          const float cw = tv * bgs, cu2 = tv * bs;
          wa[a].x = fmaf(cw, kv.x, wa[a].x); wa[a].y = fmaf(cw, kv.y, wa[a].y);
          wa[a].z = fmaf(cw, kv.z, wa[a].z); wa[a].w = fmaf(cw, kv.w, wa[a].w);
          ua[a].x = fmaf(cu2, vv.x, ua[a].x); ua[a].y = fmaf(cu2, vv.y, ua[a].y);
          ua[a].z = fmaf(cu2, vv.z, ua[a].z); ua[a].w = fmaf(cu2, vv.w, ua[a].w);
        }
      }
      __syncthreads();   // every read of V is done: U goes over it
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        *reinterpret_cast<float4*>(sh.W + (tw + 16 * a) * kLdk + 4 * d4) = wa[a];
        *reinterpret_cast<float4*>(sh.V + (tw + 16 * a) * kLdk + 4 * d4) = ua[a];
      }
    }
    __syncthreads();

    // ---- Delta_ti = U_ti - W_t . S_i (row i, four lanes); lane cq keeps
    //      t = 4u + cq (loops unrolled so that dk stays in registers) ----
    float dk[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
#pragma unroll
      for (int tt = 0; tt < 4; ++tt) {
        const int t = 4 * u + tt;
        float p = 0.f;
#pragma unroll
        for (int m = 0; m < 8; ++m)
          p += dot4(ld4(sh.W + t * kLdk + 4 * (cq + 4 * m)),
                    make_float4(S[4 * m], S[4 * m + 1], S[4 * m + 2], S[4 * m + 3]));
        p += __shfl_xor_sync(0xffffffffu, p, 1);
        p += __shfl_xor_sync(0xffffffffu, p, 2);
        const float d = sh.V[t * kLdk + i] - p;
        if (tt == cq) dk[u] = d;
      }
    }
    __syncthreads();   // every read of U and W is done
#pragma unroll
    for (int u = 0; u < 16; ++u) sh.V[(4 * u + cq) * kLdk + i] = dk[u];
    __syncthreads();

    // ---- O_ti = scale (e^{G_t} q_t . S_i + sum_{s<=t} M_ts Delta_si), staged over W ----
    {
      float ok[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
#pragma unroll
        for (int tt = 0; tt < 4; ++tt) {
          const int t = 4 * u + tt;
          float p = 0.f;
#pragma unroll
          for (int m = 0; m < 8; ++m)
            p += dot4(ld4(sh.Q + t * kLdk + 4 * (cq + 4 * m)),
                      make_float4(S[4 * m], S[4 * m + 1], S[4 * m + 2], S[4 * m + 3]));
          p += __shfl_xor_sync(0xffffffffu, p, 1);
          p += __shfl_xor_sync(0xffffffffu, p, 2);
          if (tt == cq) ok[u] = sh.gam[t] * p;
        }
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int t = 4 * u + cq;
        float acc = ok[u];
        for (int s = 0; s <= t; ++s) acc = fmaf(sh.M[t * kLdt + s], sh.V[s * kLdk + i], acc);
        sh.W[t * kLdk + i] = scale * acc;
      }
    }
    // ---- S <- e^{G_L} S + Delta^T diag(e^{G_L - G}) K ----
    {
      const float gL = sh.gL;
#pragma unroll
      for (int j = 0; j < 32; ++j) S[j] *= gL;
#pragma unroll 4
      for (int t = 0; t < kChunk; ++t) {
        const float dd = sh.V[t * kLdk + i] * sh.tail[t];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const float4 kv = ld4(sh.K + t * kLdk + 4 * (cq + 4 * m));
          S[4 * m] = fmaf(dd, kv.x, S[4 * m]);
          S[4 * m + 1] = fmaf(dd, kv.y, S[4 * m + 1]);
          S[4 * m + 2] = fmaf(dd, kv.z, S[4 * m + 2]);
          S[4 * m + 3] = fmaf(dd, kv.w, S[4 * m + 3]);
        }
      }
    }
    __syncthreads();   // the staged outputs are complete
    for (int idx = tid; idx < L * 32; idx += kF32Threads) {
      const int r = idx >> 5, c4 = idx & 31;
      const float4 val = ld4(sh.W + r * kLdk + 4 * c4);
      To* dst = o + ((t0 + r) * H_v + h) * kHeadDim + 4 * c4;
      if constexpr (sizeof(To) == 4) {
        *reinterpret_cast<float4*>(dst) = val;
      } else {
        const __nv_bfloat162 lo = __floats2bfloat162_rn(val.x, val.y);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(val.z, val.w);
        *reinterpret_cast<uint2*>(dst) = make_uint2(*reinterpret_cast<const uint32_t*>(&lo),
                                                    *reinterpret_cast<const uint32_t*>(&hi));
      }
    }
    __syncthreads();   // the next chunk overwrites every tile
  }

  if (state_out) {
    float* dst = state_out + (nh * kHeadDim + i) * kHeadDim;
#pragma unroll
    for (int m = 0; m < 8; ++m)
      *reinterpret_cast<float4*>(dst + 4 * (cq + 4 * m)) =
          make_float4(S[4 * m], S[4 * m + 1], S[4 * m + 2], S[4 * m + 3]);
  }
}

template <class Tin, class Tg, class To>
cudaError_t launch_typed(const RecurArgs& a) {
  auto kern = chunked_f32_kernel<Tin, Tg, To>;
  const int smem = (int)sizeof(F32Smem);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (int64_t)a.N * a.H_v;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  kern<<<(unsigned)blocks, kF32Threads, smem, a.stream>>>(
      static_cast<const Tin*>(a.q), static_cast<const Tin*>(a.k), static_cast<const Tin*>(a.v),
      a.q_row_stride, a.k_row_stride, a.v_row_stride, static_cast<const Tg*>(a.g),
      static_cast<const Tg*>(a.beta), a.state_in, a.state_out, a.cu_seqlens, a.T_total, a.H_k,
      a.H_v, a.scale, static_cast<To*>(a.o));
  return cudaGetLastError();
}

template <class Tin, class Tg>
cudaError_t pick_o(const RecurArgs& a) {
  return a.o_dtype == GDN_F32 ? launch_typed<Tin, Tg, float>(a)
                              : launch_typed<Tin, Tg, __nv_bfloat16>(a);
}
template <class Tin>
cudaError_t pick_g(const RecurArgs& a) {
  return a.gate_dtype == GDN_F32 ? pick_o<Tin, float>(a) : pick_o<Tin, __nv_bfloat16>(a);
}

}  // namespace

cudaError_t launch_prefill_chunked_f32(const RecurArgs& a) {
  if (a.N == 0) return cudaSuccess;
  return a.qkv_dtype == GDN_F32 ? pick_g<float>(a) : pick_g<__nv_bfloat16>(a);
}

}  // namespace gdn
