// One decode step of the whole delta-rule layer in one kernel: the conv-cache
// roll with the kernel-4 causal conv, SiLU and the q/k L2 norm, the stepwise
// gated delta rule on a pooled state, and the gated RMS-norm of the output
// (the stepwise decode path, "delta_rule_stepwise": "Agnes-3.0-Flash Preview"
// leaderboard commentary, section 二.1; conv k=4 in front, gated RMS-norm,
// fp32 state: model card, 架构 table).
//
// Per sequence n (pool slot p = state_idx[n]) and token x_n:
//   y[c]  = SiLU(sum_j w[c,j] h_j[c] (+ b[c])), h = (cache[p] rows 0..2, x_n)
//   cache[p] <- (h_1, h_2, x_n)                    (rolled in place)
//   q, k  <- q / |q|, k / |k| per 128-channel head
//   per value head h:  S <- g S (I - beta k k^T) + beta v k^T ;  o = scale S q
//   out   = o / sqrt(mean(o^2) + eps) * w_n * SiLU(z)
//
// Launch: one 512-thread CTA per (sequence, value head), owning that head's
// 64 KiB state (8 lanes per 512-byte row, two rows per lane group, registers),
// streamed as in the plain decode kernel. Every load that does not depend on
// the pool slot (gates, z, the norm weight, the token's conv inputs and taps)
// is issued at the very top, then the slot-dependent ones (the state, all
// issued before anything is computed, and the conv-cache rows), so a CTA's
// life is one round of load latency plus its arithmetic. Each CTA computes q
// and k of its key head itself (256 channels: a few KB next to 64 KiB of
// state) and its own 128 v channels, so no CTA waits on another. A head's v
// cache rows have one reader, its CTA, which rolls them in place; the q/k
// cache rows are read by all H_v / H_k CTAs of the key head, so a second,
// tiny kernel queued right behind on the same stream rolls them.

#include "gdn_common.cuh"
#include "launch.h"

namespace gdn {
namespace {

constexpr int kLayThreads = 512;

__device__ __forceinline__ float dot4(float4 a, float4 b) {
  return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}

// the four taps of channel c (one 16-byte or 8-byte load)
__device__ __forceinline__ float4 taps4(const float* w, int c) {
  return __ldg(reinterpret_cast<const float4*>(w) + c);
}
__device__ __forceinline__ float4 taps4(const __nv_bfloat16* w, int c) {
  const uint2 u = __ldg(reinterpret_cast<const uint2*>(w) + c);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
struct LayerParams {
  const void* x; int64_t xs;
  const void* w; const void* bias;
  void* cache;
  const void* g; const void* beta;
  float* state;
  const int32_t* idx;
  int N, P, H_k, H_v, C;
  int ahead;            // CTAs resident at once: the state of CTA b + ahead is prefetched
  float scale, l2_eps;
  const void* z; const void* nw; float norm_eps;
  void* y;
};

// Tx: x, the conv cache and z; Tw: conv weights, bias and the norm weight
template <class Tx, class Tw, class Tg, class Ty>
__global__ void __launch_bounds__(kLayThreads, 2)
decode_layer_kernel(const LayerParams p) {
  const int64_t nh = blockIdx.x;
  const int n = (int)(nh / p.H_v), h = (int)(nh % p.H_v);
  const int kh = h / (p.H_v / p.H_k);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = tid >> 3, sub = tid & 7;        // rows row and row + 64
  const int part = tid >> 7, j = tid & (kHeadDim - 1);   // conv: q | k | v | idle

  __shared__ __align__(16) float k_s[kHeadDim], q_s[kHeadDim];
  __shared__ float v_s[kHeadDim], o_s[kHeadDim], red[16];

  // ---- loads that do not depend on the slot ----
  const int slot_raw = __ldg(p.idx + n);
  const float gg = to_f32(static_cast<const Tg*>(p.g)[nh]);
  const float bb = to_f32(static_cast<const Tg*>(p.beta)[nh]);
  float zz = 0.f, wn = 0.f;
  if (tid < kHeadDim) {
    zz = to_f32(static_cast<const Tx*>(p.z)[nh * kHeadDim + tid]);
    wn = to_f32(static_cast<const Tw*>(p.nw)[tid]);
  }
  const int C = p.C;
  const int c = part < 2 ? part * p.H_k * kHeadDim + kh * kHeadDim + j
                         : 2 * p.H_k * kHeadDim + h * kHeadDim + j;
  const Tx* xrow = static_cast<const Tx*>(p.x) + (int64_t)n * p.xs;
  Tx xr{};
  float4 wc = make_float4(0.f, 0.f, 0.f, 0.f);
  float bc = 0.f;
  if (part < 3) {
    xr = xrow[c];
    wc = taps4(static_cast<const Tw*>(p.w), c);
    if (p.bias) bc = to_f32(static_cast<const Tw*>(p.bias)[c]);
  }
  Ty* yrow = static_cast<Ty*>(p.y) + nh * kHeadDim;
  if (slot_raw < 0 || slot_raw >= p.P) {   // padding
    if (tid < kHeadDim) yrow[tid] = from_f32<Ty>(0.f);
    return;
  }
  const int64_t slot = slot_raw;

  // ---- the slot's state (every load issued first, evict-first) and cache rows ----
  float* S = p.state + (slot * p.H_v + h) * kHeadDim * kHeadDim;
  float4 s[2][4];
#pragma unroll
  for (int pp = 0; pp < 2; ++pp)
#pragma unroll
    for (int m = 0; m < 4; ++m)
      s[pp][m] = __ldcs(reinterpret_cast<const float4*>(S + (pp * 64 + row) * kHeadDim + (sub + 8 * m) * 4));
  // the head a CTA of the next wave will take: its state into L2 now, so that
  // CTA's loads wait for L2, not for HBM (more bytes in flight than registers hold)
  if (tid == 0 && nh + p.ahead < (int64_t)p.N * p.H_v) {
    const int64_t nx = nh + p.ahead;
    const int sx = __ldg(p.idx + nx / p.H_v);
    if (sx >= 0 && sx < p.P)
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(
                       p.state + ((int64_t)sx * p.H_v + nx % p.H_v) * kHeadDim * kHeadDim),
                   "r"((uint32_t)(kHeadDim * kHeadDim * 4))
                   : "memory");
  }
  Tx* cache = static_cast<Tx*>(p.cache) + slot * 3 * C;
  Tx c0{}, c1{}, c2{};
  if (part < 3) {
    c0 = cache[c];
    c1 = cache[C + c];
    c2 = cache[2 * C + c];
  }

  // ---- conv + SiLU; the v channels' cache rows are rolled here ----
  float val = 0.f;
  if (part < 3) {
    float a = bc;
    a = fmaf(wc.x, to_f32(c0), a);
    a = fmaf(wc.y, to_f32(c1), a);
    a = fmaf(wc.z, to_f32(c2), a);
    a = fmaf(wc.w, to_f32(xr), a);
    val = silu(a);
  }
  if (part == 2) {   // this CTA is the only reader of these rows
    cache[c] = c1;
    cache[C + c] = c2;
    cache[2 * C + c] = xr;
    v_s[j] = val;
  }
  float ss = val * val;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  if (lane == 0) red[warp] = ss;
  __syncthreads();
  if (part < 2) {    // L2 norm of q (warps 0-3) and k (warps 4-7)
    const float tot = red[4 * part] + red[4 * part + 1] + red[4 * part + 2] + red[4 * part + 3];
    (part ? k_s : q_s)[j] = val * rsqrtf(tot + p.l2_eps);
  }
  __syncthreads();

  // ---- the recurrence on the head's 128 rows (8 lanes per row) ----
  const float4* k4 = reinterpret_cast<const float4*>(k_s);
  const float4* q4 = reinterpret_cast<const float4*>(q_s);
#pragma unroll
  for (int pp = 0; pp < 2; ++pp) {
    float sk = 0.f;
#pragma unroll
    for (int m = 0; m < 4; ++m) sk += dot4(s[pp][m], k4[sub + 8 * m]);
    sk += __shfl_xor_sync(0xffffffffu, sk, 1);
    sk += __shfl_xor_sync(0xffffffffu, sk, 2);
    sk += __shfl_xor_sync(0xffffffffu, sk, 4);
    const float cc = bb * (v_s[pp * 64 + row] - gg * sk);
    float so = 0.f;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const float4 kk = k4[sub + 8 * m];
      float4 u = s[pp][m];
      u.x = fmaf(gg, u.x, cc * kk.x);
      u.y = fmaf(gg, u.y, cc * kk.y);
      u.z = fmaf(gg, u.z, cc * kk.z);
      u.w = fmaf(gg, u.w, cc * kk.w);
      so += dot4(u, q4[sub + 8 * m]);
      __stcs(reinterpret_cast<float4*>(S + (pp * 64 + row) * kHeadDim + (sub + 8 * m) * 4), u);
    }
    so += __shfl_xor_sync(0xffffffffu, so, 1);
    so += __shfl_xor_sync(0xffffffffu, so, 2);
    so += __shfl_xor_sync(0xffffffffu, so, 4);
    if (sub == 0) o_s[pp * 64 + row] = p.scale * so;
  }
  __syncthreads();
  // ---- gated RMS-norm over the head's 128 outputs ----
  if (warp < 4) {
    float sq = o_s[tid] * o_s[tid];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
    if (lane == 0) red[8 + warp] = sq;
  }
  __syncthreads();
  if (tid < kHeadDim) {
    const float inv = rsqrtf((red[8] + red[9] + red[10] + red[11]) * (1.0f / kHeadDim) + p.norm_eps);
    yrow[tid] = from_f32<Ty>(o_s[tid] * inv * wn * silu(zz));
  }
}

// Rolls the q and k channels of each live slot's conv cache once every CTA of
// decode_layer_kernel has read them: rows become (row 1, row 2, x). One thread
// per (sequence, 16-byte column chunk of the q | k channels).
__global__ void qk_cache_roll_kernel(const char* __restrict__ x, int64_t xs_bytes, char* cache,
                                     int64_t row_bytes, const int32_t* __restrict__ idx, int N,
                                     int P, int qk_chunks) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (int64_t)N * qk_chunks) return;
  const int n = (int)(t / qk_chunks);
  const int64_t off = (t % qk_chunks) * 16;
  const int slot = __ldg(idx + n);
  if (slot < 0 || slot >= P) return;
  char* cs = cache + (int64_t)slot * 3 * row_bytes + off;
  const uint4 r1 = *reinterpret_cast<const uint4*>(cs + row_bytes);
  const uint4 r2 = *reinterpret_cast<const uint4*>(cs + 2 * row_bytes);
  const uint4 xv = *reinterpret_cast<const uint4*>(x + n * xs_bytes + off);
  *reinterpret_cast<uint4*>(cs) = r1;
  *reinterpret_cast<uint4*>(cs + row_bytes) = r2;
  *reinterpret_cast<uint4*>(cs + 2 * row_bytes) = xv;
}

template <class Tx, class Tw, class Tg, class Ty>
cudaError_t launch_typed(const DecodeLayerArgs& a) {
  int dev = 0, nsm = 0, per_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_layer_kernel<Tx, Tw, Tg, Ty>,
                                                    kLayThreads, 0);
  if (e != cudaSuccess) return e;
  LayerParams p{a.x, a.x_row_stride, a.conv_w, a.conv_bias, a.conv_state, a.g, a.beta,
                a.state, a.state_idx, a.N, a.P, a.H_k, a.H_v,
                2 * a.H_k * kHeadDim + a.H_v * kHeadDim, nsm * (per_sm > 0 ? per_sm : 1),
                a.scale, a.l2_eps, a.z, a.norm_w, a.norm_eps, a.y};
  const int64_t blocks = (int64_t)a.N * a.H_v;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  decode_layer_kernel<Tx, Tw, Tg, Ty><<<(unsigned)blocks, kLayThreads, 0, a.stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int eb = (int)sizeof(Tx);
  const int qk_chunks = 2 * a.H_k * kHeadDim * eb / 16;
  const int64_t threads = (int64_t)a.N * qk_chunks;
  qk_cache_roll_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, a.stream>>>(
      static_cast<const char*>(a.x), a.x_row_stride * eb, static_cast<char*>(a.conv_state),
      (int64_t)p.C * eb, a.state_idx, a.N, a.P, qk_chunks);
  return cudaGetLastError();
}

template <class Tx, class Tw, class Tg>
cudaError_t pick_y(const DecodeLayerArgs& a) {
  return a.y_dtype == GDN_F32 ? launch_typed<Tx, Tw, Tg, float>(a)
                              : launch_typed<Tx, Tw, Tg, __nv_bfloat16>(a);
}
template <class Tx, class Tw>
cudaError_t pick_g(const DecodeLayerArgs& a) {
  return a.gate_dtype == GDN_F32 ? pick_y<Tx, Tw, float>(a) : pick_y<Tx, Tw, __nv_bfloat16>(a);
}
template <class Tx>
cudaError_t pick_w(const DecodeLayerArgs& a) {
  return a.w_dtype == GDN_F32 ? pick_g<Tx, float>(a) : pick_g<Tx, __nv_bfloat16>(a);
}

}  // namespace

cudaError_t launch_decode_layer(const DecodeLayerArgs& a) {
  if (a.N == 0) return cudaSuccess;
  return a.x_dtype == GDN_F32 ? pick_w<float>(a) : pick_w<__nv_bfloat16>(a);
}

}  // namespace gdn
