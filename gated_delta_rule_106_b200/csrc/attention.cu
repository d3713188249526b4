// Global-attention layer of the hybrid decoder: the quarter of its layers
// that keep a KV cache (Agnes-3.0-Flash Preview model card, section 架构,
// rows 全局注意力 and 位置编码; leaderboard commentary, section 二.1):
// 24 query / 4 key-value heads (GQA 6 : 1), head dim 256, RMS-norm on q and k,
// three-axis rotary (text / height / width interleaved, base 1e7) on the first
// 64 dims, causal softmax attention, sigmoid gate on each head's output.
//
// Prefill is two launches:
//  * attn_qk_prologue_kernel: per (token, head) row, RMS-norm with the weight
//    vector and rotary (angles in fp64, shared by all heads of a token); writes
//    rotated q into the workspace and rotated k where the caller wants its KV
//    cache, both in fp16: after the norm every element is at most
//    16 * sqrt(2) * max|w| in magnitude, well inside fp16's range, and fp16
//    keeps three more significand bits than bf16 for the score product. The
//    values go to fp16 as well (the value cache's dtype): a bf16 value in
//    fp16's normal range converts exactly, so P V can take P in fp16 too.
//  * attn_prefill_kernel: causal flash attention on tcgen05. A CTA owns 64
//    query tokens of two query heads that share a key-value head (128 rows),
//    walks 64-key blocks up to the diagonal. S = Q K^T (128 x 64, K = 256) and
//    O += P V (128 x 256, K = 64) take fp16 operands and accumulate in TMEM.
//    The online softmax runs in 8 warps (two per TMEM lane quadrant, each on
//    half of a row's columns; row maxima and sums meet in shared memory) and
//    rescales O in TMEM only when a row's running max grows by more than 2^8;
//    the epilogue divides by the row sum and applies sigmoid(gate).
#include <cudaTypedefs.h>
#include <math.h>

#include "gdn_common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int kAD = 256;        // head dim of the attention layer
constexpr int kTileTok = 64;    // query tokens per tile (two heads -> 128 rows)
constexpr int kBlk = 64;        // keys per block
constexpr uint64_t kAttnLimitNs = 2000000000ull;

// --------------------------------------------------------------- prologue --

constexpr int kProTok = 4;      // tokens per prologue CTA

struct ProParams {
  const __nv_bfloat16* q; const __nv_bfloat16* k; int64_t q_stride, k_stride;
  const void* wq; const void* wk;
  const int32_t* cu; int N; int64_t T;
  const int32_t* positions;     // [3][T] or null
  const int32_t* pos0;          // [N] or null
  int Hq, Hkv; float eps; int R; double log2_base;
  const __nv_bfloat16* v; int64_t v_stride;
  __half* q_out; __half* k_out; __half* v_out;   // [T][H][256] dense
};

__device__ __forceinline__ float ldw(const float* w, int i) { return w[i]; }
__device__ __forceinline__ float ldw(const __nv_bfloat16* w, int i) {
  return __bfloat162float(w[i]);
}

// Sequence of token t: the n with cu[n] <= t < cu[n + 1].
__device__ __forceinline__ int seq_of(const int32_t* cu, int N, int64_t t) {
  int lo = 0, hi = N;        // cu[lo] <= t, answer in [lo, hi)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cu[mid] <= t) lo = mid; else hi = mid;
  }
  return lo;
}

__device__ __forceinline__ void store8h(__half* p, const float (&f)[8]) {
  uint4 u;
  __half2* h = reinterpret_cast<__half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}

// bf16 -> fp16 for a value row: exact in fp16's normal range; beyond +-65504
// the value saturates there.
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 u) {
  const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
  uint4 r;
  __half2* h = reinterpret_cast<__half2*>(&r);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(b[i]);
    f.x = fminf(fmaxf(f.x, -65504.f), 65504.f);
    f.y = fminf(fmaxf(f.y, -65504.f), 65504.f);
    h[i] = __floats2half2_rn(f.x, f.y);
  }
  return r;
}

// One (token, head) row of 256 by one warp: RMS-norm with weight w, then
// rotary on dims [0, R) with the token's (cos, sin) per pair; lane l returns
// dims 8l .. 8l + 7. `row` is this warp's 256-float staging area.
template <class Tw>
__device__ __forceinline__ void norm_rope_vals(const Tw* w, const float2* cs, float* row, int R,
                                               float eps, int lane, float (&x)[8]) {
  const int half = R >> 1;
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) ss += x[i] * x[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = rsqrtf(ss * (1.0f / kAD) + eps);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    x[i] = x[i] * inv * ldw(w, lane * 8 + i);
    row[lane * 8 + i] = x[i];
  }
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int d = lane * 8 + i;
    if (d < half) {
      const float2 a = cs[d];
      x[i] = row[d] * a.x - row[d + half] * a.y;
    } else if (d < R) {
      const float2 a = cs[d - half];
      x[i] = row[d] * a.x + row[d - half] * a.y;
    }
  }
  __syncwarp();
}
template <class Tw>
__device__ __forceinline__ void norm_rope_row(const __nv_bfloat16* src, const Tw* w,
                                              const float2* cs, float* row, int R, float eps,
                                              int lane, float (&x)[8]) {
  load8(src + lane * 8, x);
  norm_rope_vals(w, cs, row, R, eps, lane, x);
}

// (cos, sin) of rotary pair i at position pos, angle in fp64.
__device__ __forceinline__ float2 rope_cs(int64_t pos, int i, int R, double log2_base) {
  const double theta = (double)pos * exp2(-(2.0 * i / R) * log2_base);
  double s, c;
  sincos(theta, &s, &c);
  return make_float2((float)c, (float)s);
}

template <class Tw>
__global__ void __launch_bounds__(256) attn_qk_prologue_kernel(const ProParams p) {
  __shared__ float2 cs[kProTok][32];       // (cos, sin) per token and rotary pair
  __shared__ float row[8][kAD];            // one staged row per warp
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t t0 = (int64_t)blockIdx.x * kProTok;
  const int half = p.R >> 1;
  if (tid < kProTok * 32) {
    const int tt = tid >> 5, i = tid & 31;
    const int64_t t = t0 + tt;
    if (t < p.T && i < half) {
      const int axis = i % 3;
      int64_t pos;
      if (p.positions) {
        pos = p.positions[(int64_t)axis * p.T + t];
      } else {
        const int n = seq_of(p.cu, p.N, t);
        pos = t - p.cu[n] + (p.pos0 ? p.pos0[n] : 0);
      }
      cs[tt][i] = rope_cs(pos, i, p.R, p.log2_base);
    }
  }
  __syncthreads();
  const int H = p.Hq + p.Hkv;
  const Tw* wq = static_cast<const Tw*>(p.wq);
  const Tw* wk = static_cast<const Tw*>(p.wk);
  // two rows per warp and round, both loaded before either is normed
  for (int r0 = warp; r0 < kProTok * H; r0 += 16) {
    uint4 raw[2];
    bool live[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int r = r0 + 8 * u;
      const int tt = r / H, hh = r % H;
      const int64_t t = t0 + tt;
      live[u] = r < kProTok * H && t < p.T;
      const __nv_bfloat16* src = hh < p.Hq ? p.q + t * p.q_stride + (int64_t)hh * kAD
                                           : p.k + t * p.k_stride + (int64_t)(hh - p.Hq) * kAD;
      raw[u] = live[u] ? __ldg(reinterpret_cast<const uint4*>(src + lane * 8))
                       : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (!live[u]) continue;     // warp-uniform
      const int r = r0 + 8 * u;
      const int tt = r / H, hh = r % H;
      const int64_t t = t0 + tt;
      const bool isq = hh < p.Hq;
      float x[8];
      {
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&raw[u]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(b2[e]);
          x[2 * e] = f.x;
          x[2 * e + 1] = f.y;
        }
      }
      norm_rope_vals(isq ? wq : wk, cs[tt], row[warp], p.R, p.eps, lane, x);
      if (isq) {
        store8h(p.q_out + (t * p.Hq + hh) * kAD + lane * 8, x);
      } else {
        const int g = hh - p.Hq;
        const int64_t o = (t * p.Hkv + g) * kAD + lane * 8;
        store8h(p.k_out + o, x);
        *reinterpret_cast<uint4*>(p.v_out + o) = bf16x8_to_f16x8(
            *reinterpret_cast<const uint4*>(p.v + t * p.v_stride + (int64_t)g * kAD + lane * 8));
      }
    }
  }
}

// ---------------------------------------------------------- flash attention --

// Shared memory (offsets from a 1024-byte aligned base). Operand tiles are
// 128-byte-swizzled rows of 64 bf16, as the TMA writes them.
constexpr uint32_t A_Q = 0;          // 4 dim chunks x [128 rows][128 B] (16 KB each)
constexpr uint32_t A_K = 65536;      // 2 slots x 4 dim chunks x [64 keys][128 B]
constexpr uint32_t A_V = 131072;     // 2 slots x 4 dim chunks x [64 keys][128 B]
constexpr uint32_t A_P = 196608;     // [128 rows][64 keys] fp16 (P_j is written after
                                     // O_{j-1} has read P_{j-1})
constexpr uint32_t A_RED = 212992;   // [2 block parities][2 column halves][128 rows] fp32
constexpr uint32_t A_BAR = 215040;
constexpr uint32_t A_SMEM = A_BAR + 256 + 1024;   // + alignment slack
constexpr int kAttnThreads = 384;    // producer, MMA, TMEM, idle, 8 softmax warps

// TMEM columns: O accumulator [0, 256), S buffers at 256 and 320.
constexpr uint32_t T_O = 0, T_S = 256;

struct AttnBars {
  uint64_t q_full, k_full[2], v_full[2], s_full[2], o_done[2], p_full[2];
  uint32_t tmem;
  int n, tile;          // item: sequence and query tile (n < 0: nothing to do)
};

struct AttnParams {
  const int32_t* cu; int N; int64_t T; int Hq, Hkv;
  int grid_tiles;       // tiles the grid was sized for (>= the real count)
  float sl2;            // softmax scale * log2(e)
  const __nv_bfloat16* gate; int64_t gate_stride;
  __nv_bfloat16* o;     // [T][Hq][256]
  int* status;          // set to 1 when a wait ran out
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void fail(const AttnParams& p) { atomicExch(p.status, 1); }

// Locate tile u (counted over all sequences, ceil(len / 64) tiles each) with
// one warp: returns (n, tile) or n = -1 when u is past the last tile.
__device__ __forceinline__ int cu_at(const int32_t* cu, int n, int64_t T) {
  const int64_t c = cu[n];
  return (int)(c < 0 ? 0 : (c > T ? T : c));
}

__device__ void find_tile(const int32_t* cu, int N, int64_t T, int u, int lane, int* n_out,
                          int* t_out) {
  int base = 0;
  for (int n0 = 0; n0 < N; n0 += 32) {
    const int n = n0 + lane;
    const int len = n < N ? max(cu_at(cu, n + 1, T) - cu_at(cu, n, T), 0) : 0;
    const int tiles = (len + kTileTok - 1) / kTileTok;
    int incl = tiles;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int excl = incl - tiles;
    if (n < N && u >= base + excl && u < base + incl) {
      *n_out = n;
      *t_out = u - base - excl;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
    __syncwarp();
  }
}

__global__ void __launch_bounds__(kAttnThreads, 1)
attn_prefill_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sa = smem_u32(sm);
  AttnBars& B = *reinterpret_cast<AttnBars*>(sm + A_BAR);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int pairs = p.Hq >> 1;
  const int pair = blockIdx.x % pairs;
  const int u = p.grid_tiles - 1 - (int)(blockIdx.x / pairs);   // heaviest tiles first

  if (tid == 0) {
    B.n = -1;
    mbar_init(&B.q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&B.k_full[i], 1);
      mbar_init(&B.v_full[i], 1);
      mbar_init(&B.s_full[i], 1);
      mbar_init(&B.o_done[i], 1);
      mbar_init(&B.p_full[i], 256);
    }
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == 0) {
    int n = -1, t = 0;
    find_tile(p.cu, p.N, p.T, u, lane, &n, &t);
    // the lane that found it holds the answer; share through shared memory
    if (n >= 0) { B.n = n; B.tile = t; }
  }
  if (warp == 2) {
    tmem_alloc(&B.tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int n = B.n;
  const uint32_t tmem = B.tmem;
  if (n >= 0) {
    const int tile = B.tile;
    const int s0 = cu_at(p.cu, n, p.T), s1 = max(cu_at(p.cu, n + 1, p.T), s0);
    const int q0 = s0 + tile * kTileTok;
    const int nb = tile + 1;                    // key blocks up to the diagonal
    const int h0 = 2 * pair;
    const int g = h0 / (p.Hq / p.Hkv);

    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------- producer
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      mbar_arrive_expect_tx(&B.q_full, 65536);
      for (int c = 0; c < 4; ++c)
        for (int hh = 0; hh < 2; ++hh)
          tma_load_2d(sm + A_Q + c * 16384 + hh * 8192, &tm_q, (h0 + hh) * kAD + c * 64, q0,
                      &B.q_full);
      bool ok = true;
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < nb && ok; ++j) {
        const int sl = j & 1;
        const uint32_t par = (uint32_t)(((j - 2) >> 1) & 1);
        if (j >= 2) ok = mbar_wait_bounded(&B.s_full[sl], par, kAttnLimitNs);   // S_{j-2} read K
        if (!ok) break;
        mbar_arrive_expect_tx(&B.k_full[sl], 32768);
        for (int c = 0; c < 4; ++c)
          tma_load_2d(sm + A_K + sl * 32768 + c * 8192, &tm_k, g * kAD + c * 64, s0 + j * kBlk,
                      &B.k_full[sl]);
        k_issued = j + 1;
        if (j >= 2) ok = mbar_wait_bounded(&B.o_done[sl], par, kAttnLimitNs);   // O_{j-2} read V
        if (!ok) break;
        mbar_arrive_expect_tx(&B.v_full[sl], 32768);
        for (int c = 0; c < 4; ++c)
          tma_load_2d(sm + A_V + sl * 32768 + c * 8192, &tm_v, g * kAD + c * 64, s0 + j * kBlk,
                      &B.v_full[sl]);
        v_issued = j + 1;
      }
      if (!ok) fail(p);
      // leave only once every copy issued here has landed
      mbar_wait_bounded(&B.q_full, 0, kAttnLimitNs);
      for (int j = (k_issued > 2 ? k_issued - 2 : 0); j < k_issued; ++j)
        mbar_wait_bounded(&B.k_full[j & 1], (uint32_t)((j >> 1) & 1), kAttnLimitNs);
      for (int j = (v_issued > 2 ? v_issued - 2 : 0); j < v_issued; ++j)
        mbar_wait_bounded(&B.v_full[j & 1], (uint32_t)((j >> 1) & 1), kAttnLimitNs);
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------------- MMA issuer
      const uint32_t id_s = idesc_f16(128, kBlk, false, false);
      const uint32_t id_o = idesc_f16(128, kAD, false, true);
      auto issue_s = [&](int j) {
        const int sl = j & 1;
        const uint32_t kb = sa + A_K + sl * 32768;
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
          const uint32_t off_q = (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint32_t off_k = (kk >> 2) * 8192 + (kk & 3) * 32;
          mma_f16(tmem + T_S + sl * kBlk, sw128_desc(sa + A_Q + off_q, 16, 1024),
                  sw128_desc(kb + off_k, 16, 1024), id_s, kk > 0);
        }
        mma_commit(&B.s_full[sl]);
      };
      bool ok = mbar_wait_bounded(&B.q_full, 0, kAttnLimitNs);
      for (int j = 0; j < 2 && j < nb && ok; ++j) {
        ok = mbar_wait_bounded(&B.k_full[j], 0, kAttnLimitNs);
        if (ok) {
          tc_fence_after();
          issue_s(j);
        }
      }
      for (int j = 0; j < nb && ok; ++j) {
        const int sl = j & 1;
        const uint32_t par = (uint32_t)((j >> 1) & 1);
        ok = mbar_wait_bounded(&B.p_full[sl], par, kAttnLimitNs) &&
             mbar_wait_bounded(&B.v_full[sl], par, kAttnLimitNs);
        if (!ok) break;
        tc_fence_after();
        const uint32_t pb = sa + A_P, vb = sa + A_V + sl * 32768;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f16(tmem + T_O, sw128_desc(pb + kk * 32, 16, 1024),
                  sw128_desc(vb + kk * 2048, 8192, 1024), id_o, (j > 0 || kk > 0));
        mma_commit(&B.o_done[sl]);
        if (j + 2 < nb) {
          ok = mbar_wait_bounded(&B.k_full[sl], (uint32_t)(((j + 2) >> 1) & 1), kAttnLimitNs);
          if (!ok) break;
          tc_fence_after();
          issue_s(j + 2);
        }
      }
      if (!ok) fail(p);
    } else if (warp >= 4) {
      // ------------------------------------------- softmax, then epilogue
      // Two warps per TMEM lane quadrant: `half` 0 takes score columns 0..31
      // and output columns 0..127, `half` 1 the rest; they exchange row maxima
      // (and, at the end, row sums) through shared memory.
      const int quad = warp & 3, half = (warp - 4) >> 2;
      const int r = quad * 32 + lane;           // row = TMEM lane
      const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
      float* red = reinterpret_cast<float*>(sm + A_RED);
      const int tq_off = r & 63;               // token offset within the tile
      float m = -INFINITY, l = 0.f;
      // A wait that runs out clears `ok`; the loop still runs to the end with
      // no further waits, so that both warps of a pair pass the same named
      // barriers (what it computes then is discarded: the status word is set).
      bool ok = true;
      for (int j = 0; j < nb; ++j) {
        const int sl = j & 1;
        if (ok) ok = mbar_wait_bounded(&B.s_full[sl], (uint32_t)((j >> 1) & 1), kAttnLimitNs);
        ok = __all_sync(0xffffffffu, ok);
        tc_fence_after();
        uint32_t sr[32];
        tmem_ld32_nowait(trow + T_S + sl * kBlk + half * 32, sr);
        tmem_wait_ld();
        float s[32];
        const bool diag = (j == nb - 1);
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          s[c] = (diag && half * 32 + c > tq_off) ? -INFINITY : __uint_as_float(sr[c]);
          mx = fmaxf(mx, s[c]);
        }
        float* rb = red + (j & 1) * 256;
        rb[half * 128 + r] = mx;
        bar_sync_n(1 + quad, 64);
        mx = fmaxf(mx, rb[(1 - half) * 128 + r]);
        const float mb = mx * p.sl2;
        bool o_prev_done = false;
        if (j == 0) {
          m = mb;
        } else {
          const bool need = mb > m + 8.0f;
          if (__any_sync(0xffffffffu, need) && ok) {   // the partner warp decides the same
            const float m_new = fmaxf(m, mb);
            const float f = ex2(m - m_new);
            m = m_new;
            l *= f;
            // O holds P_0..P_{j-1} V: wait for the last of them, rescale this half
            ok = __all_sync(0xffffffffu,
                            mbar_wait_bounded(&B.o_done[(j - 1) & 1],
                                              (uint32_t)(((j - 1) >> 1) & 1), kAttnLimitNs));
            o_prev_done = true;
            tc_fence_after();
#pragma unroll 1
            for (int cc = 0; cc < 4 && ok; ++cc) {
              uint32_t ov[32];
              const uint32_t ta = trow + T_O + half * 128 + cc * 32;
              tmem_ld32_nowait(ta, ov);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * f);
              tmem_st32(ta, ov);
            }
            tmem_wait_st();
          }
        }
        // P in registers first, so the exponentials overlap O_{j-1}
        uint32_t w[16];
        float sum = 0.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float a = ex2(fmaf(s[2 * e], p.sl2, -m));
          const float b = ex2(fmaf(s[2 * e + 1], p.sl2, -m));
          sum += a + b;
          __half2 h2 = __floats2half2_rn(a, b);
          w[e] = *reinterpret_cast<uint32_t*>(&h2);
        }
        l += sum;
        // one P buffer: O_{j-1} must have read P_{j-1}
        if (j >= 1 && !o_prev_done && ok)
          ok = __all_sync(0xffffffffu,
                          mbar_wait_bounded(&B.o_done[(j - 1) & 1],
                                            (uint32_t)(((j - 1) >> 1) & 1), kAttnLimitNs));
        uint8_t* prow = sm + A_P + r * 128;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int c16 = half * 4 + q4;
          *reinterpret_cast<uint4*>(prow + ((c16 ^ (r & 7)) << 4)) =
              make_uint4(w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2], w[4 * q4 + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&B.p_full[sl]);
      }
      {
        float* rb = red + (nb & 1) * 256;
        rb[half * 128 + r] = l;
        bar_sync_n(1 + quad, 64);
        l += rb[(1 - half) * 128 + r];
      }
      if (ok)
        ok = mbar_wait_bounded(&B.o_done[(nb - 1) & 1], (uint32_t)(((nb - 1) >> 1) & 1),
                               kAttnLimitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (lane == 0) fail(p);
      } else {
        tc_fence_after();
        const int tq = q0 + tq_off;
        const int h = h0 + (r >> 6);
        const bool valid = tq < s1;
        const float inv_l = 1.0f / l;
        const __nv_bfloat16* gp =
            p.gate + (int64_t)tq * p.gate_stride + (int64_t)h * kAD + half * 128;
        __nv_bfloat16* op = p.o + ((int64_t)tq * p.Hq + h) * kAD + half * 128;
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t ov[32];
          tmem_ld32_nowait(trow + T_O + half * 128 + cc * 32, ov);
          tmem_wait_ld();
          if (valid) {
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8) {
              float gt[8], y[8];
              load8(gp + cc * 32 + q8 * 8, gt);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                y[i] = __uint_as_float(ov[q8 * 8 + i]) * inv_l / (1.0f + __expf(-gt[i]));
              store8(op + cc * 32 + q8 * 8, y);
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ decode --
//
// One new token per sequence against a pooled KV cache [P][L_max][Hkv][256]:
//  * attn_decode_prologue_kernel (one CTA per sequence): norm + rotary of the
//    new q and k at position cache_len[n] (or the given three-axis
//    positions); rotated q to the workspace in fp32, rotated k and v appended
//    to the sequence's cache slot at row cache_len[n];
//  * attn_decode_split_kernel (one warp per sequence, key-value head and unit
//    of kUnit cached tokens): the G query heads of the group share every K / V
//    row the warp streams; writes the unit's un-normalised output with its
//    running max and sum;
//  * attn_decode_combine_kernel (one CTA per sequence and query head): merges
//    the splits, divides by the sum, applies sigmoid(gate), and advances
//    cache_len[n] by one.

struct DecParams {
  const __nv_bfloat16* q; const __nv_bfloat16* k; const __nv_bfloat16* v;
  const __nv_bfloat16* gate;
  int64_t q_stride, k_stride, v_stride, gate_stride;   // per sequence row (elements)
  const void* wq; const void* wk;
  __half* kc; __half* vc;                 // [P][L_max][Hkv][256]
  const int32_t* idx;                     // [N] slots, or null (slot n)
  int32_t* len;                           // [N] cached tokens before this step
  const int32_t* positions;               // [3][N] or null
  int N, P, L_max, Hq, Hkv; float eps; int R; double log2_base; float sl2;
  float* q_rot;                           // [N][Hq][256]
  float* part_ml;                         // [N][Hq][S][2]: max (log2 units), sum
  float* part_o;                          // [N][Hq][S][256]
  int S;                                  // units per (sequence, key-value head)
  __nv_bfloat16* o;                       // [N][Hq][256]
  int* status;                            // 2: a sequence's slot or length was out of range
};

__device__ __forceinline__ bool dec_valid(const DecParams& p, int n, int* slot, int* L) {
  *slot = p.idx ? p.idx[n] : n;
  *L = p.len[n];
  return *slot >= 0 && *slot < p.P && *L >= 0 && *L < p.L_max;
}

template <class Tw>
__global__ void __launch_bounds__(256) attn_decode_prologue_kernel(const DecParams p) {
  __shared__ float2 cs[32];
  __shared__ float row[8][kAD];
  const int n = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int slot, L;
  const bool ok = dec_valid(p, n, &slot, &L);
  if (!ok) {
    if (tid == 0) atomicExch(p.status, 2);
    return;
  }
  if (tid < (p.R >> 1)) {
    const int64_t pos = p.positions ? p.positions[(int64_t)(tid % 3) * p.N + n] : L;
    cs[tid] = rope_cs(pos, tid, p.R, p.log2_base);
  }
  __syncthreads();
  const Tw* wq = static_cast<const Tw*>(p.wq);
  const Tw* wk = static_cast<const Tw*>(p.wk);
  for (int r = warp; r < p.Hq + p.Hkv; r += 8) {
    float x[8];
    if (r < p.Hq) {
      norm_rope_row(p.q + n * p.q_stride + (int64_t)r * kAD, wq, cs, row[warp], p.R, p.eps,
                    lane, x);
      float* dst = p.q_rot + ((int64_t)n * p.Hq + r) * kAD + lane * 8;
      store8(dst, x);
    } else {
      const int g = r - p.Hq;
      norm_rope_row(p.k + n * p.k_stride + (int64_t)g * kAD, wk, cs, row[warp], p.R, p.eps,
                    lane, x);
      const int64_t crow = (((int64_t)slot * p.L_max + L) * p.Hkv + g) * kAD + lane * 8;
      store8h(p.kc + crow, x);
      *reinterpret_cast<uint4*>(p.vc + crow) = bf16x8_to_f16x8(
          *reinterpret_cast<const uint4*>(p.v + n * p.v_stride + (int64_t)g * kAD + lane * 8));
    }
  }
}

// ---- split kernel: one warp streams kUnit cached tokens of one (sequence,
// key-value head) in groups of 16 through a two-stage cp.async ring in its own
// shared memory, and runs both products on the tensor cores (mma.sync
// m16n8k16, fp16 in, fp32 accumulate): S = Q K^T with the G query heads of the
// group as rows (rows G..15 zero), then O += P V with P taken straight from the
// S registers. Online softmax per row with the same lazy rescale as prefill.
// Each warp writes its own partial (max, sum, un-normalised O); no CTA-wide
// synchronisation.
constexpr int kGrp = 16;                     // tokens per group
constexpr int kUnit = 512;                   // tokens per warp
constexpr int kRowB = 528;                   // smem row stride: 512 B + 16 (no bank conflicts)
constexpr int kStageB = 2 * kGrp * kRowB;    // K and V rows of one group
constexpr int kDecWarps = 2;                 // warps (units) per CTA; they share Q
constexpr int kQB = 8 * kRowB;               // Q rows 0..7 in fp16 (rows >= G zero)
constexpr int kDecSmem = kQB + kDecWarps * 2 * kStageB;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// d += A B, A rows 8..15 zero (a1 = a3 = 0)
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <int G>
__global__ void __launch_bounds__(32 * kDecWarps, 3) attn_decode_split_kernel(const DecParams p) {
  extern __shared__ __align__(16) uint8_t dsm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int unit = blockIdx.x * kDecWarps + warp, g = blockIdx.y, n = blockIdx.z;
  const int64_t hq0 = (int64_t)n * p.Hq + g * G;
  int slot, L;
  const bool ok = dec_valid(p, n, &slot, &L);
  // Q of the group's G heads -> fp16 rows of shared memory (rows G..7 zero)
  const uint32_t qbase = smem_u32(dsm);
  for (int i = threadIdx.x; i < 8 * kAD / 2; i += 32 * kDecWarps) {
    const int r = i / (kAD / 2), c = 2 * (i % (kAD / 2));
    uint32_t v = 0u;
    if (ok && r < G) {
      const float* qr = p.q_rot + (hq0 + r) * kAD + c;
      v = pack_h2(qr[0], qr[1]);
    }
    *reinterpret_cast<uint32_t*>(dsm + r * kRowB + c * 2) = v;
  }
  __syncthreads();
  if (unit >= p.S) return;
  const int t_beg = unit * kUnit;
  const int n_tok = ok ? min(kUnit, L + 1 - t_beg) : 0;
  if (n_tok <= 0) {
    if (lane < G) {
      float* ml = p.part_ml + ((hq0 + lane) * p.S + unit) * 2;
      ml[0] = ok ? -INFINITY : 0.f;
      ml[1] = ok ? 0.f : __int_as_float(0x7fc00000);
    }
    return;
  }
  const uint32_t sbase = qbase + kQB + warp * 2 * kStageB;
  const int row = lane >> 2, qd = lane & 3;     // fragment row (query head) and quad
  const bool live = row < G;
  const int64_t tok_stride = (int64_t)p.Hkv * kAD;
  const int64_t base = (((int64_t)slot * p.L_max + t_beg) * p.Hkv + g) * kAD;
  const __half* kb = p.kc + base;
  const __half* vb = p.vc + base;
  const int n_grp = (n_tok + kGrp - 1) / kGrp;
  const __half* kl = kb + lane * 8;
  const __half* vl = vb + lane * 8;
  auto issue = [&](int gi) {
    const uint32_t st = sbase + (gi & 1) * kStageB + lane * 16;
#pragma unroll
    for (int r = 0; r < kGrp; ++r) {          // 16 rows x 32 chunks of 16 B, K then V
      const int t = gi * kGrp + r;
      const bool valid = t < n_tok;
      const int64_t off = (int64_t)(valid ? t : 0) * tok_stride;
      cp_async16(st + r * kRowB, kl + off, valid);
      cp_async16(st + (kGrp + r) * kRowB, vl + off, valid);
    }
    cp_async_commit();
  };
  float o[32][4];
#pragma unroll
  for (int j = 0; j < 32; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m = -INFINITY, l = 0.f;
  issue(0);
  if (n_grp > 1) issue(1);
  // ldmatrix row addresses: matrix j = lane / 8, row i = lane % 8
  const int mj = lane >> 3, mi = lane & 7;
  const uint32_t k_off = (uint32_t)(((mj >> 1) * 8 + mi) * kRowB + (mj & 1) * 16);
  const uint32_t q_off = (uint32_t)(mi * kRowB + (mj & 1) * 16);   // x2: lanes 0..15
  const uint32_t v_off = (uint32_t)(((mj & 1) * 8 + mi) * kRowB + (mj >> 1) * 16);
  for (int gi = 0; gi < n_grp; ++gi) {
    if (gi + 1 < n_grp) cp_async_wait<1>(); else cp_async_wait<0>();
    __syncwarp();
    const uint32_t kst = sbase + (gi & 1) * kStageB, vst = kst + kGrp * kRowB;
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      uint32_t b[4], a0, a2;
      ldsm_x2(qbase + q_off + kk * 32, a0, a2);
      ldsm_x4(kst + k_off + kk * 32, b);
      mma16816(s0, a0, a2, b[0], b[1]);
      mma16816(s1, a0, a2, b[2], b[3]);
    }
    // this lane's scores: row `row`, tokens 2qd, 2qd+1 (s0) and 8+2qd, 9+2qd (s1)
    const int t0 = gi * kGrp + 2 * qd;
    float x[4] = {t0 < n_tok ? s0[0] * p.sl2 : -INFINITY,
                  t0 + 1 < n_tok ? s0[1] * p.sl2 : -INFINITY,
                  t0 + 8 < n_tok ? s1[0] * p.sl2 : -INFINITY,
                  t0 + 9 < n_tok ? s1[1] * p.sl2 : -INFINITY};
    float mb = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
    mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 1));
    mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 2));
    if (mb > m + 8.0f) {               // same for the 4 lanes of a row
      const float f = ex2(m - mb);
      m = mb;
      l *= f;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        o[j][0] *= f;
        o[j][1] *= f;
      }
    }
    float pv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      pv[e] = ex2(x[e] - m);
      l += pv[e];
    }
    const uint32_t pa0 = pack_h2(pv[0], pv[1]), pa2 = pack_h2(pv[2], pv[3]);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      uint32_t b[4];
      ldsm_x4_t(vst + v_off + j * 32, b);
      mma16816(o[2 * j], pa0, pa2, b[0], b[1]);
      mma16816(o[2 * j + 1], pa0, pa2, b[2], b[3]);
    }
    __syncwarp();
    if (gi + 2 < n_grp) issue(gi + 2);
  }
  l += __shfl_xor_sync(0xffffffffu, l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);
  if (live) {
    float* po = p.part_o + ((hq0 + row) * p.S + unit) * kAD + 2 * qd;
#pragma unroll
    for (int j = 0; j < 32; ++j)
      *reinterpret_cast<float2*>(po + j * 8) = make_float2(o[j][0], o[j][1]);
    if (qd == 0) {
      float* ml = p.part_ml + ((hq0 + row) * p.S + unit) * 2;
      ml[0] = m;
      ml[1] = l;
    }
  }
}

__global__ void __launch_bounds__(256) attn_decode_combine_kernel(const DecParams p) {
  const int h = blockIdx.x, n = blockIdx.y, d = threadIdx.x;
  const int64_t hq = (int64_t)n * p.Hq + h;
  const float* ml = p.part_ml + hq * p.S * 2;
  float M = -INFINITY;
  for (int s = 0; s < p.S; ++s)
    if (ml[2 * s + 1] > 0.f) M = fmaxf(M, ml[2 * s]);
  float Lsum = 0.f, acc = 0.f;
  for (int s = 0; s < p.S; ++s) {
    const float l = ml[2 * s + 1];
    if (l > 0.f) {
      const float w = ex2(ml[2 * s] - M);
      Lsum += w * l;
      acc += w * p.part_o[(hq * p.S + s) * kAD + d];
    }
  }
  const float gt = __bfloat162float(p.gate[n * p.gate_stride + (int64_t)h * kAD + d]);
  const float y = (Lsum > 0.f ? acc / Lsum : __int_as_float(0x7fc00000)) / (1.0f + __expf(-gt));
  p.o[hq * kAD + d] = __float2bfloat16_rn(y);
  if (h == 0 && d == 0) {
    int slot, L;
    if (dec_valid(p, n, &slot, &L)) p.len[n] = L + 1;
  }
}

// ------------------------------------------------------------------ host --

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// [rows][cols] 16-bit elements with a row stride, 64 x 64 boxes, 128-byte swizzle.
bool make_attn_map(CUtensorMap* m, const void* base, int64_t cols, int64_t rows,
                   int64_t stride_elems, CUtensorMapDataType type) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(stride_elems * 2)};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, type, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace

size_t attention_prefill_workspace(int64_t T, int Hq) {
  return 256 + (size_t)T * Hq * kAD * 2;
}

cudaError_t launch_attention_prefill(const AttnPrefillArgs& a) {
  if (a.T == 0) return cudaSuccess;
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  int* status = reinterpret_cast<int*>(ws);
  __half* q_rot = reinterpret_cast<__half*>(ws + 256);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), a.stream);
  if (e != cudaSuccess) return e;

  ProParams pp{static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
               a.q_row_stride, a.k_row_stride, a.wq, a.wk, a.cu_seqlens, a.N, a.T,
               a.positions, a.pos0, a.Hq, a.Hkv, a.eps, a.rope_dims, log2((double)a.rope_base),
               static_cast<const __nv_bfloat16*>(a.v), a.v_row_stride, q_rot,
               static_cast<__half*>(a.k_rot), static_cast<__half*>(a.v_h)};
  const unsigned pgrid = (unsigned)((a.T + kProTok - 1) / kProTok);
  if (a.w_dtype == GDN_F32)
    attn_qk_prologue_kernel<float><<<pgrid, 256, 0, a.stream>>>(pp);
  else
    attn_qk_prologue_kernel<__nv_bfloat16><<<pgrid, 256, 0, a.stream>>>(pp);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  CUtensorMap mq, mk, mv;
  if (!make_attn_map(&mq, q_rot, (int64_t)a.Hq * kAD, a.T, (int64_t)a.Hq * kAD,
                     CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
      !make_attn_map(&mk, a.k_rot, (int64_t)a.Hkv * kAD, a.T, (int64_t)a.Hkv * kAD,
                     CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
      !make_attn_map(&mv, a.v_h, (int64_t)a.Hkv * kAD, a.T, (int64_t)a.Hkv * kAD,
                     CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
    return cudaErrorInvalidValue;
  const int grid_tiles = (int)((a.T + kTileTok - 1) / kTileTok) + a.N;
  AttnParams ap{a.cu_seqlens, a.N, a.T, a.Hq, a.Hkv, grid_tiles,
                a.scale * 1.4426950408889634f, static_cast<const __nv_bfloat16*>(a.gate),
                a.gate_row_stride, static_cast<__nv_bfloat16*>(a.o), status};
  static bool attr_set = false;
  if (!attr_set) {
    e = cudaFuncSetAttribute(attn_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)A_SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const unsigned grid = (unsigned)grid_tiles * (unsigned)(a.Hq / 2);
  attn_prefill_kernel<<<grid, kAttnThreads, A_SMEM, a.stream>>>(mq, mk, mv, ap);
  return cudaGetLastError();
}

cudaError_t attention_status_word(const void* workspace, cudaStream_t stream, int* word) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  return cudaMemcpy(word, workspace, sizeof(int), cudaMemcpyDeviceToHost);
}

size_t attention_decode_workspace(int N, int Hq, int L_max) {
  const size_t S = (size_t)((L_max + kUnit - 1) / kUnit);
  return 256 + (size_t)N * Hq * kAD * 4 + (size_t)N * Hq * S * 2 * 4 +
         (size_t)N * Hq * S * kAD * 4;
}

template <int G>
cudaError_t launch_split(const DecParams& dp, dim3 grid, cudaStream_t stream) {
  const size_t smem = (size_t)kDecSmem;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn_decode_split_kernel<G>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  attn_decode_split_kernel<G><<<grid, 32 * kDecWarps, smem, stream>>>(dp);
  return cudaGetLastError();
}

cudaError_t launch_attention_decode(const AttnDecodeArgs& a) {
  if (a.N == 0) return cudaSuccess;
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  int* status = reinterpret_cast<int*>(ws);
  const int S = (a.L_max + kUnit - 1) / kUnit;
  float* q_rot = reinterpret_cast<float*>(ws + 256);
  float* part_ml = q_rot + (size_t)a.N * a.Hq * kAD;
  float* part_o = part_ml + (size_t)a.N * a.Hq * S * 2;
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), a.stream);
  if (e != cudaSuccess) return e;
  DecParams dp{static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
               static_cast<const __nv_bfloat16*>(a.v), static_cast<const __nv_bfloat16*>(a.gate),
               a.q_row_stride, a.k_row_stride, a.v_row_stride, a.gate_row_stride, a.wq, a.wk,
               static_cast<__half*>(a.k_cache), static_cast<__half*>(a.v_cache),
               a.cache_idx, a.cache_len, a.positions, a.N, a.P, a.L_max, a.Hq, a.Hkv, a.eps,
               a.rope_dims, log2((double)a.rope_base), a.scale * 1.4426950408889634f, q_rot,
               part_ml, part_o, S, static_cast<__nv_bfloat16*>(a.o), status};
  if (a.w_dtype == GDN_F32)
    attn_decode_prologue_kernel<float><<<a.N, 256, 0, a.stream>>>(dp);
  else
    attn_decode_prologue_kernel<__nv_bfloat16><<<a.N, 256, 0, a.stream>>>(dp);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((S + kDecWarps - 1) / kDecWarps), (unsigned)a.Hkv, (unsigned)a.N);
  switch (a.Hq / a.Hkv) {
    case 1: e = launch_split<1>(dp, grid, a.stream); break;
    case 2: e = launch_split<2>(dp, grid, a.stream); break;
    case 4: e = launch_split<4>(dp, grid, a.stream); break;
    case 6: e = launch_split<6>(dp, grid, a.stream); break;
    case 8: e = launch_split<8>(dp, grid, a.stream); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  attn_decode_combine_kernel<<<dim3((unsigned)a.Hq, (unsigned)a.N), kAD, 0, a.stream>>>(dp);
  return cudaGetLastError();
}

}  // namespace gdn
