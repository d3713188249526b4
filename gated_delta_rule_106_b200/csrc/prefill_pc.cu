// Chunked gated delta rule on B200: a persistent producer/consumer kernel.
//
// The chunked prefill path ("delta_rule_chunked", chunk = 64: "Agnes-3.0-
// Flash Preview" leaderboard commentary, section 二.1; fp32 recurrent state:
// model card, 架构 table) splits, per 64-token chunk, into work that does not
// depend on the state entering the chunk and work that does. With
// G_t = sum_{s<=t} log g_s and S0 the state entering a chunk of L tokens:
//   state-free:  A_ts = beta_t e^{G_t-G_s} k_t.k_s (s<t);  T = (I + A)^{-1}
//                W = T diag(beta e^G) K;  U = T diag(beta) V;
//                M_ts = e^{G_t-G_s} q_t.k_s (s<=t)
//   state chain: Delta = U - W S0^T
//                O     = scale (diag(e^G) Q S0^T + M Delta)
//                S_L   = e^{G_L} S0 + (diag(e^{G_L-G}) Delta)^T K
//
// One cooperative launch, one CTA per SM, two roles:
//  * state CTAs (about a third of the SMs) each own a list of (sequence,
//    value head) items and run their chunks in order. Per chunk: D1 = S0
//    [-W ; Q~]^T (N = 128: the S0 part of Delta and S0 q~ per token together,
//    Q~ = diag(e^G) Q), the Delta readout, then P = Delta'^T K (the state
//    update with Delta' = diag(e^{G_L-G}) Delta as binary16 high and low parts
//    against the exact binary16 image of the bf16 keys) and the M Delta
//    products, which accumulate onto S0 q~ in TMEM; the fp32 state stays in
//    registers (four threads per row). Few wide MMAs matter because each tcgen05.mma instruction costs
//    about the same time whether N is 64 or 128. A chunk's outputs are read
//    during the next chunk and leave as one TMA tensor store.
//  * prep CTAs run two independent 256-thread pipelines each; a pipeline claims
//    (item, chunk) work in chunk order from a global counter and computes the
//    state-free part: bf16 TMA tiles of K, Q, V; the Gram [K;Q] K^T on the
//    tensor cores (bf16, exact products: K K^T for A, Q K^T for M); decays; the
//    UT solve in fp32; W and U as bf16 hi/lo MMAs (~17 significant bits, unit
//    diagonal included); it writes binary16 images of [-W ; Q~] and
//    [K | M hi | M lo], U in fp32 and the chunk's decays straight into a ring
//    slot in the caller's workspace (6 slots per state CTA, ~97 KB each, L2-resident) and releases
//    its flag; the state CTA acquires it, bulk-copies the operand images into
//    shared memory and releases the slot once read.
// Deadlock freedom: all CTAs are co-resident (cooperative launch); a prep CTA
// works on claims in increasing order and a claim only waits on the
// consumption of an earlier step of the same state CTA. Every wait is
// bounded: waits on another CTA's flag by a settable limit (2 s unless
// gdn_set_wait_limit_ns changed it), waits on this CTA's own copies and MMAs
// by 2 s. On a timeout the CTA raises the abort word in the workspace, every
// CTA leaves its loops, waits for its own copies in flight and frees its
// tensor memory; a state CTA then writes NaN to the outputs (o and state_out)
// of every (sequence, head) it did not finish. gdn_chunked_prefill_status
// reads the abort word.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "gdn_common.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int kPcThreads = 512;
constexpr int kRing = 6;            // slots per state CTA: how far prep may run ahead
constexpr uint64_t kLimitNs = 2000000000ull;   // own copies and MMAs; default for flags

// ---- ring slot (global), 1024-aligned sections ---------------------------
// B operand of S0 [-W ; Q~]^T: K-major, [2 d_k blocks][128 rows][64], rows 0-63 = -W
// (token t), rows 64-127 = Q~ = diag(e^G) Q (token t), binary16.
constexpr uint32_t SL_WQ = 0;
// Four 8 KB blocks: K, MN-major [64 tokens s][64 d_k] (d_k 0-63, 64-127; the B
// operand of P = Delta'^T K; bf16 keys are exact in binary16), then the lower triangle of M
// (M[t][s] = M_ts for s <= t) as binary16 high and low parts, K-major [64 t][64 s]
// (the B operands of the M Delta products).
constexpr uint32_t SL_BKM = 32768;
constexpr uint32_t SL_OPS = 65536;     // bytes of the operand images above
// fp32 [0] = e^{G_L} (the chunk's total decay), [1 + t] = e^{G_L - G_t}
constexpr uint32_t SL_VEC = 65536;
constexpr uint32_t SL_VEC_BYTES = 272;  // 65 floats, rounded up to 16 bytes
constexpr uint32_t SL_UT = 66560;      // U fp32 [64 t][128 i] (copied to shared memory separately)
constexpr uint32_t SLOT_BYTES = 99328;
// state CTA use of a slot image buffer once its MMAs are done: the [-W ; Q~] area
// stages that step's outputs (o's dtype), the K/M area receives the next step's U
constexpr uint32_t S_STG_OFF = SL_WQ, S_UT_OFF = SL_BKM;

constexpr uint32_t CTRL_BYTES = 16384; // counter, abort word, per-state-CTA flags
constexpr int kFlagStride = 16;        // ints per state CTA: full[kRing], consumed

// ---- prep CTA shared memory ---------------------------------------------
// A prep CTA runs two independent pipelines of kPipeThreads threads (named
// barriers 1 and 2), each working on its own item, so that one pipeline's
// latency-bound phases overlap the other's. Per pipeline:
constexpr int kPipeThreads = kPcThreads / 2;
constexpr uint32_t PIPE_BYTES = 100352;
constexpr uint32_t PP_TILES = 0;       // [K0 8K | Q0 8K | K1 8K | Q1 8K | V0 8K | V1 8K] bf16,
                                       // TMA 128B swizzle; the solve scratch reuses Q0
constexpr int kLd = 68;                // row stride (floats) of the fp32 A and T tiles
constexpr uint32_t PP_AF = 49152;      // fp32 A [64][kLd]; after the solve: bf16 T' hi | lo
constexpr uint32_t PP_TF = 66560;      // fp32 T [64][kLd]
constexpr uint32_t PP_T2 = 83968;      // bf16 T'' hi | lo [64][64] each
constexpr uint32_t P_SMALL = 2 * PIPE_BYTES;
// ---- state CTA shared memory --------------------------------------------
constexpr uint32_t S_BUF = 0;          // 2 x slot operand images (SL_OPS each)
constexpr uint32_t S_VEC = 131072;     // 2 x slot decay vectors (512 bytes each)
constexpr uint32_t S_S0 = 132096;      // binary16 state, K-major [2 blocks][128 rows]
constexpr uint32_t S_DTH = 164864;     // Delta^T high, K-major A [128 d_v][64 t]
constexpr uint32_t S_DTL = 181248;     // Delta^T low
constexpr uint32_t S_DPH = 197632;     // Delta'^T high, Delta' = diag(e^{G_L-G}) Delta
constexpr uint32_t S_DPL = 214016;     // Delta'^T low
constexpr uint32_t S_SMALL = 230400;
constexpr uint32_t PC_SMEM_BYTES = S_SMALL + 1024;   // the state role needs the most
constexpr uint32_t PC_SMEM_ALLOC = PC_SMEM_BYTES + 1024;   // 227 KB: the sm_100 limit
static_assert(PC_SMEM_ALLOC <= 232448, "over the shared memory of a CTA");

// TMEM columns
// prep, per pipeline (256 columns each): Gram [128 x 64] at 0, then W^T as
// [hi part | lo part] column halves at 0 and U^T the same way at 128
constexpr uint32_t PT_GR = 0, PT_W = 0, PT_U = 128, PT_PIPE = 256, PT_COLS = 512;
// state: D1 = S0 [-W ; Q~]^T -> [Delta^T - U^T | OA = S0 Q~^T], in one of two column
//        sets by step parity (a step's outputs outlive the next step's D1), and
//        Delta_lo^T M_hi^T accumulated onto OA;  P = Delta'^T K (hi and lo parts);
//        OB = Delta_hi^T [M hi ; M lo]^T -> [OB_hh | OB_hl] (M with its diagonal).
//        o^T = scale (OA + OB_hh + OB_hl)
constexpr uint32_t ST_D1A = 0, ST_P = 128, ST_D1B = 256, ST_OB = 384, ST_COLS = 512;

struct PcParams {
  const void* g; const void* beta;
  const float* state_in; float* state_out;
  const int32_t* cu; int64_t T; int N; int H_k; int H_v; float scale;
  void* o;
  uint8_t* ws;          // workspace base
  int NS;               // state CTAs
  uint64_t wait_ns;     // limit of a wait on another CTA's flag
  // the whole layer (gdn_prefill_layer): pre-conv x [T, C] bf16 with row stride xs,
  // conv taps cw [C, 4] and bias cb (conv weight dtype), carried conv history
  // cs_in [N, 3, C] (bf16, may be null), q/k L2 epsilon; gated RMS-norm gate z
  // [T, H_v, 128] bf16, weight nw [128] (conv weight dtype), epsilon
  const void* x; int64_t xs; const void* cw; const void* cb; const void* cs_in; int C;
  float l2_eps;
  const void* z; const void* nw; float norm_eps;
};

constexpr int kCuCache = 513;   // sequences whose boundaries the prep CTAs keep on chip
struct PipeSmall {
  float G[64], beta[64], gamma[64], bg[64], tail[64];
  float gL;
  int claim;
  int ok;
  int abort;
  uint64_t bar_tma, bar_mma;
};
struct PrepSmall {
  int cu[kCuCache];
  int max_steps;
  uint32_t tmem;
  PipeSmall pipe[2];
};
struct StateSmall {
  uint32_t tmem;
  int ok;
  int pf;     // step r+1's slot was seen released (acquire) during step r
  uint64_t bar_slot[2], bar_ut[2], bar_dt, bar_p, bar_o;
};

__device__ __forceinline__ uint32_t swz(int r, int c) {
  return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}
__device__ __forceinline__ uint4 pack_half8(const float* f) {
  uint4 u;
  __half2* h = reinterpret_cast<__half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
  return u;
}
// hi/lo splits without round trips through the conversion unit (its
// throughput is a fraction of the ALU's): float(hi) is rebuilt from the bits.
// bf16 round-to-nearest-even with integer operations (finite inputs).
__device__ __forceinline__ uint32_t bf16_bits_rn(float x) {
  uint32_t u = __float_as_uint(x);
  u += 0x7fffu + ((u >> 16) & 1u);
  return u >> 16;
}
// 8 values -> bf16 high parts and bf16 low parts (x - hi), packed
__device__ __forceinline__ void split_bf8(const float* f, uint4& hi, uint4& lo) {
  uint32_t h[8], l[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    h[j] = bf16_bits_rn(f[j]);
    l[j] = bf16_bits_rn(f[j] - __uint_as_float(h[j] << 16));
  }
  hi = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16), h[6] | (h[7] << 16));
  lo = make_uint4(l[0] | (l[1] << 16), l[2] | (l[3] << 16), l[4] | (l[5] << 16), l[6] | (l[7] << 16));
}
// value of a finite binary16 given by its bits (low 16 bits of hb); exact
__device__ __forceinline__ float half_bits_value(uint32_t hb) {
  const float mag = __uint_as_float((hb & 0x7fffu) << 13) * 5.192296858534828e33f;  // * 2^112
  return __uint_as_float(__float_as_uint(mag) | ((hb & 0x8000u) << 16));
}
// 8 values -> binary16 high parts and binary16 low parts (x - hi), packed
__device__ __forceinline__ void split_half8(const float* f, uint4& hi, uint4& lo) {
  uint32_t hw[4], lw[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2 h2 = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
    const uint32_t hb = *reinterpret_cast<const uint32_t*>(&h2);
    const __half2 l2 = __floats2half2_rn(f[2 * i] - half_bits_value(hb & 0xffffu),
                                         f[2 * i + 1] - half_bits_value(hb >> 16));
    hw[i] = hb;
    lw[i] = *reinterpret_cast<const uint32_t*>(&l2);
  }
  hi = make_uint4(hw[0], hw[1], hw[2], hw[3]);
  lo = make_uint4(lw[0], lw[1], lw[2], lw[3]);
}

__device__ __forceinline__ int* flags_of(uint8_t* ws, int s) {
  return reinterpret_cast<int*>(ws + 128) + s * kFlagStride;
}
__device__ __forceinline__ uint8_t* slot_of(uint8_t* ws, int s, int r) {
  return ws + CTRL_BYTES + ((size_t)s * kRing + (size_t)(r % kRing)) * SLOT_BYTES;
}

// chunks of sequence n (clamped cu_seqlens)
__device__ __forceinline__ int seq_chunks(const int32_t* cu, int64_t T, int n, int64_t* s0,
                                          int64_t* s1) {
  int64_t a = clamp_t(cu[n], T), b = clamp_t(cu[n + 1], T);
  if (b < a) b = a;
  *s0 = a;
  *s1 = b;
  return (int)((b - a + kChunk - 1) / kChunk);
}
__device__ int steps_of(const PcParams& p, const int32_t* cu, int s) {
  int total = 0;
  int64_t a, b;
  for (int i = s; i < p.N * p.H_v; i += p.NS) total += seq_chunks(cu, p.T, i / p.H_v, &a, &b);
  return total;
}
// step r of state CTA s -> item i and chunk c (false if r is past its steps)
__device__ bool locate(const PcParams& p, const int32_t* cu, int s, int r, int* item, int* chunk) {
  int64_t a, b;
  for (int i = s; i < p.N * p.H_v; i += p.NS) {
    const int nc = seq_chunks(cu, p.T, i / p.H_v, &a, &b);
    if (r < nc) {
      *item = i;
      *chunk = r;
      return true;
    }
    r -= nc;
  }
  return false;
}

// One merge level of the blocked inverse of a 64x64 unit lower-triangular
// matrix: for each pair of b x b diagonal blocks already inverted (T11, T22),
// T21 = -T22 (A21 T11). T holds zeros above its diagonal; rows of A, T and
// X are read four floats at a time; at b = 32 each thread makes two adjacent
// outputs.
template <int b>
__device__ __forceinline__ void merge_level(const float* Af, float* Tf, float* Xs, int tid,
                                             uint32_t bar) {
  // Each active thread makes an RI x 2 block of outputs (rows i..i+RI-1,
  // columns j, j+1): row segments of A / T are read four floats at a time and
  // column pairs of T / X two at a time, so loads per FMA stay low.
  constexpr int bb = b * b, pairs = 64 / (2 * b);
  constexpr int RI = b >= 32 ? 4 : 2, RJ = 2;
  constexpr int tiles_i = b / RI, tiles_j = b / RJ;
  constexpr int threads = pairs * tiles_i * tiles_j;   // b=8: 64, 16: 128, 32: 128
  static_assert(threads <= kPipeThreads, "too many threads");
  const int pr = tid / (tiles_i * tiles_j);
  const int ti = (tid / tiles_j) % tiles_i, tj = tid % tiles_j;
  const int i0 = ti * RI, j0 = tj * RJ, o = 2 * b * pr;
  if (tid < threads) {
    float acc[RI][RJ];
#pragma unroll
    for (int a = 0; a < RI; ++a)
#pragma unroll
      for (int c = 0; c < RJ; ++c) acc[a][c] = 0.f;
#pragma unroll 2
    for (int m4 = 0; m4 < b / 4; ++m4) {
      float av[RI][4];
#pragma unroll
      for (int a = 0; a < RI; ++a) {
        const float4 v = reinterpret_cast<const float4*>(Af + (o + b + i0 + a) * kLd + o)[m4];
        av[a][0] = v.x; av[a][1] = v.y; av[a][2] = v.z; av[a][3] = v.w;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 t2 = *reinterpret_cast<const float2*>(Tf + (o + 4 * m4 + u) * kLd + o + j0);
#pragma unroll
        for (int a = 0; a < RI; ++a) {
          acc[a][0] = fmaf(av[a][u], t2.x, acc[a][0]);
          acc[a][1] = fmaf(av[a][u], t2.y, acc[a][1]);
        }
      }
    }
#pragma unroll
    for (int a = 0; a < RI; ++a)
      *reinterpret_cast<float2*>(Xs + pr * bb + (i0 + a) * b + j0) = make_float2(acc[a][0], acc[a][1]);
  }
  bar_sync_n(bar, kPipeThreads);
  if (tid < threads) {
    float acc[RI][RJ];
#pragma unroll
    for (int a = 0; a < RI; ++a)
#pragma unroll
      for (int c = 0; c < RJ; ++c) acc[a][c] = 0.f;
#pragma unroll 2
    for (int m4 = 0; m4 < b / 4; ++m4) {
      float tv[RI][4];
#pragma unroll
      for (int a = 0; a < RI; ++a) {
        const float4 v = reinterpret_cast<const float4*>(Tf + (o + b + i0 + a) * kLd + o + b)[m4];
        tv[a][0] = v.x; tv[a][1] = v.y; tv[a][2] = v.z; tv[a][3] = v.w;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 x2 = *reinterpret_cast<const float2*>(Xs + pr * bb + (4 * m4 + u) * b + j0);
#pragma unroll
        for (int a = 0; a < RI; ++a) {
          acc[a][0] = fmaf(tv[a][u], x2.x, acc[a][0]);
          acc[a][1] = fmaf(tv[a][u], x2.y, acc[a][1]);
        }
      }
    }
#pragma unroll
    for (int a = 0; a < RI; ++a)
      *reinterpret_cast<float2*>(Tf + (o + b + i0 + a) * kLd + o + j0) =
          make_float2(-acc[a][0], -acc[a][1]);
  }
  bar_sync_n(bar, kPipeThreads);
}

// The layer's prologue inside a prep pipeline: the V tile (value head h) of
// the chunk at t0 (L tokens of sequence n, which starts at s0) from the
// pre-conv input: causal conv k=4 (+ bias) over rows t0-3 .. t0+63 and SiLU,
// rounded to bf16 into the 128-byte-swizzled [64 tokens][64 channels] blocks
// that the tensor cores read (the layout the tensor-map loads of the plain
// path produce). The q and k heads, which all value heads of a key head share,
// come convolved and normed from a separate conv launch into a scratch buffer
// and load by TMA. Rows before the sequence start come from the carried conv
// history (zeros if none); tokens at or past L are written as zeros. Warps 0-3
// take 16 tokens each; lane = 4 channels. The arithmetic (and its order) is the
// conv kernel's, so the tile holds exactly the values that kernel would store.
template <class Tw>
__device__ __forceinline__ void conv_fill_v(const PcParams& p, uint8_t* vv, int n, int h,
                                            int64_t s0, int64_t t0, int L, int warp, int lane) {
  const int c = (2 * p.H_k + h) * kHeadDim + lane * 4;
  const Tw* w = static_cast<const Tw*>(p.cw);
  const Tw* bias = static_cast<const Tw*>(p.cb);
  float wt[4][4], b[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    b[e] = bias ? to_f32(bias[c + e]) : 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) wt[e][j] = to_f32(w[(c + e) * 4 + j]);
  }
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(p.x);
  const __nv_bfloat16* cs = static_cast<const __nv_bfloat16*>(p.cs_in);
  // the pre-conv row of chunk token tt (tt may be -3..-1), as loaded (4 bf16)
  auto load_row = [&](int tt) -> uint2 {
    const int64_t tg = t0 + tt;
    if (tg >= s0 && tg < p.T) return __ldg(reinterpret_cast<const uint2*>(x + tg * p.xs + c));
    if (tg < s0 && cs)
      return __ldg(reinterpret_cast<const uint2*>(cs + ((int64_t)n * 3 + 3 + (tg - s0)) * p.C + c));
    return make_uint2(0u, 0u);
  };
  auto unpack = [](uint2 u, float (&f)[4]) {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 bb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    f[0] = a.x; f[1] = a.y; f[2] = bb.x; f[3] = bb.y;
  };
  uint8_t* tile = vv + (lane >> 4) * 8192;
  const int chunk = (lane & 15) >> 1, sub = (lane & 1) * 8;
  const int tb = warp * 16;
  uint2 raw[19];
#pragma unroll
  for (int i = 0; i < 19; ++i) raw[i] = load_row(tb - 3 + i);   // every load issued first
  float h0[4], h1[4], h2[4];
  unpack(raw[0], h0);
  unpack(raw[1], h1);
  unpack(raw[2], h2);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int tt = tb + i;
    float h3[4], out[4];
    unpack(raw[3 + i], h3);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float a = fmaf(wt[e][3], h3[e], fmaf(wt[e][2], h2[e], fmaf(wt[e][1], h1[e], fmaf(wt[e][0], h0[e], b[e]))));
      out[e] = silu(a);
    }
    const bool live = tt < L;
    const __nv_bfloat162 lo = __floats2bfloat162_rn(live ? out[0] : 0.f, live ? out[1] : 0.f);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(live ? out[2] : 0.f, live ? out[3] : 0.f);
    *reinterpret_cast<uint2*>(tile + swz(tt, chunk) + sub) =
        make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      h0[e] = h1[e];
      h1[e] = h2[e];
      h2[e] = h3[e];
    }
  }
}

// ===================================================================== prep ==
template <class Tg, bool Fused, class Tw>
__device__ void prep_role(const PcParams& p, const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                          const CUtensorMap* tm_v, uint8_t* sm) {
  PrepSmall& sh = *reinterpret_cast<PrepSmall*>(sm + P_SMALL);
  int* ctrl = reinterpret_cast<int*>(p.ws);         // [0] claim counter, [1] abort word

  const int tid = threadIdx.x, lane = tid & 31;
  const int pl = tid / kPipeThreads;                // pipeline
  const int ptid = tid % kPipeThreads, warp = ptid >> 5;
  const int q4 = warp & 3, cg = warp >> 2;          // TMEM lane quadrant, column half
  const int row = (q4 << 5) | lane;
  const uint32_t lane_base = (uint32_t)(q4 << 5) << 16;
  const uint32_t bar = 1 + pl;
  // lane 0 of the pipeline's last warp claims the next item during the solve
  // (where that warp is idle) and starts its tile loads once the current
  // item's tiles are no longer read
  constexpr int kIssuer = kPipeThreads - 32;
  PipeSmall& ss = sh.pipe[pl];
  uint8_t* pb = sm + pl * PIPE_BYTES;
  float* Af = reinterpret_cast<float*>(pb + PP_AF);
  float* Tf = reinterpret_cast<float*>(pb + PP_TF);
  float* Xs = reinterpret_cast<float*>(pb + PP_TILES + 8192);   // over Q0 once it is dead
  uint8_t* kq = pb + PP_TILES;                      // [K0 | Q0 | K1 | Q1]
  uint8_t* vv = kq + 32768;                         // [V0 | V1]

  if (tid < 32) {
    tmem_alloc(&sh.tmem, PT_COLS);
    tmem_relinquish();
  }
  if (tid == 32) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.pipe[i].bar_tma, 1);
      mbar_init(&sh.pipe[i].bar_mma, 1);
    }
    fence_mbar_init();
  }
  if (tid == 64) {
    prefetch_tmap(tm_q);
    prefetch_tmap(tm_k);
    prefetch_tmap(tm_v);
  }
  if (tid == 0) sh.max_steps = 0;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem + pl * PT_PIPE;
  const bool cu_on_chip = p.N + 1 <= kCuCache;
  if (cu_on_chip)
    for (int i = tid; i <= p.N; i += kPcThreads) sh.cu[i] = __ldg(p.cu + i);
  __syncthreads();
  const int32_t* cu = cu_on_chip ? sh.cu : p.cu;
  for (int s = tid; s < p.NS; s += kPcThreads) atomicMax(&sh.max_steps, steps_of(p, cu, s));
  __syncthreads();
  const int64_t E = (int64_t)p.NS * sh.max_steps;

  // next existing (state CTA, step) item, in global claim order (one thread)
  auto claim = [&]() -> int {
    int x, it_, c_;
    do {
      x = atomicAdd(&ctrl[0], 1);
    } while (x < E && !locate(p, cu, x % p.NS, x / p.NS, &it_, &c_));
    return x;
  };
  // TMA of item x's K, Q (key head) and V (value head) tiles; the layer's form
  // loads K and Q from the q/k conv scratch and convolves V itself
  auto issue_tiles = [&](int x) {
    int it_, c_;
    locate(p, cu, x % p.NS, x / p.NS, &it_, &c_);
    const int n_ = it_ / p.H_v, h_ = it_ % p.H_v, kh_ = h_ / (p.H_v / p.H_k);
    int64_t a_, b_;
    seq_chunks(cu, p.T, n_, &a_, &b_);
    const int y = (int)(a_ + (int64_t)c_ * kChunk);
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(&ss.bar_tma, (Fused ? 4 : 6) * 8192);
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      tma_load_2d(kq + b * 16384, tm_k, kh_ * kHeadDim + b * 64, y, &ss.bar_tma);
      tma_load_2d(kq + b * 16384 + 8192, tm_q, kh_ * kHeadDim + b * 64, y, &ss.bar_tma);
      if (!Fused) tma_load_2d(vv + b * 8192, tm_v, h_ * kHeadDim + b * 64, y, &ss.bar_tma);
    }
  };
  bool pend = false;   // kIssuer: tile loads in flight that no item has waited on
  int next = 0;        // kIssuer: the claimed next item
  if (ptid == kIssuer) {
    const int x = claim();
    ss.claim = x;
    if (x < E) {
      issue_tiles(x);
      pend = true;
    }
  }
  bar_sync_n(bar, kPipeThreads);
  int e = ss.claim;
  uint32_t tma_par = 0, mma_par = 0;
  const uint32_t a_kq = smem_u32(kq), a_v = smem_u32(vv);
  const uint32_t a_t1 = smem_u32(pb + PP_AF), a_t2 = smem_u32(pb + PP_T2);
  const uint32_t id_gram = idesc_bf16(128, 64, false, false);
  const uint32_t id_mn = idesc_bf16(128, 128, true, false);

  while (e < E) {
    const int s = e % p.NS, r = e / p.NS;
    int item = 0, c = 0;
    locate(p, cu, s, r, &item, &c);
    const int n = item / p.H_v, h = item % p.H_v;
    int64_t s0, s1;
    seq_chunks(cu, p.T, n, &s0, &s1);
    const int64_t t0 = s0 + (int64_t)c * kChunk;
    const int L = (int)((s1 - t0) < kChunk ? (s1 - t0) : kChunk);
    uint8_t* slot = slot_of(p.ws, s, r);
    bool ok = true;

    // the slot is written directly: wait until step r - kRing has been consumed
    // (the layer's form waits in warp 6, which has no share of the conv)
    if (ptid == (Fused ? 192 : 0))
      ss.ok = wait_flag_ge(flags_of(p.ws, s) + kRing, r + 1 - kRing, &ctrl[1], p.wait_ns);
    if constexpr (Fused) {   // the chunk's v tile from the pre-conv input
      if (warp < 4) conv_fill_v<Tw>(p, vv, n, h, s0, t0, L, warp, lane);
    }
    if (warp == (Fused ? 7 : 1)) {   // gates: cumulative log-decay and derived vectors
      const Tg* g = static_cast<const Tg*>(p.g);
      const Tg* bt = static_cast<const Tg*>(p.beta);
      float lg[2], be[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int t = 2 * lane + j;
        lg[j] = 0.f;
        be[j] = 0.f;
        if (t < L) {
          const int64_t idx = (t0 + t) * p.H_v + h;
          lg[j] = logf(fmaxf(to_f32(g[idx]), 1.17549435e-38f));
          be[j] = to_f32(bt[idx]);
        }
      }
      float incl = lg[0] + lg[1];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      const float excl = incl - (lg[0] + lg[1]);
      const float Gl = __shfl_sync(0xffffffffu, incl, 31);
      const float Gt[2] = {excl + lg[0], excl + lg[0] + lg[1]};
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int t = 2 * lane + j;
        const float gam = __expf(Gt[j]);
        ss.G[t] = Gt[j];
        ss.beta[t] = be[j];
        ss.gamma[t] = gam;
        ss.bg[t] = be[j] * gam;
        ss.tail[t] = __expf(Gl - Gt[j]);
      }
      if (lane == 0) ss.gL = __expf(Gl);
    }
    if constexpr (Fused) fence_proxy_async_smem();   // the tensor cores read the v tile
    ok = mbar_wait_bounded(&ss.bar_tma, tma_par, kLimitNs);
    if (ok) {   // a phase seen complete by this thread
      tma_par ^= 1;
      if (ptid == kIssuer) pend = false;
    }
    bar_sync_n(bar, kPipeThreads);
    ok = ok && ss.ok;
    if (bar_or_n(bar, kPipeThreads, !ok)) goto fail;

    if (L < kChunk) {   // rows past the sequence end hold other data: zero them
      // (the layer's v tile has them zero already)
      for (int idx = ptid; idx < (Fused ? 2048 : 3072); idx += kPipeThreads) {
        const int rr = (idx & 511) >> 3;
        if (rr >= L) {
          uint8_t* ptr = idx < 2048 ? kq + idx * 16 : vv + (idx - 2048) * 16;
          *reinterpret_cast<uint4*>(ptr) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      bar_sync_n(bar, kPipeThreads);
    }
    // ---- Gram [K;Q] K^T (bf16, exact products): rows 0-63 give K K^T, rows
    //      64-127 the query-key products Q K^T ----
    if (ptid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
        mma_f16(tmem + PT_GR, sw128_desc(a_kq + off, 16, 1024),
                sw128_desc(a_kq + off, 16, 1024), id_gram, kk > 0);
      }
      mma_commit(&ss.bar_mma);
    }
    // meanwhile: binary16 images of K (exact: bf16 values) and Q~ = diag(gamma) Q,
    // straight to the slot
#pragma unroll 2
    for (int idx = ptid; idx < 2048; idx += kPipeThreads) {
      const int which = idx >> 10, b = (idx >> 9) & 1, x = idx & 511;
      const uint8_t* src = kq + b * 16384 + which * 8192 + x * 16;
      float f[8];
      load8(reinterpret_cast<const __nv_bfloat16*>(src), f);
      const float sc = which == 0 ? 1.f : ss.gamma[x >> 3];
#pragma unroll
      for (int u = 0; u < 8; ++u) f[u] *= sc;
      uint8_t* dst = which == 0 ? slot + SL_BKM + b * 8192 + x * 16
                                : slot + SL_WQ + b * 16384 + 8192 + x * 16;
      *reinterpret_cast<uint4*>(dst) = pack_half8(f);
    }
    ok = mbar_wait_bounded(&ss.bar_mma, mma_par, kLimitNs);
    mma_par ^= 1;
    tc_fence_after();
    if (q4 < 2) {
      // lanes 0-63 (key token s = row), columns x = 32cg..32cg+31:
      // A[s][x] = beta_s e^{G_s-G_x} k_s.k_x for x < s (the solve reads no other entry)
      const int s2 = row, c0 = 32 * cg;
      if (!(q4 == 0 && cg == 1)) {
        const float Gs = ss.G[s2], bs = ss.beta[s2];
        float v[32];
        tmem_ld32(tmem + lane_base + PT_GR + c0, v);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float a4[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int x = c0 + 4 * q + u;
            a4[u] = (x < s2) ? bs * __expf(Gs - ss.G[x]) * v[4 * q + u] : 0.f;
          }
          *reinterpret_cast<float4*>(Af + s2 * kLd + c0 + 4 * q) = make_float4(a4[0], a4[1], a4[2], a4[3]);
        }
      }
    } else {
      // lanes 64-127 (query token t = row - 64), columns s = 32cg..32cg+31:
      // M[t][s] = e^{G_t-G_s} q_t.k_s for s <= t as binary16 high and low parts
      const int t = row - 64, c0 = 32 * cg;
      uint8_t* mh = slot + SL_BKM + 2 * 8192;
      uint8_t* ml = slot + SL_BKM + 3 * 8192;
      if (q4 == 2 && cg == 1) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          *reinterpret_cast<uint4*>(mh + swz(t, 4 * cg + q)) = make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(ml + swz(t, 4 * cg + q)) = make_uint4(0, 0, 0, 0);
        }
      } else {
        const float Gt = ss.G[t];
        float v[32];
        tmem_ld32(tmem + lane_base + PT_GR + c0, v);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float m8[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int s2 = c0 + 8 * q + u;
            m8[u] = (s2 <= t) ? __expf(Gt - ss.G[s2]) * v[8 * q + u] : 0.f;
          }
          uint4 hi, lo;
          split_half8(m8, hi, lo);
          *reinterpret_cast<uint4*>(mh + swz(t, 4 * cg + q)) = hi;
          *reinterpret_cast<uint4*>(ml + swz(t, 4 * cg + q)) = lo;
        }
      }
    }
    tc_fence_before();
    if (bar_or_n(bar, kPipeThreads, !ok)) goto fail;

    if (ptid == kIssuer) {
      next = claim();
      ss.claim = next;
    }
    // ---- T = (I + A)^{-1}: 8x8 diagonal blocks by forward substitution,
    //      then pairwise merges 8 -> 16 -> 32 -> 64:  T21 = -T22 A21 T11 ----
    for (int idx = ptid; idx < 16 * kLd; idx += kPipeThreads)
      reinterpret_cast<float4*>(Tf)[idx] = make_float4(0.f, 0.f, 0.f, 0.f);
    bar_sync_n(bar, kPipeThreads);
    if (ptid < 64) {
      const int B = ptid >> 3, j = ptid & 7;
      float a[8][8], x[8];
#pragma unroll
      for (int rr = 1; rr < 8; ++rr)
#pragma unroll
        for (int m = 0; m < rr; ++m) a[rr][m] = Af[(8 * B + rr) * kLd + 8 * B + m];
#pragma unroll
      for (int rr = 0; rr < 8; ++rr) {
        float acc = (rr == j) ? 1.f : 0.f;
#pragma unroll
        for (int m = 0; m < rr; ++m) acc = fmaf(-a[rr][m], x[m], acc);
        x[rr] = acc;
      }
#pragma unroll
      for (int rr = 0; rr < 8; ++rr) Tf[(8 * B + rr) * kLd + 8 * B + j] = x[rr];
    }
    bar_sync_n(bar, kPipeThreads);
    merge_level<8>(Af, Tf, Xs, ptid, bar);
    merge_level<16>(Af, Tf, Xs, ptid, bar);
    merge_level<32>(Af, Tf, Xs, ptid, bar);
    // T' = T diag(beta e^G) (over A, which is no longer read), T'' = T diag(beta)
    // (unit diagonal included) as bf16 hi/lo K-major B images [t][s]
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int t = (ptid >> 3) + 32 * h2, c8 = ptid & 7;
      float pa[8], pb2[8];
      const float4 t0v = *reinterpret_cast<const float4*>(Tf + t * kLd + c8 * 8);
      const float4 t1v = *reinterpret_cast<const float4*>(Tf + t * kLd + c8 * 8 + 4);
      const float tv[8] = {t0v.x, t0v.y, t0v.z, t0v.w, t1v.x, t1v.y, t1v.z, t1v.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int s2 = c8 * 8 + j;
        const float val = (s2 < t) ? tv[j] : (s2 == t ? 1.f : 0.f);
        pa[j] = val * ss.bg[s2];
        pb2[j] = val * ss.beta[s2];
      }
      uint4 hi, lo;
      split_bf8(pa, hi, lo);
      *reinterpret_cast<uint4*>(pb + PP_AF + swz(t, c8)) = hi;
      *reinterpret_cast<uint4*>(pb + PP_AF + 8192 + swz(t, c8)) = lo;
      split_bf8(pb2, hi, lo);
      *reinterpret_cast<uint4*>(pb + PP_T2 + swz(t, c8)) = hi;
      *reinterpret_cast<uint4*>(pb + PP_T2 + 8192 + swz(t, c8)) = lo;
    }
    fence_proxy_async_smem();
    bar_sync_n(bar, kPipeThreads);
    // ---- W^T = K^T T'^T, U^T = V^T T''^T: B = [hi ; lo] stacked (N = 128), the
    //      two column halves are summed in the readout ----
    if (ptid == 0) {
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint64_t ak = sw128_desc(a_kq + ks * 2048, 16384, 1024);
        const uint64_t av = sw128_desc(a_v + ks * 2048, 8192, 1024);
        mma_f16(tmem + PT_W, ak, sw128_desc(a_t1 + ks * 32, 16, 1024), id_mn, ks > 0);
        mma_f16(tmem + PT_U, av, sw128_desc(a_t2 + ks * 32, 16, 1024), id_mn, ks > 0);
      }
      mma_commit(&ss.bar_mma);
    }
    ok = mbar_wait_bounded(&ss.bar_mma, mma_par, kLimitNs);
    mma_par ^= 1;
    tc_fence_after();
    // the tiles are free: start the next item's loads
    if (ptid == kIssuer && ok && next < E) {
      issue_tiles(next);
      pend = true;
    }
    {
      float* ut = reinterpret_cast<float*>(slot + SL_UT);
      // -W, K-major: row = token t, 64 d_k per block (this thread's d_k column = row)
      uint8_t* blk = slot + SL_WQ + (row >> 6) * 16384;
      const uint32_t col = (row & 7) * 2;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int tb0 = 32 * cg + 16 * hh;
        float v[16], vl[16];
        tmem_ld16(tmem + lane_base + PT_W + tb0, v);
        tmem_ld16(tmem + lane_base + PT_W + 64 + tb0, vl);
#pragma unroll
        for (int j = 0; j < 16; j += 2) {
          const int t = tb0 + j;
          const __half2 h2 = __floats2half2_rn(-(v[j] + vl[j]), -(v[j + 1] + vl[j + 1]));
          const uint32_t hb = *reinterpret_cast<const uint32_t*>(&h2);
          *reinterpret_cast<uint16_t*>(blk + swz(t, (row & 63) >> 3) + col) = (uint16_t)(hb & 0xffffu);
          *reinterpret_cast<uint16_t*>(blk + swz(t + 1, (row & 63) >> 3) + col) = (uint16_t)(hb >> 16);
        }
        tmem_ld16(tmem + lane_base + PT_U + tb0, v);
        tmem_ld16(tmem + lane_base + PT_U + 64 + tb0, vl);
#pragma unroll
        for (int j = 0; j < 16; ++j) ut[(tb0 + j) * kHeadDim + row] = v[j] + vl[j];
      }
      float* vec = reinterpret_cast<float*>(slot + SL_VEC);
      if (ptid == 0) vec[0] = ss.gL;
      if (ptid < kChunk) vec[1 + ptid] = ss.tail[ptid];
    }
    fence_proxy_async_all();   // the state CTA reads the slot with a bulk copy
    tc_fence_before();
    if (ptid == 0) ss.abort = ld_acquire(&ctrl[1]);
    if (bar_or_n(bar, kPipeThreads, !ok)) goto fail;
    // every thread's slot writes precede this release (barrier, then gpu fence)
    if (ptid == 0) {
      __threadfence();
      st_release(flags_of(p.ws, s) + (r % kRing), r + 1);
    }
    e = ss.claim;
    if (ss.abort != 0) break;
    continue;
  fail:
    if (ptid == 0) atomicExch(&ctrl[1], 1);
    break;
  }
  if (ptid == kIssuer && pend) mbar_wait_bounded(&ss.bar_tma, tma_par, kLimitNs);
  tc_fence_before();
  __syncthreads();
  if (tid < 32) tmem_dealloc(sh.tmem, PT_COLS);
}

// ==================================================================== state ==
template <class To, bool Fused, class Tw>
__device__ void state_role(const PcParams& p, const CUtensorMap* tm_o, uint8_t* sm, int s) {
  StateSmall& ss = *reinterpret_cast<StateSmall*>(sm + S_SMALL);
  int* ctrl = reinterpret_cast<int*>(p.ws);
  int* flags = flags_of(p.ws, s);
  To* o = static_cast<To*>(p.o);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3, cg = warp >> 2;     // TMEM lane quadrant, column group (0..3)
  const int row = (q4 << 5) | lane;            // state row (d_v index)
  const uint32_t lane_base = (uint32_t)(q4 << 5) << 16;

  if (warp == 0) {
    tmem_alloc(&ss.tmem, ST_COLS);
    tmem_relinquish();
  }
  if (tid == 32) {
    mbar_init(&ss.bar_slot[0], 1);
    mbar_init(&ss.bar_slot[1], 1);
    mbar_init(&ss.bar_ut[0], 1);
    mbar_init(&ss.bar_ut[1], 1);
    mbar_init(&ss.bar_dt, 1);
    mbar_init(&ss.bar_p, 1);
    mbar_init(&ss.bar_o, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ss.tmem;
  const int total = steps_of(p, p.cu, s);
  const uint32_t a_s0 = smem_u32(sm + S_S0), a_dth = smem_u32(sm + S_DTH);
  const uint32_t a_dtl = smem_u32(sm + S_DTL);
  const uint32_t a_dph = smem_u32(sm + S_DPH), a_dpl = smem_u32(sm + S_DPL);
  const uint32_t id_d1 = idesc_f16(128, 128, false, false);
  const uint32_t id_p = idesc_f16(128, 128, false, true);
  const uint32_t id_ob = idesc_f16(128, 128, false, false);
  const uint32_t id_d3 = idesc_f16(128, 64, false, false);

  int issued = 0;                 // slot image copies issued (thread 32's view)
  int ut_issued = 0;              // U^T copies issued (thread 32's view)
  uint32_t par_dt = 0, par_p = 0, par_o = 0;
  bool ok = true;
  int r = 0;
  // Copy the operand image of `step` into its buffer; unless `acquired`, first
  // wait (bounded) for the producer's release of that slot.
  auto issue_copy = [&](int step, bool acquired) -> bool {
    int* full = flags + (step % kRing);
    if (!acquired && !wait_flag_ge(full, step + 1, &ctrl[1], p.wait_ns)) return false;
    fence_proxy_async_all();
    bulk_wait_read_all();   // an output store of this thread may still read the buffer
    uint64_t* bar = &ss.bar_slot[step & 1];
    uint8_t* src = slot_of(p.ws, s, step);
    mbar_arrive_expect_tx(bar, SL_OPS + SL_VEC_BYTES);
    bulk_g2s(sm + S_BUF + (step & 1) * SL_OPS, src, SL_OPS, bar);
    bulk_g2s(sm + S_VEC + (step & 1) * 512, src + SL_VEC, SL_VEC_BYTES, bar);
    return true;
  };
  // U^T of `step` goes to the other buffer's K/M area, free once step-1's output
  // MMAs are done (the caller has acquired the slot and fenced the async proxy)
  auto issue_ut = [&](int step) {
    const int ub = (step + 1) & 1;
    mbar_arrive_expect_tx(&ss.bar_ut[ub], 32768);
    bulk_g2s(sm + S_BUF + ub * SL_OPS + S_UT_OFF, slot_of(p.ws, s, step) + SL_UT, 32768,
             &ss.bar_ut[ub]);
  };
  // staged outputs of an earlier step (o's dtype, [64 t][128 rows] over a buffer's
  // [-W ; Q~] area): a whole bf16 chunk leaves as one tensor store issued by thread
  // 32, which waits for its read before it next copies into that buffer; a ragged
  // chunk (whose box would reach the next sequence) or fp32 goes as 16-byte rows
  auto emit_out = [&](const uint8_t* stage, int64_t ot0, int oL, int oh) {
    if (sizeof(To) == 2 && oL == kChunk) {
      if (tid == 32) {
        tma_store_2d(tm_o, oh * kHeadDim, (int)ot0, stage);
        bulk_commit();
      }
      return;
    }
    constexpr int kRowChunks = kHeadDim * (int)sizeof(To) / 16;
#pragma unroll
    for (int ci = tid; ci < kChunk * kRowChunks; ci += kPcThreads) {
      const int t = ci / kRowChunks, part = ci % kRowChunks;
      if (t < oL)
        *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(o + ((ot0 + t) * p.H_v + oh) * kHeadDim) +
                                  part * 16) = *reinterpret_cast<const uint4*>(stage + ci * 16);
    }
  };
  // this thread's 16 outputs (row, tokens 16cg..16cg+15) of the step whose D1
  // went to column set d1c: o^T = scale (OA + OB_hh + OB_hl)
  auto load_out = [&](uint32_t d1c, float (&ov)[16]) {
    float part[16];
    tmem_ld16(tmem + lane_base + d1c + 64 + 16 * cg, ov);
    tmem_ld16(tmem + lane_base + ST_OB + 16 * cg, part);
#pragma unroll
    for (int j = 0; j < 16; ++j) ov[j] += part[j];
    tmem_ld16(tmem + lane_base + ST_OB + 64 + 16 * cg, part);
#pragma unroll
    for (int j = 0; j < 16; ++j) ov[j] = p.scale * (ov[j] + part[j]);
  };
  // [64 t][128 rows] stage in o's dtype over a buffer's [-W ; Q~] area
  auto stage_out = [&](uint8_t* sbuf, const float (&ov)[16]) {
    if constexpr (sizeof(To) == 2) {
      uint16_t* stg = reinterpret_cast<uint16_t*>(sbuf + S_STG_OFF);
#pragma unroll
      for (int j = 0; j < 16; j += 2) {
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(ov[j], ov[j + 1]);
        const uint32_t hb = *reinterpret_cast<const uint32_t*>(&h2);
        stg[(16 * cg + j) * kHeadDim + row] = (uint16_t)(hb & 0xffffu);
        stg[(16 * cg + j + 1) * kHeadDim + row] = (uint16_t)(hb >> 16);
      }
    } else {
      float* stg = reinterpret_cast<float*>(sbuf + S_STG_OFF);
#pragma unroll
      for (int j = 0; j < 16; ++j) stg[(16 * cg + j) * kHeadDim + row] = ov[j];
    }
  };
  // the layer's epilogue: gated RMS-norm of a staged [64 t][128 i] output tile in
  // place, y = o / sqrt(mean(o^2) + eps) * w * SiLU(z) per token (8 threads per
  // token, 16 channels each); the staged o is already in o's dtype, as the plain
  // path would store it
  auto norm_stage = [&](uint8_t* stage, int64_t ot0, int oL, int oh) {
    const int t = tid >> 3, c0 = (tid & 7) * 16;
    To* sv = reinterpret_cast<To*>(stage) + t * kHeadDim + c0;
    float ssum = 0.f;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      float v[8];
      load8(sv + 8 * q, v);
#pragma unroll
      for (int j = 0; j < 8; ++j) ssum = fmaf(v[j], v[j], ssum);
    }
    ssum += __shfl_xor_sync(0xffffffffu, ssum, 1);
    ssum += __shfl_xor_sync(0xffffffffu, ssum, 2);
    ssum += __shfl_xor_sync(0xffffffffu, ssum, 4);
    if (t < oL) {
      const float inv = rsqrtf(ssum * (1.0f / kHeadDim) + p.norm_eps);
      const __nv_bfloat16* zr =
          static_cast<const __nv_bfloat16*>(p.z) + ((ot0 + t) * p.H_v + oh) * kHeadDim + c0;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        float v[8], zz[8], wv[8];
        load8(sv + 8 * q, v);
        load8(zr + 8 * q, zz);
        load8(static_cast<const Tw*>(p.nw) + c0 + 8 * q, wv);
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = v[j] * inv * wv[j] * silu(zz[j]);
        store8(sv + 8 * q, v);
      }
    }
  };
  bool staged = false;            // (fused) a normed tile waits in the stage of buffer r & 1
  int64_t stg_t0 = 0;
  int stg_L = 0, stg_h = 0;
  bool pend = false;              // a step's outputs wait in TMEM
  int64_t pend_t0 = 0;
  int pend_L = 0, pend_h = 0;
  int fail_item = -1;             // the item being worked on when a wait gave up

  for (int i = s; i < p.N * p.H_v && ok; i += p.NS) {
    const int n = i / p.H_v, h = i % p.H_v;
    int64_t s0, s1;
    const int nch = seq_chunks(p.cu, p.T, n, &s0, &s1);
    const int64_t nh = (int64_t)n * p.H_v + h;
    float S[32];
    {
      const float* src = p.state_in ? p.state_in + (nh * kHeadDim + row) * kHeadDim + cg * 32 : nullptr;
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        float4 v = src ? *reinterpret_cast<const float4*>(src + j) : make_float4(0.f, 0.f, 0.f, 0.f);
        S[j] = v.x; S[j + 1] = v.y; S[j + 2] = v.z; S[j + 3] = v.w;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4*>(sm + S_S0 + (cg >> 1) * 16384 + swz(row, (cg & 1) * 4 + q)) =
            pack_half8(S + 8 * q);
    }
    fence_proxy_async_smem();
    __syncthreads();

    for (int c = 0; c < nch; ++c, ++r) {
      const int b = r & 1;
      uint8_t* buf = sm + S_BUF + b * SL_OPS;
      const uint32_t a_buf = smem_u32(buf);
      const int64_t t0 = s0 + (int64_t)c * kChunk;
      const int L = (int)((s1 - t0) < kChunk ? (s1 - t0) : kChunk);
      if (tid == 32) {
        ss.ok = 1;
        if (issued == r) {
          if (issue_copy(r, false)) issued = r + 1;
          else ss.ok = 0;
        }
        if (ss.ok && ut_issued == r) {
          issue_ut(r);
          ut_issued = r + 1;
        }
      }
      __syncthreads();
      if (!ss.ok) { ok = false; break; }
      uint8_t* ubuf = sm + S_BUF + ((r + 1) & 1) * SL_OPS;   // U^T of step r
      const uint32_t d1 = (r & 1) ? ST_D1B : ST_D1A;
      const uint32_t ut_par = (uint32_t)((r >> 1) & 1);        // step r is its r>>1-th use
      if (!mbar_wait_bounded(&ss.bar_slot[b], (uint32_t)((r >> 1) & 1), kLimitNs)) ok = false;
      if (__syncthreads_or(!ok)) { ok = false; break; }
      // ---- D1 = S0 [-W ; Q~]^T: Delta^T - U^T and OA (critical path) ----
      if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_f16(tmem + d1, sw128_desc(a_s0 + off, 16, 1024),
                  sw128_desc(a_buf + SL_WQ + off, 16, 1024), id_d1, kk > 0);
        }
        mma_commit(&ss.bar_dt);
      }
      // gpu-scope flag work, in the shadow of D1 (each access costs a memory
      // round trip): release slot r (its image is in shared memory, its U^T loads
      // were issued above) and look, with acquire, whether step r+1 is published;
      // the barrier after the readout carries that to thread 32, which copies
      if (tid == 64) {
        if (mbar_wait_bounded(&ss.bar_ut[(r + 1) & 1], ut_par, kLimitNs))
          st_release(flags + kRing, r + 1);
        else
          ok = false;
      }
      if (tid == 96)
        ss.pf = (r + 1 < total && ld_acquire(flags + ((r + 1) % kRing)) >= r + 2) ? 1 : 0;
      // step r-1's outputs (its MMAs completed before the last barrier)
      float ov[16];
      if (pend) {
        tc_fence_after();
        load_out((r & 1) ? ST_D1A : ST_D1B, ov);
      }
      if (!mbar_wait_bounded(&ss.bar_ut[(r + 1) & 1], ut_par, kLimitNs)) ok = false;
      if (!mbar_wait_bounded(&ss.bar_dt, par_dt, kLimitNs)) ok = false;
      par_dt ^= 1;
      tc_fence_after();
      // ---- Delta = U - W S0^T (for the outputs) and Delta' = diag(e^{G_L-G})
      //      Delta (for the state update), each as binary16 high and low parts ----
      const float* vec = reinterpret_cast<const float*>(sm + S_VEC + b * 512);
      {
        float v[16], d[16];
        tmem_ld16(tmem + lane_base + d1 + 16 * cg, v);
        const float* ut = reinterpret_cast<const float*>(ubuf + S_UT_OFF);
#pragma unroll
        for (int j = 0; j < 16; ++j) d[j] = v[j] + ut[(16 * cg + j) * kHeadDim + row];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          uint4 hi, lo;
          split_half8(d + 8 * q, hi, lo);
          *reinterpret_cast<uint4*>(sm + S_DTH + swz(row, 2 * cg + q)) = hi;
          *reinterpret_cast<uint4*>(sm + S_DTL + swz(row, 2 * cg + q)) = lo;
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) d[j] *= vec[1 + 16 * cg + j];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          uint4 hi, lo;
          split_half8(d + 8 * q, hi, lo);
          *reinterpret_cast<uint4*>(sm + S_DPH + swz(row, 2 * cg + q)) = hi;
          *reinterpret_cast<uint4*>(sm + S_DPL + swz(row, 2 * cg + q)) = lo;
        }
      }
      // stage step r-1's outputs over this step's [-W ; Q~] image (D1 is done)
      if (pend) stage_out(buf, ov);
      fence_proxy_async_smem();
      tc_fence_before();
      if (__syncthreads_or(!ok)) { ok = false; break; }
      // ---- P = Delta'_hi^T K + Delta'_lo^T K (critical path), then Delta_hi^T
      //      [M hi ; M lo]^T and Delta_lo^T M_hi^T (onto OA) for the output, read
      //      during the next step ----
      if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_f16(tmem + ST_P, sw128_desc(a_dph + ks * 32, 16, 1024),
                  sw128_desc(a_buf + SL_BKM + ks * 2048, 8192, 1024), id_p, ks > 0);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_f16(tmem + ST_P, sw128_desc(a_dpl + ks * 32, 16, 1024),
                  sw128_desc(a_buf + SL_BKM + ks * 2048, 8192, 1024), id_p, 1);
        mma_commit(&ss.bar_p);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t bm = sw128_desc(a_buf + SL_BKM + 2 * 8192 + ks * 32, 16, 1024);
          mma_f16(tmem + ST_OB, sw128_desc(a_dth + ks * 32, 16, 1024), bm, id_ob, ks > 0);
          mma_f16(tmem + d1 + 64, sw128_desc(a_dtl + ks * 32, 16, 1024), bm, id_d3, true);
        }
        mma_commit(&ss.bar_o);
      }
      // copy step r+1's slot into the other buffer (its stage was copied out and its
      // U^T read before the barrier above) if it was seen published, in the shadow of P
      if (tid == 32 && issued == r + 1 && ss.pf) {
        issue_copy(r + 1, true);
        issued = r + 2;
      }
      // and step r-1's outputs leave from the stage (the layer's form first normalises
      // them there and leaves them after the step's last barrier)
      if (pend) {
        if constexpr (Fused) {
          norm_stage(buf + S_STG_OFF, pend_t0, pend_L, pend_h);
          fence_proxy_async_smem();
          staged = true;
          stg_t0 = pend_t0;
          stg_L = pend_L;
          stg_h = pend_h;
        } else {
          emit_out(buf + S_STG_OFF, pend_t0, pend_L, pend_h);
        }
        pend = false;
      }
      if (!mbar_wait_bounded(&ss.bar_p, par_p, kLimitNs)) ok = false;
      par_p ^= 1;
      tc_fence_after();
      {
        const float gL = vec[0];
        float pv[32];
        tmem_ld32(tmem + lane_base + ST_P + 32 * cg, pv);
#pragma unroll
        for (int j = 0; j < 32; ++j) S[j] = fmaf(gL, S[j], pv[j]);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4*>(sm + S_S0 + (cg >> 1) * 16384 + swz(row, (cg & 1) * 4 + q)) =
              pack_half8(S + 8 * q);
        fence_proxy_async_smem();   // the next step's D1 reads S0
      }
      if (!mbar_wait_bounded(&ss.bar_o, par_o, kLimitNs)) ok = false;
      par_o ^= 1;
      tc_fence_after();
      // step r+1's U^T into this buffer's K/M area, which the output MMAs have
      // finished reading
      if (tid == 32 && issued == r + 2 && ut_issued == r + 1) {
        issue_ut(r + 1);
        ut_issued = r + 2;
      }
      tc_fence_before();
      if (__syncthreads_or(!ok)) { ok = false; break; }
      if (Fused && staged) {   // the normed tile of step r-1, staged in this step's buffer
        emit_out(buf + S_STG_OFF, stg_t0, stg_L, stg_h);
        staged = false;
      }
      pend = true;
      pend_t0 = t0;
      pend_L = L;
      pend_h = h;
    }
    if (!ok) {
      fail_item = i;
      break;
    }
    if (p.state_out) {
      float* dst = p.state_out + (nh * kHeadDim + row) * kHeadDim + cg * 32;
#pragma unroll
      for (int j = 0; j < 32; j += 4)
        *reinterpret_cast<float4*>(dst + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
    }
  }
  if (ok && pend) {   // the last step's outputs
    float ov[16];
    tc_fence_after();
    load_out(((r - 1) & 1) ? ST_D1B : ST_D1A, ov);
    // an earlier tile store may still read this buffer's stage
    if (tid == 32) bulk_wait_read_all();
    __syncthreads();
    uint8_t* lbuf = sm + S_BUF + ((r - 1) & 1) * SL_OPS;
    stage_out(lbuf, ov);
    fence_proxy_async_smem();
    __syncthreads();
    if constexpr (Fused) {
      norm_stage(lbuf + S_STG_OFF, pend_t0, pend_L, pend_h);
      fence_proxy_async_smem();
      __syncthreads();
    }
    emit_out(lbuf + S_STG_OFF, pend_t0, pend_L, pend_h);
  }
  if (!ok && tid == 0) atomicExch(&ctrl[1], 1);
  // drain our own copies before leaving (bounded)
  if (tid == 32) {
    for (int st = r; st < issued; ++st)
      mbar_wait_bounded(&ss.bar_slot[st & 1], (uint32_t)((st >> 1) & 1), kLimitNs);
    for (int st = r; st < ut_issued; ++st)
      mbar_wait_bounded(&ss.bar_ut[(st + 1) & 1], (uint32_t)((st >> 1) & 1), kLimitNs);
    bulk_wait_all();   // output stores complete
    fence_proxy_async_all();
  }
  tc_fence_before();
  __syncthreads();
  if (fail_item >= 0) {   // every unfinished (sequence, head): outputs and state NaN
    const float qnan = __int_as_float(0x7fc00000);
    for (int i = fail_item; i < p.N * p.H_v; i += p.NS) {
      const int n = i / p.H_v, h = i % p.H_v;
      int64_t s0, s1;
      seq_chunks(p.cu, p.T, n, &s0, &s1);
      for (int64_t e = tid; e < (s1 - s0) * kHeadDim; e += kPcThreads)
        o[((s0 + e / kHeadDim) * p.H_v + h) * kHeadDim + e % kHeadDim] = from_f32<To>(qnan);
      if (p.state_out)
        for (int e = tid; e < kHeadDim * kHeadDim; e += kPcThreads)
          p.state_out[((int64_t)n * p.H_v + h) * kHeadDim * kHeadDim + e] = qnan;
    }
  }
  if (warp == 0) tmem_dealloc(tmem, ST_COLS);
}

template <class Tg, class To, bool Fused, class Tw>
__global__ void __launch_bounds__(kPcThreads, 1)
prefill_pc_kernel(const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ CUtensorMap tm_o, const PcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if ((int)blockIdx.x < p.NS) state_role<To, Fused, Tw>(p, &tm_o, sm, blockIdx.x);
  else prep_role<Tg, Fused, Tw>(p, &tm_q, &tm_k, &tm_v, sm);
}

// ------------------------------------------------------------------ host --

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

bool make_map(CUtensorMap* m, const void* base, int64_t cols, int64_t rows, int64_t stride) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(stride * 2)};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 output [rows][cols] (dense), 128 x 64 boxes, unswizzled
bool make_out_map(CUtensorMap* m, void* base, int64_t cols, int64_t rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(cols * 2)};
  cuuint32_t box[2] = {(cuuint32_t)kHeadDim, (cuuint32_t)kChunk};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

template <class Tg, class To, bool Fused, class Tw>
cudaError_t launch_kernel(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                          const CUtensorMap& mo, const PcParams& p, int nsm, void* workspace,
                          cudaStream_t stream);

template <class Tg, class To>
cudaError_t launch_typed(const RecurArgs& a, int nsm, int NS) {
  CUtensorMap mq, mk, mv, mo;
  if (!make_map(&mq, a.q, (int64_t)a.H_k * kHeadDim, a.T_total, a.q_row_stride) ||
      !make_map(&mk, a.k, (int64_t)a.H_k * kHeadDim, a.T_total, a.k_row_stride) ||
      !make_map(&mv, a.v, (int64_t)a.H_v * kHeadDim, a.T_total, a.v_row_stride))
    return cudaErrorInvalidValue;
  if (sizeof(To) == 2) {   // whole-chunk output tiles [64 tokens][128] leave by TMA
    if (!make_out_map(&mo, a.o, (int64_t)a.H_v * kHeadDim, a.T_total)) return cudaErrorInvalidValue;
  } else {
    mo = mv;   // unused: fp32 outputs are stored by the threads
  }
  PcParams p{a.g, a.beta, a.state_in, a.state_out, a.cu_seqlens, a.T_total, a.N,
             a.H_k, a.H_v, a.scale, a.o, static_cast<uint8_t*>(a.workspace), NS,
             wait_limit_ns()};
  return launch_kernel<Tg, To, false, float>(mq, mk, mv, mo, p, nsm, a.workspace, a.stream);
}

// one cooperative launch of the kernel, one CTA per SM
template <class Tg, class To, bool Fused, class Tw>
cudaError_t launch_kernel(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                          const CUtensorMap& mo, const PcParams& p, int nsm, void* workspace,
                          cudaStream_t stream) {
  auto kern = prefill_pc_kernel<Tg, To, Fused, Tw>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)PC_SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(workspace, 0, CTRL_BYTES, stream);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)nsm);
  cfg.blockDim = dim3(kPcThreads);
  cfg.dynamicSmemBytes = PC_SMEM_ALLOC;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, mo, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <class Tg>
cudaError_t pick_o(const RecurArgs& a, int nsm, int NS) {
  return a.o_dtype == GDN_F32 ? launch_typed<Tg, float>(a, nsm, NS)
                              : launch_typed<Tg, __nv_bfloat16>(a, nsm, NS);
}

// State CTAs: about a third of the SMs (a multiple of H_v when that fits, so
// that every state CTA gets the same heads of every sequence), at most one per
// item; the remaining SMs prepare chunks.
int state_ctas(int64_t items, int H_v, int nsm) {
  int base = nsm / 3;
  if (base < 1) base = 1;
  if (items <= base) return (int)items;
  if (H_v <= base) return (base / H_v) * H_v;
  return base;
}

std::atomic<uint64_t> g_wait_ns{kLimitNs};

// ---- library-owned scratch for callers that cannot allocate --------------
// Room for the rings of 49 state CTAs (a third of a 148-SM B200). Every GPU
// that loads the library holds this array until the process exits.
constexpr int kNoAllocStateCtas = 49;
constexpr size_t kNoAllocScratchBytes =
    CTRL_BYTES + (size_t)kNoAllocStateCtas * kRing * SLOT_BYTES;   // 29 218 816 B
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (the host-side symbol is only a stand-in, never a device address).
cudaError_t noalloc_scratch(void** out) {
  static std::mutex mu;
  static void* addr[256] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 256) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = ptr;
  }
  *out = addr[dev];
  return cudaSuccess;
}

}  // namespace

void set_wait_limit_ns(uint64_t ns) { g_wait_ns.store(ns ? ns : kLimitNs); }
uint64_t wait_limit_ns() { return g_wait_ns.load(); }

cudaError_t prefill_abort_word(const void* workspace, cudaStream_t stream, int* word) {
  const void* ws = workspace;
  if (!ws) {
    void* scratch = nullptr;
    cudaError_t e = noalloc_scratch(&scratch);
    if (e != cudaSuccess) return e;
    ws = scratch;
  }
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  return cudaMemcpy(word, static_cast<const int*>(ws) + 1, sizeof(int), cudaMemcpyDeviceToHost);
}

size_t prefill_noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

cudaError_t launch_prefill_pc_noalloc(const RecurArgs& args) {
  void* scratch = nullptr;
  cudaError_t e = noalloc_scratch(&scratch);
  if (e != cudaSuccess) return e;
  RecurArgs a = args;
  a.workspace = scratch;
  a.workspace_bytes = kNoAllocScratchBytes;
  return launch_prefill_pc(a);
}

size_t prefill_pc_workspace(int N, int64_t T_total, int H_v) {
  const int nsm = sm_count();
  if (nsm < 2 || N <= 0 || T_total <= 0) return 0;
  const int NS = state_ctas((int64_t)N * H_v, H_v, nsm);
  return CTRL_BYTES + (size_t)NS * kRing * SLOT_BYTES;
}

cudaError_t launch_prefill_pc(const RecurArgs& a) {
  if (a.N == 0) return cudaSuccess;
  if (a.T_total == 0) return launch_prefill_chunked_f32(a);   // only state copies
  const int nsm = sm_count();
  if (nsm < 2) return cudaErrorInvalidDevice;
  const int NS = state_ctas((int64_t)a.N * a.H_v, a.H_v, nsm);
  if (a.workspace_bytes < CTRL_BYTES + (size_t)NS * kRing * SLOT_BYTES || !a.workspace)
    return cudaErrorInvalidValue;
  return a.gate_dtype == GDN_F32 ? pick_o<float>(a, nsm, NS) : pick_o<__nv_bfloat16>(a, nsm, NS);
}

namespace {

template <class Tg, class To, class Tw>
cudaError_t launch_layer_typed(const LayerPrefillArgs& a, int nsm, int NS) {
  const int64_t C = 2 * (int64_t)a.H_k * kHeadDim + (int64_t)a.H_v * kHeadDim;
  const int64_t Cqk = 2 * (int64_t)a.H_k * kHeadDim;
  // q and k once per key head: conv + SiLU + L2 of the leading 2 H_k heads into
  // the scratch behind the ring (all value heads of a key head read them)
  __nv_bfloat16* qk = reinterpret_cast<__nv_bfloat16*>(
      static_cast<uint8_t*>(a.workspace) + CTRL_BYTES + (size_t)NS * kRing * SLOT_BYTES);
  ConvArgs ca{a.x, a.x_row_stride, GDN_BF16, a.conv_w, a.w_dtype, a.conv_bias, (int)Cqk,
              (int)Cqk, a.l2_eps, a.cu_seqlens, a.N, a.T_total, a.conv_state_in, nullptr, qk,
              Cqk, GDN_BF16, a.stream, C};
  cudaError_t e = launch_conv1d_silu(ca);
  if (e != cudaSuccess) return e;
  CUtensorMap mx, mq, mk, mo;
  // the v map of the plain path is not read in the layer's form; a valid map
  // over x stands in its place
  if (!make_map(&mx, a.x, C, a.T_total, a.x_row_stride) ||
      !make_map(&mq, qk, (int64_t)a.H_k * kHeadDim, a.T_total, Cqk) ||
      !make_map(&mk, qk + (int64_t)a.H_k * kHeadDim, (int64_t)a.H_k * kHeadDim, a.T_total, Cqk))
    return cudaErrorInvalidValue;
  if (sizeof(To) == 2) {
    if (!make_out_map(&mo, a.y, (int64_t)a.H_v * kHeadDim, a.T_total)) return cudaErrorInvalidValue;
  } else {
    mo = mx;
  }
  PcParams p{a.g, a.beta, a.state_in, a.state_out, a.cu_seqlens, a.T_total, a.N, a.H_k, a.H_v,
             a.scale, a.y, static_cast<uint8_t*>(a.workspace), NS, wait_limit_ns(),
             a.x, a.x_row_stride, a.conv_w, a.conv_bias, a.conv_state_in, (int)C, a.l2_eps,
             a.z, a.norm_w, a.norm_eps};
  return launch_kernel<Tg, To, true, Tw>(mq, mk, mx, mo, p, nsm, a.workspace, a.stream);
}
template <class Tg, class To>
cudaError_t layer_pick_w(const LayerPrefillArgs& a, int nsm, int NS) {
  return a.w_dtype == GDN_F32 ? launch_layer_typed<Tg, To, float>(a, nsm, NS)
                              : launch_layer_typed<Tg, To, __nv_bfloat16>(a, nsm, NS);
}
template <class Tg>
cudaError_t layer_pick_o(const LayerPrefillArgs& a, int nsm, int NS) {
  return a.y_dtype == GDN_F32 ? layer_pick_w<Tg, float>(a, nsm, NS)
                              : layer_pick_w<Tg, __nv_bfloat16>(a, nsm, NS);
}

}  // namespace

size_t prefill_layer_workspace(int N, int64_t T_total, int H_k, int H_v) {
  const int nsm = sm_count();
  if (nsm < 2) return 0;
  const int NS = state_ctas((int64_t)N * H_v, H_v, nsm);
  return CTRL_BYTES + (size_t)NS * kRing * SLOT_BYTES +
         (size_t)T_total * 2 * H_k * kHeadDim * 2;
}

cudaError_t launch_prefill_layer(const LayerPrefillArgs& a) {
  if (a.N == 0) return cudaSuccess;
  cudaError_t e = cudaSuccess;
  if (a.T_total > 0) {
    const int nsm = sm_count();
    if (nsm < 2) return cudaErrorInvalidDevice;
    const int NS = state_ctas((int64_t)a.N * a.H_v, a.H_v, nsm);
    if (a.workspace_bytes < prefill_layer_workspace(a.N, a.T_total, a.H_k, a.H_v) ||
        !a.workspace)
      return cudaErrorInvalidValue;
    e = a.gate_dtype == GDN_F32 ? layer_pick_o<float>(a, nsm, NS)
                                : layer_pick_o<__nv_bfloat16>(a, nsm, NS);
  } else {   // no tokens: the states pass through
    RecurArgs r{a.x, a.x, a.x, GDN_BF16, a.x_row_stride, a.x_row_stride, a.x_row_stride,
                a.g, a.beta, a.gate_dtype, a.state_in, a.state_out, a.cu_seqlens, a.N, 0,
                a.H_k, a.H_v, a.scale, a.y, a.y_dtype, nullptr, 0, a.stream};
    e = launch_prefill_chunked_f32(r);
  }
  if (e != cudaSuccess || !a.conv_state_out) return e;
  // the carried conv history for the next call: each sequence's last three
  // pre-conv rows (after the kernel, which read conv_state_in: they may alias)
  return launch_conv_state_roll(a.x, a.x_row_stride, GDN_BF16,
                                2 * a.H_k * kHeadDim + a.H_v * kHeadDim, a.cu_seqlens, a.N,
                                a.T_total, a.conv_state_in, a.conv_state_out, a.stream);
}

}  // namespace gdn
