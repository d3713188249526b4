// Gated delta-rule layer: plain, slow, fp64 CPU oracle.
//
// TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or
// load this file; only the test suite, the package smoke check and the
// bench's CPU-baseline leg use it. It shares no code, header, table or
// constant with the CUDA library.
//
// Sources (page titles and sections):
//  * "Agnes-3.0-Flash Preview" leaderboard commentary (discosf.com), section
//    二.1 "72 层里只有 18 层吃 KV cache": the delta-rule layer is recurrent,
//    16 key / 48 value heads, head dim 128, a kernel-4 causal conv in front,
//    fp32 recurrent state; a chunked prefill path (chunk 64) and a stepwise
//    decode path compute the same recurrence.
//  * Agnes-3.0-Flash Preview model card (modelscope.cn README_zh), section
//    架构 (architecture table): causal conv kernel 4, gated RMS-norm, fp32
//    recurrent state, state size independent of sequence length.
//  The pages name the layer but print no equations. The recurrence is the
//  published gated delta rule,
//      S_t = g_t * S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
//      o_t = scale * S_t q_t,
//  with S in R^{d_v x d_k}. Points the pages leave open are read plainly:
//  value head h uses key/query head h / (H_v/H_k); the conv history before a
//  sequence's start is the carried conv state (zeros when absent); the gated
//  RMS-norm normalises first and then multiplies by w and SiLU(z).
//
//  The hybrid decoder's other layer type, global attention (model card,
//  section 架构, rows 全局注意力 and 位置编码; commentary section 二.1): 24
//  query / 4 key-value heads (GQA 6 : 1), head dim 256, RMS-norm on q and k,
//  a sigmoid gate on the output, and three-axis rotary (text / height /
//  width, interleaved 11 : 11 : 10, base 1e7) on the first 64 dims of each
//  head. Read plainly: the norms are per head over the head dim with a weight
//  vector; rotary pair i couples dims i and i + 32 (rotate-half); the gate is
//  elementwise on each head's output; softmax scale is D^-1/2; attention is
//  causal within each packed sequence.
//
// Every function is the plain definition written out in fp64, with no
// blocking, fusion or reordering beyond it. Work is split over independent
// (sequence, value head) pairs with std::thread only.
//
// Parity is pinned by tests/test_oracle_*.py against brute-force ordered
// matrix products, closed forms and invariants (none of which call back into
// this file's formulas).

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

int resolve_threads(int requested, int64_t work_items) {
  int hw = (int)std::thread::hardware_concurrency();
  if (hw <= 0) hw = 1;
  int n = requested > 0 ? requested : hw;
  if ((int64_t)n > work_items) n = (int)(work_items > 0 ? work_items : 1);
  return n;
}

template <class F>
void parallel_for(int64_t items, int threads, F&& body) {
  std::atomic<int64_t> next{0};
  auto worker = [&]() {
    for (;;) {
      int64_t i = next.fetch_add(1);
      if (i >= items) return;
      body(i);
    }
  };
  if (threads <= 1) {
    worker();
    return;
  }
  std::vector<std::thread> pool;
  pool.reserve(threads);
  for (int i = 0; i < threads; ++i) pool.emplace_back(worker);
  for (auto& t : pool) t.join();
}

double silu(double a) { return a / (1.0 + std::exp(-a)); }

}  // namespace

extern "C" {

// Number of hardware threads the host reports.
int oracle_hardware_threads(void) {
  int hw = (int)std::thread::hardware_concurrency();
  return hw > 0 ? hw : 1;
}

// Causal depthwise conv (kernel 4) + SiLU, then per-128-channel L2
// normalisation of the leading `l2_channels` channels (the q and k heads).
//
//   y[t,c] = SiLU( bias[c] + sum_{j=0..3} w[c,j] * xh(t-3+j, c) )
//
// where xh(p, c) is the pre-conv input at sequence-local position p; for
// p < 0 it is the carried history conv_state_in[n, 3+p, c] (zeros when
// conv_state_in is null). Tap j=3 multiplies the current token. Then for
// every head group [128*m, 128*m+128) with 128*m < l2_channels:
//   y <- y / sqrt(sum y^2 + l2_eps).
// conv_state_out[n, r, c] = xh(len_n - 3 + r, c), r = 0..2 (oldest first).
//
// Layouts (row-major, dense): x, y [T_total, C]; w [C, 4]; bias [C];
// conv_state_* [N, 3, C]; cu_seqlens [N+1].
void oracle_conv1d_silu_l2(const double* x, int64_t T_total, int C,
                           const double* w, const double* bias,
                           const int32_t* cu_seqlens, int N,
                           const double* conv_state_in, int l2_channels,
                           double l2_eps, double* y, double* conv_state_out,
                           int threads) {
  (void)T_total;
  int nt = resolve_threads(threads, N);
  parallel_for(N, nt, [&](int64_t n) {
    const int64_t t0 = cu_seqlens[n];
    const int64_t len = (int64_t)cu_seqlens[n + 1] - t0;
    auto xh = [&](int64_t p, int c) -> double {
      if (p >= 0) return x[(t0 + p) * C + c];
      if (!conv_state_in) return 0.0;
      return conv_state_in[(n * 3 + (3 + p)) * (int64_t)C + c];
    };
    for (int64_t p = 0; p < len; ++p) {
      double* yr = y + (t0 + p) * C;
      for (int c = 0; c < C; ++c) {
        double acc = bias ? bias[c] : 0.0;
        for (int j = 0; j < 4; ++j) acc += w[c * 4 + j] * xh(p - 3 + j, c);
        yr[c] = silu(acc);
      }
      for (int h0 = 0; h0 < l2_channels; h0 += 128) {
        double ss = 0.0;
        for (int c = h0; c < h0 + 128; ++c) ss += yr[c] * yr[c];
        double inv = 1.0 / std::sqrt(ss + l2_eps);
        for (int c = h0; c < h0 + 128; ++c) yr[c] *= inv;
      }
    }
    if (conv_state_out) {
      for (int r = 0; r < 3; ++r)
        for (int c = 0; c < C; ++c)
          conv_state_out[(n * 3 + r) * (int64_t)C + c] = xh(len - 3 + r, c);
    }
  });
}

// Stepwise gated delta rule over packed variable-length sequences.
//
// For each sequence n and value head h (key/query head kh = h / (H_v/H_k)),
// starting from S = state_in[n,h] (or 0), for every token t in order:
//   S <- g_t S (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
//   o_t = scale * S q_t
// S is [d, d] = [d_v, d_k], row-major, (S k)_i = sum_j S_ij k_j.
//
// Layouts: q, k [T_total, H_k, d]; v, o [T_total, H_v, d]; g, beta
// [T_total, H_v]; state_in/state_out [N, H_v, d, d] (state_in nullable).
void oracle_recurrence(const double* q, const double* k, const double* v,
                       const double* g, const double* beta,
                       const double* state_in, const int32_t* cu_seqlens,
                       int N, int H_k, int H_v, int d, double scale,
                       double* o, double* state_out, int threads) {
  const int group = H_v / H_k;
  const int64_t pairs = (int64_t)N * H_v;
  int nt = resolve_threads(threads, pairs);
  parallel_for(pairs, nt, [&](int64_t idx) {
    const int n = (int)(idx / H_v);
    const int h = (int)(idx % H_v);
    const int kh = h / group;
    std::vector<double> S((size_t)d * d, 0.0), Sk(d);
    if (state_in)
      std::memcpy(S.data(), state_in + idx * (int64_t)d * d,
                  sizeof(double) * d * d);
    for (int64_t t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
      const double* qt = q + (t * H_k + kh) * d;
      const double* kt = k + (t * H_k + kh) * d;
      const double* vt = v + (t * H_v + h) * d;
      const double gt = g[t * H_v + h];
      const double bt = beta[t * H_v + h];
      // S <- g S
      for (int64_t e = 0; e < (int64_t)d * d; ++e) S[e] *= gt;
      // S <- S (I - beta k k^T) = S - beta (S k) k^T
      for (int i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int j = 0; j < d; ++j) acc += S[(size_t)i * d + j] * kt[j];
        Sk[i] = acc;
      }
      for (int i = 0; i < d; ++i)
        for (int j = 0; j < d; ++j)
          S[(size_t)i * d + j] -= bt * Sk[i] * kt[j];
      // S <- S + beta v k^T
      for (int i = 0; i < d; ++i)
        for (int j = 0; j < d; ++j)
          S[(size_t)i * d + j] += bt * vt[i] * kt[j];
      // o_t = scale * S q
      double* ot = o + (t * H_v + h) * d;
      for (int i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int j = 0; j < d; ++j) acc += S[(size_t)i * d + j] * qt[j];
        ot[i] = scale * acc;
      }
    }
    if (state_out)
      std::memcpy(state_out + idx * (int64_t)d * d, S.data(),
                  sizeof(double) * d * d);
  });
}

// Gated RMS-norm over rows of `dim` channels:
//   y = x / sqrt(mean(x^2) + eps) * w * SiLU(z)
// Layouts: x, z, y [rows, dim]; w [dim].
void oracle_gated_rmsnorm(const double* x, const double* z, const double* w,
                          int64_t rows, int dim, double eps, double* y,
                          int threads) {
  int nt = resolve_threads(threads, rows);
  parallel_for(rows, nt, [&](int64_t r) {
    const double* xr = x + r * dim;
    const double* zr = z + r * dim;
    double ss = 0.0;
    for (int c = 0; c < dim; ++c) ss += xr[c] * xr[c];
    double inv = 1.0 / std::sqrt(ss / dim + eps);
    for (int c = 0; c < dim; ++c)
      y[r * dim + c] = xr[c] * inv * w[c] * silu(zr[c]);
  });
}

// Global-attention layer of the same hybrid decoder (the fourth layer of each
// four: "Agnes-3.0-Flash Preview" model card, 架构 table; leaderboard
// commentary, section 二.1): 24 query / 4 key-value heads (each kv head shared
// by 6 query heads), head dim 256, RMS-norm on q and on k, rotary position
// encoding on the first 64 dims (base 1e7; the three-axis interleaved form of
// the pages gives every frequency the same angle when the text, height and
// width positions coincide, as they do for text tokens), causal softmax
// attention, and a sigmoid gate on the output. Per sequence n (tokens
// cu[n] .. cu[n+1]-1, position p = t - cu[n] + pos0[n]) and token t:
//   qn[h] = q[t,h] / sqrt(mean(q[t,h]^2) + eps) * wq          (per head, D dims)
//   kn[g] = k[t,g] / sqrt(mean(k[t,g]^2) + eps) * wk
//   rotary on dims [0, R): for i < R/2, theta = p * base^(-2i/R),
//     (x_i, x_{i+R/2}) <- (x_i cos theta - x_{i+R/2} sin theta,
//                          x_{i+R/2} cos theta + x_i sin theta)
//   for query head h (kv head g = h / (Hq/Hkv)):
//     s_j = scale * qr[t,h] . kr[j,g] for the sequence's tokens j <= t
//     o[t,h] = sum_j softmax(s)_j v[j,g]
//   out[t,h] = o[t,h] * sigmoid(gate[t,h])                      (elementwise)
// q_rot / k_rot (nullable) receive qr and kr.
// Layouts: q, gate, out, q_rot [T, Hq, D]; k, v, k_rot [T, Hkv, D]; wq, wk [D];
// pos0 [N] (nullable: 0).
void oracle_attention(const double* q, const double* k, const double* v,
                      const double* gate, const int32_t* cu_seqlens, const int64_t* pos0,
                      const int64_t* pos3, int N, int64_t T, int Hq, int Hkv, int D,
                      const double* wq, const double* wk, double eps, int R, double base,
                      double scale, const uint8_t* want, double* out, double* q_rot,
                      double* k_rot, int threads) {
  // Per-head RMS-norm with weight w, then rotary on dims [0, R): pair i couples
  // dims i and i + R/2 and turns by theta_i = p * base^(-2i/R), where p is the
  // token's position on axis i mod 3 (text, height, width interleaved, which
  // gives the 11 : 11 : 10 split of the 32 pairs at R = 64). Without explicit
  // per-axis positions all three axes carry the index within the sequence.
  std::vector<double> qr((size_t)T * Hq * D), kr((size_t)T * Hkv * D);
  auto prep = [&](const double* x, const double* w, double* y, const int64_t* p) {
    double ss = 0.0;
    for (int d = 0; d < D; ++d) ss += x[d] * x[d];
    const double inv = 1.0 / std::sqrt(ss / D + eps);
    for (int d = 0; d < D; ++d) y[d] = x[d] * inv * w[d];
    for (int i = 0; i < R / 2; ++i) {
      const double theta = (double)p[i % 3] * std::pow(base, -2.0 * i / R);
      const double c = std::cos(theta), s = std::sin(theta);
      const double a = y[i], b = y[i + R / 2];
      y[i] = a * c - b * s;
      y[i + R / 2] = b * c + a * s;
    }
  };
  int nt = resolve_threads(threads, N);
  parallel_for(N, nt, [&](int64_t n) {
    for (int64_t t = cu_seqlens[n]; t < cu_seqlens[n + 1]; ++t) {
      int64_t p[3];
      for (int ax = 0; ax < 3; ++ax)
        p[ax] = pos3 ? pos3[ax * T + t] : t - cu_seqlens[n] + (pos0 ? pos0[n] : 0);
      for (int h = 0; h < Hq; ++h) prep(q + (t * Hq + h) * D, wq, qr.data() + (t * Hq + h) * D, p);
      for (int g = 0; g < Hkv; ++g) prep(k + (t * Hkv + g) * D, wk, kr.data() + (t * Hkv + g) * D, p);
    }
  });
  if (q_rot) std::memcpy(q_rot, qr.data(), sizeof(double) * qr.size());
  if (k_rot) std::memcpy(k_rot, kr.data(), sizeof(double) * kr.size());
  // causal softmax attention per (sequence, query head)
  const int group = Hq / Hkv;
  const int64_t pairs = (int64_t)N * Hq;
  nt = resolve_threads(threads, pairs);
  parallel_for(pairs, nt, [&](int64_t idx) {
    const int n = (int)(idx / Hq), h = (int)(idx % Hq), g = h / group;
    const int64_t s0 = cu_seqlens[n], s1 = cu_seqlens[n + 1];
    std::vector<double> sc((size_t)(s1 - s0)), o(D);
    for (int64_t t = s0; t < s1; ++t) {
      if (want && !want[t]) continue;   // output row not asked for
      const double* qt = qr.data() + (t * Hq + h) * D;
      double m = -INFINITY;
      for (int64_t j = s0; j <= t; ++j) {
        const double* kj = kr.data() + (j * Hkv + g) * D;
        double acc = 0.0;
        for (int d = 0; d < D; ++d) acc += qt[d] * kj[d];
        sc[j - s0] = scale * acc;
        if (sc[j - s0] > m) m = sc[j - s0];
      }
      double l = 0.0;
      for (int64_t j = s0; j <= t; ++j) l += std::exp(sc[j - s0] - m);
      for (int d = 0; d < D; ++d) o[d] = 0.0;
      for (int64_t j = s0; j <= t; ++j) {
        const double pj = std::exp(sc[j - s0] - m) / l;
        const double* vj = v + (j * Hkv + g) * D;
        for (int d = 0; d < D; ++d) o[d] += pj * vj[d];
      }
      const double* gt = gate + (t * Hq + h) * D;
      double* ot = out + (t * Hq + h) * D;
      for (int d = 0; d < D; ++d) ot[d] = o[d] / (1.0 + std::exp(-gt[d]));
    }
  });
}

}  // extern "C"
