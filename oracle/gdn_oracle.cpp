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

}  // extern "C"
