// C-ABI entry points of libgdn.so: host-side validation, then dispatch to the
// kernels. Nothing is launched when validation fails. The declarations, with
// the passages each operation follows, are in include/gdn.h.
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn.h"
#include "gdn_common.cuh"
#include "launch.h"

namespace {

using gdn::kHeadDim;

bool valid_dtype(gdn_dtype t) { return t == GDN_BF16 || t == GDN_F32; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned_to(const void* p, int bytes) {
  return (reinterpret_cast<uintptr_t>(p) % (uintptr_t)bytes) == 0;
}
bool stride_ok(int64_t stride_elems, gdn_dtype t) {
  return (stride_elems * gdn::elem_bytes(t)) % 16 == 0;
}
gdn_status from_cuda(cudaError_t e) { return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA; }

// [a, a+na) and [b, b+nb) overlap without being identical ranges
bool partial_overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  uintptr_t a0 = (uintptr_t)a, b0 = (uintptr_t)b;
  if (a0 == b0 && na == nb) return false;
  return a0 < b0 + nb && b0 < a0 + na;
}

// Checks shared by the prefill and decode recurrences.
gdn_status check_recurrence(const void* q, const void* k, const void* v,
                            gdn_dtype qkv_dtype, int64_t qs, int64_t ks,
                            int64_t vs, const void* g, const void* beta,
                            gdn_dtype gate_dtype, int H_k, int H_v, void* o,
                            gdn_dtype o_dtype, bool have_tokens) {
  if (!valid_dtype(qkv_dtype) || !valid_dtype(gate_dtype) || !valid_dtype(o_dtype))
    return GDN_ERR_INVALID_ARG;
  if (H_k <= 0 || H_v <= 0 || H_v % H_k != 0) return GDN_ERR_INVALID_ARG;
  if (qs < (int64_t)H_k * kHeadDim || ks < (int64_t)H_k * kHeadDim ||
      vs < (int64_t)H_v * kHeadDim)
    return GDN_ERR_INVALID_ARG;
  if (!have_tokens) return GDN_OK;
  if (!q || !k || !v || !g || !beta || !o) return GDN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return GDN_ERR_MISALIGNED;
  if (!stride_ok(qs, qkv_dtype) || !stride_ok(ks, qkv_dtype) || !stride_ok(vs, qkv_dtype))
    return GDN_ERR_MISALIGNED;
  const int gb = gdn::elem_bytes(gate_dtype);
  if (!aligned_to(g, gb) || !aligned_to(beta, gb)) return GDN_ERR_MISALIGNED;
  return GDN_OK;
}

}  // namespace

extern "C" {

const char* gdn_status_string(gdn_status s) {
  switch (s) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG: invalid argument";
    case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED: unsupported shape or option";
    case GDN_ERR_MISALIGNED: return "GDN_ERR_MISALIGNED: pointer or stride not 16-byte aligned";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA: CUDA launch failed";
    case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT: a bounded wait in a kernel gave up";
  }
  return "unknown gdn_status";
}

const char* gdn_version(void) { return "0.1.0"; }

gdn_status gdn_conv1d_silu(const void* x, int64_t x_row_stride,
                           gdn_dtype x_dtype, const void* w, gdn_dtype w_dtype,
                           const void* bias, int channels, int l2norm_channels,
                           float l2_eps, const int32_t* cu_seqlens, int N,
                           int64_t T_total, const void* conv_state_in,
                           void* conv_state_out, void* y, int64_t y_row_stride,
                           gdn_dtype y_dtype, cudaStream_t stream) {
  if (!valid_dtype(x_dtype) || !valid_dtype(w_dtype) || !valid_dtype(y_dtype))
    return GDN_ERR_INVALID_ARG;
  if (N < 0 || T_total < 0 || channels <= 0 || channels % 8 != 0)
    return GDN_ERR_INVALID_ARG;
  if (l2norm_channels < 0 || l2norm_channels % kHeadDim != 0 ||
      l2norm_channels > channels || !(l2_eps >= 0.f))
    return GDN_ERR_INVALID_ARG;
  if (N == 0) return T_total == 0 ? GDN_OK : GDN_ERR_INVALID_ARG;
  if (!cu_seqlens || !w) return GDN_ERR_INVALID_ARG;
  if (T_total > 0) {
    if (!x || !y) return GDN_ERR_INVALID_ARG;
    if (x_row_stride < channels || y_row_stride < channels) return GDN_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y)) return GDN_ERR_MISALIGNED;
    if (!stride_ok(x_row_stride, x_dtype) || !stride_ok(y_row_stride, y_dtype))
      return GDN_ERR_MISALIGNED;
  }
  if (!aligned16(w) || (bias && !aligned16(bias)) ||
      (conv_state_in && !aligned16(conv_state_in)) ||
      (conv_state_out && !aligned16(conv_state_out)))
    return GDN_ERR_MISALIGNED;
  const size_t cs_bytes = (size_t)N * 3 * channels * gdn::elem_bytes(x_dtype);
  if (partial_overlap(conv_state_in, cs_bytes, conv_state_out, cs_bytes))
    return GDN_ERR_INVALID_ARG;
  gdn::ConvArgs a{x, x_row_stride, x_dtype, w, w_dtype, bias, channels,
                  l2norm_channels, l2_eps, cu_seqlens, N, T_total,
                  conv_state_in, conv_state_out, y, y_row_stride, y_dtype,
                  stream};
  return from_cuda(gdn::launch_conv1d_silu(a));
}

size_t gdn_chunked_prefill_workspace(int N, int64_t T_total, int H_k, int H_v) {
  (void)H_k;
  if (N <= 0 || T_total <= 0 || H_v <= 0) return 0;
  return gdn::prefill_pc_workspace(N, T_total, H_v);
}

gdn_status gdn_chunked_prefill(const void* q, const void* k, const void* v,
                               gdn_dtype qkv_dtype, int64_t q_row_stride,
                               int64_t k_row_stride, int64_t v_row_stride,
                               const void* g, const void* beta,
                               gdn_dtype gate_dtype, const float* state_in,
                               float* state_out, const int32_t* cu_seqlens,
                               int N, int64_t T_total, int H_k, int H_v,
                               float scale, void* o, gdn_dtype o_dtype,
                               void* workspace, size_t workspace_bytes,
                               cudaStream_t stream) {
  if (N < 0 || T_total < 0) return GDN_ERR_INVALID_ARG;
  gdn_status st = check_recurrence(q, k, v, qkv_dtype, q_row_stride, k_row_stride,
                                   v_row_stride, g, beta, gate_dtype, H_k, H_v,
                                   o, o_dtype, T_total > 0);
  if (st != GDN_OK) return st;
  if (N == 0) return T_total == 0 ? GDN_OK : GDN_ERR_INVALID_ARG;
  if (!cu_seqlens) return GDN_ERR_INVALID_ARG;
  if ((state_in && !aligned16(state_in)) || (state_out && !aligned16(state_out)))
    return GDN_ERR_MISALIGNED;
  const size_t st_bytes = (size_t)N * H_v * kHeadDim * kHeadDim * sizeof(float);
  if (partial_overlap(state_in, st_bytes, state_out, st_bytes)) return GDN_ERR_INVALID_ARG;
  if (qkv_dtype == GDN_BF16 && T_total > 0) {
    if (workspace_bytes < gdn_chunked_prefill_workspace(N, T_total, H_k, H_v) ||
        (workspace_bytes > 0 && !workspace))
      return GDN_ERR_INVALID_ARG;
    if (!aligned16(workspace)) return GDN_ERR_MISALIGNED;
  }
  gdn::RecurArgs a{q, k, v, qkv_dtype, q_row_stride, k_row_stride, v_row_stride,
                   g, beta, gate_dtype, state_in, state_out, cu_seqlens, N,
                   T_total, H_k, H_v, scale, o, o_dtype, workspace,
                   workspace_bytes, stream};
  return from_cuda(qkv_dtype == GDN_BF16 ? gdn::launch_prefill_pc(a)
                                         : gdn::launch_prefill_chunked_f32(a));
}

gdn_status gdn_prefill_layer(const void* x, int64_t x_row_stride, const void* conv_w,
                             gdn_dtype w_dtype, const void* conv_bias,
                             const void* conv_state_in, void* conv_state_out,
                             const void* g, const void* beta, gdn_dtype gate_dtype,
                             const float* state_in, float* state_out,
                             const int32_t* cu_seqlens, int N, int64_t T_total, int H_k,
                             int H_v, float scale, float l2_eps, const void* z,
                             const void* norm_w, float norm_eps, void* y, gdn_dtype y_dtype,
                             void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!valid_dtype(w_dtype) || !valid_dtype(gate_dtype) || !valid_dtype(y_dtype))
    return GDN_ERR_INVALID_ARG;
  if (N < 0 || T_total < 0 || H_k <= 0 || H_v <= 0 || H_v % H_k != 0 || !(l2_eps >= 0.f) ||
      !(norm_eps >= 0.f))
    return GDN_ERR_INVALID_ARG;
  const int64_t C = 2 * (int64_t)H_k * kHeadDim + (int64_t)H_v * kHeadDim;
  if (x_row_stride < C) return GDN_ERR_INVALID_ARG;
  if (N == 0) return T_total == 0 ? GDN_OK : GDN_ERR_INVALID_ARG;
  if (!cu_seqlens || !conv_w || !norm_w) return GDN_ERR_INVALID_ARG;
  if (T_total > 0 && (!x || !g || !beta || !z || !y)) return GDN_ERR_INVALID_ARG;
  if ((x && !aligned16(x)) || !aligned16(conv_w) || (conv_bias && !aligned16(conv_bias)) ||
      (conv_state_in && !aligned16(conv_state_in)) ||
      (conv_state_out && !aligned16(conv_state_out)) || (z && !aligned16(z)) ||
      !aligned16(norm_w) || (y && !aligned16(y)) || (state_in && !aligned16(state_in)) ||
      (state_out && !aligned16(state_out)))
    return GDN_ERR_MISALIGNED;
  if (!stride_ok(x_row_stride, GDN_BF16)) return GDN_ERR_MISALIGNED;
  const int gb = gdn::elem_bytes(gate_dtype);
  if ((g && !aligned_to(g, gb)) || (beta && !aligned_to(beta, gb))) return GDN_ERR_MISALIGNED;
  const size_t st_bytes = (size_t)N * H_v * kHeadDim * kHeadDim * sizeof(float);
  if (partial_overlap(state_in, st_bytes, state_out, st_bytes)) return GDN_ERR_INVALID_ARG;
  const size_t cs_bytes = (size_t)N * 3 * C * 2;
  if (partial_overlap(conv_state_in, cs_bytes, conv_state_out, cs_bytes))
    return GDN_ERR_INVALID_ARG;
  if (T_total > 0) {
    if (workspace_bytes < gdn_prefill_layer_workspace(N, T_total, H_k, H_v) || !workspace)
      return GDN_ERR_INVALID_ARG;
    if (!aligned16(workspace)) return GDN_ERR_MISALIGNED;
  }
  gdn::LayerPrefillArgs a{x, x_row_stride, conv_w, w_dtype, conv_bias, conv_state_in,
                          conv_state_out, g, beta, gate_dtype, state_in, state_out,
                          cu_seqlens, N, T_total, H_k, H_v, scale, l2_eps, z, norm_w,
                          norm_eps, y, y_dtype, workspace, workspace_bytes, stream};
  return from_cuda(gdn::launch_prefill_layer(a));
}

size_t gdn_prefill_layer_workspace(int N, int64_t T_total, int H_k, int H_v) {
  if (N < 0 || T_total < 0 || H_k <= 0 || H_v <= 0 || H_v % H_k != 0) return 0;
  if (T_total == 0) return 0;
  return gdn::prefill_layer_workspace(N, T_total, H_k, H_v);
}

gdn_status gdn_chunked_prefill_status(const void* workspace, cudaStream_t stream) {
  if (workspace && !aligned16(workspace)) return GDN_ERR_MISALIGNED;
  int word = 0;
  if (gdn::prefill_abort_word(workspace, stream, &word) != cudaSuccess) return GDN_ERR_CUDA;
  return word ? GDN_ERR_TIMEOUT : GDN_OK;
}

void gdn_set_wait_limit_ns(uint64_t ns) { gdn::set_wait_limit_ns(ns); }

gdn_status gdn_stepwise_prefill(const void* q, const void* k, const void* v,
                                gdn_dtype qkv_dtype, int64_t q_row_stride,
                                int64_t k_row_stride, int64_t v_row_stride,
                                const void* g, const void* beta,
                                gdn_dtype gate_dtype, const float* state_in,
                                float* state_out, const int32_t* cu_seqlens,
                                int N, int64_t T_total, int H_k, int H_v,
                                float scale, void* o, gdn_dtype o_dtype,
                                cudaStream_t stream) {
  if (N < 0 || T_total < 0) return GDN_ERR_INVALID_ARG;
  gdn_status st = check_recurrence(q, k, v, qkv_dtype, q_row_stride, k_row_stride,
                                   v_row_stride, g, beta, gate_dtype, H_k, H_v,
                                   o, o_dtype, T_total > 0);
  if (st != GDN_OK) return st;
  if (N == 0) return T_total == 0 ? GDN_OK : GDN_ERR_INVALID_ARG;
  if (!cu_seqlens) return GDN_ERR_INVALID_ARG;
  if ((state_in && !aligned16(state_in)) || (state_out && !aligned16(state_out)))
    return GDN_ERR_MISALIGNED;
  const size_t st_bytes = (size_t)N * H_v * kHeadDim * kHeadDim * sizeof(float);
  if (partial_overlap(state_in, st_bytes, state_out, st_bytes)) return GDN_ERR_INVALID_ARG;
  gdn::RecurArgs a{q, k, v, qkv_dtype, q_row_stride, k_row_stride, v_row_stride,
                   g, beta, gate_dtype, state_in, state_out, cu_seqlens, N,
                   T_total, H_k, H_v, scale, o, o_dtype, nullptr, 0, stream};
  return from_cuda(gdn::launch_prefill_stepwise(a));
}

gdn_status gdn_chunked_prefill_noalloc(const void* q, const void* k, const void* v,
                                       gdn_dtype qkv_dtype, int64_t q_row_stride,
                                       int64_t k_row_stride, int64_t v_row_stride,
                                       const void* g, const void* beta,
                                       gdn_dtype gate_dtype, const float* state_in,
                                       float* state_out, const int32_t* cu_seqlens,
                                       int N, int64_t T_total, int H_k, int H_v,
                                       float scale, void* o, gdn_dtype o_dtype,
                                       cudaStream_t stream) {
  if (N < 0 || T_total < 0) return GDN_ERR_INVALID_ARG;
  gdn_status st = check_recurrence(q, k, v, qkv_dtype, q_row_stride, k_row_stride,
                                   v_row_stride, g, beta, gate_dtype, H_k, H_v,
                                   o, o_dtype, T_total > 0);
  if (st != GDN_OK) return st;
  if (N == 0) return T_total == 0 ? GDN_OK : GDN_ERR_INVALID_ARG;
  if (!cu_seqlens) return GDN_ERR_INVALID_ARG;
  if ((state_in && !aligned16(state_in)) || (state_out && !aligned16(state_out)))
    return GDN_ERR_MISALIGNED;
  const size_t st_bytes = (size_t)N * H_v * kHeadDim * kHeadDim * sizeof(float);
  if (partial_overlap(state_in, st_bytes, state_out, st_bytes)) return GDN_ERR_INVALID_ARG;
  if (qkv_dtype == GDN_BF16 && T_total > 0 &&
      gdn_chunked_prefill_workspace(N, T_total, H_k, H_v) > gdn::prefill_noalloc_scratch_bytes())
    return GDN_ERR_UNSUPPORTED;
  gdn::RecurArgs a{q, k, v, qkv_dtype, q_row_stride, k_row_stride, v_row_stride,
                   g, beta, gate_dtype, state_in, state_out, cu_seqlens, N,
                   T_total, H_k, H_v, scale, o, o_dtype, nullptr, 0, stream};
  return from_cuda(qkv_dtype == GDN_BF16 ? gdn::launch_prefill_pc_noalloc(a)
                                         : gdn::launch_prefill_chunked_f32(a));
}

size_t gdn_chunked_prefill_noalloc_scratch_bytes(void) {
  return gdn::prefill_noalloc_scratch_bytes();
}

gdn_status gdn_decode_step(const void* q, const void* k, const void* v,
                           gdn_dtype qkv_dtype, int64_t q_row_stride,
                           int64_t k_row_stride, int64_t v_row_stride,
                           const void* g, const void* beta,
                           gdn_dtype gate_dtype, float* state, int N, int H_k,
                           int H_v, float scale, void* o, gdn_dtype o_dtype,
                           cudaStream_t stream) {
  if (N < 0) return GDN_ERR_INVALID_ARG;
  gdn_status st = check_recurrence(q, k, v, qkv_dtype, q_row_stride, k_row_stride,
                                   v_row_stride, g, beta, gate_dtype, H_k, H_v,
                                   o, o_dtype, N > 0);
  if (st != GDN_OK) return st;
  if (N == 0) return GDN_OK;
  if (!state) return GDN_ERR_INVALID_ARG;
  if (!aligned16(state)) return GDN_ERR_MISALIGNED;
  gdn::RecurArgs a{q, k, v, qkv_dtype, q_row_stride, k_row_stride, v_row_stride,
                   g, beta, gate_dtype, state, state, nullptr, N, N, H_k, H_v,
                   scale, o, o_dtype, nullptr, 0, stream};
  return from_cuda(gdn::launch_decode_step(a));
}

gdn_status gdn_decode_layer_step(const void* x, int64_t x_row_stride, gdn_dtype x_dtype,
                                 const void* conv_w, gdn_dtype w_dtype,
                                 const void* conv_bias, void* conv_state,
                                 const void* g, const void* beta, gdn_dtype gate_dtype,
                                 float* state, const int32_t* state_idx, int N, int P,
                                 int H_k, int H_v, float scale, float l2_eps,
                                 const void* z, const void* norm_w, float norm_eps,
                                 void* y, gdn_dtype y_dtype, cudaStream_t stream) {
  if (!valid_dtype(x_dtype) || !valid_dtype(w_dtype) || !valid_dtype(gate_dtype) ||
      !valid_dtype(y_dtype))
    return GDN_ERR_INVALID_ARG;
  if (N < 0 || P < 0 || H_k <= 0 || H_v <= 0 || H_v % H_k != 0 || !(l2_eps >= 0.f) ||
      !(norm_eps >= 0.f))
    return GDN_ERR_INVALID_ARG;
  if (H_v / H_k > 8) return GDN_ERR_UNSUPPORTED;
  const int64_t C = 2 * (int64_t)H_k * kHeadDim + (int64_t)H_v * kHeadDim;
  if (x_row_stride < C) return GDN_ERR_INVALID_ARG;
  if (N == 0) return GDN_OK;
  if (P == 0 || !x || !conv_w || !conv_state || !g || !beta || !state || !state_idx || !z ||
      !norm_w || !y)
    return GDN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(conv_w) || (conv_bias && !aligned16(conv_bias)) ||
      !aligned16(conv_state) || !aligned16(state) || !aligned16(z) || !aligned16(norm_w) ||
      !aligned16(y) || !aligned_to(state_idx, 4))
    return GDN_ERR_MISALIGNED;
  if (!stride_ok(x_row_stride, x_dtype)) return GDN_ERR_MISALIGNED;
  const int gb = gdn::elem_bytes(gate_dtype);
  if (!aligned_to(g, gb) || !aligned_to(beta, gb)) return GDN_ERR_MISALIGNED;
  gdn::DecodeLayerArgs a{x, x_row_stride, x_dtype, conv_w, w_dtype, conv_bias, conv_state,
                         g, beta, gate_dtype, state, state_idx, N, P, H_k, H_v, scale,
                         l2_eps, z, norm_w, norm_eps, y, y_dtype, stream};
  return from_cuda(gdn::launch_decode_layer(a));
}

gdn_status gdn_gated_rmsnorm(const void* x, gdn_dtype x_dtype, const void* z,
                             gdn_dtype z_dtype, const void* w,
                             gdn_dtype w_dtype, int64_t rows, int dim,
                             float eps, void* y, gdn_dtype y_dtype,
                             cudaStream_t stream) {
  if (!valid_dtype(x_dtype) || !valid_dtype(z_dtype) || !valid_dtype(w_dtype) ||
      !valid_dtype(y_dtype) || rows < 0 || !(eps >= 0.f))
    return GDN_ERR_INVALID_ARG;
  if (dim != kHeadDim) return GDN_ERR_UNSUPPORTED;
  if (rows == 0) return GDN_OK;
  if (!x || !z || !w || !y) return GDN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(z) || !aligned16(w) || !aligned16(y))
    return GDN_ERR_MISALIGNED;
  if (x == y && x_dtype != y_dtype) return GDN_ERR_INVALID_ARG;
  gdn::NormArgs a{x, x_dtype, z, z_dtype, w, w_dtype, rows, dim, eps, y, y_dtype,
                  stream};
  return from_cuda(gdn::launch_gated_rmsnorm(a));
}

// ---------------------------------------------------------- global attention

namespace {

constexpr int kAttnHeadDim = 256;

gdn_status check_attn_common(int H_q, int H_kv, int head_dim, int rope_dims, float rope_base,
                             float eps, gdn_dtype w_dtype) {
  if (head_dim != kAttnHeadDim) return GDN_ERR_UNSUPPORTED;
  if (H_q <= 0 || H_kv <= 0 || H_q % H_kv != 0) return GDN_ERR_INVALID_ARG;
  if (rope_dims < 0 || rope_dims > 64 || rope_dims % 2 != 0) return GDN_ERR_UNSUPPORTED;
  if (rope_dims > 0 && !(rope_base > 1.0f)) return GDN_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || !valid_dtype(w_dtype)) return GDN_ERR_INVALID_ARG;
  return GDN_OK;
}

bool attn_stride_ok(int64_t stride, int H) {
  return stride >= (int64_t)H * kAttnHeadDim && stride % 8 == 0;
}

}  // namespace

size_t gdn_attention_prefill_workspace(int64_t T_total, int H_q, int head_dim) {
  if (T_total < 0 || H_q <= 0 || head_dim != kAttnHeadDim) return 0;
  return gdn::attention_prefill_workspace(T_total, H_q);
}

gdn_status gdn_attention_prefill(const void* q, int64_t q_row_stride, const void* k,
                                 int64_t k_row_stride, const void* v, int64_t v_row_stride,
                                 const void* gate, int64_t gate_row_stride,
                                 const void* q_norm_w, const void* k_norm_w, gdn_dtype w_dtype,
                                 const int32_t* cu_seqlens, const int32_t* positions,
                                 const int32_t* pos0, int N, int64_t T_total, int H_q, int H_kv,
                                 int head_dim, float eps, int rope_dims, float rope_base,
                                 float scale, void* o, void* k_rot, void* v_h, void* workspace,
                                 size_t workspace_bytes, cudaStream_t stream) {
  gdn_status st = check_attn_common(H_q, H_kv, head_dim, rope_dims, rope_base, eps, w_dtype);
  if (st != GDN_OK) return st;
  if ((H_q / H_kv) % 2 != 0) return GDN_ERR_UNSUPPORTED;   // query heads go in pairs
  if (N < 0 || T_total < 0 || T_total > (int64_t)1 << 30) return GDN_ERR_INVALID_ARG;
  if (N == 0 && T_total > 0) return GDN_ERR_INVALID_ARG;
  if (!attn_stride_ok(q_row_stride, H_q) || !attn_stride_ok(gate_row_stride, H_q) ||
      !attn_stride_ok(k_row_stride, H_kv) || !attn_stride_ok(v_row_stride, H_kv))
    return GDN_ERR_MISALIGNED;
  if (T_total == 0) return GDN_OK;
  if (!q || !k || !v || !gate || !q_norm_w || !k_norm_w || !cu_seqlens || !o || !k_rot ||
      !v_h || !workspace)
    return GDN_ERR_INVALID_ARG;
  if (workspace_bytes < gdn::attention_prefill_workspace(T_total, H_q)) return GDN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(gate) || !aligned16(o) ||
      !aligned16(k_rot) || !aligned16(v_h) || !aligned16(workspace))
    return GDN_ERR_MISALIGNED;
  const int wb = gdn::elem_bytes(w_dtype);
  if (!aligned_to(q_norm_w, wb) || !aligned_to(k_norm_w, wb)) return GDN_ERR_MISALIGNED;
  gdn::AttnPrefillArgs a{q, k, v, gate, q_row_stride, k_row_stride, v_row_stride,
                         gate_row_stride, q_norm_w, k_norm_w, w_dtype, cu_seqlens, positions,
                         pos0, N, T_total, H_q, H_kv, eps, rope_dims, rope_base, scale, o,
                         k_rot, v_h, workspace, stream};
  return from_cuda(gdn::launch_attention_prefill(a));
}

size_t gdn_attention_decode_workspace(int N, int H_q, int L_max, int head_dim) {
  if (N < 0 || H_q <= 0 || L_max <= 0 || head_dim != kAttnHeadDim) return 0;
  return gdn::attention_decode_workspace(N, H_q, L_max);
}

gdn_status gdn_attention_decode(const void* q, int64_t q_row_stride, const void* k,
                                int64_t k_row_stride, const void* v, int64_t v_row_stride,
                                const void* gate, int64_t gate_row_stride,
                                const void* q_norm_w, const void* k_norm_w, gdn_dtype w_dtype,
                                void* k_cache, void* v_cache, const int32_t* cache_idx,
                                int32_t* cache_len, const int32_t* positions, int N, int P,
                                int L_max, int H_q, int H_kv, int head_dim, float eps,
                                int rope_dims, float rope_base, float scale, void* o,
                                void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  gdn_status st = check_attn_common(H_q, H_kv, head_dim, rope_dims, rope_base, eps, w_dtype);
  if (st != GDN_OK) return st;
  const int G = H_q / H_kv;
  if (G != 1 && G != 2 && G != 4 && G != 6 && G != 8) return GDN_ERR_UNSUPPORTED;
  if (N < 0 || N > 65535 || P < 0 || L_max <= 0 || H_q > 65535) return GDN_ERR_INVALID_ARG;
  if (!attn_stride_ok(q_row_stride, H_q) || !attn_stride_ok(gate_row_stride, H_q) ||
      !attn_stride_ok(k_row_stride, H_kv) || !attn_stride_ok(v_row_stride, H_kv))
    return GDN_ERR_MISALIGNED;
  if (N == 0) return GDN_OK;
  if (P == 0) return GDN_ERR_INVALID_ARG;
  if (!q || !k || !v || !gate || !q_norm_w || !k_norm_w || !k_cache || !v_cache ||
      !cache_len || !o || !workspace)
    return GDN_ERR_INVALID_ARG;
  if (workspace_bytes < gdn::attention_decode_workspace(N, H_q, L_max))
    return GDN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(gate) || !aligned16(o) ||
      !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(workspace))
    return GDN_ERR_MISALIGNED;
  const int wb = gdn::elem_bytes(w_dtype);
  if (!aligned_to(q_norm_w, wb) || !aligned_to(k_norm_w, wb)) return GDN_ERR_MISALIGNED;
  gdn::AttnDecodeArgs a{q, k, v, gate, q_row_stride, k_row_stride, v_row_stride,
                        gate_row_stride, q_norm_w, k_norm_w, w_dtype, k_cache, v_cache,
                        cache_idx, cache_len, positions, N, P, L_max, H_q, H_kv, eps,
                        rope_dims, rope_base, scale, o, workspace, stream};
  return from_cuda(gdn::launch_attention_decode(a));
}

gdn_status gdn_attention_status(const void* workspace, cudaStream_t stream) {
  if (!workspace) return GDN_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return GDN_ERR_MISALIGNED;
  int word = 0;
  if (gdn::attention_status_word(workspace, stream, &word) != cudaSuccess) return GDN_ERR_CUDA;
  if (word == 1) return GDN_ERR_TIMEOUT;
  if (word == 2) return GDN_ERR_INVALID_ARG;
  return GDN_OK;
}

}  // extern "C"
