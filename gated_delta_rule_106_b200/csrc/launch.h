// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
// Arguments arrive here already validated.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "gdn.h"

namespace gdn {

struct ConvArgs {
  const void* x; int64_t x_row_stride; gdn_dtype x_dtype;
  const void* w; gdn_dtype w_dtype; const void* bias;
  int channels; int l2norm_channels; float l2_eps;
  const int32_t* cu_seqlens; int N; int64_t T_total;
  const void* conv_state_in; void* conv_state_out;
  void* y; int64_t y_row_stride; gdn_dtype y_dtype;
  cudaStream_t stream;
  // elements per row of conv_state_in when it holds more channels than are
  // convolved here (the layer's q/k-only conv); 0: `channels`
  int64_t cs_row_stride;
};

struct RecurArgs {
  const void* q; const void* k; const void* v; gdn_dtype qkv_dtype;
  int64_t q_row_stride, k_row_stride, v_row_stride;
  const void* g; const void* beta; gdn_dtype gate_dtype;
  const float* state_in; float* state_out;   // decode: both = state
  const int32_t* cu_seqlens;                 // decode: unused
  int N; int64_t T_total; int H_k; int H_v; float scale;
  void* o; gdn_dtype o_dtype;
  void* workspace; size_t workspace_bytes;
  cudaStream_t stream;
};

// Fused decode step of the layer (conv roll + SiLU + q/k L2, recurrence on a
// pooled state, gated RMS-norm). x, the conv cache and z share x_dtype; the
// conv weights, bias and norm weight share w_dtype.
struct DecodeLayerArgs {
  const void* x; int64_t x_row_stride; gdn_dtype x_dtype;
  const void* conv_w; gdn_dtype w_dtype; const void* conv_bias;
  void* conv_state;                  // [P, 3, C] pool
  const void* g; const void* beta; gdn_dtype gate_dtype;
  float* state;                      // [P, H_v, 128, 128] pool
  const int32_t* state_idx;          // [N] slots (device)
  int N; int P; int H_k; int H_v; float scale; float l2_eps;
  const void* z; const void* norm_w; float norm_eps;
  void* y; gdn_dtype y_dtype;
  cudaStream_t stream;
};

// The whole prefill layer in the chunk kernel: conv + SiLU + q/k L2 from the
// pre-conv x (bf16) in the load stage, gated RMS-norm of the outputs before
// they leave. Conv weights, bias and the norm weight share w_dtype; z is bf16.
struct LayerPrefillArgs {
  const void* x; int64_t x_row_stride;
  const void* conv_w; gdn_dtype w_dtype; const void* conv_bias;
  const void* conv_state_in; void* conv_state_out;
  const void* g; const void* beta; gdn_dtype gate_dtype;
  const float* state_in; float* state_out;
  const int32_t* cu_seqlens; int N; int64_t T_total; int H_k; int H_v;
  float scale; float l2_eps;
  const void* z; const void* norm_w; float norm_eps;
  void* y; gdn_dtype y_dtype;
  void* workspace; size_t workspace_bytes;
  cudaStream_t stream;
};

// Global-attention prefill: q/k RMS-norm + rotary, then causal GQA flash
// attention with the sigmoid output gate. q, k, v, gate and o are bf16 with
// head dim 256; the rotated keys k_rot and the values v_h (as the KV cache
// holds them) are fp16; the norm weights are w_dtype.
struct AttnPrefillArgs {
  const void* q; const void* k; const void* v; const void* gate;
  int64_t q_row_stride, k_row_stride, v_row_stride, gate_row_stride;
  const void* wq; const void* wk; gdn_dtype w_dtype;
  const int32_t* cu_seqlens; const int32_t* positions; const int32_t* pos0;
  int N; int64_t T; int Hq; int Hkv;
  float eps; int rope_dims; float rope_base; float scale;
  void* o; void* k_rot; void* v_h;
  void* workspace;
  cudaStream_t stream;
};

// Global-attention decode: one new token per sequence against a pooled KV
// cache [P][L_max][Hkv][256] (fp16 keys and values); cache_len[n] is read, the new k / v go to
// that row, and it is advanced by one.
struct AttnDecodeArgs {
  const void* q; const void* k; const void* v; const void* gate;
  int64_t q_row_stride, k_row_stride, v_row_stride, gate_row_stride;
  const void* wq; const void* wk; gdn_dtype w_dtype;
  void* k_cache; void* v_cache; const int32_t* cache_idx; int32_t* cache_len;
  const int32_t* positions;
  int N; int P; int L_max; int Hq; int Hkv;
  float eps; int rope_dims; float rope_base; float scale;
  void* o; void* workspace;
  cudaStream_t stream;
};

struct NormArgs {
  const void* x; gdn_dtype x_dtype; const void* z; gdn_dtype z_dtype;
  const void* w; gdn_dtype w_dtype; int64_t rows; int dim; float eps;
  void* y; gdn_dtype y_dtype; cudaStream_t stream;
};

cudaError_t launch_conv1d_silu(const ConvArgs& a);
// conv_state_out[n] = the last three pre-conv rows of sequence n (shifted in
// from conv_state_in when shorter); conv_state_out may alias conv_state_in.
cudaError_t launch_conv_state_roll(const void* x, int64_t x_row_stride, gdn_dtype x_dtype,
                                   int channels, const int32_t* cu, int N, int64_t T,
                                   const void* cs_in, void* cs_out, cudaStream_t stream);
cudaError_t launch_prefill_layer(const LayerPrefillArgs& a);
// Workspace of gdn_prefill_layer: the chunk ring plus a bf16 [T, 2 H_k 128]
// scratch for the q/k conv output.
size_t prefill_layer_workspace(int N, int64_t T_total, int H_k, int H_v);
cudaError_t launch_gated_rmsnorm(const NormArgs& a);
cudaError_t launch_decode_step(const RecurArgs& a);
cudaError_t launch_decode_layer(const DecodeLayerArgs& a);
// Stepwise fp32 recurrence on the CUDA cores (any input dtype).
cudaError_t launch_prefill_stepwise(const RecurArgs& a);
// Chunk-64 recurrence on the CUDA cores in fp32 (fp32 inputs; any input dtype).
cudaError_t launch_prefill_chunked_f32(const RecurArgs& a);
// Chunk-64 tensor-core prefill (bf16 inputs), persistent producer/consumer
// kernel over all SMs; needs prefill_pc_workspace() bytes of workspace.
cudaError_t launch_prefill_pc(const RecurArgs& a);
size_t prefill_pc_workspace(int N, int64_t T_total, int H_v);
// The same kernel on the library-owned static scratch (no workspace argument).
cudaError_t launch_prefill_pc_noalloc(const RecurArgs& a);
size_t prefill_noalloc_scratch_bytes();
cudaError_t launch_attention_prefill(const AttnPrefillArgs& a);
size_t attention_prefill_workspace(int64_t T, int Hq);
cudaError_t launch_attention_decode(const AttnDecodeArgs& a);
size_t attention_decode_workspace(int N, int Hq, int L_max);
// Synchronises `stream`, then reads the status word the last attention call
// left in `workspace` (1: a wait inside the kernel ran out).
cudaError_t attention_status_word(const void* workspace, cudaStream_t stream, int* word);
// Limit of the chunk kernel's waits on another CTA's flag (0 restores 2 s).
void set_wait_limit_ns(uint64_t ns);
uint64_t wait_limit_ns();
// Synchronises `stream`, then reads the abort word of the workspace (NULL: the
// library-owned scratch) that the last chunk-kernel call on it left.
cudaError_t prefill_abort_word(const void* workspace, cudaStream_t stream, int* word);

}  // namespace gdn
