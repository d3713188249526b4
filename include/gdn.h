/*
 * gdn.h -- C ABI of the gated delta-rule layer library (libgdn.so, sm_100a).
 *
 * The layer is the recurrent ("delta-rule") layer of the Agnes-3.0-Flash
 * Preview hybrid decoder. Sources, cited by page and section:
 *   [P2]  "Agnes-3.0-Flash Preview" leaderboard commentary (discosf.com),
 *         section 二.1 "72 层里只有 18 层吃 KV cache": delta-rule layers are
 *         recurrent with 16 key / 48 value heads and head dim 128, a kernel-4
 *         causal conv comes first, the recurrent state is fp32
 *         (mamba_ssm_dtype float32), and the modeling code has a chunked
 *         prefill path (chunk = 64) and a stepwise decode path.
 *   [P3]  Agnes-3.0-Flash Preview model card (modelscope.cn README_zh),
 *         section 架构, architecture table: 3 of every 4 layers are gated
 *         delta-rule layers (54 of 72), state size independent of sequence
 *         length, causal conv (kernel 4) in front, gated RMS-norm, fp32 state.
 * The pages name the operations but print neither equations nor an
 * interface. The recurrence implemented is the gated delta rule
 *     S_t = g_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t = scale * S_t q_t
 * with S_t in R^{d_v x d_k} per (sequence, value head). Value head h reads
 * key/query head h / (H_v / H_k) (contiguous groups).
 *
 * Conventions for every entry point:
 *   - Every pointer is a DEVICE pointer on the current device, unless the
 *     parameter says otherwise. The caller owns all memory; the library never
 *     allocates, frees or synchronises, and launches only on `stream`.
 *   - Data pointers must be 16-byte aligned and row strides (given in
 *     ELEMENTS) must be multiples of 16 bytes; otherwise GDN_ERR_MISALIGNED.
 *   - Arguments are validated on the host before anything is launched; on
 *     any error nothing is launched and the outputs are untouched.
 *     GDN_ERR_CUDA reports a launch failure (cudaGetLastError after launch).
 *   - Head dim is fixed at 128 (d_k = d_v = 128) and H_v % H_k == 0.
 *   - Packed variable-length batches: tokens of N sequences are concatenated
 *     into T_total rows; cu_seqlens (device, int32, N+1 entries) holds the
 *     prefix sums with cu_seqlens[0] = 0, cu_seqlens[N] = T_total and
 *     non-decreasing entries (empty sequences allowed). cu_seqlens is read on
 *     the device only (no device-to-host copy). Entries outside [0, T_total]
 *     are clamped, so no access leaves the buffers, but the results for a
 *     malformed cu_seqlens are unspecified.
 *   - Recurrent states are fp32, [N, H_v, d_v=128, d_k=128], row-major
 *     (d_k contiguous): row i of a head's state is an independent 512-byte
 *     line.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GDN_OK = 0,
  GDN_ERR_INVALID_ARG = -1, /* null pointer, negative size, bad dtype ...  */
  GDN_ERR_UNSUPPORTED = -2, /* valid but not implemented (head dim != 128) */
  GDN_ERR_MISALIGNED = -3,  /* pointer or stride not 16-byte aligned        */
  GDN_ERR_CUDA = -4,        /* a CUDA launch or query failed               */
  GDN_ERR_TIMEOUT = -5      /* a bounded wait inside a kernel gave up      */
} gdn_status;

typedef enum { GDN_BF16 = 0, GDN_F32 = 1 } gdn_dtype;

/* Human-readable name of a status code (static string, never NULL). */
const char* gdn_status_string(gdn_status status);

/* Library version as "major.minor.patch" (static string). */
const char* gdn_version(void);

/*
 * gdn_conv1d_silu -- fused causal depthwise conv (kernel 4) + SiLU + per-head
 * L2 normalisation of the q and k channels.            [P2 二.1], [P3 架构]
 *
 *   y[t,c] = SiLU( bias[c] + sum_{j=0..3} w[c,j] * xh(t-3+j, c) )
 *   then for each 128-channel group m with 128*m < l2norm_channels:
 *   y[t, group] <- y[t, group] / sqrt(sum(y[t, group]^2) + l2_eps)
 *
 * xh(p, c) is the pre-conv input of the same sequence at position p; for
 * positions before the sequence's first token it is the carried history
 * conv_state_in[n, 3 + p_local, c] (p_local = -3..-1), or 0 when
 * conv_state_in is NULL. Tap j = 3 multiplies the current token.
 *
 *   x               [T_total, channels], x_dtype, row stride x_row_stride.
 *   w               [channels, 4], w_dtype (contiguous).
 *   bias            [channels], w_dtype, or NULL (no bias).
 *   channels        multiple of 8 (10240 = q 2048 | k 2048 | v 6144 here).
 *   l2norm_channels leading channels normalised per 128 (4096 = q|k), a
 *                   multiple of 128 and <= channels; 0 disables.
 *   cu_seqlens      [N+1] int32 (device), see conventions.
 *   conv_state_in   [N, 3, channels], x_dtype, oldest row first, or NULL.
 *   conv_state_out  [N, 3, channels], x_dtype, or NULL. Receives the last
 *                   three pre-conv rows of each sequence (shifted in from
 *                   conv_state_in for sequences shorter than 3). It may alias
 *                   conv_state_in (in-place roll for decode).
 *   y               [T_total, channels], y_dtype, row stride y_row_stride.
 *                   Must not overlap x.
 * T_total == 0 is valid (only the conv state is rolled, i.e. copied).
 * Decode uses the same call with one token per sequence.
 */
gdn_status gdn_conv1d_silu(const void* x, int64_t x_row_stride,
                           gdn_dtype x_dtype, const void* w, gdn_dtype w_dtype,
                           const void* bias, int channels, int l2norm_channels,
                           float l2_eps, const int32_t* cu_seqlens, int N,
                           int64_t T_total, const void* conv_state_in,
                           void* conv_state_out, void* y, int64_t y_row_stride,
                           gdn_dtype y_dtype, cudaStream_t stream);

/*
 * gdn_chunked_prefill -- the gated delta rule over packed sequences, computed
 * chunk by chunk (chunk = 64 tokens, the chunked prefill path of [P2 二.1]).
 * Results equal the stepwise recurrence above up to rounding.
 *
 *   q, k        [T_total, H_k, 128], qkv_dtype, token row strides
 *               q_row_stride / k_row_stride (elements; heads contiguous).
 *   v           [T_total, H_v, 128], qkv_dtype, row stride v_row_stride.
 *               (Strides let the call read the packed conv output in place.)
 *   g           [T_total, H_v] multiplicative decay in (0, 1], gate_dtype.
 *   beta        [T_total, H_v] write strength, gate_dtype.
 *   state_in    [N, H_v, 128, 128] fp32, or NULL for zero initial states.
 *   state_out   [N, H_v, 128, 128] fp32, or NULL (not written). May alias
 *               state_in exactly (in-place update); no partial overlap.
 *   scale       multiplies every output (1.0 for the plain rule).
 *   o           [T_total, H_v, 128] contiguous, o_dtype.
 *   workspace   device scratch of gdn_chunked_prefill_workspace(...) bytes
 *               (may be NULL when that is 0).
 * Numerics: with qkv_dtype == GDN_BF16 the chunk products run on the tensor
 * cores with binary16 operands and fp32 accumulation (bf16 inputs convert to
 * binary16 exactly when |x| lies in [2^-14, 65504]; smaller magnitudes keep
 * an absolute error below 2^-25); the state is carried in fp32. Inputs,
 * states and outputs must stay well inside the binary16 range (|x| < 6e4).
 * With qkv_dtype == GDN_F32 the same chunk-64 form runs on the CUDA cores
 * with every product in fp32 (one CTA per sequence and value head); it needs
 * no workspace.
 */
gdn_status gdn_chunked_prefill(const void* q, const void* k, const void* v,
                               gdn_dtype qkv_dtype, int64_t q_row_stride,
                               int64_t k_row_stride, int64_t v_row_stride,
                               const void* g, const void* beta,
                               gdn_dtype gate_dtype, const float* state_in,
                               float* state_out, const int32_t* cu_seqlens,
                               int N, int64_t T_total, int H_k, int H_v,
                               float scale, void* o, gdn_dtype o_dtype,
                               void* workspace, size_t workspace_bytes,
                               cudaStream_t stream);

/* Device scratch bytes gdn_chunked_prefill needs for these sizes (host). */
size_t gdn_chunked_prefill_workspace(int N, int64_t T_total, int H_k, int H_v);

/*
 * gdn_prefill_layer -- the whole prefill of the delta-rule layer as two
 * launches: the causal conv (kernel 4) + SiLU + per-head L2 norm of the q and k
 * heads ([P2 二.1], [P3 架构]) once per key head into a workspace scratch, then
 * the tensor-core chunk kernel, which convolves each value head's v channels in
 * its load stage from the pre-conv input, runs the chunked (chunk = 64) gated
 * delta rule ([P2 二.1]) as in gdn_chunked_prefill, and applies the gated
 * RMS-norm ([P3 架构]) to each output tile before it leaves. The result equals
 * gdn_conv1d_silu -> gdn_chunked_prefill (o in y_dtype) -> gdn_gated_rmsnorm:
 * the conv values enter the chunk products rounded to bf16 exactly as the conv
 * kernel stores them, and the norm reads the outputs in y_dtype. Neither the v
 * conv output nor the un-normed output is written to memory. Additional entry
 * point (fused form of the three calls).
 *
 *   x            [T_total, C] bf16, row stride x_row_stride: pre-conv q | k | v,
 *                C = 2*H_k*128 + H_v*128.
 *   conv_w       [C, 4] w_dtype (tap 3 = current token); conv_bias [C] w_dtype or NULL.
 *   conv_state_in   [N, 3, C] bf16 history before each sequence, or NULL (zeros).
 *   conv_state_out  [N, 3, C] bf16 or NULL: each sequence's last three pre-conv
 *                rows (may alias conv_state_in; written after the kernel has read it).
 *   g, beta, state_in, state_out, cu_seqlens, N, T_total, H_k, H_v, scale:
 *                as gdn_chunked_prefill.
 *   workspace    gdn_prefill_layer_workspace(N, T_total, H_k, H_v) bytes, 16-byte
 *                aligned: the chunk ring and a bf16 [T_total, 2*H_k*128] q/k scratch.
 *   l2_eps       q/k L2 epsilon: y / sqrt(sum y^2 + l2_eps).
 *   z            [T_total, H_v, 128] bf16 gate; norm_w [128] w_dtype; norm_eps.
 *   y            [T_total, H_v, 128] contiguous, y_dtype: the normed output.
 * A bounded wait that gives up is reported by gdn_chunked_prefill_status.
 */
size_t gdn_prefill_layer_workspace(int N, int64_t T_total, int H_k, int H_v);
gdn_status gdn_prefill_layer(const void* x, int64_t x_row_stride, const void* conv_w,
                             gdn_dtype w_dtype, const void* conv_bias,
                             const void* conv_state_in, void* conv_state_out,
                             const void* g, const void* beta, gdn_dtype gate_dtype,
                             const float* state_in, float* state_out,
                             const int32_t* cu_seqlens, int N, int64_t T_total, int H_k,
                             int H_v, float scale, float l2_eps, const void* z,
                             const void* norm_w, float norm_eps, void* y, gdn_dtype y_dtype,
                             void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * gdn_chunked_prefill_status -- did the last gdn_chunked_prefill (bf16 inputs)
 * that worked in `workspace` complete? Its CTAs hand chunks to one another
 * through flags in the workspace, and every wait on such a flag is bounded
 * (gdn_set_wait_limit_ns); a wait that runs out makes the whole call give up:
 * each CTA leaves, the outputs o and state_out of every (sequence, head) not
 * finished are written as NaN, and the workspace's abort word is set. This
 * call waits for `stream` (it synchronises: it is not meant for the hot path),
 * reads that word and returns GDN_OK or GDN_ERR_TIMEOUT (GDN_ERR_CUDA if the
 * synchronisation or the 4-byte read fails). workspace == NULL reads the
 * library-owned array of gdn_chunked_prefill_noalloc instead. The word is
 * cleared by the next call that uses the workspace. Additional entry point.
 */
gdn_status gdn_chunked_prefill_status(const void* workspace, cudaStream_t stream);

/*
 * gdn_set_wait_limit_ns -- the bound, in nanoseconds, on each wait of the
 * chunked prefill kernel for a flag that another CTA sets (0 restores the
 * default, 2 s). A lower bound makes a stuck call give up sooner; the waits of
 * a CTA on its own copies and tensor-core products keep their 2 s bound.
 * Process-wide; read at each launch. Additional entry point.
 */
void gdn_set_wait_limit_ns(uint64_t ns);

/*
 * gdn_stepwise_prefill -- the same packed-sequence recurrence advanced token by
 * token (the stepwise path of [P2 二.1], which the modeling code uses for
 * decode), for any prompt length: the recurrence written out, in fp32 on the
 * CUDA cores. A warp owns 32 rows of one (sequence, value head) state and
 * keeps them in registers for the whole sequence, so the state crosses HBM
 * once per call; the time grows with the longest sequence (one dependent
 * update per token). It is the reference-grade path next to the chunked one:
 * both compute the same recurrence and must agree up to rounding.
 * Arguments, layouts and errors are those of gdn_chunked_prefill without the
 * workspace. Additional entry point (the pages name the path, not the call).
 */
gdn_status gdn_stepwise_prefill(const void* q, const void* k, const void* v,
                                gdn_dtype qkv_dtype, int64_t q_row_stride,
                                int64_t k_row_stride, int64_t v_row_stride,
                                const void* g, const void* beta,
                                gdn_dtype gate_dtype, const float* state_in,
                                float* state_out, const int32_t* cu_seqlens,
                                int N, int64_t T_total, int H_k, int H_v,
                                float scale, void* o, gdn_dtype o_dtype,
                                cudaStream_t stream);

/*
 * gdn_chunked_prefill_noalloc -- gdn_chunked_prefill with no workspace
 * argument: the library supplies the working memory itself. It is meant for
 * callers that cannot hand the library device memory at the call site -- for
 * example an operator plugged into a host framework whose allocator the plugin
 * cannot reach, or a serving loop whose memory plan forbids any allocation
 * after start-up. The pages have no counterpart to this call; it exists only
 * for such callers.
 *
 * Arguments, results and numerics are those of gdn_chunked_prefill. The
 * working memory is one static device array of
 * gdn_chunked_prefill_noalloc_scratch_bytes() bytes (29 218 816: the chunk
 * rings of 49 state CTAs) that every GPU which loads the library holds until
 * the process exits. A problem whose working memory would exceed it returns
 * GDN_ERR_UNSUPPORTED without launching (on a 148-SM B200 none does). The
 * call itself never allocates or frees memory.
 * The first call on a device looks up the array's device address with that
 * device current; make that first call before any stream capture begins.
 * Every call uses the same array and leaves its contents behind (the next
 * call clears what must start at zero): calls whose executions overlap on the
 * GPU -- on different streams or from different host threads -- race and give
 * undefined results.
 */
gdn_status gdn_chunked_prefill_noalloc(const void* q, const void* k, const void* v,
                                       gdn_dtype qkv_dtype, int64_t q_row_stride,
                                       int64_t k_row_stride, int64_t v_row_stride,
                                       const void* g, const void* beta,
                                       gdn_dtype gate_dtype, const float* state_in,
                                       float* state_out, const int32_t* cu_seqlens,
                                       int N, int64_t T_total, int H_k, int H_v,
                                       float scale, void* o, gdn_dtype o_dtype,
                                       cudaStream_t stream);

/* Bytes of the static device array gdn_chunked_prefill_noalloc works in. */
size_t gdn_chunked_prefill_noalloc_scratch_bytes(void);

/*
 * gdn_decode_step -- one stepwise update of the gated delta rule for N
 * sequences, one token each (the stepwise decode path of [P2 二.1]):
 *   S <- g S (I - beta k k^T) + beta v k^T ;  o = scale * S q
 * The state is read and written in place; each head's 64 KiB state crosses
 * HBM once per call.
 *
 *   q, k    [N, H_k, 128], qkv_dtype, row strides q_row_stride/k_row_stride.
 *   v       [N, H_v, 128], qkv_dtype, row stride v_row_stride.
 *   g, beta [N, H_v], gate_dtype.
 *   state   [N, H_v, 128, 128] fp32, updated in place.
 *   o       [N, H_v, 128] contiguous, o_dtype.
 * N == 0 is valid (nothing is launched).
 */
gdn_status gdn_decode_step(const void* q, const void* k, const void* v,
                           gdn_dtype qkv_dtype, int64_t q_row_stride,
                           int64_t k_row_stride, int64_t v_row_stride,
                           const void* g, const void* beta,
                           gdn_dtype gate_dtype, float* state, int N, int H_k,
                           int H_v, float scale, void* o, gdn_dtype o_dtype,
                           cudaStream_t stream);

/*
 * gdn_decode_layer_step -- one decode token of the whole delta-rule layer for
 * N sequences in one launch: the causal conv (kernel 4) over the conv cache
 * with the cache rolled in place, SiLU and the per-head L2 norm of q and k, the
 * stepwise gated delta rule on the sequence's fp32 state, and the gated
 * RMS-norm of the output (the stepwise decode path of [P2 二.1]; conv k=4,
 * gated RMS-norm and fp32 state: [P3 架构]). The result equals
 * gdn_conv1d_silu -> gdn_decode_step -> gdn_gated_rmsnorm except that q, k, v
 * stay in fp32 between the stages (they are not stored in x_dtype).
 * Additional entry point (fused form of the three calls, for serving).
 *
 * States and conv caches live in pools indexed by a slot per sequence, as a
 * server keeps them:
 *   x           [N, C] x_dtype, row stride x_row_stride: the new token's
 *               pre-conv channels q | k | v, C = 2*H_k*128 + H_v*128.
 *   conv_w      [C, 4] w_dtype (tap 3 = current token); conv_bias [C] w_dtype
 *               or NULL.
 *   conv_state  [P, 3, C] x_dtype pool, oldest row first; slot state_idx[n]
 *               is read and rolled in place (its rows become h1, h2, x_n).
 *   g, beta     [N, H_v] gate_dtype.
 *   state       [P, H_v, 128, 128] fp32 pool; slot state_idx[n] is updated in
 *               place.
 *   state_idx   [N] int32 (device): the pool slot of sequence n, the same in
 *               both pools. Slots of different sequences must differ. A slot
 *               outside [0, P) marks padding: nothing of it is read or
 *               written except its output rows, which are set to 0.
 *   scale       multiplies o (1.0 for the plain rule); l2_eps: the q/k norm's
 *               epsilon, y / sqrt(sum y^2 + l2_eps).
 *   z           [N, H_v, 128] x_dtype, the output gate; norm_w [128] w_dtype;
 *               norm_eps: out = o / sqrt(mean(o^2) + norm_eps) * norm_w * SiLU(z).
 *   y           [N, H_v, 128] contiguous, y_dtype: the normed output.
 * Two launches on `stream`: the layer kernel (one CTA per sequence and value
 * head; each computes q and k of its key head itself and rolls its own v
 * cache rows) and a small kernel that then rolls the q/k cache rows, which
 * every value head of a key head reads. H_v / H_k must be at most 8, else
 * GDN_ERR_UNSUPPORTED. N == 0 is valid.
 */
gdn_status gdn_decode_layer_step(const void* x, int64_t x_row_stride, gdn_dtype x_dtype,
                                 const void* conv_w, gdn_dtype w_dtype,
                                 const void* conv_bias, void* conv_state,
                                 const void* g, const void* beta, gdn_dtype gate_dtype,
                                 float* state, const int32_t* state_idx, int N, int P,
                                 int H_k, int H_v, float scale, float l2_eps,
                                 const void* z, const void* norm_w, float norm_eps,
                                 void* y, gdn_dtype y_dtype, cudaStream_t stream);

/*
 * gdn_gated_rmsnorm -- gated RMS-norm on the layer output ([P3 架构]):
 *   y = x / sqrt(mean(x^2) + eps) * w * SiLU(z)
 * over rows of `dim` channels (one row per token and value head).
 *
 *   x  [rows, dim] x_dtype; z [rows, dim] z_dtype; w [dim] w_dtype (shared by
 *   all rows); y [rows, dim] y_dtype (may alias x when the dtypes match).
 *   dim must be 128. rows == 0 is valid.
 */
gdn_status gdn_gated_rmsnorm(const void* x, gdn_dtype x_dtype, const void* z,
                             gdn_dtype z_dtype, const void* w,
                             gdn_dtype w_dtype, int64_t rows, int dim,
                             float eps, void* y, gdn_dtype y_dtype,
                             cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Global-attention layer: the hybrid decoder's other layer type, one of
 * every four layers (18 of 72) and the only one holding a KV cache ([P3 架构],
 * rows 全局注意力 and 位置编码; [P2 二.1], attn_output_gate true). Per token:
 *   qn = q / sqrt(mean(q^2) + eps) * q_norm_w   (per head over head_dim)
 *   kn = k / sqrt(mean(k^2) + eps) * k_norm_w
 *   rotary on dims [0, rope_dims): pair i couples dims i and i + rope_dims/2
 *     and turns (counter-clockwise: (a, b) -> (a c - b s, b c + a s)) by
 *     theta_i = p_{i mod 3} * rope_base^(-2i / rope_dims), where (p_0, p_1,
 *     p_2) are the token's text, height and width positions (the pages'
 *     interleaved 11 : 11 : 10 split of the 32 pairs at rope_dims = 64);
 *   o_h = sum_j softmax_j(scale * qn_h . kn_j) v_j over the earlier tokens j
 *     of the same sequence and itself, query head h reading key-value head
 *     h / (H_q / H_kv);
 *   out_h = o_h * sigmoid(gate_h)   (elementwise).
 * The model's sizes are H_q = 24, H_kv = 4, head_dim = 256, rope_dims = 64,
 * rope_base = 1e7; head_dim must be 256 and rope_dims even and <= 64
 * (GDN_ERR_UNSUPPORTED otherwise). q, k, v, gate and o are bf16. The KV
 * cache is fp16: the normed, rotated keys are bounded by
 * 16 * sqrt(2) * max|k_norm_w|, inside fp16's range, and fp16 keeps three
 * more significand bits than bf16 for the score product; a bf16 value in
 * fp16's normal range converts to fp16 exactly (beyond +-65504 it saturates),
 * and fp16 values let the softmax weights P enter P V in fp16 as well. The
 * norm weights are w_dtype (bf16 or fp32). Row strides are per
 * token (prefill) or per sequence (decode), in elements, multiples of 8 and
 * at least H * 256; each head's 256 values are contiguous.
 * ---------------------------------------------------------------------- */

/*
 * gdn_attention_prefill -- causal attention over a packed batch of prompts.
 *   q, gate [T_total, H_q, 256]; k, v [T_total, H_kv, 256] (row strides as
 *   given); cu_seqlens as for the delta-rule layer.
 *   positions  [3, T_total] int32 (text, height, width) or NULL: then every
 *              axis carries the token's index within its sequence plus
 *              pos0[n] (pos0 [N] int32, or NULL for 0) -- a prompt that
 *              continues a cached prefix passes the prefix length there.
 *   o          [T_total, H_q, 256] contiguous: the gated output.
 *   k_rot      [T_total, H_kv, 256] contiguous fp16: the normed, rotated
 *              keys, as the key cache holds them.
 *   v_h        [T_total, H_kv, 256] contiguous fp16: v as the value cache
 *              holds it.
 *   workspace  gdn_attention_prefill_workspace(T_total, H_q, 256) bytes,
 *              16-byte aligned (the rotated queries and a status word).
 * (H_q / H_kv) must be even: a CTA works on two query heads of one group.
 * Each attention CTA's waits on its own copies and tensor-core products are
 * bounded (2 s); gdn_attention_status reports one that ran out. Additional
 * entry point (the pages describe the layer, not an interface).
 */
size_t gdn_attention_prefill_workspace(int64_t T_total, int H_q, int head_dim);
gdn_status gdn_attention_prefill(const void* q, int64_t q_row_stride, const void* k,
                                 int64_t k_row_stride, const void* v, int64_t v_row_stride,
                                 const void* gate, int64_t gate_row_stride,
                                 const void* q_norm_w, const void* k_norm_w, gdn_dtype w_dtype,
                                 const int32_t* cu_seqlens, const int32_t* positions,
                                 const int32_t* pos0, int N, int64_t T_total, int H_q, int H_kv,
                                 int head_dim, float eps, int rope_dims, float rope_base,
                                 float scale, void* o, void* k_rot, void* v_h, void* workspace,
                                 size_t workspace_bytes, cudaStream_t stream);

/*
 * gdn_attention_decode -- one new token for each of N sequences against a
 * pooled KV cache.
 *   q, gate [N, H_q, 256]; k, v [N, H_kv, 256] (row strides per sequence).
 *   k_cache, v_cache  [P, L_max, H_kv, 256] fp16 pools; sequence n lives in
 *              slot cache_idx[n] (cache_idx NULL: slot n) and has
 *              cache_len[n] tokens cached (rotated keys, as
 *              gdn_attention_prefill's k_rot and v_h). The new token's
 *              rotated k and its v (in fp16) are written at row cache_len[n], the token attends to
 *              rows 0 .. cache_len[n], and cache_len[n] is then advanced by
 *              one on the device (the caller's copy of it stays in step).
 *   positions  [3, N] int32 or NULL (then cache_len[n] on every axis).
 *   o          [N, H_q, 256] contiguous.
 *   workspace  gdn_attention_decode_workspace(N, H_q, L_max, 256) bytes.
 * H_q / H_kv must be 1, 2, 4, 6 or 8. A sequence whose slot is outside
 * [0, P) or whose cache_len is outside [0, L_max) is skipped: its cache and
 * cache_len stay untouched, its output is NaN, and gdn_attention_status
 * returns GDN_ERR_INVALID_ARG. Distinct sequences must use distinct slots.
 * Additional entry point.
 */
size_t gdn_attention_decode_workspace(int N, int H_q, int L_max, int head_dim);
gdn_status gdn_attention_decode(const void* q, int64_t q_row_stride, const void* k,
                                int64_t k_row_stride, const void* v, int64_t v_row_stride,
                                const void* gate, int64_t gate_row_stride,
                                const void* q_norm_w, const void* k_norm_w, gdn_dtype w_dtype,
                                void* k_cache, void* v_cache, const int32_t* cache_idx,
                                int32_t* cache_len, const int32_t* positions, int N, int P,
                                int L_max, int H_q, int H_kv, int head_dim, float eps,
                                int rope_dims, float rope_base, float scale, void* o,
                                void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * gdn_attention_status -- waits for `stream` (it synchronises), then reads the
 * status word that the last attention call working in `workspace` left:
 * GDN_OK; GDN_ERR_TIMEOUT when a bounded wait inside the prefill kernel ran
 * out (the affected output tiles are left unwritten); GDN_ERR_INVALID_ARG when
 * a decode sequence had an out-of-range slot or length. Additional entry point.
 */
gdn_status gdn_attention_status(const void* workspace, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
