/*
 * fp8attn -- on-the-fly FP8 (E4M3) quantisation of Q/K/V with per-tensor
 * scales, followed by a varlen, non-causal FP8 flash-attention forward, for
 * NVIDIA B200 (sm_100a).  Plain C ABI: device pointers are raw CUDA device
 * addresses, host pointers are ordinary host memory, streams are
 * `cudaStream_t` values passed as `void*` (NULL = the legacy default stream).
 *
 * Method (web pages on FP8 ViT / DiT attention):
 *   - vLLM docs, "FP8 ViT encoder attention": Q/K/V are quantised to FP8 on
 *     the fly right before the attention call (introduction); by default a
 *     circular buffer of 16 observed Q/K/V amax values drives the per-forward
 *     scale update (usage section); static per-layer scales can be calibrated
 *     once -- 16 dynamic passes, then the learned scales are saved multiplied
 *     by a save margin, default 1.5 -- and reused (usage section, scale file
 *     format section); the reference cost is three quantisation launches plus
 *     an unpadding step (notes).
 *   - vLLM-Omni docs, "Quantized KV Cache": eligible full (non-causal)
 *     attention forwards use FP8; layers named by a selector of
 *     comma-separated integers and inclusive ranges keep the native dtype
 *     (parameters table).
 *   - Ascend quantisation chapter: FP8 formats E4M3 / E5M2 (names only).
 *
 * Readings where the pages are silent (each is fixed here):
 *   - E4M3 is the OCP "FN" format: max 448, no infinities; casts round to
 *     nearest even and saturate to +-448; NaN casts to 0x7F.
 *   - amax = max |x| over the valid (unpadded) tokens of one tensor; NaN is
 *     ignored; an infinite amax is reported (FP8ATTN_ERR_NONFINITE) and not
 *     pushed.
 *   - Dynamic scaling is current-inclusive: the pass's amax is pushed into
 *     the 16-entry ring first, then A = max over the filled slots.
 *   - qs = fl32(448 / A), ds = fl32(A / 448) (each one correctly rounded fp32
 *     division); A == 0 gives qs = ds = 1.  code = e4m3(fl32(x * qs)).
 *   - Static values are bounds A in activation units with the margin already
 *     applied (the margin multiplies saved values once, at export).
 *   - Attention: s = q8.k8 * ds_q * ds_k * softmax_scale, t = s log2(e);
 *     per 128-key block, P for the PV product is e4m3(2^(t - r + 5)) with r
 *     the row's reference max (block 0's max, moved to a later block's max
 *     only when that exceeds r by more than 3, so P <= 256); the row sum l
 *     accumulates the unquantised 2^(t - r + 5) carried to a common max;
 *     out = bf16(O * ds_v / l).  The bf16 entry point takes r = the running
 *     max and P = bf16(2^(t - r)).
 *
 * Layouts: bf16 sources are addressed as (token, head, channel) with the
 * channel contiguous (head_dim == 128) and element strides `tok_stride`,
 * `head_stride` (multiples of 8; 16-byte aligned base), so packed [T,H,D],
 * padded [B,S_max,H,D] and interleaved [T,3,H,D] sources all work.  FP8
 * outputs and attention inputs/outputs are packed [T,H,D] with
 * T = total_tokens (the row count of those buffers).
 *
 * Errors: host-detectable problems return a status at once and launch
 * nothing.  Problems found on the device (inconsistent cu_seqlens, a wait
 * that ran past its time limit, a non-finite amax) set a device error word
 * and the kernel skips the affected work without trapping;
 * fp8attn_get_error() reports and clears it.
 *
 * Ownership: the caller allocates and owns every buffer, including the
 * context's device workspace; a context owns only a small host struct.
 * All launches are asynchronous on the given stream; functions that read
 * results back to the host synchronise that stream and say so.
 */
#ifndef FP8ATTN_H_
#define FP8ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FP8ATTN_OK = 0,
  FP8ATTN_ERR_INVALID = 1,     /* bad argument (null, negative, out of range) */
  FP8ATTN_ERR_CUDA = 2,        /* a CUDA runtime / driver call failed */
  FP8ATTN_ERR_TIMEOUT = 3,     /* a device-side wait gave up (work skipped) */
  FP8ATTN_ERR_UNSUPPORTED = 4, /* valid but unsupported (head_dim != 128, ...) */
  FP8ATTN_ERR_NONFINITE = 5,   /* an observed amax was infinite (not pushed) */
  FP8ATTN_ERR_SEQLENS = 6      /* cu_seqlens inconsistent with batch/max_seqlen */
} fp8attn_status;

/* Per-layer quantisation mode (host-side selection). */
typedef enum {
  FP8ATTN_DYNAMIC = 0, /* amax ring, current pass included */
  FP8ATTN_STATIC = 1,  /* static bounds set by fp8attn_set_static_scales */
  FP8ATTN_SKIP = 2,    /* native bf16 attention, no quantisation */
  FP8ATTN_RING = 3     /* cast with the layer's current ring scales (the last ring
                          update), no amax pass, ring unchanged: the cast step of a
                          head-sharded dynamic pass (fp8attn_amax_qkv) */
} fp8attn_mode;

typedef struct fp8attn_ctx fp8attn_ctx;

/* Human-readable name of a status code (static string). */
const char* fp8attn_status_string(int status);

/* Entries per amax ring: 16 (vLLM FP8 ViT page, usage section). */
int fp8attn_ring_length(void);

/* Bytes of device workspace a context for `num_layers` layers needs (ring,
 * scales, static bounds, grid-barrier words, error word). 0 if num_layers<1. */
size_t fp8attn_workspace_bytes(int num_layers);

/* Create a context over caller-owned device workspace `d_workspace` of at
 * least fp8attn_workspace_bytes(num_layers) bytes (256-byte aligned).  The
 * workspace is zeroed on `stream` (empty rings, no static scales).  The
 * current CUDA device must be the workspace's device.  *out receives the
 * context.  Errors: INVALID (null pointers, too small, misaligned), CUDA. */
fp8attn_status fp8attn_create(int num_layers, void* d_workspace, size_t workspace_bytes,
                              void* stream, fp8attn_ctx** out);

/* Free the host struct (the workspace stays the caller's). */
fp8attn_status fp8attn_destroy(fp8attn_ctx* ctx);

/* Fused amax-reduce + ring/scale update + E4M3 cast + unpad of Q, K and V
 * for one layer, in a single launch (replaces the pages' three quantisation
 * launches plus unpadding).
 *   mode DYNAMIC: amax of each tensor over its valid tokens; push into the
 *     layer's ring; A = ring max; cast with qs = 448/A.  STATIC: cast with the
 *     layer's static bounds (error INVALID if none were set).  RING: cast with
 *     the layer's current scales, ring unchanged.  SKIP: INVALID.
 *   q, k, v: bf16 sources; element (t_src, h, d) at base + t_src*tok_stride
 *     + h*head_stride + d.  d_src_seq_start: NULL if the source is packed
 *     (t_src = t); else int32[batch], the source row of each sequence's first
 *     token (padded source).  d_cu_seqlens: int32[batch+1], non-decreasing,
 *     cu[0] = 0, each length <= max_seqlen, cu[batch] == total_tokens.
 *   q8, k8, v8: E4M3 outputs, packed [total_tokens, num_heads, head_dim].
 * The layer's scales (fp8attn_descale_ptr) are updated on the device.
 * Errors: INVALID, UNSUPPORTED (head_dim != 128, misaligned strides), CUDA;
 * device-side: SEQLENS (nothing written), NONFINITE, TIMEOUT. */
fp8attn_status fp8attn_quantize_qkv(fp8attn_ctx* ctx, int layer, int mode, const void* q,
                                    const void* k, const void* v, int64_t tok_stride,
                                    int64_t head_stride, const int32_t* d_src_seq_start,
                                    const int32_t* d_cu_seqlens, int batch, int max_seqlen,
                                    int64_t total_tokens, int num_heads, int head_dim, void* q8,
                                    void* k8, void* v8, void* stream);

/* The cast of fp8attn_quantize_qkv (modes STATIC and RING only) writing each
 * output head-grouped: q8, k8, v8 are [groups][total_tokens][num_heads /
 * groups][head_dim], group g holding heads [g H/groups, (g+1) H/groups) of
 * every token, i.e. the send buffer of the all-to-all that hands group g to
 * rank g in sequence-parallel (Ulysses) attention (vLLM-Omni "Quantized KV
 * Cache", Configuration: the DiT sharded over a Ulysses degree).  One launch
 * for all groups; the codes equal those of fp8attn_quantize_qkv, regrouped.
 * groups must divide num_heads (groups = 1 is the packed layout).  Sources,
 * scales and errors as fp8attn_quantize_qkv; INVALID for mode DYNAMIC or
 * SKIP (a sharded dynamic pass reduces its amax across ranks first, then
 * casts with RING) and for a bad group count. */
fp8attn_status fp8attn_quantize_qkv_grouped(fp8attn_ctx* ctx, int layer, int mode, const void* q,
                                            const void* k, const void* v, int64_t tok_stride,
                                            int64_t head_stride, const int32_t* d_src_seq_start,
                                            const int32_t* d_cu_seqlens, int batch,
                                            int max_seqlen, int64_t total_tokens, int num_heads,
                                            int head_dim, int groups, void* q8, void* k8,
                                            void* v8, void* stream);

/* Per-tensor amax of Q, K and V over their valid tokens into d_amax3 (device
 * float[3]; NaN ignored, an infinite amax stays infinite), without casting
 * and without touching any ring (vLLM FP8 ViT page, usage section: the ring
 * holds observed Q/K/V amax values).  With heads sharded across GPUs, each
 * rank runs this on its shard, the three values are all-reduced with MAX,
 * pushed with fp8attn_amax_ring_update, and each shard is cast with mode
 * FP8ATTN_RING: codes, scales and ring then equal those of one DYNAMIC pass
 * over all heads.  Sources and errors as fp8attn_quantize_qkv (no outputs);
 * uses the context's reduction words, so it must not overlap another call
 * on the same context. */
fp8attn_status fp8attn_amax_qkv(fp8attn_ctx* ctx, const void* q, const void* k, const void* v,
                                int64_t tok_stride, int64_t head_stride,
                                const int32_t* d_src_seq_start, const int32_t* d_cu_seqlens,
                                int batch, int max_seqlen, int64_t total_tokens, int num_heads,
                                int head_dim, float* d_amax3, void* stream);

/* Push three externally observed amax values (device float[3]: q, k, v) into
 * the layer's rings and recompute its scales, on the device (vLLM FP8 ViT
 * page, usage section: the ring drives the per-forward scale).  A NaN or
 * infinite value is not pushed and sets NONFINITE.  Errors: INVALID, CUDA. */
fp8attn_status fp8attn_amax_ring_update(fp8attn_ctx* ctx, int layer, const float* d_amax3,
                                        void* stream);

/* Set a layer's static bounds (values as stored in a scale file: q, k, v,
 * margin already applied; vLLM FP8 ViT page, scale file format section).
 * Enqueues a small host->device copy on `stream`.  Errors: INVALID
 * (negative or non-finite value, bad layer), CUDA. */
fp8attn_status fp8attn_set_static_scales(fp8attn_ctx* ctx, int layer, float q, float k,
                                         float v, void* stream);

/* Forget a layer's static bounds (host-side flag only). */
fp8attn_status fp8attn_clear_static_scales(fp8attn_ctx* ctx, int layer);

/* 1 if the layer has static bounds, 0 if not, -1 on a bad argument. */
int fp8attn_has_static_scales(const fp8attn_ctx* ctx, int layer);

/* Export the calibrated static values for every layer: h_out[l*3 + t] =
 * fl32(max(ring of tensor t of layer l) * margin), t = q, k, v (vLLM FP8 ViT
 * page, usage section: saved scales are multiplied by the save margin,
 * default 1.5).  Synchronises `stream`.  Errors: INVALID, CUDA. */
fp8attn_status fp8attn_export_static_scales(fp8attn_ctx* ctx, float margin, float* h_out,
                                            void* stream);

/* Device pointer to the layer's current descales {ds_q, ds_k, ds_v} (fp32),
 * as written by the last quantisation of that layer -- the scale argument of
 * fp8attn_varlen_fwd.  NULL on a bad argument. */
const float* fp8attn_descale_ptr(fp8attn_ctx* ctx, int layer);

/* Device pointer to the layer's current quantisation scales {qs_q, qs_k, qs_v}. */
const float* fp8attn_quant_scale_ptr(fp8attn_ctx* ctx, int layer);

/* Copy the layer's ring state to the host: h_slots float[3][16],
 * h_meta uint32[3][2] = {head, count} per tensor.  Synchronises `stream`. */
fp8attn_status fp8attn_get_ring_state(fp8attn_ctx* ctx, int layer, float* h_slots,
                                      uint32_t* h_meta, void* stream);

/* Restore a ring state saved by fp8attn_get_ring_state (resume) and
 * recompute the layer's dynamic scales from it.  Synchronises `stream`. */
fp8attn_status fp8attn_set_ring_state(fp8attn_ctx* ctx, int layer, const float* h_slots,
                                      const uint32_t* h_meta, void* stream);

/* Copy the layer's current {qs_q, qs_k, qs_v, ds_q, ds_k, ds_v} to the host.
 * Synchronises `stream`. */
fp8attn_status fp8attn_get_scales(fp8attn_ctx* ctx, int layer, float* h_out6, void* stream);

/* Varlen, non-causal FP8 attention forward (vLLM-Omni "Quantized KV Cache"
 * overview: the quantised Q/K/V feed the attention operator; vLLM FP8 ViT
 * page: per-tensor scales).  q8, k8, v8: E4M3 packed [T, num_heads, 128]
 * with T = total_tokens (the buffers' row count; the kernel never reads past
 * it); d_cu_seqlens int32[batch+1] with cu[batch] <= T; d_descale_qkv: device float[3] {ds_q, ds_k,
 * ds_v}; softmax_scale: 0 selects 1/sqrt(head_dim); out: bf16 [T, num_heads,
 * 128].  Each token attends to every token of its own sequence.  The base
 * pointers must be 16-byte aligned.  d_error: optional device int32 that
 * receives FP8ATTN_ERR_SEQLENS / FP8ATTN_ERR_TIMEOUT bits (may be NULL).
 * Errors: INVALID, UNSUPPORTED (head_dim != 128), CUDA. */
fp8attn_status fp8attn_varlen_fwd(const void* q8, const void* k8, const void* v8,
                                  const int32_t* d_cu_seqlens, int batch, int max_seqlen,
                                  int64_t total_tokens, int num_heads, int head_dim,
                                  const float* d_descale_qkv,
                                  float softmax_scale, void* out, int32_t* d_error,
                                  void* stream);

/* The rule that turns the softmax numerators into the E4M3 P operand of the
 * PV product (the pages give none; both are defined in full here).  With
 * c = ds_q ds_k softmax_scale log2(e), a per-row reference m (log2 units; the
 * first 128-key block's max of s c, moved to a later block's max only when
 * that exceeds m by more than 3) and t = s c - m + 5 <= 8:
 *   FP8ATTN_P_LINEAR_LOG: code = RNE(8 t + 56) clamped to [0, 128] -- the
 *     E4M3 bit pattern read as a fixed-point log2 (Mitchell's / Schraudolph's
 *     piecewise-linear 2^t, exponent and mantissa filled linearly from t);
 *     no exponential is evaluated.  NaN scores give code 0.  The row sum l
 *     adds the E4M3 values of the codes.
 *   FP8ATTN_P_EXP2: code = e4m3_rne(2^t) (2^t evaluated to about 2^-22
 *     relative); l adds the unquantised 2^t.
 * Both: out = (sum_j P_j v_j) ds_v / l, with P carried across moves of m by
 * 2^(m_old - m_new). */
typedef enum {
  FP8ATTN_P_LINEAR_LOG = 0,
  FP8ATTN_P_EXP2 = 1
} fp8attn_p_rule;

/* Static-scale quantisation and FP8 attention in one launch: the result of
 * fp8attn_quantize_qkv(ctx, layer, FP8ATTN_STATIC, q, k, v, tok_stride,
 * head_stride, NULL, ...) followed by fp8attn_varlen_fwd on its codes with
 * fp8attn_descale_ptr(ctx, layer), bit for bit, without the E4M3 copies of
 * Q, K and V in device memory: the kernel casts Q as each CTA starts and K
 * and V tile by tile between their TMA loads and the tensor-core products
 * (vLLM FP8 ViT page, Notes: the separate quantisation launches are what
 * costs small inputs their FP8 gain).
 *   q, k, v: packed bf16 sources (one row per token, no padding); element
 *     (t, h, d) at base + t*tok_stride + h*head_stride + d, strides in
 *     elements, multiples of 8, head_stride >= head_dim and tok_stride >=
 *     num_heads*head_stride (e.g. [T, H, 128], or an interleaved [T, 3, H,
 *     128] projection output).  Other arguments as fp8attn_varlen_fwd_rule;
 *     the work schedule is FP8ATTN_SCHED_AUTO.
 * The layer's current scales become its static ones, as after the cast.
 * Device-side errors (SEQLENS, TIMEOUT) go to the context's error word
 * (fp8attn_get_error).  Errors: INVALID (no static scales for the layer,
 * bad arguments), UNSUPPORTED (head_dim != 128, strides), CUDA.  With
 * total_tokens == 0 nothing is launched.
 * Speed: up to about 300 tokens a sequence this matches the two launches;
 * beyond, every 256-query CTA of a head casts all of that head's K and V
 * again, and the two launches are faster (2-3x at 2048-8192 tokens). */
fp8attn_status fp8attn_varlen_fwd_static(fp8attn_ctx* ctx, int layer, const void* q,
                                         const void* k, const void* v, int64_t tok_stride,
                                         int64_t head_stride, const int32_t* d_cu_seqlens,
                                         int batch, int max_seqlen, int64_t total_tokens,
                                         int num_heads, int head_dim, float softmax_scale,
                                         int p_rule, void* out, void* stream);

/* How fp8attn_varlen_fwd_sched lays the work units (256 query rows of one
 * head of one sequence, computed as two 128-row tiles) on the GPU.  Each
 * output row is computed the same way under every schedule (same key
 * blocks, order and P rule), so the results are bit-identical.
 *   FP8ATTN_SCHED_AUTO: one CTA per unit, except that when the last wave of
 *     units would fill at most half of the SMs, each of those units runs as
 *     two CTAs of one tile each, so that the tiles fill that wave (a lone
 *     tile's blocks run faster than a CTA's two interleaved tiles); those
 *     CTAs form a second launch that starts as SMs free up.  When every
 *     unit fits in that one wave (short sequences, few heads), all units
 *     run that way, in one launch.
 *   FP8ATTN_SCHED_WHOLE: one CTA per unit.
 *   FP8ATTN_SCHED_SPLIT: every unit as two single-tile CTAs. */
typedef enum {
  FP8ATTN_SCHED_AUTO = 0,
  FP8ATTN_SCHED_WHOLE = 1,
  FP8ATTN_SCHED_SPLIT = 2
} fp8attn_schedule;

/* fp8attn_varlen_fwd with an explicit P rule (fp8attn_varlen_fwd uses
 * FP8ATTN_P_LINEAR_LOG, which evaluates no exponential per score and is the
 * faster of the two on B200, where the exponential unit is otherwise the
 * bottleneck; FP8ATTN_P_EXP2 rounds the exact exponential).  Errors as
 * fp8attn_varlen_fwd, and INVALID for an unknown rule. */
fp8attn_status fp8attn_varlen_fwd_rule(const void* q8, const void* k8, const void* v8,
                                       const int32_t* d_cu_seqlens, int batch, int max_seqlen,
                                       int64_t total_tokens, int num_heads, int head_dim,
                                       const float* d_descale_qkv, float softmax_scale,
                                       int p_rule, void* out, int32_t* d_error, void* stream);

/* fp8attn_varlen_fwd_rule with an explicit work schedule (fp8attn_schedule;
 * the other two entry points use FP8ATTN_SCHED_AUTO).  Errors as
 * fp8attn_varlen_fwd, and INVALID for an unknown rule or schedule. */
fp8attn_status fp8attn_varlen_fwd_sched(const void* q8, const void* k8, const void* v8,
                                        const int32_t* d_cu_seqlens, int batch, int max_seqlen,
                                        int64_t total_tokens, int num_heads, int head_dim,
                                        const float* d_descale_qkv, float softmax_scale,
                                        int p_rule, int schedule, void* out, int32_t* d_error,
                                        void* stream);

/* Native-dtype attention for skipped layers (vLLM-Omni "Quantized KV Cache",
 * parameters table: selected layers keep the native dtype): the same
 * computation on bf16 q, k, v [T, num_heads, 128] with no quantisation. */
fp8attn_status fp8attn_varlen_fwd_bf16(const void* q, const void* k, const void* v,
                                       const int32_t* d_cu_seqlens, int batch, int max_seqlen,
                                       int64_t total_tokens, int num_heads, int head_dim,
                                       float softmax_scale,
                                       void* out, int32_t* d_error, void* stream);

/* Read and clear the context's device error word (synchronises `stream`).
 * Returns OK or the most severe device-side status seen since the last call.
 * After a TIMEOUT the context's grid-barrier words are reset. */
fp8attn_status fp8attn_get_error(fp8attn_ctx* ctx, void* stream);

/* Read and clear a caller-owned device error word as filled by
 * fp8attn_varlen_fwd (synchronises `stream`). */
fp8attn_status fp8attn_read_error_word(int32_t* d_error, void* stream);

/* Parse a layer/step selector: comma-separated non-negative integers and
 * inclusive ranges "a-b" (vLLM-Omni "Quantized KV Cache", parameters table,
 * e.g. "0,1,4-6" and "0-2,10").  Spaces around items are allowed; NULL or
 * an empty string selects nothing.  mask_out: uint8[max_index], set to 1 for
 * selected indices, 0 otherwise.  Errors: INVALID for malformed items,
 * reversed ranges or indices >= max_index (mask_out then all zero). */
fp8attn_status fp8attn_parse_selector(const char* text, int max_index, uint8_t* mask_out);

/* Mode of a layer: SKIP if skip_mask[layer] (skip_mask may be NULL),
 * else STATIC if the context has static bounds for it, else DYNAMIC.
 * -1 on a bad argument. */
int fp8attn_select_mode(const fp8attn_ctx* ctx, const uint8_t* skip_mask, int layer);

/* Mode of one attention call inside a denoising loop (vLLM-Omni docs,
 * parameters table: kv_cache_skip_steps and kv_cache_skip_layers; listed
 * steps or layers skip FP8 attention): SKIP if skip_steps[step] or
 * skip_layers[layer], else as fp8attn_select_mode.  Either mask may be NULL;
 * skip_steps holds num_steps entries (a fp8attn_parse_selector mask).  -1 on
 * a bad argument (layer out of range, or step outside [0, num_steps) when
 * skip_steps is given). */
int fp8attn_select_mode_at_step(const fp8attn_ctx* ctx, const uint8_t* skip_layers, int layer,
                                const uint8_t* skip_steps, int num_steps, int step);

/* E4M3 cast helper: d_out[i] = e4m3(fl32(d_in[i] * scale)), fp32 device
 * input, n elements, the same conversion the quantisation kernel uses. */
fp8attn_status fp8attn_e4m3_encode(const float* d_in, int64_t n, float scale, void* d_out,
                                   void* stream);

/* Head-group regrouping for sequence-parallel (Ulysses) attention
 * (vLLM-Omni docs, "Quantized KV Cache", Configuration: the offline
 * diffusion example shards the DiT's sequence over a Ulysses degree of 4).
 * Each rank holds a contiguous slice of the tokens; an all-to-all gives every
 * rank all tokens of num_heads/groups heads and a second one returns the
 * attention output.  An all-to-all moves one contiguous chunk per rank, so:
 *   to_groups = 1: d_src [tokens, num_heads, head_bytes] ->
 *                  d_dst [groups, tokens, num_heads/groups, head_bytes]
 *   to_groups = 0: the inverse ([groups, tokens, H/groups, hb] -> [tokens, H, hb]).
 * head_bytes is the byte size of one head row (256 for bf16 with
 * head_dim 128, 128 for E4M3 codes).  Device buffers, caller-owned, must not
 * overlap.  Asynchronous on `stream`.  Errors: INVALID (negative tokens,
 * groups < 1, num_heads not a multiple of groups, to_groups not 0/1, null or
 * overlapping buffers), UNSUPPORTED (head_bytes not a multiple of 16, buffers
 * not 16-byte aligned), CUDA.  tokens == 0 is a no-op. */
fp8attn_status fp8attn_regroup_heads(const void* d_src, void* d_dst, int64_t tokens,
                                    int num_heads, int groups, int head_bytes, int to_groups,
                                    void* stream);

/* Self-test of the bounded waits (failure detection without a GPU fault).
 * The pages have no counterpart: every wait inside this library's kernels
 * (mbarrier waits of the attention kernels, the grid barrier of the
 * quantisation kernels) gives up after a time limit and reports
 * FP8ATTN_ERR_TIMEOUT instead of hanging.  This runs two probes on `stream`
 * whose waits nothing ever completes -- an mbarrier wait with limit
 * `mbar_limit_ns` (0 < limit <= 1 s) and a two-CTA grid barrier that one CTA
 * leaves before arriving (limit 1 s) -- synchronises the stream, and stores
 * in *h_gave_up how many of the two waits gave up (2 when the bounds work).
 * Returns FP8ATTN_ERR_INVALID for a bad limit or null output,
 * FP8ATTN_ERR_CUDA on a CUDA error.  Takes about 1 s. */
int fp8attn_selftest_bounded_waits(uint64_t mbar_limit_ns, int* h_gave_up, void* stream);

/* ------------------------------------------------------------------ */
/* Static scale map (vLLM docs, "FP8 ViT encoder attention": scale file */
/* format section -- a JSON object mapping each layer name to its      */
/* {"q", "k", "v"} values, "q_scale"/"k_scale"/"v_scale" accepted as    */
/* aliases; usage section -- saved values are multiplied by the save    */
/* margin, 1.5 by default).  Host-only functions, no GPU needed.        */
/* ------------------------------------------------------------------ */

/* Bytes reserved per layer name in the name arrays below (including the
 * terminating NUL). */
#define FP8ATTN_SCALE_NAME_MAX 256

/* h_out[i] = fl32(h_in[i] * margin) for i < n (one fp32 rounding each): the
 * save margin applied to exported values, or (the other reading of the
 * page) to stored values when a map is read.  margin must be finite and
 * > 0; h_in and h_out may be the same array.  Errors: INVALID. */
fp8attn_status fp8attn_apply_margin(const float* h_in, int64_t n, float margin, float* h_out);

/* Parse a scale map from JSON text (text_len bytes, no NUL needed).  Each
 * layer's three values are read as doubles, rounded once to fp32 and
 * multiplied by `margin` (1.0 leaves them as stored); the short key wins
 * when a layer has both it and its alias; other keys are ignored.  Layers
 * are returned in file order: names_out [max_layers][FP8ATTN_SCALE_NAME_MAX]
 * NUL-terminated, values_out [max_layers][3] {q, k, v}; *n_layers_out the
 * count.  The caller owns every buffer.  Errors: INVALID (malformed JSON, a
 * missing q/k/v value, a name of FP8ATTN_SCALE_NAME_MAX bytes or more, more
 * than max_layers layers, a bad margin); *n_layers_out is 0 then. */
fp8attn_status fp8attn_scale_map_parse(const char* json_text, size_t text_len, float margin,
                                       int max_layers, char* names_out, float* values_out,
                                       int* n_layers_out);

/* Write a scale map as JSON text: n_layers names (FP8ATTN_SCALE_NAME_MAX-byte
 * slots, NUL-terminated) with their {q, k, v} values (finite), each value as
 * the shortest decimal that reads back as the same fp32 number.  *written
 * receives the bytes needed including the NUL; if buf is NULL or buf_size is
 * smaller than that, nothing is written and INVALID is returned (call again
 * with a larger buffer).  Errors: INVALID. */
fp8attn_status fp8attn_scale_map_format(int n_layers, const char* names, const float* values,
                                        char* buf, size_t buf_size, size_t* written);

/* Self-test of the score product (no counterpart in the pages; it checks
 * the accumulation error that the tests' tie model assumes).  For each of
 * `tiles` pairs of 128 x 128 E4M3 tiles -- rows [128 t, 128 t + 128) of
 * d_q8 and d_k8, each [tiles * 128, 128] codes, 16-byte aligned -- writes
 * S = Q K^T as fp32 to d_scores [tiles, 128, 128], computed with the FP8
 * attention kernel's shared-memory layout, descriptors and MMA sequence.
 * d_error: optional device int32 receiving FP8ATTN_ERR_TIMEOUT bits.
 * Errors: INVALID (null pointers, tiles < 1, misaligned), CUDA. */
fp8attn_status fp8attn_selftest_qk_scores(const void* d_q8, const void* d_k8, int64_t tiles,
                                          float* d_scores, int32_t* d_error, void* stream);

/* Allocation-free one-shot dynamic quantisation.  The pages have no
 * counterpart to this entry point; it exists for callers that cannot
 * allocate device memory -- for example an operator that an inference
 * runtime hands only its input and output buffers under a fixed memory
 * plan, or code that must not call cudaMalloc/cudaFree because those calls
 * synchronise the device -- and so cannot provide the context workspace of
 * fp8attn_quantize_qkv.
 *
 * It performs the fused amax + scale + E4M3 cast + unpad of Q, K and V in
 * one launch, with the scales taken from this call's amax alone (no ring;
 * identical to the first DYNAMIC pass of a freshly created context), and
 * writes {ds_q, ds_k, ds_v} to d_descale_out (device float[3]) and, if
 * d_scale_out is not NULL, {qs_q, qs_k, qs_v} to it.  All other arguments
 * and layouts are those of fp8attn_quantize_qkv.
 *
 * Scratch: a library-owned, file-scope device array of 16,640 bytes holding
 * one partial maximum per CTA (up to 1,024 CTAs) and the grid-barrier and
 * error words; every GPU that loads the library holds one until the process
 * exits.  A launch that would need more than 1,024 CTAs is refused with
 * FP8ATTN_ERR_UNSUPPORTED (on B200 the launch uses at most 148 x 4).  The
 * call performs no allocation of any kind.  The first call on a device looks
 * up the array's device address (once per device); make that first call
 * before any stream capture.  All calls share the one array, so calls whose
 * kernels overlap on the GPU (different streams, or concurrent graphs) race
 * and give wrong results: serialise them.  Device-side errors accumulate in
 * the array until read with fp8attn_quantize_qkv_noalloc_error().  After a
 * device-side TIMEOUT the grid-barrier words may be left mid-count, so every
 * later call on that device returns from its kernel at once, writing
 * nothing, until fp8attn_quantize_qkv_noalloc_error() has reported the
 * timeout and reset them.  The array belongs to the device current at the
 * call (cudaGetDevice): make the inputs' device current before calling.
 * Returns an fp8attn_status. */
int fp8attn_quantize_qkv_noalloc(const void* q, const void* k, const void* v, int64_t tok_stride,
                                 int64_t head_stride, const int32_t* d_src_seq_start,
                                 const int32_t* d_cu_seqlens, int batch, int max_seqlen,
                                 int64_t total_tokens, int num_heads, int head_dim, void* q8,
                                 void* k8, void* v8, float* d_descale_out, float* d_scale_out,
                                 void* stream);

/* Read and clear the device-side error word of the allocation-free entry
 * point for the current device (synchronises `stream`); after a TIMEOUT the
 * barrier words are reset too.  Returns an fp8attn_status. */
int fp8attn_quantize_qkv_noalloc_error(void* stream);

/* Number of kernels the library has launched in this process (a counter
 * incremented on every successful launch; for accounting in benchmarks). */
uint64_t fp8attn_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8ATTN_H_ */
