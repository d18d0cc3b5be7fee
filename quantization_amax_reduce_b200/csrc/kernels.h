// Internal launcher interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

namespace fp8attn {

struct QuantLaunch {
  const void* src[3];            // bf16 q, k, v
  void* dst[3];                  // E4M3 q8, k8, v8 (packed [T, H, 128])
  int64_t tok_stride;            // elements
  int64_t head_stride;           // elements
  const int32_t* cu;             // device [batch + 1]
  const int32_t* src_seq_start;  // device [batch] or null
  int batch, heads, max_seqlen;
  int64_t total_tokens;          // must equal cu[batch]
  int kind;                      // a QuantKind
  float* amax_out;               // kQuantAmaxOnly: device float[3]
  void* gs;                      // GlobalState*
  void* ls;                      // LayerState*
  int dst_groups = 1;            // static / ring cast: > 1 writes [groups][T][H/groups][128]
};

enum QuantKind {
  kQuantStatic = 0,     // cast with the static bounds
  kQuantDynamic = 1,    // fused amax + ring push + cast (current pass included)
  kQuantRing = 2,       // cast with the layer's current ring scales, ring unchanged
  kQuantAmaxOnly = 3,   // per-tensor amax into amax_out, nothing cast or pushed
};

cudaError_t launch_quantize(const QuantLaunch& q, cudaStream_t stream);
cudaError_t launch_ring_update(void* ls, void* gs, const float* amax3, cudaStream_t stream);
cudaError_t launch_rescale_from_ring(void* ls, cudaStream_t stream);
cudaError_t launch_encode(const float* in, int64_t n, float scale, void* out,
                          cudaStream_t stream);

struct AttnLaunch {
  const void* q;                 // E4M3 or bf16 [T, H, 128]
  const void* k;
  const void* v;
  const int32_t* cu;             // device [batch + 1]
  int batch, heads, max_seqlen;
  const float* descale;          // device {ds_q, ds_k, ds_v} (fp8 only)
  float softmax_scale;
  void* out;                     // bf16 [T, H, 128]
  int32_t* err;                  // device error word or null
  int bf16;                      // 1 = native bf16 inputs (skip-layer path)
  int p_rule;                    // FP8 only: kPRuleLinearLog or kPRuleExp2
  int schedule;                  // FP8 only: kSchedAuto, kSchedWhole or kSchedSplit
  // FP8 with the static cast inside the kernel: q, k, v are bf16 sources
  // (element (t, h, d) at base + t * tok_stride + h * head_stride + d), cast
  // with qscale {qs_q, qs_k, qs_v}; the first CTA copies qscale and descale
  // to cur_qs / cur_ds (the layer's current scales)
  int fused = 0;
  int64_t tok_stride = 0, head_stride = 0;
  const float* qscale = nullptr;
  float* cur_qs = nullptr;
  float* cur_ds = nullptr;
};

// P rules of the FP8 kernel (the values of fp8attn_p_rule in fp8attn.h).
constexpr int kPRuleLinearLog = 0;
constexpr int kPRuleExp2 = 1;

// Work schedules of the FP8 kernel (the values of fp8attn_schedule).
constexpr int kSchedAuto = 0;    // split the units of a last wave at most half full
constexpr int kSchedWhole = 1;   // one CTA per unit (256 query rows, two tiles)
constexpr int kSchedSplit = 2;   // every unit as two single-tile CTAs

cudaError_t launch_attention(const AttnLaunch& p, int64_t total_tokens, cudaStream_t stream);

// S = Q K^T for `tiles` 128 x 128 tiles of E4M3 codes ([tiles * 128, 128]
// each), with the FP8 attention kernel's MMA sequence; fp32 [tiles, 128, 128].
cudaError_t launch_qk_scores_probe(const void* q8, const void* k8, int64_t tiles, float* scores,
                                   int32_t* err, cudaStream_t stream);

// Counts one successful kernel launch (fp8attn_launch_count).
void note_launch();

// [T, H, hb] <-> [G, T, H/G, hb] (to_groups = 1 / 0); hb a multiple of 16,
// H a multiple of G, 16-byte aligned, non-overlapping buffers.
cudaError_t launch_regroup_heads(const void* src, void* dst, int64_t tokens, int heads,
                                 int groups, int head_bytes, int to_groups, cudaStream_t stream);

}  // namespace fp8attn
