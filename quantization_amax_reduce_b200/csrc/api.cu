// C ABI of the fp8attn library: argument checks, context and workspace
// handling, selector parsing, static-scale import/export and the launches.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstring>
#include <new>
#include <vector>

#include "fp8attn.h"
#include "kernels.h"
#include "state.cuh"

using namespace fp8attn;

struct fp8attn_ctx {
  int layers;
  int device;
  GlobalState* gs;
  LayerState* ls;
  std::vector<uint8_t> has_static;
};

namespace {

std::atomic<uint64_t> g_launches{0};

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

inline bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

inline bool layer_ok(const fp8attn_ctx* c, int layer) {
  return c && layer >= 0 && layer < c->layers;
}

fp8attn_status status_of_bits(uint32_t bits) {
  if (bits & kErrTimeout) return FP8ATTN_ERR_TIMEOUT;
  if (bits & kErrSeqlens) return FP8ATTN_ERR_SEQLENS;
  if (bits & kErrNonfinite) return FP8ATTN_ERR_NONFINITE;
  return FP8ATTN_OK;
}

__global__ void set_static_kernel(LayerState* ls, float q, float k, float v) {
  if (threadIdx.x != 0) return;
  const float A[3] = {q, k, v};
  for (int t = 0; t < 3; ++t) {
    ls->static_bound[t] = A[t];
    scales_from_bound(A[t], &ls->static_qs[t], &ls->static_ds[t]);
  }
}

// shared shape checks of the attention entry points
fp8attn_status check_attention(const void* q, const void* k, const void* v,
                               const int32_t* cu, int batch, int max_seqlen,
                               int64_t total_tokens, int num_heads, int head_dim, void* out) {
  if (batch < 1 || max_seqlen < 0 || num_heads < 1 || total_tokens < 0) return FP8ATTN_ERR_INVALID;
  if (head_dim != kHeadDim) return FP8ATTN_ERR_UNSUPPORTED;
  if (!cu) return FP8ATTN_ERR_INVALID;
  if (total_tokens > static_cast<int64_t>(batch) * max_seqlen) return FP8ATTN_ERR_INVALID;
  if (total_tokens > 0x7FFFFFFFLL) return FP8ATTN_ERR_UNSUPPORTED;
  if (total_tokens == 0) return FP8ATTN_OK;
  if (!q || !k || !v || !out) return FP8ATTN_ERR_INVALID;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
    return FP8ATTN_ERR_INVALID;
  return FP8ATTN_OK;
}

fp8attn_status run_attention(const void* q, const void* k, const void* v, const int32_t* cu,
                             int batch, int max_seqlen, int64_t total_tokens, int num_heads,
                             int head_dim, const float* descale, float softmax_scale, void* out,
                             int32_t* err, void* stream, int bf16, int p_rule,
                             int schedule) {
  if (p_rule != FP8ATTN_P_LINEAR_LOG && p_rule != FP8ATTN_P_EXP2) return FP8ATTN_ERR_INVALID;
  if (schedule != FP8ATTN_SCHED_AUTO && schedule != FP8ATTN_SCHED_WHOLE &&
      schedule != FP8ATTN_SCHED_SPLIT)
    return FP8ATTN_ERR_INVALID;
  fp8attn_status st = check_attention(q, k, v, cu, batch, max_seqlen, total_tokens, num_heads,
                                      head_dim, out);
  if (st != FP8ATTN_OK || total_tokens == 0) return st;
  if (!bf16 && !descale) return FP8ATTN_ERR_INVALID;
  if (!(softmax_scale >= 0.0f) || std::isinf(softmax_scale)) return FP8ATTN_ERR_INVALID;
  AttnLaunch a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.cu = cu;
  a.batch = batch;
  a.heads = num_heads;
  a.max_seqlen = max_seqlen;
  a.descale = descale;
  a.softmax_scale = softmax_scale == 0.0f ? 1.0f / std::sqrt(static_cast<float>(head_dim))
                                          : softmax_scale;
  a.out = out;
  a.err = err;
  a.bf16 = bf16;
  a.p_rule = p_rule == FP8ATTN_P_EXP2 ? kPRuleExp2 : kPRuleLinearLog;
  a.schedule = schedule == FP8ATTN_SCHED_WHOLE   ? kSchedWhole
               : schedule == FP8ATTN_SCHED_SPLIT ? kSchedSplit
                                                 : kSchedAuto;
  const cudaError_t e = launch_attention(a, total_tokens, as_stream(stream));
  if (e != cudaSuccess) return FP8ATTN_ERR_CUDA;
  g_launches.fetch_add(1);
  return FP8ATTN_OK;
}

}  // namespace

void fp8attn::note_launch() { g_launches.fetch_add(1); }

extern "C" {

const char* fp8attn_status_string(int status) {
  switch (status) {
    case FP8ATTN_OK: return "ok";
    case FP8ATTN_ERR_INVALID: return "invalid argument";
    case FP8ATTN_ERR_CUDA: return "CUDA error";
    case FP8ATTN_ERR_TIMEOUT: return "device wait timed out";
    case FP8ATTN_ERR_UNSUPPORTED: return "unsupported configuration";
    case FP8ATTN_ERR_NONFINITE: return "non-finite amax";
    case FP8ATTN_ERR_SEQLENS: return "inconsistent cu_seqlens";
    default: return "unknown status";
  }
}

int fp8attn_ring_length(void) { return kRing; }

size_t fp8attn_workspace_bytes(int num_layers) {
  return num_layers < 1 ? 0 : workspace_bytes_for(num_layers);
}

fp8attn_status fp8attn_create(int num_layers, void* d_workspace, size_t workspace_bytes,
                              void* stream, fp8attn_ctx** out) {
  if (!out) return FP8ATTN_ERR_INVALID;
  *out = nullptr;
  if (num_layers < 1 || !d_workspace || !aligned(d_workspace, 256) ||
      workspace_bytes < workspace_bytes_for(num_layers))
    return FP8ATTN_ERR_INVALID;
  fp8attn_ctx* c = new (std::nothrow) fp8attn_ctx;
  if (!c) return FP8ATTN_ERR_INVALID;
  c->layers = num_layers;
  c->gs = static_cast<GlobalState*>(d_workspace);
  c->ls = reinterpret_cast<LayerState*>(static_cast<char*>(d_workspace) + sizeof(GlobalState));
  c->has_static.assign(num_layers, 0);
  if (cudaGetDevice(&c->device) != cudaSuccess ||
      cudaMemsetAsync(d_workspace, 0, workspace_bytes_for(num_layers), as_stream(stream)) !=
          cudaSuccess) {
    delete c;
    return FP8ATTN_ERR_CUDA;
  }
  // empty rings: unit scales until the first pass
  std::vector<LayerState> init(num_layers);
  std::memset(init.data(), 0, sizeof(LayerState) * num_layers);
  for (auto& l : init)
    for (int t = 0; t < 3; ++t) l.qs[t] = l.ds[t] = l.static_qs[t] = l.static_ds[t] = 1.0f;
  if (cudaMemcpyAsync(c->ls, init.data(), sizeof(LayerState) * num_layers,
                      cudaMemcpyHostToDevice, as_stream(stream)) != cudaSuccess ||
      cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) {
    delete c;
    return FP8ATTN_ERR_CUDA;
  }
  *out = c;
  return FP8ATTN_OK;
}

fp8attn_status fp8attn_destroy(fp8attn_ctx* ctx) {
  if (!ctx) return FP8ATTN_ERR_INVALID;
  delete ctx;
  return FP8ATTN_OK;
}

fp8attn_status fp8attn_quantize_qkv(fp8attn_ctx* ctx, int layer, int mode, const void* q,
                                    const void* k, const void* v, int64_t tok_stride,
                                    int64_t head_stride, const int32_t* d_src_seq_start,
                                    const int32_t* d_cu_seqlens, int batch, int max_seqlen,
                                    int64_t total_tokens, int num_heads, int head_dim, void* q8,
                                    void* k8, void* v8, void* stream) {
  if (!layer_ok(ctx, layer)) return FP8ATTN_ERR_INVALID;
  if (mode != FP8ATTN_DYNAMIC && mode != FP8ATTN_STATIC && mode != FP8ATTN_RING)
    return FP8ATTN_ERR_INVALID;
  if (mode == FP8ATTN_STATIC && !ctx->has_static[layer]) return FP8ATTN_ERR_INVALID;
  if (batch < 1 || max_seqlen < 0 || num_heads < 1 || total_tokens < 0 || !d_cu_seqlens)
    return FP8ATTN_ERR_INVALID;
  if (head_dim != kHeadDim) return FP8ATTN_ERR_UNSUPPORTED;
  if (total_tokens > static_cast<int64_t>(batch) * max_seqlen) return FP8ATTN_ERR_INVALID;
  if (!q || !k || !v || !q8 || !k8 || !v8) return FP8ATTN_ERR_INVALID;
  if (tok_stride <= 0 || head_stride <= 0 || (tok_stride % 8) || (head_stride % 8))
    return FP8ATTN_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(q8, 16) ||
      !aligned(k8, 16) || !aligned(v8, 16))
    return FP8ATTN_ERR_UNSUPPORTED;
  QuantLaunch L;
  L.src[0] = q;
  L.src[1] = k;
  L.src[2] = v;
  L.dst[0] = q8;
  L.dst[1] = k8;
  L.dst[2] = v8;
  L.tok_stride = tok_stride;
  L.head_stride = head_stride;
  L.cu = d_cu_seqlens;
  L.src_seq_start = d_src_seq_start;
  L.batch = batch;
  L.heads = num_heads;
  L.max_seqlen = max_seqlen;
  L.total_tokens = total_tokens;
  L.kind = mode == FP8ATTN_DYNAMIC ? kQuantDynamic : mode == FP8ATTN_RING ? kQuantRing
                                                                           : kQuantStatic;
  L.amax_out = nullptr;
  L.gs = ctx->gs;
  L.ls = ctx->ls + layer;
  const cudaError_t e = launch_quantize(L, as_stream(stream));
  if (e != cudaSuccess) return FP8ATTN_ERR_CUDA;
  g_launches.fetch_add(1);
  return FP8ATTN_OK;
}

fp8attn_status fp8attn_quantize_qkv_grouped(fp8attn_ctx* ctx, int layer, int mode, const void* q,
                                            const void* k, const void* v, int64_t tok_stride,
                                            int64_t head_stride, const int32_t* d_src_seq_start,
                                            const int32_t* d_cu_seqlens, int batch,
                                            int max_seqlen, int64_t total_tokens, int num_heads,
                                            int head_dim, int groups, void* q8, void* k8,
                                            void* v8, void* stream) {
  if (mode != FP8ATTN_STATIC && mode != FP8ATTN_RING) return FP8ATTN_ERR_INVALID;
  if (groups < 1 || num_heads < 1 || num_heads % groups) return FP8ATTN_ERR_INVALID;
  if (!layer_ok(ctx, layer)) return FP8ATTN_ERR_INVALID;
  if (mode == FP8ATTN_STATIC && !ctx->has_static[layer]) return FP8ATTN_ERR_INVALID;
  if (batch < 1 || max_seqlen < 0 || total_tokens < 0 || !d_cu_seqlens)
    return FP8ATTN_ERR_INVALID;
  if (head_dim != kHeadDim) return FP8ATTN_ERR_UNSUPPORTED;
  if (total_tokens > static_cast<int64_t>(batch) * max_seqlen) return FP8ATTN_ERR_INVALID;
  if (!q || !k || !v || !q8 || !k8 || !v8) return FP8ATTN_ERR_INVALID;
  if (tok_stride <= 0 || head_stride <= 0 || (tok_stride % 8) || (head_stride % 8))
    return FP8ATTN_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(q8, 16) ||
      !aligned(k8, 16) || !aligned(v8, 16))
    return FP8ATTN_ERR_UNSUPPORTED;
  QuantLaunch L;
  L.src[0] = q;
  L.src[1] = k;
  L.src[2] = v;
  L.dst[0] = q8;
  L.dst[1] = k8;
  L.dst[2] = v8;
  L.tok_stride = tok_stride;
  L.head_stride = head_stride;
  L.cu = d_cu_seqlens;
  L.src_seq_start = d_src_seq_start;
  L.batch = batch;
  L.heads = num_heads;
  L.max_seqlen = max_seqlen;
  L.total_tokens = total_tokens;
  L.kind = mode == FP8ATTN_RING ? kQuantRing : kQuantStatic;
  L.amax_out = nullptr;
  L.gs = ctx->gs;
  L.ls = ctx->ls + layer;
  L.dst_groups = groups;
  const cudaError_t e = launch_quantize(L, as_stream(stream));
  if (e != cudaSuccess) return FP8ATTN_ERR_CUDA;
  g_launches.fetch_add(1);
  return FP8ATTN_OK;
}

fp8attn_status fp8attn_amax_qkv(fp8attn_ctx* ctx, const void* q, const void* k, const void* v,
                                int64_t tok_stride, int64_t head_stride,
                                const int32_t* d_src_seq_start, const int32_t* d_cu_seqlens,
                                int batch, int max_seqlen, int64_t total_tokens, int num_heads,
                                int head_dim, float* d_amax3, void* stream) {
  if (!ctx || !d_amax3 || !aligned(d_amax3, 4)) return FP8ATTN_ERR_INVALID;
  if (batch < 1 || max_seqlen < 0 || num_heads < 1 || total_tokens < 0 || !d_cu_seqlens)
    return FP8ATTN_ERR_INVALID;
  if (head_dim != kHeadDim) return FP8ATTN_ERR_UNSUPPORTED;
  if (total_tokens > static_cast<int64_t>(batch) * max_seqlen) return FP8ATTN_ERR_INVALID;
  if (!q || !k || !v) return FP8ATTN_ERR_INVALID;
  if (tok_stride <= 0 || head_stride <= 0 || (tok_stride % 8) || (head_stride % 8))
    return FP8ATTN_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16)) return FP8ATTN_ERR_UNSUPPORTED;
  QuantLaunch L;
  L.src[0] = q;
  L.src[1] = k;
  L.src[2] = v;
  L.dst[0] = L.dst[1] = L.dst[2] = nullptr;
  L.tok_stride = tok_stride;
  L.head_stride = head_stride;
  L.cu = d_cu_seqlens;
  L.src_seq_start = d_src_seq_start;
  L.batch = batch;
  L.heads = num_heads;
  L.max_seqlen = max_seqlen;
  L.total_tokens = total_tokens;
  L.kind = kQuantAmaxOnly;
  L.amax_out = d_amax3;
  L.gs = ctx->gs;
  L.ls = ctx->ls;
  const cudaError_t e = launch_quantize(L, as_stream(stream));
  if (e != cudaSuccess) return FP8ATTN_ERR_CUDA;
  g_launches.fetch_add(1);
  return FP8ATTN_OK;
}

fp8attn_status fp8attn_amax_ring_update(fp8attn_ctx* ctx, int layer, const float* d_amax3,
                                        void* stream) {
  if (!layer_ok(ctx, layer) || !d_amax3) return FP8ATTN_ERR_INVALID;
  const cudaError_t e = launch_ring_update(ctx->ls + layer, ctx->gs, d_amax3, as_stream(stream));
  if (e != cudaSuccess) return FP8ATTN_ERR_CUDA;
  g_launches.fetch_add(1);
  return FP8ATTN_OK;
}

fp8attn_status fp8attn_set_static_scales(fp8attn_ctx* ctx, int layer, float q, float k,
                                         float v, void* stream) {
  if (!layer_ok(ctx, layer)) return FP8ATTN_ERR_INVALID;
  for (float x : {q, k, v})
    if (!std::isfinite(x) || x < 0.0f) return FP8ATTN_ERR_INVALID;
  set_static_kernel<<<1, 32, 0, as_stream(stream)>>>(ctx->ls + layer, q, k, v);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return FP8ATTN_ERR_CUDA;
  g_launches.fetch_add(1);
  ctx->has_static[layer] = 1;
  return FP8ATTN_OK;
}

fp8attn_status fp8attn_clear_static_scales(fp8attn_ctx* ctx, int layer) {
  if (!layer_ok(ctx, layer)) return FP8ATTN_ERR_INVALID;
  ctx->has_static[layer] = 0;
  return FP8ATTN_OK;
}

int fp8attn_has_static_scales(const fp8attn_ctx* ctx, int layer) {
  if (!layer_ok(ctx, layer)) return -1;
  return ctx->has_static[layer] ? 1 : 0;
}

fp8attn_status fp8attn_export_static_scales(fp8attn_ctx* ctx, float margin, float* h_out,
                                            void* stream) {
  if (!ctx || !h_out || !std::isfinite(margin) || margin <= 0.0f) return FP8ATTN_ERR_INVALID;
  std::vector<LayerState> host(ctx->layers);
  cudaError_t e = cudaMemcpyAsync(host.data(), ctx->ls, sizeof(LayerState) * ctx->layers,
                                  cudaMemcpyDeviceToHost, as_stream(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return FP8ATTN_ERR_CUDA;
  for (int l = 0; l < ctx->layers; ++l)
    for (int t = 0; t < 3; ++t) {
      float A = 0.0f;
      for (uint32_t i = 0; i < host[l].count[t] && i < static_cast<uint32_t>(kRing); ++i)
        A = std::fmax(A, host[l].ring[t][i]);
      volatile float prod = A * margin;   // one fp32 multiply
      h_out[l * 3 + t] = prod;
    }
  return FP8ATTN_OK;
}

const float* fp8attn_descale_ptr(fp8attn_ctx* ctx, int layer) {
  if (!layer_ok(ctx, layer)) return nullptr;
  return ctx->ls[layer].ds;
}

const float* fp8attn_quant_scale_ptr(fp8attn_ctx* ctx, int layer) {
  if (!layer_ok(ctx, layer)) return nullptr;
  return ctx->ls[layer].qs;
}

fp8attn_status fp8attn_get_ring_state(fp8attn_ctx* ctx, int layer, float* h_slots,
                                      uint32_t* h_meta, void* stream) {
  if (!layer_ok(ctx, layer) || !h_slots || !h_meta) return FP8ATTN_ERR_INVALID;
  LayerState host;
  cudaError_t e = cudaMemcpyAsync(&host, ctx->ls + layer, sizeof(LayerState),
                                  cudaMemcpyDeviceToHost, as_stream(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return FP8ATTN_ERR_CUDA;
  std::memcpy(h_slots, host.ring, sizeof(host.ring));
  for (int t = 0; t < 3; ++t) {
    h_meta[2 * t] = host.head[t];
    h_meta[2 * t + 1] = host.count[t];
  }
  return FP8ATTN_OK;
}

fp8attn_status fp8attn_set_ring_state(fp8attn_ctx* ctx, int layer, const float* h_slots,
                                      const uint32_t* h_meta, void* stream) {
  if (!layer_ok(ctx, layer) || !h_slots || !h_meta) return FP8ATTN_ERR_INVALID;
  for (int t = 0; t < 3; ++t) {
    const uint32_t head = h_meta[2 * t], count = h_meta[2 * t + 1];
    if (count > static_cast<uint32_t>(kRing) || head >= static_cast<uint32_t>(kRing))
      return FP8ATTN_ERR_INVALID;
    if (count < static_cast<uint32_t>(kRing) && head != count) return FP8ATTN_ERR_INVALID;
    for (int i = 0; i < kRing; ++i)
      if (!std::isfinite(h_slots[t * kRing + i]) || h_slots[t * kRing + i] < 0.0f)
        return FP8ATTN_ERR_INVALID;
  }
  LayerState host;
  cudaError_t e = cudaMemcpyAsync(&host, ctx->ls + layer, sizeof(LayerState),
                                  cudaMemcpyDeviceToHost, as_stream(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return FP8ATTN_ERR_CUDA;
  std::memcpy(host.ring, h_slots, sizeof(host.ring));
  for (int t = 0; t < 3; ++t) {
    host.head[t] = h_meta[2 * t];
    host.count[t] = h_meta[2 * t + 1];
  }
  e = cudaMemcpyAsync(ctx->ls + layer, &host, sizeof(LayerState), cudaMemcpyHostToDevice,
                      as_stream(stream));
  if (e == cudaSuccess) e = launch_rescale_from_ring(ctx->ls + layer, as_stream(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return FP8ATTN_ERR_CUDA;
  g_launches.fetch_add(1);
  return FP8ATTN_OK;
}

fp8attn_status fp8attn_get_scales(fp8attn_ctx* ctx, int layer, float* h_out6, void* stream) {
  if (!layer_ok(ctx, layer) || !h_out6) return FP8ATTN_ERR_INVALID;
  LayerState host;
  cudaError_t e = cudaMemcpyAsync(&host, ctx->ls + layer, sizeof(LayerState),
                                  cudaMemcpyDeviceToHost, as_stream(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return FP8ATTN_ERR_CUDA;
  for (int t = 0; t < 3; ++t) {
    h_out6[t] = host.qs[t];
    h_out6[3 + t] = host.ds[t];
  }
  return FP8ATTN_OK;
}

fp8attn_status fp8attn_varlen_fwd(const void* q8, const void* k8, const void* v8,
                                  const int32_t* d_cu_seqlens, int batch, int max_seqlen,
                                  int64_t total_tokens, int num_heads, int head_dim,
                                  const float* d_descale_qkv, float softmax_scale, void* out,
                                  int32_t* d_error, void* stream) {
  return run_attention(q8, k8, v8, d_cu_seqlens, batch, max_seqlen, total_tokens, num_heads,
                       head_dim, d_descale_qkv, softmax_scale, out, d_error, stream, 0,
                       FP8ATTN_P_LINEAR_LOG, FP8ATTN_SCHED_AUTO);
}

fp8attn_status fp8attn_varlen_fwd_rule(const void* q8, const void* k8, const void* v8,
                                       const int32_t* d_cu_seqlens, int batch, int max_seqlen,
                                       int64_t total_tokens, int num_heads, int head_dim,
                                       const float* d_descale_qkv, float softmax_scale,
                                       int p_rule, void* out, int32_t* d_error, void* stream) {
  return run_attention(q8, k8, v8, d_cu_seqlens, batch, max_seqlen, total_tokens, num_heads,
                       head_dim, d_descale_qkv, softmax_scale, out, d_error, stream, 0, p_rule,
                       FP8ATTN_SCHED_AUTO);
}

fp8attn_status fp8attn_varlen_fwd_sched(const void* q8, const void* k8, const void* v8,
                                        const int32_t* d_cu_seqlens, int batch, int max_seqlen,
                                        int64_t total_tokens, int num_heads, int head_dim,
                                        const float* d_descale_qkv, float softmax_scale,
                                        int p_rule, int schedule, void* out, int32_t* d_error,
                                        void* stream) {
  return run_attention(q8, k8, v8, d_cu_seqlens, batch, max_seqlen, total_tokens, num_heads,
                       head_dim, d_descale_qkv, softmax_scale, out, d_error, stream, 0, p_rule,
                       schedule);
}

fp8attn_status fp8attn_varlen_fwd_static(fp8attn_ctx* ctx, int layer, const void* q,
                                         const void* k, const void* v, int64_t tok_stride,
                                         int64_t head_stride, const int32_t* d_cu_seqlens,
                                         int batch, int max_seqlen, int64_t total_tokens,
                                         int num_heads, int head_dim, float softmax_scale,
                                         int p_rule, void* out, void* stream) {
  if (!layer_ok(ctx, layer) || !ctx->has_static[layer]) return FP8ATTN_ERR_INVALID;
  if (p_rule != FP8ATTN_P_LINEAR_LOG && p_rule != FP8ATTN_P_EXP2) return FP8ATTN_ERR_INVALID;
  fp8attn_status st = check_attention(q, k, v, d_cu_seqlens, batch, max_seqlen, total_tokens,
                                      num_heads, head_dim, out);
  if (st != FP8ATTN_OK || total_tokens == 0) return st;
  if (!(softmax_scale >= 0.0f) || std::isinf(softmax_scale)) return FP8ATTN_ERR_INVALID;
  // rows of heads of 128 channels, heads within a row, no overlap; strides in
  // 16-byte units (the TMA map's rule)
  if (tok_stride <= 0 || head_stride <= 0 || (tok_stride % 8) || (head_stride % 8) ||
      head_stride < head_dim || tok_stride < static_cast<int64_t>(num_heads) * head_stride)
    return FP8ATTN_ERR_UNSUPPORTED;
  LayerState* ls = ctx->ls + layer;
  AttnLaunch a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.cu = d_cu_seqlens;
  a.batch = batch;
  a.heads = num_heads;
  a.max_seqlen = max_seqlen;
  a.descale = ls->static_ds;
  a.softmax_scale = softmax_scale == 0.0f ? 1.0f / std::sqrt(static_cast<float>(head_dim))
                                          : softmax_scale;
  a.out = out;
  a.err = reinterpret_cast<int32_t*>(&ctx->gs->error);
  a.bf16 = 0;
  a.p_rule = p_rule == FP8ATTN_P_EXP2 ? kPRuleExp2 : kPRuleLinearLog;
  a.schedule = kSchedAuto;
  a.fused = 1;
  a.tok_stride = tok_stride;
  a.head_stride = head_stride;
  a.qscale = ls->static_qs;
  a.cur_qs = ls->qs;
  a.cur_ds = ls->ds;
  const cudaError_t e = launch_attention(a, total_tokens, as_stream(stream));
  if (e != cudaSuccess) return FP8ATTN_ERR_CUDA;
  g_launches.fetch_add(1);
  return FP8ATTN_OK;
}

fp8attn_status fp8attn_selftest_qk_scores(const void* d_q8, const void* d_k8, int64_t tiles,
                                          float* d_scores, int32_t* d_error, void* stream) {
  if (!d_q8 || !d_k8 || !d_scores || tiles < 1 || tiles > 0x7FFFFFFF / 128)
    return FP8ATTN_ERR_INVALID;
  if (!aligned(d_q8, 16) || !aligned(d_k8, 16) || !aligned(d_scores, 16))
    return FP8ATTN_ERR_INVALID;
  if (launch_qk_scores_probe(d_q8, d_k8, tiles, d_scores, d_error, as_stream(stream)) !=
      cudaSuccess)
    return FP8ATTN_ERR_CUDA;
  g_launches.fetch_add(1);
  return FP8ATTN_OK;
}

fp8attn_status fp8attn_varlen_fwd_bf16(const void* q, const void* k, const void* v,
                                       const int32_t* d_cu_seqlens, int batch, int max_seqlen,
                                       int64_t total_tokens, int num_heads, int head_dim,
                                       float softmax_scale, void* out, int32_t* d_error,
                                       void* stream) {
  return run_attention(q, k, v, d_cu_seqlens, batch, max_seqlen, total_tokens, num_heads,
                       head_dim, nullptr, softmax_scale, out, d_error, stream, 1,
                       FP8ATTN_P_EXP2, FP8ATTN_SCHED_WHOLE);
}

fp8attn_status fp8attn_get_error(fp8attn_ctx* ctx, void* stream) {
  if (!ctx) return FP8ATTN_ERR_INVALID;
  GlobalState host;
  cudaError_t e = cudaMemcpyAsync(&host, ctx->gs, sizeof(GlobalState), cudaMemcpyDeviceToHost,
                                  as_stream(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return FP8ATTN_ERR_CUDA;
  const fp8attn_status st = status_of_bits(host.error);
  if (host.error) {
    // clear the error; after a timeout also reset the reduction words
    if (host.error & kErrTimeout) {
      e = cudaMemsetAsync(ctx->gs, 0, sizeof(GlobalState), as_stream(stream));
    } else {
      e = cudaMemsetAsync(&ctx->gs->error, 0, sizeof(uint32_t), as_stream(stream));
    }
    if (e == cudaSuccess) e = cudaStreamSynchronize(as_stream(stream));
    if (e != cudaSuccess) return FP8ATTN_ERR_CUDA;
  }
  return st;
}

fp8attn_status fp8attn_read_error_word(int32_t* d_error, void* stream) {
  if (!d_error) return FP8ATTN_ERR_INVALID;
  int32_t bits = 0;
  cudaError_t e = cudaMemcpyAsync(&bits, d_error, sizeof(int32_t), cudaMemcpyDeviceToHost,
                                  as_stream(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(as_stream(stream));
  if (e == cudaSuccess && bits) {
    e = cudaMemsetAsync(d_error, 0, sizeof(int32_t), as_stream(stream));
    if (e == cudaSuccess) e = cudaStreamSynchronize(as_stream(stream));
  }
  if (e != cudaSuccess) return FP8ATTN_ERR_CUDA;
  return status_of_bits(static_cast<uint32_t>(bits));
}

fp8attn_status fp8attn_parse_selector(const char* text, int max_index, uint8_t* mask_out) {
  if (max_index < 0 || (max_index > 0 && !mask_out)) return FP8ATTN_ERR_INVALID;
  if (max_index > 0) std::memset(mask_out, 0, static_cast<size_t>(max_index));
  if (!text) return FP8ATTN_OK;
  std::vector<uint8_t> mask(static_cast<size_t>(max_index), 0);
  const char* s = text;
  auto skip_ws = [&]() { while (*s == ' ' || *s == '\t') ++s; };
  auto read_int = [&](long* v) {
    if (*s < '0' || *s > '9') return false;
    long x = 0;
    while (*s >= '0' && *s <= '9') {
      x = x * 10 + (*s - '0');
      if (x > 1000000000L) return false;
      ++s;
    }
    *v = x;
    return true;
  };
  skip_ws();
  if (*s == '\0') return FP8ATTN_OK;   // empty selector
  for (;;) {
    long lo = 0, hi = 0;
    skip_ws();
    if (!read_int(&lo)) return FP8ATTN_ERR_INVALID;
    hi = lo;
    skip_ws();
    if (*s == '-') {
      ++s;
      skip_ws();
      if (!read_int(&hi)) return FP8ATTN_ERR_INVALID;
      skip_ws();
    }
    if (hi < lo || hi >= max_index) return FP8ATTN_ERR_INVALID;
    for (long i = lo; i <= hi; ++i) mask[static_cast<size_t>(i)] = 1;
    if (*s == ',') { ++s; continue; }
    if (*s == '\0') break;
    return FP8ATTN_ERR_INVALID;
  }
  if (max_index > 0) std::memcpy(mask_out, mask.data(), mask.size());
  return FP8ATTN_OK;
}

int fp8attn_select_mode(const fp8attn_ctx* ctx, const uint8_t* skip_mask, int layer) {
  if (!layer_ok(ctx, layer)) return -1;
  if (skip_mask && skip_mask[layer]) return FP8ATTN_SKIP;
  return ctx->has_static[layer] ? FP8ATTN_STATIC : FP8ATTN_DYNAMIC;
}

int fp8attn_select_mode_at_step(const fp8attn_ctx* ctx, const uint8_t* skip_layers, int layer,
                                const uint8_t* skip_steps, int num_steps, int step) {
  if (!layer_ok(ctx, layer)) return -1;
  if (skip_steps && (step < 0 || step >= num_steps)) return -1;
  if (skip_steps && skip_steps[step]) return FP8ATTN_SKIP;
  return fp8attn_select_mode(ctx, skip_layers, layer);
}

fp8attn_status fp8attn_e4m3_encode(const float* d_in, int64_t n, float scale, void* d_out,
                                   void* stream) {
  if (n < 0 || (n > 0 && (!d_in || !d_out))) return FP8ATTN_ERR_INVALID;
  if (n == 0) return FP8ATTN_OK;
  const cudaError_t e = launch_encode(d_in, n, scale, d_out, as_stream(stream));
  if (e != cudaSuccess) return FP8ATTN_ERR_CUDA;
  g_launches.fetch_add(1);
  return FP8ATTN_OK;
}

fp8attn_status fp8attn_regroup_heads(const void* d_src, void* d_dst, int64_t tokens,
                                    int num_heads, int groups, int head_bytes, int to_groups,
                                    void* stream) {
  if (tokens < 0 || num_heads < 1 || groups < 1 || head_bytes < 1) return FP8ATTN_ERR_INVALID;
  if (num_heads % groups) return FP8ATTN_ERR_INVALID;
  if (to_groups != 0 && to_groups != 1) return FP8ATTN_ERR_INVALID;
  if (head_bytes % 16) return FP8ATTN_ERR_UNSUPPORTED;
  if (tokens == 0) return FP8ATTN_OK;
  if (!d_src || !d_dst) return FP8ATTN_ERR_INVALID;
  if (!aligned(d_src, 16) || !aligned(d_dst, 16)) return FP8ATTN_ERR_UNSUPPORTED;
  const uintptr_t bytes = static_cast<uintptr_t>(tokens) * num_heads * head_bytes;
  const uintptr_t s0 = reinterpret_cast<uintptr_t>(d_src), d0 = reinterpret_cast<uintptr_t>(d_dst);
  if (s0 < d0 + bytes && d0 < s0 + bytes) return FP8ATTN_ERR_INVALID;   // overlap
  const cudaError_t e = launch_regroup_heads(d_src, d_dst, tokens, num_heads, groups, head_bytes,
                                             to_groups, as_stream(stream));
  if (e != cudaSuccess) return FP8ATTN_ERR_CUDA;
  g_launches.fetch_add(1);
  return FP8ATTN_OK;
}

uint64_t fp8attn_launch_count(void) { return g_launches.load(); }

}  // extern "C"
