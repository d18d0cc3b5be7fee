// Fused amax-reduce + ring/scale update + E4M3 cast + unpad (one launch for
// Q, K and V of one layer), the standalone ring update, and an E4M3 cast
// helper.
//
// The pages' reference path spends three quantisation launches plus an
// unpadding step before the attention call (vLLM docs, "FP8 ViT encoder
// attention", notes) and keeps the 16-entry amax ring on the host side,
// which is why dynamic scaling there cannot be captured in a CUDA graph.
// Here one persistent, co-resident grid does it all on the device:
//   dynamic, per tensor: (1) grid-stride 16-byte loads of the valid tokens,
//   |x| max on bf16 bit patterns (NaN lanes dropped), warp/block reduction,
//   one atomicMax per CTA; (2) a bounded-spin grid barrier; (3) every CTA
//   derives the same bound A from the ring plus this pass's amax; (4) a
//   grid-stride re-read in reverse order (the most recently read data is
//   still in L2), x * qs in fp32, cvt.rn.satfinite to E4M3, packed 8-byte
//   stores.  The last CTA to finish commits the ring and the scales.
//   static: a single read-cast-store sweep over all three tensors.
#include <cuda_runtime.h>

#include "kernels.h"
#include "sm100_ptx.cuh"
#include "state.cuh"

namespace fp8attn {

namespace {

struct QuantArgs {
  const uint16_t* src[3];
  uint8_t* dst[3];
  int64_t tok_stride;     // elements
  int64_t head_stride;    // elements
  const int32_t* cu;      // [B + 1]
  const int32_t* src_seq_start;  // [B] or null
  int B, H, max_seqlen;
  int64_t T;              // expected cu[B]
  GlobalState* gs;
  LayerState* ls;
};

constexpr int kThreads = 512;
constexpr int kUnroll = 4;

// cu_seqlens must start at 0, never decrease, and keep every length within
// max_seqlen.  Every CTA checks it the same way and reaches the same verdict.
__device__ bool seqlens_ok(const QuantArgs& a) {
  int bad = 0;
  if (threadIdx.x == 0 && (__ldg(a.cu) != 0 || __ldg(a.cu + a.B) != a.T)) bad = 1;
  for (int b = threadIdx.x; b < a.B; b += blockDim.x) {
    const int l = __ldg(a.cu + b + 1) - __ldg(a.cu + b);
    if (l < 0 || l > a.max_seqlen) bad = 1;
  }
  return __syncthreads_or(bad) == 0;
}

__device__ __forceinline__ uint4 ld_vec(const uint16_t* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// Element offset of 16-byte vector `v` of the source (8 bf16 per vector,
// 16 vectors per (token, head) row).
template <bool kContig>
__device__ __forceinline__ int64_t src_offset(const QuantArgs& a, int64_t v) {
  if (kContig) return v * 8;
  const int64_t row = v >> 4;
  const int c = static_cast<int>(v & 15);
  const int64_t t = row / a.H;
  const int h = static_cast<int>(row - t * a.H);
  int64_t srow = t;
  if (a.src_seq_start) {
    // sequence of token t: largest b with cu[b] <= t
    int lo = 0, hi = a.B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(a.cu + mid) <= t) lo = mid; else hi = mid - 1;
    }
    srow = static_cast<int64_t>(__ldg(a.src_seq_start + lo)) + (t - __ldg(a.cu + lo));
  }
  return srow * a.tok_stride + h * a.head_stride + c * 8;
}

// max of |x| over 8 bf16 lanes, as bf16 magnitude bits; NaN lanes dropped.
__device__ __forceinline__ uint32_t absmax_bits(uint4 x, uint32_t m2) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t a = w[i] & 0x7FFF7FFFu;
    const uint32_t nan = __vcmpgtu2(a, 0x7F807F80u);
    a &= ~nan;
    m2 = __vmaxu2(m2, a);
  }
  return m2;
}

// 8 bf16 -> 8 E4M3 codes of fl32(x * qs).
__device__ __forceinline__ uint2 cast8(uint4 x, float qs) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  uint32_t h[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = __uint_as_float(w[i] << 16);
    const float hi = __uint_as_float(w[i] & 0xFFFF0000u);
    h[i] = cvt_e4m3x2(__fmul_rn(lo, qs), __fmul_rn(hi, qs));
  }
  return make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
}

template <bool kContig>
__device__ uint32_t amax_sweep(const QuantArgs& a, int t, int64_t nvec) {
  const uint16_t* src = a.src[t];
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  uint32_t m2 = 0;
  for (int64_t v0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v0 < nvec;
       v0 += stride * kUnroll) {
    uint4 x[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t v = v0 + u * stride;
      x[u] = v < nvec ? ld_vec(src + src_offset<kContig>(a, v)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) m2 = absmax_bits(x[u], m2);
  }
  return max(m2 & 0xFFFFu, m2 >> 16);
}

// Cast sweep; `reverse` walks the vectors from the end (L2 reuse after an
// amax sweep that ended there).
template <bool kContig>
__device__ void cast_sweep(const QuantArgs& a, int t, int64_t nvec, float qs, bool reverse) {
  const uint16_t* src = a.src[t];
  uint2* dst = reinterpret_cast<uint2*>(a.dst[t]);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t v0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v0 < nvec;
       v0 += stride * kUnroll) {
    uint4 x[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      int64_t v = v0 + u * stride;
      if (reverse) v = nvec - 1 - v;
      x[u] = (v >= 0 && v < nvec) ? ld_vec(src + src_offset<kContig>(a, v)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      int64_t v = v0 + u * stride;
      if (reverse) v = nvec - 1 - v;
      if (v >= 0 && v < nvec) dst[v] = cast8(x[u], qs);
    }
  }
}

// Block-wide max, result valid in thread 0.
__device__ uint32_t block_max(uint32_t m, uint32_t* red) {
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = m;
  __syncthreads();
  if (warp == 0) {
    m = lane < static_cast<int>(blockDim.x >> 5) ? red[lane] : 0u;
    m = __reduce_max_sync(0xFFFFFFFFu, m);
  }
  __syncthreads();
  return m;
}

// Grid-wide barrier over co-resident CTAs (cooperative launch).  Bounded:
// returns false if the other CTAs did not arrive within the wait limit.
__device__ bool grid_barrier(GlobalState* gs, int* s_ok) {
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile uint32_t* gen = &gs->bar_gen;
    const uint32_t my_gen = *gen;
    __threadfence();
    const uint32_t arrived = atomicAdd(&gs->bar_count, 1u) + 1u;
    int ok = 1;
    if (arrived == gridDim.x) {
      gs->bar_count = 0;
      __threadfence();
      atomicAdd(&gs->bar_gen, 1u);
    } else {
      const uint64_t t0 = global_timer_ns();
      uint32_t it = 0;
      while (*gen == my_gen) {
        if ((++it & 255u) == 0 && global_timer_ns() - t0 > kWaitLimitNs) { ok = 0; break; }
        __nanosleep(64);
      }
    }
    __threadfence();
    *s_ok = ok;
  }
  __syncthreads();
  return *s_ok != 0;
}

template <bool kContig>
__global__ void __launch_bounds__(kThreads) quant_dynamic_kernel(QuantArgs a) {
  __shared__ uint32_t red[kThreads / 32];
  __shared__ int s_ok;
  if (!seqlens_ok(a)) {
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(&a.gs->error, kErrSeqlens);
    return;
  }
  const int64_t T = __ldg(a.cu + a.B);
  const int64_t nvec = T * a.H * 16;
  LayerState* ls = a.ls;
  for (int t = 0; t < 3; ++t) {
    uint32_t m = amax_sweep<kContig>(a, t, nvec);
    m = block_max(m, red);
    if (threadIdx.x == 0 && m != 0) atomicMax(&a.gs->amax_bits[t], m);
    if (!grid_barrier(a.gs, &s_ok)) {
      if (threadIdx.x == 0) atomicOr(&a.gs->error, kErrTimeout);
      return;
    }
    // every CTA derives the same bound from the (not yet updated) ring
    const uint32_t bits = *reinterpret_cast<volatile uint32_t*>(&a.gs->amax_bits[t]);
    const float amax = __uint_as_float(bits << 16);
    const bool finite = bits < 0x7F80u;
    const uint32_t count = ls->count[t], head = ls->head[t];
    float A = finite ? amax : 0.0f;
    for (uint32_t i = 0; i < count; ++i)
      if (!finite || i != head) A = fmaxf(A, ls->ring[t][i]);
    float qs, ds;
    scales_from_bound(A, &qs, &ds);
    cast_sweep<kContig>(a, t, nvec, qs, true);
  }
  // the last CTA out commits the ring and the scales and clears the words
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t done = atomicAdd(&a.gs->done_count, 1u) + 1u;
    if (done == gridDim.x) {
      __threadfence();
      for (int t = 0; t < 3; ++t) {
        const uint32_t bits = *reinterpret_cast<volatile uint32_t*>(&a.gs->amax_bits[t]);
        const bool finite = bits < 0x7F80u;
        if (finite) {
          ls->ring[t][ls->head[t]] = __uint_as_float(bits << 16);
          ls->head[t] = (ls->head[t] + 1) % kRing;
          if (ls->count[t] < kRing) ls->count[t] += 1;
        } else {
          atomicOr(&a.gs->error, kErrNonfinite);
        }
        float A = 0.0f;
        for (uint32_t i = 0; i < ls->count[t]; ++i) A = fmaxf(A, ls->ring[t][i]);
        scales_from_bound(A, &ls->qs[t], &ls->ds[t]);
        a.gs->amax_bits[t] = 0;
      }
      a.gs->done_count = 0;
      __threadfence();
    }
  }
}

template <bool kContig>
__global__ void __launch_bounds__(kThreads) quant_static_kernel(QuantArgs a) {
  if (!seqlens_ok(a)) {
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(&a.gs->error, kErrSeqlens);
    return;
  }
  const int64_t T = __ldg(a.cu + a.B);
  const int64_t nvec = T * a.H * 16;
  for (int t = 0; t < 3; ++t) cast_sweep<kContig>(a, t, nvec, a.ls->static_qs[t], false);
  if (blockIdx.x == 0 && threadIdx.x < 3) {
    a.ls->qs[threadIdx.x] = a.ls->static_qs[threadIdx.x];
    a.ls->ds[threadIdx.x] = a.ls->static_ds[threadIdx.x];
  }
}

// Standalone ring update from three device-side amax values.
__global__ void ring_update_kernel(LayerState* ls, GlobalState* gs, const float* amax3) {
  const int t = threadIdx.x;
  if (t >= 3) return;
  const float v = amax3[t];
  if (isfinite(v) && v >= 0.0f) {
    ls->ring[t][ls->head[t]] = v;
    ls->head[t] = (ls->head[t] + 1) % kRing;
    if (ls->count[t] < kRing) ls->count[t] += 1;
  } else {
    atomicOr(&gs->error, kErrNonfinite);
  }
  float A = 0.0f;
  for (uint32_t i = 0; i < ls->count[t]; ++i) A = fmaxf(A, ls->ring[t][i]);
  scales_from_bound(A, &ls->qs[t], &ls->ds[t]);
}

// Recompute a layer's dynamic scales from its ring (after a state restore).
__global__ void rescale_from_ring_kernel(LayerState* ls) {
  const int t = threadIdx.x;
  if (t >= 3) return;
  float A = 0.0f;
  for (uint32_t i = 0; i < ls->count[t]; ++i) A = fmaxf(A, ls->ring[t][i]);
  scales_from_bound(A, &ls->qs[t], &ls->ds[t]);
}

__global__ void encode_kernel(const float* in, int64_t n, float scale, uint8_t* out) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; 2 * i < n;
       i += stride) {
    const float lo = __fmul_rn(in[2 * i], scale);
    const float hi = 2 * i + 1 < n ? __fmul_rn(in[2 * i + 1], scale) : 0.0f;
    const uint16_t c = cvt_e4m3x2(lo, hi);
    out[2 * i] = static_cast<uint8_t>(c & 0xFF);
    if (2 * i + 1 < n) out[2 * i + 1] = static_cast<uint8_t>(c >> 8);
  }
}

template <typename K>
int max_coresident(K kernel, int threads) {
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0) != cudaSuccess)
    return 0;
  return sms * per_sm;
}

}  // namespace

cudaError_t launch_quantize(const QuantLaunch& q, cudaStream_t stream) {
  QuantArgs a;
  for (int t = 0; t < 3; ++t) {
    a.src[t] = static_cast<const uint16_t*>(q.src[t]);
    a.dst[t] = static_cast<uint8_t*>(q.dst[t]);
  }
  a.tok_stride = q.tok_stride;
  a.head_stride = q.head_stride;
  a.cu = q.cu;
  a.src_seq_start = q.src_seq_start;
  a.B = q.batch;
  a.H = q.heads;
  a.max_seqlen = q.max_seqlen;
  a.T = q.total_tokens;
  a.gs = static_cast<GlobalState*>(q.gs);
  a.ls = static_cast<LayerState*>(q.ls);
  const bool contig = q.src_seq_start == nullptr && q.head_stride == kHeadDim &&
                      q.tok_stride == static_cast<int64_t>(q.heads) * kHeadDim;
  // enough CTAs to cover the upper bound of the work, at most one full wave
  const int64_t nvec_max = q.total_tokens * q.heads * 16;
  const int64_t want = (nvec_max + static_cast<int64_t>(kThreads) * kUnroll - 1) /
                       (static_cast<int64_t>(kThreads) * kUnroll);
  void* args[] = {&a};
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  if (q.dynamic) {
    const void* fn = contig ? reinterpret_cast<const void*>(&quant_dynamic_kernel<true>)
                            : reinterpret_cast<const void*>(&quant_dynamic_kernel<false>);
    const int cap = contig ? max_coresident(quant_dynamic_kernel<true>, kThreads)
                           : max_coresident(quant_dynamic_kernel<false>, kThreads);
    if (cap <= 0) return cudaErrorInvalidConfiguration;
    const int grid = static_cast<int>(want < cap ? (want < 1 ? 1 : want) : cap);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.gridDim = dim3(grid);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelExC(&cfg, fn, args);
  }
  const void* fn = contig ? reinterpret_cast<const void*>(&quant_static_kernel<true>)
                          : reinterpret_cast<const void*>(&quant_static_kernel<false>);
  const int cap = contig ? max_coresident(quant_static_kernel<true>, kThreads)
                         : max_coresident(quant_static_kernel<false>, kThreads);
  if (cap <= 0) return cudaErrorInvalidConfiguration;
  const int grid = static_cast<int>(want < cap ? (want < 1 ? 1 : want) : cap);
  cfg.gridDim = dim3(grid);
  cfg.attrs = nullptr;
  cfg.numAttrs = 0;
  return cudaLaunchKernelExC(&cfg, fn, args);
}

cudaError_t launch_ring_update(void* ls, void* gs, const float* amax3, cudaStream_t stream) {
  ring_update_kernel<<<1, 32, 0, stream>>>(static_cast<LayerState*>(ls),
                                           static_cast<GlobalState*>(gs), amax3);
  return cudaGetLastError();
}

cudaError_t launch_rescale_from_ring(void* ls, cudaStream_t stream) {
  rescale_from_ring_kernel<<<1, 32, 0, stream>>>(static_cast<LayerState*>(ls));
  return cudaGetLastError();
}

cudaError_t launch_encode(const float* in, int64_t n, float scale, void* out,
                          cudaStream_t stream) {
  const int64_t pairs = (n + 1) / 2;
  int64_t blocks = (pairs + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  encode_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(in, n, scale,
                                                                   static_cast<uint8_t*>(out));
  return cudaGetLastError();
}

}  // namespace fp8attn
