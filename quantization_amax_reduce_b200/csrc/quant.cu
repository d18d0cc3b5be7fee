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
//   static (and ring-scale): a single read-cast-store sweep over all three
//   tensors, writing packed [T, H, 128] codes or, for sequence-parallel
//   attention, head-grouped [groups, T, H / groups, 128] send buffers.
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
  int cast_with_ring;     // static kernel: 1 = use the ring scales qs (kQuantRing)
  float* amax_out;        // amax kernel: device float[3]
  int dst_groups;         // static kernel, kGrouped: head groups of the output
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

// One read-cast-store sweep with known scales: the static bounds (which then
// become the layer's current scales), or the ring's current scales as left by
// the last ring update (a shard of a head-sharded pass, whose amax was
// reduced across ranks and pushed with fp8attn_amax_ring_update).
// Q, K and V are swept together: each step of a thread reads the same two
// 16-byte vectors (16 channels of one token and head) of all three tensors
// and writes three 16-byte code vectors, so the whole launch is one grid
// stride loop with six loads in flight per step and no per-tensor tail.
constexpr int kUnrollStatic = 2;

// Index of output vector p (16 codes: vector p % 8 of token p / (8 H), head
// (p / 8) % H) in the head-grouped layout [groups][T][H / groups][128]: the
// send buffer of a sequence-parallel all-to-all, group g going to rank g.
__device__ __forceinline__ int64_t grouped_vec(const QuantArgs& a, int64_t T, int64_t p) {
  const int64_t per_tok = static_cast<int64_t>(a.H) * 8;
  const int64_t tok = p / per_tok;
  const int rem = static_cast<int>(p - tok * per_tok);
  const int head = rem >> 3;
  const int hn = a.H / a.dst_groups;
  const int g = head / hn;
  return (static_cast<int64_t>(g) * T + tok) * (hn * 8) + (head - g * hn) * 8 + (rem & 7);
}

template <bool kContig, bool kGrouped>
__global__ void __launch_bounds__(kThreads) quant_static_kernel(QuantArgs a) {
  if (!seqlens_ok(a)) {
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(&a.gs->error, kErrSeqlens);
    return;
  }
  const int64_t T = __ldg(a.cu + a.B);
  const int64_t npair = T * a.H * 8;   // pairs of 16-byte vectors (16 rows of a channel block)
  const float* qsp = a.cast_with_ring ? a.ls->qs : a.ls->static_qs;
  const float qs[3] = {qsp[0], qsp[1], qsp[2]};
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t p0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; p0 < npair;
       p0 += stride * kUnrollStatic) {
    uint4 x[kUnrollStatic][3][2];
#pragma unroll
    for (int u = 0; u < kUnrollStatic; ++u) {
      const int64_t p = p0 + u * stride;
      // vectors 2p and 2p + 1 lie in the same 128-channel row, 8 elements apart
      const int64_t off = p < npair ? src_offset<kContig>(a, 2 * p) : 0;
#pragma unroll
      for (int t = 0; t < 3; ++t) {
        x[u][t][0] = p < npair ? ld_vec(a.src[t] + off) : make_uint4(0, 0, 0, 0);
        x[u][t][1] = p < npair ? ld_vec(a.src[t] + off + 8) : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnrollStatic; ++u) {
      const int64_t p = p0 + u * stride;
      if (p < npair) {
        const int64_t d = kGrouped ? grouped_vec(a, T, p) : p;
#pragma unroll
        for (int t = 0; t < 3; ++t) {
          const uint2 lo = cast8(x[u][t][0], qs[t]);
          const uint2 hi = cast8(x[u][t][1], qs[t]);
          reinterpret_cast<uint4*>(a.dst[t])[d] = make_uint4(lo.x, lo.y, hi.x, hi.y);
        }
      }
    }
  }
  if (!a.cast_with_ring && blockIdx.x == 0 && threadIdx.x < 3) {
    a.ls->qs[threadIdx.x] = a.ls->static_qs[threadIdx.x];
    a.ls->ds[threadIdx.x] = a.ls->static_ds[threadIdx.x];
  }
}

// Per-tensor amax only (no cast, ring untouched): every CTA folds its share
// into the global amax words; the last CTA out writes the three values as
// floats (NaN ignored, an infinite amax stays infinite) and clears the words.
template <bool kContig>
__global__ void __launch_bounds__(kThreads) quant_amax_kernel(QuantArgs a) {
  __shared__ uint32_t red[kThreads / 32];
  if (!seqlens_ok(a)) {
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(&a.gs->error, kErrSeqlens);
    return;
  }
  const int64_t T = __ldg(a.cu + a.B);
  const int64_t nvec = T * a.H * 16;
  for (int t = 0; t < 3; ++t) {
    uint32_t m = amax_sweep<kContig>(a, t, nvec);
    m = block_max(m, red);
    if (threadIdx.x == 0 && m != 0) atomicMax(&a.gs->amax_bits[t], m);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t done = atomicAdd(&a.gs->done_count, 1u) + 1u;
    if (done == gridDim.x) {
      __threadfence();
      for (int t = 0; t < 3; ++t) {
        const uint32_t bits = *reinterpret_cast<volatile uint32_t*>(&a.gs->amax_bits[t]);
        a.amax_out[t] = __uint_as_float(bits << 16);
        a.gs->amax_bits[t] = 0;
      }
      a.gs->done_count = 0;
      __threadfence();
    }
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
  a.cast_with_ring = q.kind == kQuantRing;
  a.amax_out = q.amax_out;
  a.dst_groups = q.dst_groups;
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
  if (q.kind == kQuantAmaxOnly) {
    // no grid-wide wait: any grid size works; one wave at most
    const void* fn = contig ? reinterpret_cast<const void*>(&quant_amax_kernel<true>)
                            : reinterpret_cast<const void*>(&quant_amax_kernel<false>);
    const int cap = contig ? max_coresident(quant_amax_kernel<true>, kThreads)
                           : max_coresident(quant_amax_kernel<false>, kThreads);
    if (cap <= 0) return cudaErrorInvalidConfiguration;
    cfg.gridDim = dim3(static_cast<int>(want < cap ? (want < 1 ? 1 : want) : cap));
    cfg.attrs = nullptr;
    cfg.numAttrs = 0;
    return cudaLaunchKernelExC(&cfg, fn, args);
  }
  if (q.kind == kQuantDynamic) {
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
  const bool grouped = q.dst_groups > 1;
  const void* fn =
      grouped ? (contig ? reinterpret_cast<const void*>(&quant_static_kernel<true, true>)
                        : reinterpret_cast<const void*>(&quant_static_kernel<false, true>))
              : (contig ? reinterpret_cast<const void*>(&quant_static_kernel<true, false>)
                        : reinterpret_cast<const void*>(&quant_static_kernel<false, false>));
  const int cap = grouped ? (contig ? max_coresident(quant_static_kernel<true, true>, kThreads)
                                    : max_coresident(quant_static_kernel<false, true>, kThreads))
                          : (contig ? max_coresident(quant_static_kernel<true, false>, kThreads)
                                    : max_coresident(quant_static_kernel<false, false>, kThreads));
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

// ---------------------------------------------------------------------------
// Allocation-free variant of the fused dynamic quantisation.
//
// Some callers cannot allocate device memory at all: code that runs inside a
// host-side allocator-free region (a plugin or operator that is handed only
// its input and output buffers by an inference runtime with a fixed memory
// plan), or a caller that must not touch cudaMalloc/cudaFree because those
// calls synchronise the device.  They cannot provide the context workspace
// that fp8attn_quantize_qkv uses for its grid-wide reduction, so this
// variant keeps that scratch in a fixed array inside the library and needs
// nothing but the inputs and outputs.  It computes this call's per-tensor
// amax (no ring: the scales come from this call alone, as on the first
// dynamic pass of a fresh context), casts, and writes the scales.
// ---------------------------------------------------------------------------

#include <mutex>

namespace fp8attn {

namespace {

// One partial |x|-max slot (q, k, v, pad) per CTA, then the barrier words.
constexpr int kNoAllocMaxCtas = 1024;
constexpr int kNoAllocWordBar = kNoAllocMaxCtas * 4;   // bar_count
constexpr int kNoAllocWordGen = kNoAllocWordBar + 1;   // bar_gen
constexpr int kNoAllocWordErr = kNoAllocWordBar + 2;   // error bits
constexpr int kNoAllocWords = kNoAllocWordBar + 64;    // 16,640 bytes

// Library-owned scratch; every device that loads the library holds its own
// copy until the process exits.  Zero at load time.
static __device__ __align__(256) uint32_t g_noalloc_scratch[kNoAllocWords];

struct NoAllocArgs {
  QuantArgs a;             // gs / ls unused
  uint32_t* scratch;       // device address of g_noalloc_scratch
  float* descale_out;      // [3] ds_q, ds_k, ds_v
  float* scale_out;        // [3] qs_q, qs_k, qs_v, or null
};

__device__ bool noalloc_barrier(uint32_t* scratch, int* s_ok) {
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile uint32_t* gen = scratch + kNoAllocWordGen;
    const uint32_t my_gen = *gen;
    __threadfence();
    const uint32_t arrived = atomicAdd(scratch + kNoAllocWordBar, 1u) + 1u;
    int ok = 1;
    if (arrived == gridDim.x) {
      scratch[kNoAllocWordBar] = 0;
      __threadfence();
      atomicAdd(scratch + kNoAllocWordGen, 1u);
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
__global__ void __launch_bounds__(kThreads) quant_noalloc_kernel(NoAllocArgs n) {
  __shared__ uint32_t red[kThreads / 32];
  __shared__ int s_ok;
  __shared__ float s_scale[2][3];
  const QuantArgs& a = n.a;
  uint32_t* scratch = n.scratch;
  // A call that timed out may have left the barrier words mid-count: until
  // fp8attn_quantize_qkv_noalloc_error has reported the timeout and reset
  // them, every call leaves at once (outputs untouched).
  if (*reinterpret_cast<volatile uint32_t*>(scratch + kNoAllocWordErr) & kErrTimeout) return;
  if (!seqlens_ok(a)) {
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(scratch + kNoAllocWordErr, kErrSeqlens);
    return;
  }
  const int64_t T = __ldg(a.cu + a.B);
  const int64_t nvec = T * a.H * 16;
  for (int t = 0; t < 3; ++t) {
    uint32_t m = amax_sweep<kContig>(a, t, nvec);
    m = block_max(m, red);
    // each CTA owns its slot and rewrites it on every call: nothing to clear
    if (threadIdx.x == 0) scratch[blockIdx.x * 4 + t] = m;
    if (!noalloc_barrier(scratch, &s_ok)) {
      if (threadIdx.x == 0) atomicOr(scratch + kNoAllocWordErr, kErrTimeout);
      return;
    }
    // every CTA reduces all slots the same way and gets the same bound
    uint32_t all = 0;
    for (uint32_t c = threadIdx.x; c < gridDim.x; c += blockDim.x)
      all = max(all, *reinterpret_cast<volatile uint32_t*>(scratch + c * 4 + t));
    all = block_max(all, red);
    if (threadIdx.x == 0) {
      const bool finite = all < 0x7F80u;
      float qs, ds;
      scales_from_bound(finite ? __uint_as_float(all << 16) : 0.0f, &qs, &ds);
      s_scale[0][t] = qs;
      s_scale[1][t] = ds;
      if (!finite && blockIdx.x == 0) atomicOr(scratch + kNoAllocWordErr, kErrNonfinite);
    }
    __syncthreads();
    cast_sweep<kContig>(a, t, nvec, s_scale[0][t], true);
  }
  if (blockIdx.x == 0 && threadIdx.x < 3) {
    n.descale_out[threadIdx.x] = s_scale[1][threadIdx.x];
    if (n.scale_out) n.scale_out[threadIdx.x] = s_scale[0][threadIdx.x];
  }
}

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};

// Device address of the scratch array for the current device, looked up once
// per device (host code cannot use the array's name as a device address).
cudaError_t noalloc_scratch(uint32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = p;
  }
  *out = static_cast<uint32_t*>(g_noalloc_ptr[dev]);
  return cudaSuccess;
}

}  // namespace

}  // namespace fp8attn

// ---------------------------------------------------------------------------
// Self-test of the bounded waits: failure detection without a GPU fault.
// Each probe waits on something that never completes; the wait must give up
// at its limit and report it, and the GPU stays usable.
// ---------------------------------------------------------------------------
namespace fp8attn {
namespace {

__device__ GlobalState g_probe_state;     // grid-barrier words used only here
__device__ int32_t g_probe_result[2];     // per probe: 1 = the wait completed, 2 = gave up

// An mbarrier that nothing arrives on: mbar_wait_limit (the wait of the
// attention kernels, with a caller-chosen limit) must give up.
__global__ void mbar_timeout_probe(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  const bool done = mbar_wait_limit(&bar, 0, nullptr, limit_ns);
  if (threadIdx.x == 0) g_probe_result[0] = done ? 1 : 2;
}

// The quantisation kernels' grid barrier with one of two CTAs leaving before
// it arrives: the other must give up after kWaitLimitNs.
__global__ void grid_barrier_timeout_probe() {
  __shared__ int s_ok;
  if (blockIdx.x == 1) return;
  const bool ok = grid_barrier(&g_probe_state, &s_ok);
  if (threadIdx.x == 0) g_probe_result[1] = ok ? 1 : 2;
}

}  // namespace
}  // namespace fp8attn

extern "C" {

// See include/fp8attn.h.
int fp8attn_selftest_bounded_waits(uint64_t mbar_limit_ns, int* h_gave_up, void* stream) {
  using namespace fp8attn;
  if (!h_gave_up || mbar_limit_ns == 0 || mbar_limit_ns > kWaitLimitNs) return 1;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const GlobalState zero_state{};
  const int32_t zero_result[2] = {0, 0};
  if (cudaMemcpyToSymbolAsync(g_probe_state, &zero_state, sizeof(zero_state), 0,
                              cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyToSymbolAsync(g_probe_result, zero_result, sizeof(zero_result), 0,
                              cudaMemcpyHostToDevice, s) != cudaSuccess)
    return 2;
  mbar_timeout_probe<<<1, 32, 0, s>>>(mbar_limit_ns);
  grid_barrier_timeout_probe<<<2, 32, 0, s>>>();
  if (cudaGetLastError() != cudaSuccess) return 2;
  int32_t result[2] = {0, 0};
  if (cudaMemcpyFromSymbolAsync(result, g_probe_result, sizeof(result), 0,
                                cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return 2;
  *h_gave_up = (result[0] == 2 ? 1 : 0) + (result[1] == 2 ? 1 : 0);
  return 0;
}

// See include/fp8attn.h.
int fp8attn_quantize_qkv_noalloc(const void* q, const void* k, const void* v, int64_t tok_stride,
                                 int64_t head_stride, const int32_t* d_src_seq_start,
                                 const int32_t* d_cu_seqlens, int batch, int max_seqlen,
                                 int64_t total_tokens, int num_heads, int head_dim, void* q8,
                                 void* k8, void* v8, float* d_descale_out, float* d_scale_out,
                                 void* stream) {
  using namespace fp8attn;
  auto aligned = [](const void* p, uintptr_t al) {
    return (reinterpret_cast<uintptr_t>(p) & (al - 1)) == 0;
  };
  if (batch < 1 || max_seqlen < 0 || num_heads < 1 || total_tokens < 0 || !d_cu_seqlens ||
      !d_descale_out)
    return 1;   // FP8ATTN_ERR_INVALID
  if (head_dim != kHeadDim) return 4;   // FP8ATTN_ERR_UNSUPPORTED
  if (total_tokens > static_cast<int64_t>(batch) * max_seqlen) return 1;
  if (!q || !k || !v || !q8 || !k8 || !v8) return 1;
  if (tok_stride <= 0 || head_stride <= 0 || (tok_stride % 8) || (head_stride % 8)) return 4;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(q8, 16) ||
      !aligned(k8, 16) || !aligned(v8, 16) || !aligned(d_descale_out, 4) ||
      (d_scale_out && !aligned(d_scale_out, 4)))
    return 4;
  uint32_t* scratch = nullptr;
  if (noalloc_scratch(&scratch) != cudaSuccess) return 2;   // FP8ATTN_ERR_CUDA
  NoAllocArgs n;
  QuantArgs& a = n.a;
  a.src[0] = static_cast<const uint16_t*>(q);
  a.src[1] = static_cast<const uint16_t*>(k);
  a.src[2] = static_cast<const uint16_t*>(v);
  a.dst[0] = static_cast<uint8_t*>(q8);
  a.dst[1] = static_cast<uint8_t*>(k8);
  a.dst[2] = static_cast<uint8_t*>(v8);
  a.tok_stride = tok_stride;
  a.head_stride = head_stride;
  a.cu = d_cu_seqlens;
  a.src_seq_start = d_src_seq_start;
  a.B = batch;
  a.H = num_heads;
  a.max_seqlen = max_seqlen;
  a.T = total_tokens;
  a.gs = nullptr;
  a.ls = nullptr;
  a.cast_with_ring = 0;
  a.amax_out = nullptr;
  n.scratch = scratch;
  n.descale_out = d_descale_out;
  n.scale_out = d_scale_out;
  const bool contig = d_src_seq_start == nullptr && head_stride == kHeadDim &&
                      tok_stride == static_cast<int64_t>(num_heads) * kHeadDim;
  const int cap = contig ? max_coresident(quant_noalloc_kernel<true>, kThreads)
                         : max_coresident(quant_noalloc_kernel<false>, kThreads);
  if (cap <= 0) return 2;
  const int64_t nvec_max = total_tokens * num_heads * 16;
  int64_t want = (nvec_max + static_cast<int64_t>(kThreads) * kUnroll - 1) /
                 (static_cast<int64_t>(kThreads) * kUnroll);
  if (want < 1) want = 1;
  const int64_t grid = want < cap ? want : cap;
  // the array holds one partial maximum per CTA: a launch needing more CTAs
  // than it has slots is refused
  if (grid > kNoAllocMaxCtas) return 4;   // FP8ATTN_ERR_UNSUPPORTED
  void* args[] = {&n};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.stream = static_cast<cudaStream_t>(stream);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const void* fn = contig ? reinterpret_cast<const void*>(&quant_noalloc_kernel<true>)
                          : reinterpret_cast<const void*>(&quant_noalloc_kernel<false>);
  if (cudaLaunchKernelExC(&cfg, fn, args) != cudaSuccess) return 2;
  note_launch();
  return 0;
}

// See include/fp8attn.h.
int fp8attn_quantize_qkv_noalloc_error(void* stream) {
  using namespace fp8attn;
  uint32_t* scratch = nullptr;
  if (noalloc_scratch(&scratch) != cudaSuccess) return 2;
  uint32_t bits = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(&bits, scratch + kNoAllocWordErr, sizeof(bits),
                                  cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return 2;
  if (bits) {
    // clear the error; after a timeout also reset the barrier words
    e = cudaMemsetAsync(scratch + kNoAllocWordBar, 0,
                        (bits & kErrTimeout) ? 3 * sizeof(uint32_t) : 0, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(scratch + kNoAllocWordErr, 0, sizeof(uint32_t), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return 2;
  }
  if (bits & kErrTimeout) return 3;
  if (bits & kErrSeqlens) return 6;
  if (bits & kErrNonfinite) return 5;
  return 0;
}

}  // extern "C"
