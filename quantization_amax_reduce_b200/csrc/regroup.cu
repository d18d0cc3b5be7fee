// Head-group regrouping for sequence-parallel (Ulysses) attention.
//
// vLLM-Omni docs, "Quantized KV Cache", Configuration: the offline diffusion
// example runs the DiT with a Ulysses degree of 4, i.e. each rank holds a
// contiguous slice of the sequence's tokens, and an all-to-all hands every
// rank all tokens of H/G heads before attention (and back after it).  An
// all-to-all moves contiguous per-destination chunks, so the per-rank layout
// [T, H, hb] (hb bytes per head row) has to become [G, T, H/G, hb] before the
// exchange, and the received [G, T, H/G, hb] has to become [T, H, hb] after
// the return exchange.  Both are one pass of 16-byte vector copies; every
// token's group block (H/G * hb bytes) is contiguous on both sides, so reads
// and writes stay coalesced.
#include <cuda_runtime.h>

#include "kernels.h"

namespace fp8attn {

namespace {

constexpr int kRegroupThreads = 256;
constexpr int kRegroupUnroll = 4;

struct RegroupArgs {
  const uint4* src;
  uint4* dst;
  int64_t tokens;
  int64_t row_vecs;     // H * hb / 16: vectors per token row
  int64_t group_vecs;   // row_vecs / G: vectors per token of one group
  int64_t nvec;         // tokens * row_vecs
  int to_groups;
};

// Source vector of destination vector v.
__device__ __forceinline__ int64_t regroup_src(const RegroupArgs& a, int64_t v) {
  if (a.to_groups) {
    // dst [G, T, W] <- src [T, G * W]
    const int64_t w = v % a.group_vecs;
    const int64_t r = v / a.group_vecs;      // g * T + t
    const int64_t t = r % a.tokens;
    const int64_t g = r / a.tokens;
    return t * a.row_vecs + g * a.group_vecs + w;
  }
  // dst [T, G * W] <- src [G, T, W]
  const int64_t x = v % a.row_vecs;
  const int64_t t = v / a.row_vecs;
  const int64_t g = x / a.group_vecs;
  const int64_t w = x - g * a.group_vecs;
  return (g * a.tokens + t) * a.group_vecs + w;
}

__global__ void __launch_bounds__(kRegroupThreads) regroup_kernel(RegroupArgs a) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t v0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v0 < a.nvec;
       v0 += stride * kRegroupUnroll) {
    uint4 x[kRegroupUnroll];
#pragma unroll
    for (int u = 0; u < kRegroupUnroll; ++u) {
      const int64_t v = v0 + u * stride;
      if (v < a.nvec) x[u] = __ldg(a.src + regroup_src(a, v));
    }
#pragma unroll
    for (int u = 0; u < kRegroupUnroll; ++u) {
      const int64_t v = v0 + u * stride;
      if (v < a.nvec) a.dst[v] = x[u];
    }
  }
}

}  // namespace

cudaError_t launch_regroup_heads(const void* src, void* dst, int64_t tokens, int heads,
                                 int groups, int head_bytes, int to_groups, cudaStream_t stream) {
  RegroupArgs a;
  a.src = static_cast<const uint4*>(src);
  a.dst = static_cast<uint4*>(dst);
  a.tokens = tokens;
  a.row_vecs = static_cast<int64_t>(heads) * (head_bytes / 16);
  a.group_vecs = a.row_vecs / groups;
  a.nvec = tokens * a.row_vecs;
  a.to_groups = to_groups;
  if (a.nvec == 0) return cudaSuccess;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  // up to 8 CTAs of 256 threads per SM, each thread kRegroupUnroll vectors
  // per grid-stride step
  const int64_t per_cta = static_cast<int64_t>(kRegroupThreads) * kRegroupUnroll;
  int64_t grid = (a.nvec + per_cta - 1) / per_cta;
  const int64_t cap = static_cast<int64_t>(sms) * 8;
  if (grid > cap) grid = cap;
  regroup_kernel<<<static_cast<unsigned>(grid), kRegroupThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace fp8attn
