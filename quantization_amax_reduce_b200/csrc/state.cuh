// Device-resident scale state: per-layer amax rings and scales, plus the
// words the fused quantisation kernel uses for its grid-wide reduction.
// Everything lives in caller-owned workspace memory so that a dynamic
// scaling pass needs no host round trip and can be captured in a CUDA graph.
#pragma once

#include <cstddef>
#include <cstdint>

namespace fp8attn {

constexpr int kRing = 16;       // vLLM FP8 ViT page: 16 observed amax values
constexpr int kHeadDim = 128;
constexpr float kE4M3Max = 448.0f;

// Error bits in the device error word.
constexpr uint32_t kErrTimeout = 1u;
constexpr uint32_t kErrNonfinite = 2u;
constexpr uint32_t kErrSeqlens = 4u;

struct GlobalState {
  uint32_t amax_bits[4];   // per-call |x| max as bf16 magnitude bits (q, k, v)
  uint32_t bar_count;      // grid barrier: arrivals in the current round
  uint32_t bar_gen;        // grid barrier: completed rounds
  uint32_t done_count;     // CTAs that finished reading the shared words
  uint32_t error;          // OR of kErr* bits
  uint32_t pad[56];        // 256 bytes total
};

struct LayerState {
  float ring[3][kRing];    // observed amax per tensor (q, k, v)
  uint32_t head[3];        // next slot
  uint32_t count[3];       // filled slots (<= 16)
  float qs[3];             // current quantisation scales (448 / A)
  float ds[3];             // current descales (A / 448)
  float static_qs[3];      // static-mode scales
  float static_ds[3];
  float static_bound[3];   // static bounds A as set by the caller
  uint32_t pad[11];        // 320 bytes total
};

static_assert(sizeof(GlobalState) == 256, "GlobalState layout");
static_assert(sizeof(LayerState) == 320, "LayerState layout");

inline size_t workspace_bytes_for(int layers) {
  return sizeof(GlobalState) + static_cast<size_t>(layers) * sizeof(LayerState);
}

// Scales from a bound: qs = 448 / A, ds = A / 448, each one IEEE fp32
// division (correctly rounded); A == 0 gives 1, 1.
__host__ __device__ inline void scales_from_bound(float A, float* qs, float* ds) {
#ifdef __CUDA_ARCH__
  if (A == 0.0f) { *qs = 1.0f; *ds = 1.0f; return; }
  *qs = __fdiv_rn(kE4M3Max, A);
  *ds = __fdiv_rn(A, kE4M3Max);
#else
  if (A == 0.0f) { *qs = 1.0f; *ds = 1.0f; return; }
  volatile float a = A;   // keep the division in fp32
  *qs = kE4M3Max / a;
  *ds = a / kE4M3Max;
#endif
}

}  // namespace fp8attn
