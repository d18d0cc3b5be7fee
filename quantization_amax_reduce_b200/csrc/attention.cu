// Varlen, non-causal flash-attention forward on tcgen05 tensor cores.
//
// FP8 (E4M3) instantiation: the quantised Q/K/V feed the attention operator
// (vLLM-Omni docs, "Quantized KV Cache", overview; vLLM docs, "FP8 ViT
// encoder attention": per-tensor scales).  BF16 instantiation: the same
// kernel on native bf16 inputs for skipped layers (vLLM-Omni parameters
// table: selected layers keep the native dtype).
//
// A work unit is 256 query rows (two 128-row tiles) of one (sequence, head);
// its CTA streams the sequence's 128-key K/V tiles once for both tiles:
//   warp 8        TMA producer: Q tiles once, then rings of K and V stages
//   warps 9, 10   FP8: MMA issuers for tiles 0 and 1 (one lane each):
//                 S_i = Q_i K^T into TMEM, then O_i += P_i V (V in shared
//                 memory, MN-major); bf16: warp 9 issues for both tiles
//   warps 0-3     softmax for tile 0, warps 4-7 for tile 1: one thread per
//                 query row (= TMEM lane): block max, P quantised for the
//                 PV product, row sum, O rescaled in TMEM when the max that
//                 P is taken against moves, and the bf16 epilogue.
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512).
// attn_fwd_bf16_kernel: P_i aliases the first 64 columns of S_i and PV
// reads it from TMEM; S_i(j+1) is issued after PV_i(j).
// attn_fwd_fp8_kernel: P_i goes to shared memory, so S_i(j+1) is computed
// while the softmax still works on block j.  Its <rule, 1, *> instantiation
// runs a unit as two CTAs of one tile each (the automatic schedule's fill
// for a mostly empty last wave, launched behind the whole units).  Its
// <rule, *, 1> instantiation takes bf16 Q/K/V and casts them with the
// layer's static scales inside the kernel (384 threads): every warp casts Q
// (and, for a sequence of at most 512 keys, all of K and V) straight from
// global memory before the roles start; longer sequences stream bf16 K/V
// tiles through TMA staging that the TMA warp and warp 11 cast.
//
// P rule (pages silent; fixed here), per 128-key block: c = ds_q ds_k
// softmax_scale log2(e), t = s c - r + 5 against a reference max r that
// starts at the first block's max of s c and moves to a later block's max
// only when that exceeds r by more than 3 (so t <= 8: P never saturates, and
// O is rescaled only on such moves).  FP8 linear-log rule (default): the
// E4M3 code is RNE(8 t + 56) clamped to [0, 128] and l sums the codes'
// values; FP8 exp2 rule: P = e4m3(2^t) and l sums the unquantised 2^t.
// BF16: P = bf16(2^(t - m)) with m the running max, l unquantised.
// out = O ds_v / l.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <cstdint>
#include <mutex>
#include <type_traits>

#include "kernels.h"
#include "sm100_ptx.cuh"
#include "state.cuh"

namespace fp8attn {

namespace {

constexpr int kThreadsAttn = 320;
// Pairs of columns (of every 8) whose exp2 runs on the FMA pipe (polynomial)
// instead of the MUFU, BF16 kernel (the last two of each eight).
constexpr int kPolyPairsPer8 = 2;
// FP8 kernel: every kPolyEvery-th column pair takes the polynomial (the same
// 25 %, spread evenly through the loop: measured 1 % faster there).
constexpr int kPolyEvery = 4;
// FP8 P rule: the reference max moves only past this lag (log2 units), and
// P = e4m3(2^(t - r + kPOffsetLog2)) stays at or below 2^(kRefLag + kPOffsetLog2) = 256.
constexpr float kRefLag = 3.0f;
constexpr float kPOffsetLog2 = 5.0f;
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;
constexpr float kLog2e = 1.4426950408889634f;

struct Bf16Cfg {
  static constexpr int kStages = 2;
  static constexpr int kTile = 32768;   // bytes of a 128x128 bf16 tile (two 64-column halves)
  static constexpr int kPCols = 64;     // TMEM columns of a bf16 P tile
  static constexpr int kKSteps = 8;     // MMAs per 128-deep product
  static constexpr int kSmemTiles = 2 + 2 * kStages;
  static constexpr int kSmemBytes = kSmemTiles * kTile + 1024 /*barriers*/ + 1024 /*align*/;
};

struct AttnParams {
  const int32_t* cu;
  int B, H, max_seqlen, n_qblk;   // n_qblk = query blocks of 256 rows per sequence
  int unit0;   // FP8: the launch's first work unit (256 query rows of one head)
  int64_t T;
  const float* descale;
  float softmax_scale;
  __nv_bfloat16* out;
  int32_t* err;
};

// The FP8 kernel with the static cast inside (kFused) also takes the bf16
// sources and their strides (elements), the cast scales and the layer's
// current scales.
struct AttnParamsFused : AttnParams {
  const uint16_t* qsrc;
  const uint16_t* ksrc;
  const uint16_t* vsrc;
  int64_t tok_stride, head_stride;
  const float* qscale;
  float* cur_qs;
  float* cur_ds;
};

template <int kFused>
using Fp8Params = typename std::conditional<kFused != 0, AttnParamsFused, AttnParams>::type;

struct Barriers {
  uint64_t q_full;
  uint64_t k_full[Bf16Cfg::kStages];
  uint64_t v_full[Bf16Cfg::kStages];
  uint64_t kv_empty[Bf16Cfg::kStages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_done[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <typename Bars>
__device__ __forceinline__ void note_error(AttnParams& p, Bars& bars, uint32_t bit) {
  bars.abort_flag = 1;
  if (p.err) atomicOr(reinterpret_cast<unsigned int*>(p.err), bit);
}

// Keys past the end of a sequence share the last K/V tile with the next
// sequence's first rows (or TMA zero fill past the tensor).  Their scores are
// masked to -inf, so P is 0 there, but 0 * NaN (or Inf) in the PV product is
// NaN: the rows of V at or after `valid` are zeroed in shared memory before
// the PV MMA reads them.  A row is 128 bytes of every 128B-swizzled tile (the
// swizzle permutes 16-byte chunks within a row), so the rows form one
// contiguous range.  Called by all 32 lanes of the MMA warp.
__device__ __forceinline__ void zero_tail_rows(uint8_t* tile, int valid, int lane) {
  uint4* p = reinterpret_cast<uint4*>(tile + valid * 128);
  const int n = (128 - valid) * 8;
  for (int i = lane; i < n; i += 32) p[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async();   // generic-proxy stores -> tensor-core operand reads
  __syncwarp();
}

__global__ void __launch_bounds__(kThreadsAttn, 1)
attn_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, AttnParams p) {
  using C = Bf16Cfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sq = smem;                                   // 2 tiles
  uint8_t* sk = smem + 2 * C::kTile;                    // kStages tiles
  uint8_t* sv = smem + (2 + C::kStages) * C::kTile;     // kStages tiles
  Barriers& bars = *reinterpret_cast<Barriers*>(smem + C::kSmemTiles * C::kTile);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item: (sequence b, head h, query block qb of 256 rows) ----
  const int qb = blockIdx.x % p.n_qblk;
  const int bh = blockIdx.x / p.n_qblk;
  const int h = bh % p.H;
  const int b = bh / p.H;
  const int seq0 = __ldg(p.cu + b);
  const int seq1 = __ldg(p.cu + b + 1);
  const int len = seq1 - seq0;
  if (seq0 < 0 || len < 0 || len > p.max_seqlen || static_cast<int64_t>(seq1) > p.T) {
    if (threadIdx.x == 0 && qb == 0 && p.err)
      atomicOr(reinterpret_cast<unsigned int*>(p.err), kErrSeqlens);
    return;
  }
  const int q0 = qb * 256;
  if (q0 >= len) return;
  const int nkv = (len + 127) / 128;

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bars.k_full[s], 1);
      mbar_init(&bars.v_full[s], 1);
      mbar_init(&bars.kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.p_full[i], 128);
      mbar_init(&bars.o_done[i], 1);
    }
    mbar_init(&bars.drain, 1);
    bars.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bars.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;
  const volatile int* abort_flag = &bars.abort_flag;

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ producer
    const bool leader = lane == 0;
    if (leader) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_expect_tx(&bars.q_full, 2 * C::kTile);
      for (int i = 0; i < 2; ++i) {   // two 64-column halves per tile
        tma_load_3d(sq + i * C::kTile, &tm_q, &bars.q_full, 0, h, seq0 + q0 + 128 * i);
        tma_load_3d(sq + i * C::kTile + 16384, &tm_q, &bars.q_full, 64, h, seq0 + q0 + 128 * i);
      }
    }
    int issued = 0;
    for (int j = 0; j < nkv; ++j) {
      const int st = j % C::kStages;
      if (j >= C::kStages) {
        if (!mbar_wait(&bars.kv_empty[st], ((j / C::kStages) - 1) & 1, abort_flag)) {
          if (leader) note_error(p, bars, kErrTimeout);
          break;
        }
      }
      if (leader) {
        const int tok = seq0 + 128 * j;
        mbar_expect_tx(&bars.k_full[st], C::kTile);
        tma_load_3d(sk + st * C::kTile, &tm_k, &bars.k_full[st], 0, h, tok);
        tma_load_3d(sk + st * C::kTile + 16384, &tm_k, &bars.k_full[st], 64, h, tok);
        mbar_expect_tx(&bars.v_full[st], C::kTile);
        tma_load_3d(sv + st * C::kTile, &tm_v, &bars.v_full[st], 0, h, tok);
        tma_load_3d(sv + st * C::kTile + 16384, &tm_v, &bars.v_full[st], 64, h, tok);
      }
      __syncwarp();
      issued = j + 1;
    }
    // make sure no copy is still landing when the CTA leaves
    for (int j = (issued > C::kStages ? issued - C::kStages : 0); j < issued; ++j) {
      const int st = j % C::kStages;
      mbar_wait(&bars.k_full[st], (j / C::kStages) & 1, nullptr);
      mbar_wait(&bars.v_full[st], (j / C::kStages) & 1, nullptr);
    }
    mbar_wait(&bars.q_full, 0, nullptr);
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    const bool leader = lane == 0;
    const uint32_t id_qk = make_idesc(1, 1, 128, 0);   // bf16 x bf16
    const uint32_t id_pv = make_idesc(1, 1, 128, 1);
    const uint32_t tS[2] = {tmem + 0, tmem + 128};
    const uint32_t tO[2] = {tmem + 256, tmem + 384};
    // Descriptors are built once; the 14-bit start-address field holds
    // (address >> 4), so moving to another tile, stage or K step is a plain
    // add of (byte offset >> 4) (shared addresses stay below 256 KB, so the
    // field never carries).  Built by every lane (warp-uniform values), one
    // elected lane issues.
    const uint64_t dq0 = make_sdesc_sw128(smem_u32(sq), 16, 1024);
    const uint64_t dk0 = make_sdesc_sw128(smem_u32(sk), 16, 1024);
    const uint64_t dv0 = make_sdesc_sw128(smem_u32(sv), 16384, 1024);
    constexpr uint32_t kTileStep = C::kTile >> 4;
    // Every lane builds the descriptors of a group (warp-uniform values, so
    // they can live in uniform registers); one elected lane then issues the
    // MMAs back to back with nothing else in between.
    auto issue_s = [&](int i, int st) {
      uint64_t ad[C::kKSteps], bd[C::kKSteps];
      const uint64_t dq = dq0 + static_cast<uint64_t>(i * kTileStep);
      const uint64_t dk = dk0 + static_cast<uint64_t>(st * kTileStep);
#pragma unroll
      for (int kk = 0; kk < C::kKSteps; ++kk) {
        // K-major 128B-swizzled operands: 32 bytes of K per MMA; bf16 tiles
        // hold two 64-column halves 16 KB apart
        const uint32_t koff = ((kk / 4) * 16384 + 32 * (kk % 4)) >> 4;
        ad[kk] = dq + koff;
        bd[kk] = dk + koff;
      }
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < C::kKSteps; ++kk) {
          mma_bf16_ss(tS[i], ad[kk], bd[kk], id_qk, kk > 0);
        }
        mma_commit(&bars.s_full[i]);
      }
      __syncwarp();
    };
    auto issue_pv = [&](int i, int st, int j) {
      uint64_t bd[C::kKSteps];
      const uint64_t dv = dv0 + static_cast<uint64_t>(st * kTileStep);
#pragma unroll
      for (int kk = 0; kk < C::kKSteps; ++kk) {
        // V is MN-major: K (keys) advances by 16 rows of 128 bytes; the
        // second 64-column half of the tile sits 16 KB on (LBO)
        bd[kk] = dv + ((2048 * kk) >> 4);
      }
      const uint32_t acc0 = j > 0 ? 1u : 0u;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < C::kKSteps; ++kk) {
          mma_bf16_ts(tO[i], tS[i] + 8 * kk, bd[kk], id_pv, kk > 0 ? 1u : acc0);
        }
      }
      __syncwarp();
    };
    bool ok = mbar_wait(&bars.q_full, 0, abort_flag) && mbar_wait(&bars.k_full[0], 0, abort_flag);
    if (ok) {
      tc_fence_after();
      issue_s(0, 0);
      issue_s(1, 0);
      for (int j = 0; j < nkv && ok; ++j) {
        const int st = j % C::kStages;
        const int st1 = (j + 1) % C::kStages;
        ok = mbar_wait(&bars.v_full[st], (j / C::kStages) & 1, abort_flag);
        if (ok && j + 1 == nkv && (len & 127)) {
          // both 64-column halves of the last, partial V tile
          zero_tail_rows(sv + st * C::kTile, len & 127, lane);
          zero_tail_rows(sv + st * C::kTile + 16384, len & 127, lane);
        }
        ok = ok && mbar_wait(&bars.p_full[0], j & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        issue_pv(0, st, j);
        if (j + 1 == nkv) {
          if (elect_one()) mma_commit(&bars.o_done[0]);
          __syncwarp();
        }
        if (j + 1 < nkv) {
          ok = mbar_wait(&bars.k_full[st1], ((j + 1) / C::kStages) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          issue_s(0, st1);
        }
        ok = mbar_wait(&bars.p_full[1], j & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        issue_pv(1, st, j);
        if (elect_one()) {
          mma_commit(&bars.kv_empty[st]);
          if (j + 1 == nkv) mma_commit(&bars.o_done[1]);
        }
        __syncwarp();
        if (j + 1 < nkv) issue_s(1, st1);
      }
    }
    if (!ok && leader) note_error(p, bars, kErrTimeout);
    // drain: every MMA this warp issued has completed before TMEM is freed
    if (elect_one()) mma_commit(&bars.drain);
    __syncwarp();
    mbar_wait(&bars.drain, 0, nullptr);
  } else {
    // ------------------------------------------------------------ softmax
    const int wg = warp >> 2;             // query tile 0 or 1
    const int wq = warp & 3;              // TMEM lane quadrant
    const int row = 32 * wq + lane;       // row within the query tile
    const uint32_t lane_off = static_cast<uint32_t>(32 * wq) << 16;
    const uint32_t tS = tmem + 128 * wg + lane_off;
    const uint32_t tO = tmem + 256 + 128 * wg + lane_off;
    const float cscale = p.softmax_scale * kLog2e;
    const float ds_v = 1.0f;
    const float p_off = 0.0f;   // bf16 P = 2^(t - m), no scale needed
    float m_run = -INFINITY;
    float l_run = 0.0f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      if (!mbar_wait(&bars.s_full[wg], j & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      uint32_t u[128];
      tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
      tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&u[64]));
      tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&u[96]));
      tmem_ld_wait();
      const int valid = len - 128 * j;
      if (valid < 128) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= valid) u[c] = 0xFF800000u;   // -inf: key beyond the sequence
      }
      // row max: four independent chains of 3-input max
      float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; c += 8) {
        mx0 = fmax3(mx0, __uint_as_float(u[c + 0]), __uint_as_float(u[c + 1]));
        mx1 = fmax3(mx1, __uint_as_float(u[c + 2]), __uint_as_float(u[c + 3]));
        mx2 = fmax3(mx2, __uint_as_float(u[c + 4]), __uint_as_float(u[c + 5]));
        mx3 = fmax3(mx3, __uint_as_float(u[c + 6]), __uint_as_float(u[c + 7]));
      }
      const float mx = fmax3(mx0, mx1, fmaxf(mx2, mx3));
      const float m_new = fmaxf(m_run, mx * cscale);
      const float neg = p_off - m_new;
      const uint64_t c2 = f2_pack(cscale, cscale);
      const uint64_t n2 = f2_pack(neg, neg);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
      uint32_t pw[C::kPCols];
#pragma unroll
      for (int k = 0; k < 64; ++k) {
        // exponent argument for columns 2k, 2k+1 in one packed FMA
        const uint64_t t = f2_fma(f2_pack(__uint_as_float(u[2 * k]), __uint_as_float(u[2 * k + 1])),
                                  c2, n2);
        float t0, t1;
        f2_unpack(t, t0, t1);
        uint64_t e;
        if ((k & 7) >= 8 - kPolyPairsPer8) {
          // kPolyPairsPer8 of every 8 pairs on the FMA pipe, the rest on the MUFU
          e = f2_exp2_poly(f2_pack(fmaxf(t0, -126.0f), fmaxf(t1, -126.0f)));
        } else {
          e = f2_pack(ex2_approx(t0), ex2_approx(t1));
        }
        acc[k & 3] = f2_add(acc[k & 3], e);
        float e0, e1;
        f2_unpack(e, e0, e1);
        pw[k] = cvt_bf16x2(e0, e1);
      }
      float sum;
      {
        float a0, a1, b0, b1;
        f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), a0, a1);
        (void)b0;
        (void)b1;
        sum = a0 + a1;
      }
      const float alpha = ex2_approx(m_run - m_new);   // 0 on the first tile
      l_run = l_run * alpha + sum;
      tmem_st32(tS + 0, *reinterpret_cast<const uint32_t(*)[32]>(&pw[0]));
      tmem_st32(tS + 32, *reinterpret_cast<const uint32_t(*)[32]>(&pw[32]));
      // O_i is stable here (PV_i(j-1) finished before S_i(j) was written)
      if (j > 0 && __any_sync(0xFFFFFFFFu, m_new > m_run)) {
        const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t o[64];
          tmem_ld32(tO + 64 * half, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
          tmem_ld32(tO + 64 * half + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
          tmem_ld_wait();
#pragma unroll
          for (int x = 0; x < 64; x += 2) {
            float o0, o1;
            f2_unpack(f2_mul(f2_pack(__uint_as_float(o[x]), __uint_as_float(o[x + 1])), a2), o0, o1);
            o[x] = __float_as_uint(o0);
            o[x + 1] = __float_as_uint(o1);
          }
          tmem_st32(tO + 64 * half, *reinterpret_cast<const uint32_t(*)[32]>(&o[0]));
          tmem_st32(tO + 64 * half + 32, *reinterpret_cast<const uint32_t(*)[32]>(&o[32]));
        }
      }
      m_run = m_new;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars.p_full[wg]);
    }
    if (!ok) {
      if (lane == 0) note_error(p, bars, kErrTimeout);
    } else if (mbar_wait(&bars.o_done[wg], 0, abort_flag)) {
      // ---- epilogue: out = O * ds_v / l, bf16, valid rows only
      tc_fence_after();
      const int qrow = q0 + 128 * wg + row;
      const bool store = qrow < len;
      const float inv = ds_v / l_run;
      __nv_bfloat16* dst =
          p.out + (static_cast<int64_t>(seq0 + qrow) * p.H + h) * kHeadDim;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * c, o);
        tmem_ld_wait();
        uint32_t w[16];
        const uint64_t inv2 = f2_pack(inv, inv);
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          float o0, o1;
          f2_unpack(f2_mul(f2_pack(__uint_as_float(o[2 * x]), __uint_as_float(o[2 * x + 1])), inv2),
                    o0, o1);
          w[x] = cvt_bf16x2(o0, o1);
        }
        if (store) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
          for (int x = 0; x < 4; ++x) d4[x] = make_uint4(w[4 * x], w[4 * x + 1], w[4 * x + 2], w[4 * x + 3]);
        }
      }
    } else if (lane == 0) {
      note_error(p, bars, kErrTimeout);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}


// ---------------------------------------------------------------------------
// FP8 path with P in shared memory.
//
// The softmax of query tile i hands its S columns back to the MMA warp as
// soon as it has loaded block j into registers (s_free), so S_i(j+1) is
// computed while the softmax is still working on block j: the softmax of
// consecutive key blocks runs back to back instead of waiting for its own
// PV and S round trip.  P_i(j) goes to a swizzled shared-memory buffer
// (double-buffered per tile) that the PV MMA reads as its K-major A operand.
// Ordering facts used below (MMAs of one thread complete in issue order):
//   - S_i(j+1) is issued after PV_i(j-1), so when the softmax sees S_i(j+1)
//     complete, PV_i(j-1) (and the P buffer it read) is done;
//   - the O rescale of block j needs PV_i(j-1): it waits on the P buffer's
//     barrier, which is at most one phase behind.
// ---------------------------------------------------------------------------

struct Fp8Cfg {
  static constexpr int kStages = 3;
  static constexpr int kTile = 16384;   // 128 x 128 bytes
  static constexpr int kSmemBytes = (2 + 2 * kStages + 4) * kTile + 1024 + 1024;
  // static cast inside the kernel: four tiles each for K and V, holding
  // either a whole short sequence's E4M3 K and V (up to 512 keys), or two
  // E4M3 stages plus one bf16 staging tile of 32 KB
  static constexpr int kTilesFused = 4;
  static constexpr int kSmemBytesFused = (2 + 2 * kTilesFused + 4) * kTile + 1024 + 1024;
};

// FP8 kernel warps: 0-7 softmax, 8 TMA producer, 9 and 10 MMA issuers for
// query tiles 0 and 1 (each on its own SM sub-partition, so the two issue
// streams and their barrier waits overlap instead of queueing behind each
// other; each tile's MMAs still complete in issue order).
constexpr int kThreadsFp8 = 352;
// With the static cast inside the kernel, warp 11 joins the TMA warp in
// casting the bf16 K and V tiles (each warp 64 rows of every tile).
constexpr int kThreadsFp8Fused = 384;
constexpr int kCastWarp = 11;

template <int kTiles>   // K (and V) tiles held in shared memory
struct Fp8Barriers {
  uint64_t q_full;
  uint64_t k_full[kTiles];
  uint64_t v_full[kTiles];
  uint64_t k_empty[kTiles];   // the S products that read the K stage are done
  uint64_t v_empty[kTiles];   // the PV products that read the V stage are done
  uint64_t s_full[2];       // S_i of the current block computed
  uint64_t s_free[2];       // S_i loaded by the softmax (TMEM columns free)
  uint64_t p_full[2][2];    // [tile][P buffer] P_i written
  uint64_t pv_done[2][2];   // [tile][P buffer] PV_i that read that buffer done
  uint64_t v_tail;          // the last, partial V tile's rows past the sequence are zeroed
  uint64_t drain[2];
  uint64_t stg_full[2];     // [K, V] bf16 staging tile landed (static cast inside)
  uint64_t stg_empty[2];    // [K, V] both cast warps have read the staging tile
  uint32_t tmem_base;
  int abort_flag;
};

// 16 bf16 (two 16-byte vectors, channels in order) -> 16 E4M3 codes of
// fl32(x * qs), round to nearest even, saturating: the static cast of the
// quantisation kernel.
__device__ __forceinline__ uint4 cast16_e4m3(uint4 a, uint4 b, float qs) {
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  const uint64_t qs2 = f2_pack(qs, qs);
  uint32_t h[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float lo, hi;
    f2_unpack(f2_mul(f2_pack(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u)),
                     qs2),
              lo, hi);
    h[i] = cvt_e4m3x2(lo, hi);
  }
  return make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16),
                    h[6] | (h[7] << 16));
}

// Cast rows [64 w, 64 w + 64) of a bf16 K or V tile staged by TMA (two
// 128B-swizzled boxes of 64 channels) into the E4M3 tile the MMA reads
// (128B-swizzled, 128 channels a row).  Lane l takes rows l and l + 32 of the
// half, 16 channels at a time, so that each group of 8 lanes touches 8 rows
// of one chunk (no bank conflicts on either side).
__device__ __forceinline__ void cast_tile_half(const uint8_t* stg, uint8_t* dst, int w, int lane,
                                               float qs) {
#pragma unroll 4
  for (int n = 0; n < 16; ++n) {
    const int row = 64 * w + lane + 32 * (n & 1);
    const int cp = n >> 1;                 // 16 channels: 16 * cp ..
    const int c = 2 * (cp & 3);            // first 16-byte chunk in the bf16 box
    const uint8_t* src = stg + (cp >> 2) * 16384 + row * 128;
    const uint4 a = *reinterpret_cast<const uint4*>(src + ((c ^ (row & 7)) << 4));
    const uint4 b = *reinterpret_cast<const uint4*>(src + (((c + 1) ^ (row & 7)) << 4));
    *reinterpret_cast<uint4*>(dst + row * 128 + ((cp ^ (row & 7)) << 4)) = cast16_e4m3(a, b, qs);
  }
}

// One row's 128 consecutive TMEM columns in one load (the S block the
// softmax reads; one instruction instead of four 32-column loads).
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t (&r)[128]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x128.b32 {"
      "%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
      "%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, "
      "%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63, "
      "%64, %65, %66, %67, %68, %69, %70, %71, %72, %73, %74, %75, %76, %77, %78, %79, "
      "%80, %81, %82, %83, %84, %85, %86, %87, %88, %89, %90, %91, %92, %93, %94, %95, "
      "%96, %97, %98, %99, %100, %101, %102, %103, %104, %105, %106, %107, %108, %109, %110, %111, "
      "%112, %113, %114, %115, %116, %117, %118, %119, %120, %121, %122, %123, %124, %125, %126, %127"
      "}, [%128];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]),
        "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]),
        "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]),
        "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]),
        "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]),
        "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]),
        "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]),
        "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]),
        "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
      : "r"(taddr));
}

// kSplit = 0: each CTA runs one work unit as two interleaved 128-row tiles.
// kSplit = 1: each unit runs as two CTAs of one tile each.  The two are
// separate instantiations so that each compiles with its tile count fixed.
// kFused = 1: Q, K and V arrive as bf16 and are cast with the static scales
// inside the kernel (Q by all warps before the roles start, K and V tile by
// tile by the TMA warp and warp 11 between the TMA loads and the MMAs), so
// no E4M3 copy of the inputs goes through HBM.
template <int kRule, int kSplit, int kFused>
__global__ void __launch_bounds__(kFused ? kThreadsFp8Fused : kThreadsFp8, 1)
attn_fwd_fp8_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, Fp8Params<kFused> p) {
  using C = Fp8Cfg;
  constexpr int kSt = kFused ? C::kTilesFused : C::kStages;   // K (and V) tiles in smem
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sq = smem;                                   // 2 Q tiles
  uint8_t* sk = smem + 2 * C::kTile;                    // kStages K tiles
  uint8_t* sv = sk + kSt * C::kTile;             // kStages V tiles
  uint8_t* sp = sv + kSt * C::kTile;             // P [tile][buffer]
  Fp8Barriers<kSt>& bars = *reinterpret_cast<Fp8Barriers<kSt>*>(sp + 4 * C::kTile);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // a launch of single-tile CTAs may follow this grid on the stream: let it
  // start as soon as SMs free up (it reads nothing this grid writes)
  if (kSplit == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // work unit = (query block of 256 rows, head, sequence)
  const int cta = static_cast<int>(blockIdx.x);
  if constexpr (kFused != 0) {
    if (p.unit0 == 0 && cta == 0 && threadIdx.x < 3) {
      // the cast scales become the layer's current scales (as after a cast
      // launch); one CTA of the call writes them, whatever its unit holds
      p.cur_qs[threadIdx.x] = __ldg(p.qscale + threadIdx.x);
      p.cur_ds[threadIdx.x] = __ldg(p.descale + threadIdx.x);
    }
  }
  constexpr int ntiles = kSplit ? 1 : 2;
  const int unit = p.unit0 + (kSplit ? (cta >> 1) : cta);
  const int sub = kSplit ? (cta & 1) : 0;
  const int qb = unit % p.n_qblk;
  const int bh = unit / p.n_qblk;
  const int h = bh % p.H;
  const int b = bh / p.H;
  const int seq0 = __ldg(p.cu + b);
  const int seq1 = __ldg(p.cu + b + 1);
  const int len = seq1 - seq0;
  if (seq0 < 0 || len < 0 || len > p.max_seqlen || static_cast<int64_t>(seq1) > p.T) {
    if (threadIdx.x == 0 && qb == 0 && sub == 0 && p.err)
      atomicOr(reinterpret_cast<unsigned int*>(p.err), kErrSeqlens);
    if (kSplit) asm volatile("griddepcontrol.wait;" ::: "memory");
    return;
  }
  const int q0 = qb * 256 + 128 * sub;   // first query row of this CTA's tile 0
  if (q0 >= len) {
    if (kSplit) asm volatile("griddepcontrol.wait;" ::: "memory");
    return;
  }
  const int nkv = (len + 127) / 128;
  // kFused: a sequence of up to kTilesFused key blocks is cast whole into
  // shared memory by all warps up front; longer ones stream through two
  // E4M3 stages, tiles 2-3 of each buffer staging the bf16 tile
  const bool resident = kFused && nkv <= C::kTilesFused;
  const int nst = kFused ? (resident ? C::kTilesFused : 2) : C::kStages;

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < kSt; ++s) {
      // kFused: filled by the two cast warps (one elected arrive each)
      mbar_init(&bars.k_full[s], kFused ? 2 : 1);
      mbar_init(&bars.v_full[s], kFused ? 2 : 1);
      mbar_init(&bars.k_empty[s], ntiles);   // one commit per active MMA warp
      mbar_init(&bars.v_empty[s], ntiles);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.s_free[i], 128);
      for (int q = 0; q < 2; ++q) {
        mbar_init(&bars.p_full[i][q], 128);
        mbar_init(&bars.pv_done[i][q], 1);
      }
    }
    mbar_init(&bars.v_tail, 1);
    mbar_init(&bars.drain[0], 1);
    mbar_init(&bars.drain[1], 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars.stg_full[t], 1);
      mbar_init(&bars.stg_empty[t], 2);
    }
    bars.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bars.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;
  const volatile int* abort_flag = &bars.abort_flag;

  if constexpr (kFused != 0) {
    if (!resident && warp == kTmaWarp && lane == 0) {
      // the first K and V tiles start landing (as bf16, in tiles 2-3 of the
      // K and V buffers) while Q is cast
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      for (int t = 0; t < 2; ++t) {
        const CUtensorMap* m = t ? &tm_v : &tm_k;
        uint8_t* stg = (t ? sv : sk) + 2 * C::kTile;
        mbar_expect_tx(&bars.stg_full[t], 2 * C::kTile);
        tma_load_3d(stg, m, &bars.stg_full[t], 0, h, seq0);
        tma_load_3d(stg + C::kTile, m, &bars.stg_full[t], 64, h, seq0);
      }
    }
    // Q (and, for a resident sequence, K and V): every thread casts 32-byte
    // pieces (16 channels of a row) straight from global memory, loading
    // kBatch pieces before casting any (the loads' latency overlaps); rows
    // past the sequence become zeros.  Item order: Q rows, then K, V tiles.
    constexpr int kBatch = 8;
    const int nq = ntiles * 128 * 8;
    const int nitems = nq + (resident ? nkv * 2 * 1024 : 0);
    const int tid = static_cast<int>(threadIdx.x);
    for (int it0 = tid; it0 < nitems; it0 += kBatch * kThreadsFp8Fused) {
      uint4 xa[kBatch], xb[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int it = it0 + u * kThreadsFp8Fused;
        xa[u] = xb[u] = make_uint4(0u, 0u, 0u, 0u);
        int row, t;
        if (it < nq) {
          row = q0 + (it >> 3);
          t = 0;
        } else {
          const int x = it - nq;
          row = 128 * (x >> 11) + ((x >> 3) & 127);
          t = 1 + ((x >> 10) & 1);
        }
        if (it < nitems && row < len) {
          const uint16_t* base = t == 0 ? p.qsrc : t == 1 ? p.ksrc : p.vsrc;
          const uint4* src = reinterpret_cast<const uint4*>(
              base + static_cast<int64_t>(seq0 + row) * p.tok_stride +
              static_cast<int64_t>(h) * p.head_stride + 16 * (it & 7));
          xa[u] = __ldg(src);
          xb[u] = __ldg(src + 1);
        }
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int it = it0 + u * kThreadsFp8Fused;
        if (it >= nitems) break;
        const int cp = it & 7;
        int r, row, t;
        uint8_t* dst;
        if (it < nq) {
          r = it >> 3;
          row = q0 + r;
          t = 0;
          dst = sq + (r >> 7) * C::kTile;
        } else {
          const int x = it - nq;
          const int tj = x >> 10;    // 2 j + (0 K, 1 V)
          r = (x >> 3) & 127;
          row = 128 * (tj >> 1) + r;
          t = 1 + (tj & 1);
          dst = (t == 1 ? sk : sv) + (tj >> 1) * C::kTile;
        }
        const int rr = r & 127;
        const uint4 codes = row < len ? cast16_e4m3(xa[u], xb[u], __ldg(p.qscale + t))
                                      : make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(dst + rr * 128 + ((cp ^ (rr & 7)) << 4)) = codes;
      }
    }
    fence_proxy_async();
    __syncthreads();
    if (resident && threadIdx.x == 0) {
      // every K and V tile is in place (two arrivals: the full barriers
      // count the two cast warps of the streaming form)
      for (int j = 0; j < nkv; ++j)
        for (int a = 0; a < 2; ++a) {
          mbar_arrive(&bars.k_full[j]);
          mbar_arrive(&bars.v_full[j]);
        }
    }
  }

  // ------------------------------------------------------------ K/V cast
  // Tile order K_0, V_0, K_1, V_1, ...: staging buffer 0 holds K, 1 holds
  // V.  Both warps cast their 64 rows of a staged tile into the free E4M3
  // stage, then arrive on its full barrier and on the staging buffer's
  // empty barrier; the TMA warp's lane 0 then loads the next tile of that
  // kind into the staging buffer.
  bool cast_role = false;
  if constexpr (kFused != 0) {
    cast_role = warp == kTmaWarp || warp == kCastWarp;
    if (cast_role && !resident) {
      const int w = warp == kTmaWarp ? 0 : 1;
      const bool issuer = warp == kTmaWarp;
      const float qsk = __ldg(p.qscale + 1), qsv = __ldg(p.qscale + 2);
      int issued[2] = {1, 1};   // tiles loaded into each staging buffer
      bool ok = true;
      for (int j = 0; j < nkv && ok; ++j) {
        const int st = j % nst;
        for (int t = 0; t < 2; ++t) {
          uint8_t* buf = t ? sv : sk;
          ok = mbar_wait(&bars.stg_full[t], j & 1, abort_flag);
          if (ok && j >= nst)
            ok = mbar_wait(t ? &bars.v_empty[st] : &bars.k_empty[st], ((j / nst) - 1) & 1, abort_flag);
          if (!ok) break;
          cast_tile_half(buf + 2 * C::kTile, buf + st * C::kTile, w, lane, t ? qsv : qsk);
          fence_proxy_async();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(t ? &bars.v_full[st] : &bars.k_full[st]);
            mbar_arrive(&bars.stg_empty[t]);
          }
          if (issuer && j + 1 < nkv) {
            // both warps are done reading: the next tile of this kind may land
            ok = mbar_wait(&bars.stg_empty[t], j & 1, abort_flag);
            if (!ok) break;
            if (lane == 0) {
              const CUtensorMap* m = t ? &tm_v : &tm_k;
              mbar_expect_tx(&bars.stg_full[t], 2 * C::kTile);
              tma_load_3d(buf + 2 * C::kTile, m, &bars.stg_full[t], 0, h, seq0 + 128 * (j + 1));
              tma_load_3d(buf + 3 * C::kTile, m, &bars.stg_full[t], 64, h, seq0 + 128 * (j + 1));
            }
            ++issued[t];
            __syncwarp();
          }
        }
      }
      if (!ok && lane == 0) note_error(p, bars, kErrTimeout);
      if (issuer) {
        // no copy may still be landing when the CTA leaves: wait for the last
        // tile loaded into each staging buffer (completed phases pass at once)
        for (int t = 0; t < 2; ++t)
          mbar_wait(&bars.stg_full[t], (issued[t] - 1) & 1, nullptr);
      }
    }
  }
  if (cast_role) {
    // the K/V cast above (static cast inside the kernel, streaming form)
  } else if (warp == kTmaWarp) {
    // ------------------------------------------------------------ producer
    const bool leader = lane == 0;
    if (leader) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_expect_tx(&bars.q_full, ntiles * C::kTile);
      for (int i = 0; i < ntiles; ++i)
        tma_load_3d(sq + i * C::kTile, &tm_q, &bars.q_full, 0, h, seq0 + q0 + 128 * i);
    }
    // K and V stages are released separately: a K stage as soon as the two
    // S products that read it are done, a V stage after its PV products.  K
    // therefore streams up to kStages blocks ahead of the S products while V
    // follows the (later) PV products; the producer polls both without
    // blocking, keeping V no further ahead than K.
    int jk = 0, jv = 0;
    uint64_t t_last = global_timer_ns();
    uint32_t polls = 0;
    bool ok = true;
    while (jv < nkv) {
      bool progressed = false;
      if (jk < nkv) {
        const int st = jk % kSt;
        if (jk < kSt || mbar_test_now(&bars.k_empty[st], ((jk / kSt) - 1) & 1)) {
          if (leader) {
            mbar_expect_tx(&bars.k_full[st], C::kTile);
            tma_load_3d(sk + st * C::kTile, &tm_k, &bars.k_full[st], 0, h, seq0 + 128 * jk);
          }
          ++jk;
          progressed = true;
        }
      }
      if (jv < jk) {
        const int st = jv % kSt;
        if (jv < kSt || mbar_test_now(&bars.v_empty[st], ((jv / kSt) - 1) & 1)) {
          if (leader) {
            mbar_expect_tx(&bars.v_full[st], C::kTile);
            tma_load_3d(sv + st * C::kTile, &tm_v, &bars.v_full[st], 0, h, seq0 + 128 * jv);
          }
          ++jv;
          progressed = true;
        }
      }
      __syncwarp();
      if (progressed) {
        polls = 0;
        t_last = 0;
      } else if ((++polls & 63u) == 0) {
        // bounded like every other wait: give up after kWaitLimitNs without progress
        const uint64_t now = global_timer_ns();
        if (t_last == 0) t_last = now;
        if (*abort_flag || now - t_last > kWaitLimitNs) { ok = false; break; }
      }
    }
    if (!ok && leader) note_error(p, bars, kErrTimeout);
    // make sure no copy is still landing when the CTA leaves
    for (int j = (jk > kSt ? jk - kSt : 0); j < jk; ++j)
      mbar_wait(&bars.k_full[j % kSt], (j / kSt) & 1, nullptr);
    for (int j = (jv > kSt ? jv - kSt : 0); j < jv; ++j)
      mbar_wait(&bars.v_full[j % kSt], (j / kSt) & 1, nullptr);
    mbar_wait(&bars.q_full, 0, nullptr);
  } else if ((warp == kMmaWarp || warp == kMmaWarp + 1) && warp - kMmaWarp < ntiles) {
    // ------------------------------------------------------------ MMA issuers
    const int i = warp - kMmaWarp;   // query tile of this warp
    const bool leader = lane == 0;
    const uint32_t id_qk = make_idesc(0, 0, 128, 0);
    const uint32_t id_pv = make_idesc(0, 0, 128, 1);
    const uint64_t dq = make_sdesc_sw128(smem_u32(sq), 16, 1024) + static_cast<uint64_t>(i * (C::kTile >> 4));
    const uint64_t dk0 = make_sdesc_sw128(smem_u32(sk), 16, 1024);
    const uint64_t dv0 = make_sdesc_sw128(smem_u32(sv), 16384, 1024);
    const uint64_t dp0 = make_sdesc_sw128(smem_u32(sp), 16, 1024);
    constexpr uint32_t nstep = C::kTile >> 4;
    const uint32_t tS = tmem + 128 * i, tO = tmem + 256 + 128 * i;
    auto issue_s = [&](int j) {
      uint64_t ad[4], bd[4];
      const uint64_t dk = dk0 + static_cast<uint64_t>((j % nst) * nstep);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        ad[kk] = dq + 2 * kk;   // 32 bytes of K per MMA
        bd[kk] = dk + 2 * kk;
      }
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) mma_f8_ss(tS, ad[kk], bd[kk], id_qk, kk > 0);
        mma_commit(&bars.s_full[i]);
        // the K stage is free once both tiles' S products of block j are done
        mma_commit(&bars.k_empty[j % nst]);
      }
      __syncwarp();
    };
    auto issue_pv = [&](int j) {
      uint64_t ad[4], bd[4];
      const uint64_t dp = dp0 + static_cast<uint64_t>((2 * i + (j & 1)) * nstep);
      const uint64_t dv = dv0 + static_cast<uint64_t>((j % nst) * nstep);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        ad[kk] = dp + 2 * kk;          // P is K-major: 32 keys per MMA
        bd[kk] = dv + 256 * kk;        // V is MN-major: 32 rows of 128 bytes per MMA
      }
      const uint32_t acc0 = j > 0 ? 1u : 0u;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) mma_f8_ss(tO, ad[kk], bd[kk], id_pv, kk > 0 ? 1u : acc0);
        mma_commit(&bars.pv_done[i][j & 1]);
        mma_commit(&bars.v_empty[j % nst]);
      }
      __syncwarp();
    };
    bool ok = (kFused || mbar_wait(&bars.q_full, 0, abort_flag)) &&
              mbar_wait(&bars.k_full[0], 0, abort_flag);
    if (ok) {
      tc_fence_after();
      issue_s(0);
    }
    for (int j = 0; j < nkv && ok; ++j) {
      const int st = j % nst;
      if (j + 1 < nkv) {
        const int st1 = (j + 1) % nst;
        // S_i's TMEM columns are free once the softmax has loaded block j
        ok = mbar_wait(&bars.k_full[st1], ((j + 1) / nst) & 1, abort_flag) &&
             mbar_wait(&bars.s_free[i], j & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        issue_s(j + 1);
      }
      ok = mbar_wait(&bars.v_full[st], (j / nst) & 1, abort_flag);
      if (ok && j + 1 == nkv && (len & 127)) {
        // tile 0's warp zeroes the rows past the sequence; tile 1's waits for it
        if (i == 0) {
          zero_tail_rows(sv + st * C::kTile, len & 127, lane);
          if (leader) mbar_arrive(&bars.v_tail);
        } else {
          ok = mbar_wait(&bars.v_tail, 0, abort_flag);
        }
      }
      ok = ok && mbar_wait(&bars.p_full[i][j & 1], (j >> 1) & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      issue_pv(j);
    }
    if (!ok && leader) note_error(p, bars, kErrTimeout);
    // drain: every MMA this warp issued has completed before TMEM is freed
    if (elect_one()) mma_commit(&bars.drain[i]);
    __syncwarp();
    mbar_wait(&bars.drain[i], 0, nullptr);
  } else if (warp < 4 * ntiles) {
    // ------------------------------------------------------------ softmax
    const int wg = warp >> 2;
    const int wq = warp & 3;
    const int row = 32 * wq + lane;
    const uint32_t lane_off = static_cast<uint32_t>(32 * wq) << 16;
    const uint32_t tS = tmem + 128 * wg + lane_off;
    const uint32_t tO = tmem + 256 + 128 * wg + lane_off;
    // this row's place in the 128B-swizzled K-major P tile
    uint8_t* prow0 = sp + (2 * wg) * C::kTile + (row >> 3) * 1024 + (row & 7) * 128;
    const float cscale = __ldg(p.descale + 0) * __ldg(p.descale + 1) * p.softmax_scale * kLog2e;
    const float ds_v = __ldg(p.descale + 2);
    float m_run = -INFINITY;
    float l_run = 0.0f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      if (!mbar_wait(&bars.s_full[wg], j & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      uint32_t u[128];
      if (kRule == kPRuleLinearLog) {
        tmem_ld128(tS, u);
      } else {   // (the exponential rule's register allocation is tuned on four loads)
        tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
        tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
        tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&u[64]));
        tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&u[96]));
      }
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bars.s_free[wg]);   // the MMA warp may compute S_i(j+1) now
      const int valid = len - 128 * j;
      if (valid < 128) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= valid) u[c] = 0xFF800000u;   // -inf: key beyond the sequence
      }
      float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; c += 8) {
        mx0 = fmax3(mx0, __uint_as_float(u[c + 0]), __uint_as_float(u[c + 1]));
        mx1 = fmax3(mx1, __uint_as_float(u[c + 2]), __uint_as_float(u[c + 3]));
        mx2 = fmax3(mx2, __uint_as_float(u[c + 4]), __uint_as_float(u[c + 5]));
        mx3 = fmax3(mx3, __uint_as_float(u[c + 6]), __uint_as_float(u[c + 7]));
      }
      const float mx = fmax3(mx0, mx1, fmaxf(mx2, mx3));
      // reference max: moves to this block's max only when that exceeds it
      // by more than kRefLag (always on the first block, m_run = -inf)
      const float m_blk = mx * cscale;
      const bool moved = m_blk > m_run + kRefLag;
      const float m_new = moved ? m_blk : m_run;
      uint32_t pw[32];
      float sum;
      if (kRule == kPRuleExp2) {
        const float neg = kPOffsetLog2 - m_new;
        const uint64_t c2 = f2_pack(cscale, cscale);
        const uint64_t n2 = f2_pack(neg, neg);
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int k = 0; k < 64; ++k) {
          const uint64_t t = f2_fma(f2_pack(__uint_as_float(u[2 * k]), __uint_as_float(u[2 * k + 1])),
                                    c2, n2);
          float t0, t1;
          f2_unpack(t, t0, t1);
          uint64_t e;
          if (k % kPolyEvery == kPolyEvery - 1)
            e = f2_exp2_poly(f2_pack(fmaxf(t0, -126.0f), fmaxf(t1, -126.0f)));
          else
            e = f2_pack(ex2_approx(t0), ex2_approx(t1));
          acc[k & 3] = f2_add(acc[k & 3], e);
          float e0, e1;
          f2_unpack(e, e0, e1);
          const uint32_t hh = cvt_e4m3x2(e0, e1);
          if (k & 1) pw[k >> 1] |= hh << 16;
          else pw[k >> 1] = hh;
        }
        float a0, a1;
        f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), a0, a1);
        sum = a0 + a1;
      } else {
        // Linear-log rule: code = RNE(8 t + 56) clamped to [0, 128], with
        // t = s c - m + 5, i.e. the E4M3 bit pattern read as a fixed-point
        // log2 (exponent and mantissa filled linearly from t).  Computed as
        // y = sat(s c/16 + (0.75 - m/16)) = (8 t + 56) / 128 in [0, 1] (one
        // rounding; NaN and -inf scores give 0), then y + 1.5 * 2^16 rounds
        // 128 y to an integer in the low mantissa bits.  l sums the E4M3
        // values of the codes (pairs summed exactly in f16 first where
        // representable, then in fp32).
        const float a16 = cscale * 0.0625f;
        const float b16 = 0.75f - m_new * 0.0625f;
        const uint64_t magic2 = f2_pack(98304.0f, 98304.0f);   // 1.5 * 2^16
        float lacc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        uint32_t hprev = 0;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const float y0 = fma_sat(__uint_as_float(u[4 * k + 0]), a16, b16);
          const float y1 = fma_sat(__uint_as_float(u[4 * k + 1]), a16, b16);
          const float y2 = fma_sat(__uint_as_float(u[4 * k + 2]), a16, b16);
          const float y3 = fma_sat(__uint_as_float(u[4 * k + 3]), a16, b16);
          uint32_t ra, rb, rc, rd;
          asm("mov.b64 {%0, %1}, %2;" : "=r"(ra), "=r"(rb) : "l"(f2_add(f2_pack(y0, y1), magic2)));
          asm("mov.b64 {%0, %1}, %2;" : "=r"(rc), "=r"(rd) : "l"(f2_add(f2_pack(y2, y3), magic2)));
          const uint32_t c01 = prmt(ra, rb, 0x0040u);   // code0 | code1 << 8
          const uint32_t c23 = prmt(rc, rd, 0x0040u);
          pw[k] = prmt(c01, c23, 0x5410u);
          const uint32_t h = hadd2(cvt_f16x2_from_e4m3x2(c01), cvt_f16x2_from_e4m3x2(c23));
          if (k & 1) lacc[(k >> 1) & 3] = add_f16x2_to_f32(lacc[(k >> 1) & 3], hadd2(hprev, h));
          else hprev = h;
        }
        sum = (lacc[0] + lacc[1]) + (lacc[2] + lacc[3]);
      }
      // P row -> shared memory (buffer j % 2 is free: S_i(j) complete means
      // PV_i(j-2), its last reader, is done)
      uint8_t* prow = prow0 + (j & 1) * C::kTile;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(prow + ((c ^ (row & 7)) << 4)) =
            make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
      fence_proxy_async();
      const float alpha = ex2_approx(m_run - m_new);   // 0 on the first block, 1 unless moved
      l_run = l_run * alpha + sum;
      if (j > 0 && __any_sync(0xFFFFFFFFu, moved)) {
        // O_i holds PV up to block j-1: wait for it before rescaling
        if (!mbar_wait(&bars.pv_done[wg][(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t o[64];
          tmem_ld32(tO + 64 * half, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
          tmem_ld32(tO + 64 * half + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
          tmem_ld_wait();
#pragma unroll
          for (int x = 0; x < 64; x += 2) {
            float o0, o1;
            f2_unpack(f2_mul(f2_pack(__uint_as_float(o[x]), __uint_as_float(o[x + 1])), a2), o0, o1);
            o[x] = __float_as_uint(o0);
            o[x + 1] = __float_as_uint(o1);
          }
          tmem_st32(tO + 64 * half, *reinterpret_cast<const uint32_t(*)[32]>(&o[0]));
          tmem_st32(tO + 64 * half + 32, *reinterpret_cast<const uint32_t(*)[32]>(&o[32]));
        }
        tmem_st_wait();
      }
      m_run = m_new;
      tc_fence_before();
      mbar_arrive(&bars.p_full[wg][j & 1]);
    }
    if (!ok) {
      if (lane == 0) note_error(p, bars, kErrTimeout);
    } else if (mbar_wait(&bars.pv_done[wg][(nkv - 1) & 1], ((nkv - 1) >> 1) & 1, abort_flag)) {
      tc_fence_after();
      const int qrow = q0 + 128 * wg + row;
      const bool store = qrow < len;
      const float inv = ds_v / l_run;
      __nv_bfloat16* dst = p.out + (static_cast<int64_t>(seq0 + qrow) * p.H + h) * kHeadDim;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * c, o);
        tmem_ld_wait();
        uint32_t w[16];
        const uint64_t inv2 = f2_pack(inv, inv);
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          float o0, o1;
          f2_unpack(f2_mul(f2_pack(__uint_as_float(o[2 * x]), __uint_as_float(o[2 * x + 1])), inv2),
                    o0, o1);
          w[x] = cvt_bf16x2(o0, o1);
        }
        if (store) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
          for (int x = 0; x < 4; ++x) d4[x] = make_uint4(w[4 * x], w[4 * x + 1], w[4 * x + 2], w[4 * x + 3]);
        }
      }
    } else if (lane == 0) {
      note_error(p, bars, kErrTimeout);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
  // a single-tile grid launched behind a grid of whole units finishes only
  // after that grid (later work on the stream then follows both)
  if (kSplit) asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Self-test of the score product: S = Q K^T for 128 x 128 tiles of E4M3
// codes, computed with the attention kernel's operand layout, descriptors
// and MMA sequence (4 x K=32), written out in fp32 so that the tensor cores'
// accumulation error can be checked against exact scores.
// ---------------------------------------------------------------------------

struct ProbeSmem {
  uint8_t q[128 * 128];
  uint8_t k[128 * 128];
  uint64_t tma_bar, mma_bar;
  uint32_t tmem_base;
};

__global__ void __launch_bounds__(128, 1)
qk_scores_probe_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k, float* scores, int32_t* err) {
  extern __shared__ uint8_t smem_raw[];
  ProbeSmem& sm = *reinterpret_cast<ProbeSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(&sm.tma_bar, 1);
    mbar_init(&sm.mma_bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (threadIdx.x == 0) {
    mbar_expect_tx(&sm.tma_bar, 2 * 16384);
    tma_load_3d(sm.q, &tm_q, &sm.tma_bar, 0, 0, 128 * blockIdx.x);
    tma_load_3d(sm.k, &tm_k, &sm.tma_bar, 0, 0, 128 * blockIdx.x);
  }
  bool ok = mbar_wait(&sm.tma_bar, 0, nullptr);
  if (warp == 0 && ok) {
    tc_fence_after();
    const uint32_t id_qk = make_idesc(0, 0, 128, 0);
    const uint64_t dq = make_sdesc_sw128(smem_u32(sm.q), 16, 1024);
    const uint64_t dk = make_sdesc_sw128(smem_u32(sm.k), 16, 1024);
    if (elect_one()) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) mma_f8_ss(tmem, dq + 2 * kk, dk + 2 * kk, id_qk, kk > 0);
      mma_commit(&sm.mma_bar);
    }
    __syncwarp();
  }
  ok = ok && mbar_wait(&sm.mma_bar, 0, nullptr);
  if (!ok && threadIdx.x == 0 && err) atomicOr(reinterpret_cast<unsigned int*>(err), kErrTimeout);
  if (ok) {
    tc_fence_after();
    const uint32_t lane_off = static_cast<uint32_t>(32 * warp) << 16;
    float* row = scores + (static_cast<int64_t>(blockIdx.x) * 128 + threadIdx.x) * 128;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t r[32];
      tmem_ld32(tmem + lane_off + 32 * c, r);
      tmem_ld_wait();
#pragma unroll
      for (int x = 0; x < 32; ++x) row[32 * c + x] = __uint_as_float(r[x]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Resolved once per process; the initialisation of a function-local static is
// thread-safe, so host threads may launch concurrently from the first call.
EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(f);
    return nullptr;
  }();
  return fn;
}

// [T, H, 128] tensor viewed as (channel, head, token); 128-token boxes of
// 128 bytes of channels, 128-byte swizzle.
bool make_qkv_map(CUtensorMap* m, const void* base, int64_t T, int H, bool bf16) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t esz = bf16 ? 2 : 1;
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(T)};
  cuuint64_t strides[2] = {128 * esz, static_cast<cuuint64_t>(H) * 128 * esz};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(bf16 ? 64 : 128), 1, 128};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
            const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 source [T rows][H heads][128] with row and head strides in elements
// (multiples of 8), 64-channel boxes of 128 rows, 128B swizzle.
bool make_bf16_src_map(CUtensorMap* m, const void* base, int64_t T, int H, int64_t tok_stride,
                       int64_t head_stride) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(T)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_stride) * 2,
                           static_cast<cuuint64_t>(tok_stride) * 2};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// How many of a launch's `units` (the last ones) run as two single-tile
// CTAs each.  Auto: the units of a last wave that would fill at most half
// of the SMs, so that their tiles fill that wave instead; when all units fit
// in that one wave, every unit.
int64_t split_units(int64_t units, int schedule, int dev) {
  if (schedule == kSchedWhole) return 0;
  if (schedule == kSchedSplit) return units;
  static std::mutex mu;
  static int n_sm[64] = {0};
  int sms;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (n_sm[dev] == 0 &&
        cudaDeviceGetAttribute(&n_sm[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      n_sm[dev] = 0;
      return 0;
    }
    sms = n_sm[dev];
  }
  const int64_t tail = units % sms;
  if (tail == 0 || 2 * tail > sms) return 0;
  return tail;
}

// Launches `n_units` work units from `unit0` on (kSplit: two single-tile CTAs
// per unit; `behind`: programmatic launch behind the previous kernel).
template <bool kFp8, int kRule, int kSplit, int kFused>
cudaError_t launch_attention_t(const AttnLaunch& a, int64_t T, cudaStream_t stream,
                               int64_t unit0, int64_t n_units, bool behind) {
  CUtensorMap mq, mk, mv;
  if (kFused) {
    // K and V through TMA as bf16; Q is read by the CTA's threads (map unused)
    if (!make_bf16_src_map(&mk, a.k, T, a.heads, a.tok_stride, a.head_stride) ||
        !make_bf16_src_map(&mv, a.v, T, a.heads, a.tok_stride, a.head_stride))
      return cudaErrorInvalidValue;
    mq = mk;
  } else if (!make_qkv_map(&mq, a.q, T, a.heads, !kFp8) ||
             !make_qkv_map(&mk, a.k, T, a.heads, !kFp8) ||
             !make_qkv_map(&mv, a.v, T, a.heads, !kFp8)) {
    return cudaErrorInvalidValue;
  }
  // FP8 runs the P-in-shared-memory kernel; BF16 keeps P in TMEM
  using Prm = typename std::conditional<kFp8, Fp8Params<kFused>, AttnParams>::type;
  void (*kernel)(CUtensorMap, CUtensorMap, CUtensorMap, Prm);
  if constexpr (kFp8)
    kernel = attn_fwd_fp8_kernel<kRule, kSplit, kFused>;
  else
    kernel = attn_fwd_bf16_kernel;
  const int smem_bytes =
      kFp8 ? (kFused ? Fp8Cfg::kSmemBytesFused : Fp8Cfg::kSmemBytes) : Bf16Cfg::kSmemBytes;
  // the shared-memory opt-in is a per-device function attribute: set it once
  // for each device this process launches on
  static std::mutex mu;
  static uint64_t attr_set = 0;   // bit d: done on device d (one per instantiation)
  int dev = 0;
  {
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!(attr_set >> dev & 1u)) {
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
      if (e != cudaSuccess) return e;
      attr_set |= uint64_t{1} << dev;
    }
  }
  AttnParams p;
  p.cu = a.cu;
  p.B = a.batch;
  p.H = a.heads;
  p.max_seqlen = a.max_seqlen;
  p.n_qblk = (a.max_seqlen + 255) / 256;
  p.T = T;
  p.descale = a.descale;
  p.softmax_scale = a.softmax_scale;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.err = a.err;
  p.unit0 = static_cast<int>(unit0);
  Prm prm;
  static_cast<AttnParams&>(prm) = p;
  if constexpr (kFp8 && kFused != 0) {
    prm.qsrc = static_cast<const uint16_t*>(a.q);
    prm.ksrc = static_cast<const uint16_t*>(a.k);
    prm.vsrc = static_cast<const uint16_t*>(a.v);
    prm.tok_stride = a.tok_stride;
    prm.head_stride = a.head_stride;
    prm.qscale = a.qscale;
    prm.cur_qs = a.cur_qs;
    prm.cur_ds = a.cur_ds;
  }
  const int64_t grid = kSplit ? 2 * n_units : n_units;
  const int threads = kFp8 ? (kFused ? kThreadsFp8Fused : kThreadsFp8) : kThreadsAttn;
  if (!behind) {
    kernel<<<static_cast<unsigned>(grid), threads, smem_bytes, stream>>>(mq, mk, mv, prm);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem_bytes);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, mq, mk, mv, prm);
}

}  // namespace

cudaError_t launch_qk_scores_probe(const void* q8, const void* k8, int64_t tiles, float* scores,
                                   int32_t* err, cudaStream_t stream) {
  CUtensorMap mq, mk;
  if (!make_qkv_map(&mq, q8, tiles * 128, 1, false) || !make_qkv_map(&mk, k8, tiles * 128, 1, false))
    return cudaErrorInvalidValue;
  const int smem_bytes = static_cast<int>(sizeof(ProbeSmem)) + 1024;
  cudaError_t e = cudaFuncSetAttribute(qk_scores_probe_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
  if (e != cudaSuccess) return e;
  qk_scores_probe_kernel<<<static_cast<unsigned>(tiles), 128, smem_bytes, stream>>>(mq, mk, scores,
                                                                                 err);
  return cudaGetLastError();
}

template <int kRule, int kFused>
cudaError_t launch_fp8(const AttnLaunch& a, int64_t T, cudaStream_t stream, int64_t units,
                       int64_t split) {
  // whole units first, then the split units' single-tile CTAs behind them
  const int64_t whole = units - split;
  if (whole > 0) {
    cudaError_t e = launch_attention_t<true, kRule, 0, kFused>(a, T, stream, 0, whole, false);
    if (e != cudaSuccess || split == 0) return e;
    note_launch();   // the caller counts one launch
  }
  return launch_attention_t<true, kRule, 1, kFused>(a, T, stream, whole, split, whole > 0);
}

cudaError_t launch_attention(const AttnLaunch& a, int64_t total_tokens, cudaStream_t stream) {
  const int64_t units = static_cast<int64_t>((a.max_seqlen + 255) / 256) * a.heads * a.batch;
  if (units <= 0) return cudaSuccess;
  if (units > 0x3FFFFFFF) return cudaErrorInvalidConfiguration;
  if (a.bf16)
    return launch_attention_t<false, kPRuleExp2, 0, 0>(a, total_tokens, stream, 0, units, false);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const int64_t split = split_units(units, a.schedule, dev);
  if (a.fused)
    return a.p_rule == kPRuleExp2
               ? launch_fp8<kPRuleExp2, 1>(a, total_tokens, stream, units, split)
               : launch_fp8<kPRuleLinearLog, 1>(a, total_tokens, stream, units, split);
  return a.p_rule == kPRuleExp2 ? launch_fp8<kPRuleExp2, 0>(a, total_tokens, stream, units, split)
                                : launch_fp8<kPRuleLinearLog, 0>(a, total_tokens, stream, units, split);
}


}  // namespace fp8attn
