/*
 * fp8attn CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously-correct restatement of what the FP8 attention
 * path computes, used by the tests, by the smoke check and by the benchmark's
 * CPU-baseline leg.  It shares no code, header, table or constant with the
 * CUDA library and must never be linked into, or called by, the product path.
 *
 * Sources (web pages on on-the-fly FP8 attention quantisation):
 *   [vLLM-ViT]  vLLM docs, "FP8 ViT encoder attention" -- usage section:
 *               a 16-entry circular buffer of observed Q/K/V amax values
 *               drives the per-forward scale; static per-layer {q,k,v}
 *               scale file; saved scales multiplied by a save margin
 *               (default 1.5); scale-file format section.
 *   [vLLM-Omni] vLLM-Omni docs, "Quantized KV Cache" -- overview (Q/K/V
 *               quantised dynamically before the FA operator) and the
 *               parameters table (skip selectors).
 *   [Ascend]    Ascend quantisation chapter -- names FP8 E4M3 / E5M2.
 * The pages leave the E4M3 bit layout, rounding, the scale formula, the ring
 * reduction and the P (softmax probability) rule open; the readings used here
 * are the plainest ones and are written beside each function:
 *   - E4M3 is the OCP 8-bit "FN" format (bias 7, no infinities, 0x7F/0xFF
 *     NaN, max 448); encoding rounds to nearest, ties to even, and saturates
 *     to +-448 (satfinite); NaN encodes as 0x7F.
 *   - amax is max |x| over the valid (unpadded) tokens; NaN is ignored.
 *   - the ring is reduced with max, the current pass is pushed first
 *     ("current-inclusive"), and the bound A gives qs = fl32(448/A),
 *     ds = fl32(A/448); A == 0 gives qs = ds = 1.
 *   - static values are bounds A in activation units (the margin is applied
 *     when they are saved, never again on load).
 *   - attention: P for the PV product is quantised block by block (128
 *     keys, in sequence order) as e4m3(32 exp(s - r))/32 against a reference
 *     max r that a single-pass (online-softmax) kernel keeps per row: r is
 *     the first block's max and moves to a later block's max only when that
 *     block's max exceeds r by more than 3 in log2 units (so 32 exp(s - r)
 *     stays at or below 2^8 = 256 and never saturates); each block's P is
 *     carried to the final max M exactly; the output is normalised by l =
 *     sum of the unquantised exp(s - M).
 *
 * Floating point: quantisation follows the kernel's stated fp32 rules (one
 * fp32 RN multiply, one fp32 RN division), attention is evaluated in fp64.
 * Build with -O2 -ffp-contract=off and no fast-math.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <pthread.h>
#include <unistd.h>

/* ------------------------------------------------------------------ */
/* bf16                                                                */
/* ------------------------------------------------------------------ */

static float bf16_to_f32(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* ------------------------------------------------------------------ */
/* E4M3 ([Ascend] names the format; layout from the OCP FP8 spec)      */
/* ------------------------------------------------------------------ */

/* Value of an E4M3 (FN) code: sign, 4-bit exponent (bias 7), 3-bit mantissa.
 * Exponent field 0 is subnormal (m/8 * 2^-6); field 15 with mantissa 7 is NaN.
 * There is no infinity. */
double or_e4m3_value(uint8_t code) {
    int s = (code >> 7) & 1;
    int e = (code >> 3) & 15;
    int m = code & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        mag = ldexp((double)m, -9);          /* (m/8) * 2^-6 */
    else
        mag = ldexp(8.0 + (double)m, e - 10); /* (1 + m/8) * 2^(e-7) */
    return s ? -mag : mag;
}

/* Encode a real number to E4M3: round to nearest, ties to the even
 * mantissa, saturate magnitudes >= 448 to +-448, NaN -> 0x7F.  The sign is
 * kept, so negative values that round to zero give 0x80. */
uint8_t or_e4m3_encode(double y) {
    uint8_t sign;
    double a, step, r, n, frac;
    int e2, efield, mant;
    if (isnan(y)) return 0x7F;
    sign = signbit(y) ? 0x80 : 0x00;
    a = fabs(y);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    if (a < ldexp(1.0, -6)) {
        /* subnormal binade: spacing 2^-9 */
        step = ldexp(1.0, -9);
        efield = 0;
    } else {
        /* a in [2^E, 2^(E+1)) with E = e2 - 1; spacing 2^(E-3) */
        (void)frexp(a, &e2);
        step = ldexp(1.0, (e2 - 1) - 3);
        efield = (e2 - 1) + 7;
    }
    r = a / step;              /* exact: division by a power of two */
    n = floor(r);
    frac = r - n;
    if (frac > 0.5 || (frac == 0.5 && fmod(n, 2.0) == 1.0)) n += 1.0;
    if (efield == 0) {
        /* n in [0, 8]; n == 8 is the smallest normal 2^-6 */
        if (n >= 8.0) { efield = 1; mant = 0; }
        else mant = (int)n;
    } else {
        /* n in [8, 16]; n == 16 carries into the next binade */
        if (n >= 16.0) { efield += 1; mant = 0; }
        else mant = (int)n - 8;
    }
    /* a < 448 so rounding never reaches 480 (the NaN pattern) */
    return (uint8_t)(sign | (efield << 3) | mant);
}

/* Decoded values of all 256 codes, filled from or_e4m3_value (only a
 * lookup of the same function, so the attention loops do not re-decode). */
static double dec_table[256];
static pthread_once_t dec_once = PTHREAD_ONCE_INIT;
static void fill_dec_table(void) {
    int c;
    for (c = 0; c < 256; ++c) dec_table[c] = or_e4m3_value((uint8_t)c);
}

/* Bulk encode of fp32 inputs (used by the exhaustive cast tests). */
void or_e4m3_encode_f32_array(const float* y, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = or_e4m3_encode((double)y[i]);
}

/* Bulk decode. */
void or_e4m3_value_array(const uint8_t* c, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = or_e4m3_value(c[i]);
}

/* ------------------------------------------------------------------ */
/* Valid-token addressing ("unpadding", [vLLM-ViT] notes: quant        */
/* launches + unpadding).  Output row t of sequence b reads source row */
/* t (packed) or src_seq_start[b] + (t - cu[b]) (padded source).       */
/* ------------------------------------------------------------------ */

static int64_t src_row_of(int64_t t, const int32_t* cu, int B,
                          const int32_t* src_seq_start) {
    int b;
    if (!src_seq_start) return t;
    for (b = 0; b < B; ++b)
        if (t >= cu[b] && t < cu[b + 1]) break;
    return (int64_t)src_seq_start[b] + (t - cu[b]);
}

/* Simple parallel-for over token ranges (pthreads). */
typedef struct {
    void (*fn)(void* ctx, int64_t t0, int64_t t1, int worker);
    void* ctx;
    int64_t T;
    int nthreads;
    int worker;
} pf_arg;

static void* pf_thread(void* p) {
    pf_arg* a = (pf_arg*)p;
    int64_t chunk = (a->T + a->nthreads - 1) / a->nthreads;
    int64_t t0 = (int64_t)a->worker * chunk, t1 = t0 + chunk;
    if (t1 > a->T) t1 = a->T;
    if (t0 < t1) a->fn(a->ctx, t0, t1, a->worker);
    return NULL;
}

static int parallel_for(int64_t T, int nthreads,
                        void (*fn)(void*, int64_t, int64_t, int), void* ctx) {
    pthread_t th[256];
    pf_arg args[256];
    int i;
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    for (i = 0; i < nthreads; ++i) {
        args[i].fn = fn; args[i].ctx = ctx; args[i].T = T;
        args[i].nthreads = nthreads; args[i].worker = i;
        pthread_create(&th[i], NULL, pf_thread, &args[i]);
    }
    for (i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    return nthreads;
}

typedef struct {
    const uint16_t* x;
    int64_t tok_stride, head_stride;
    const int32_t* src_seq_start;
    const int32_t* cu;
    int B, H, D;
    float qs;
    uint8_t* out;
    float part_amax[256];
    int part_inf[256];
} tensor_job;

/* amax = max |x| over every valid token, head and channel of one tensor.
 * NaN elements are ignored; an infinity is recorded as non-finite. */
static void amax_range(void* p, int64_t t0, int64_t t1, int w) {
    tensor_job* j = (tensor_job*)p;
    float amax = 0.0f;
    int inf = 0, h, d;
    int64_t t;
    for (t = t0; t < t1; ++t) {
        int64_t row = src_row_of(t, j->cu, j->B, j->src_seq_start);
        for (h = 0; h < j->H; ++h)
            for (d = 0; d < j->D; ++d) {
                float v = bf16_to_f32(j->x[row * j->tok_stride + h * j->head_stride + d]);
                float a;
                if (isnan(v)) continue;
                a = fabsf(v);
                if (isinf(a)) inf = 1;
                if (a > amax) amax = a;
            }
    }
    j->part_amax[w] = amax;
    j->part_inf[w] = inf;
}

float or_amax_bf16(const uint16_t* x, int64_t tok_stride, int64_t head_stride,
                   const int32_t* src_seq_start, const int32_t* cu, int B,
                   int H, int D, int* nonfinite, int nthreads) {
    tensor_job j;
    float amax = 0.0f;
    int n, i;
    memset(&j, 0, sizeof(j));
    j.x = x; j.tok_stride = tok_stride; j.head_stride = head_stride;
    j.src_seq_start = src_seq_start; j.cu = cu; j.B = B; j.H = H; j.D = D;
    n = parallel_for(cu[B], nthreads, amax_range, &j);
    *nonfinite = 0;
    for (i = 0; i < n; ++i) {
        if (j.part_amax[i] > amax) amax = j.part_amax[i];
        if (j.part_inf[i]) *nonfinite = 1;
    }
    return amax;
}

/* Cast: code = E4M3(fl32(x * qs)) -- one fp32 RN multiply, then RNE encode.
 * Output is packed [T][H][D]. */
static void quant_range(void* p, int64_t t0, int64_t t1, int w) {
    tensor_job* j = (tensor_job*)p;
    int64_t t;
    int h, d;
    (void)w;
    for (t = t0; t < t1; ++t) {
        int64_t row = src_row_of(t, j->cu, j->B, j->src_seq_start);
        for (h = 0; h < j->H; ++h)
            for (d = 0; d < j->D; ++d) {
                float v = bf16_to_f32(j->x[row * j->tok_stride + h * j->head_stride + d]);
                float y = v * j->qs;
                j->out[(t * j->H + h) * (int64_t)j->D + d] = or_e4m3_encode((double)y);
            }
    }
}

void or_quantize_bf16(const uint16_t* x, int64_t tok_stride, int64_t head_stride,
                      const int32_t* src_seq_start, const int32_t* cu, int B,
                      int H, int D, float qs, uint8_t* out, int nthreads) {
    tensor_job j;
    memset(&j, 0, sizeof(j));
    j.x = x; j.tok_stride = tok_stride; j.head_stride = head_stride;
    j.src_seq_start = src_seq_start; j.cu = cu; j.B = B; j.H = H; j.D = D;
    j.qs = qs; j.out = out;
    parallel_for(cu[B], nthreads, quant_range, &j);
}

/* ------------------------------------------------------------------ */
/* Amax ring and scales ([vLLM-ViT] usage: 16 observed amax values     */
/* drive the per-forward scale; save margin 1.5).                      */
/* ------------------------------------------------------------------ */

#define OR_RING 16

typedef struct {
    float slot[OR_RING];
    uint32_t head;   /* next slot to write */
    uint32_t count;  /* filled slots, <= 16 */
} or_ring;

void or_ring_reset(or_ring* r) { memset(r, 0, sizeof(*r)); }

/* Push one observed amax into the circular buffer. */
void or_ring_push(or_ring* r, float amax) {
    r->slot[r->head] = amax;
    r->head = (r->head + 1) % OR_RING;
    if (r->count < OR_RING) r->count += 1;
}

/* Bound A = max over the filled slots (0 for an empty ring). */
float or_ring_bound(const or_ring* r) {
    float a = 0.0f;
    uint32_t i;
    for (i = 0; i < r->count; ++i)
        if (r->slot[i] > a) a = r->slot[i];
    return a;
}

/* qs = fl32(448 / A), ds = fl32(A / 448); A == 0 -> 1, 1. */
void or_scales_from_bound(float A, float* qs, float* ds) {
    if (A == 0.0f) {
        *qs = 1.0f;
        *ds = 1.0f;
        return;
    }
    *qs = 448.0f / A;
    *ds = A / 448.0f;
}

/* One dynamic pass for one tensor: the current amax is pushed first (unless
 * it is not finite, in which case the ring is left as it was), then the
 * scales come from the ring's bound. */
void or_dynamic_step(or_ring* r, float amax, int nonfinite, float* qs, float* ds) {
    if (!nonfinite) or_ring_push(r, amax);
    or_scales_from_bound(or_ring_bound(r), qs, ds);
}

/* Exported static value = fl32(bound * margin). */
float or_export_value(const or_ring* r, float margin) {
    return or_ring_bound(r) * margin;
}

/* ------------------------------------------------------------------ */
/* Attention (fp64), non-causal, per sequence of cu_seqlens            */
/* ([vLLM-Omni] overview: Q/K/V quantised before the FA operator;      */
/* eligible forwards are full, non-causal attention).                  */
/* ------------------------------------------------------------------ */

typedef struct {
    int kind;                 /* 0 = fp8 codes, 1 = bf16 */
    const void* q;
    const void* k;
    const void* v;
    const int32_t* cu;
    int B, H, D;
    double ds_q, ds_k, ds_v;
    double scale;             /* softmax scale (1/sqrt(D) by default) */
    int pquant;               /* 0: p~ = p, 1: exp2 rule, 2: linear-log rule (both with the
                                 block rule's lagged reference max) */
    int lrule;                /* 0: l = sum p, 1: l = sum p~ */
    const int64_t* rows;      /* token indices to evaluate (or NULL: all) */
    int64_t nrows;
    double* out;              /* [nrows][H][D] */
    double* amb;              /* [nrows][H][D] ambiguity allowance, or NULL */
    double* alt;              /* [nrows][H][D] the other correct result (NaN: none), or NULL */
    double* alt_amb;          /* its ambiguity allowance */
    int64_t next;             /* work counter (rows*H items) */
    pthread_mutex_t lock;
} att_job;

static double elem(const att_job* j, const void* base, int64_t t, int h, int d) {
    int64_t idx = ((int64_t)t * j->H + h) * j->D + d;
    if (j->kind == 0) return dec_table[((const uint8_t*)base)[idx]];
    return (double)bf16_to_f32(((const uint16_t*)base)[idx]);
}

/* P rule: the PV product takes P in blocks of OR_P_BLOCK keys, visited in
 * order from the start of the sequence; each block's p are quantised as
 * e4m3(OR_P_SCALE exp(s - r_t)) / OR_P_SCALE against the row's reference max
 * r_t, then carried to the final max M by the exact factor exp(r_t - M).
 * r_0 is block 0's max; r_t is block t's max when that exceeds r_{t-1} by
 * more than OR_P_LAG_LOG2 in log2 units, else r_{t-1}.  With the lag at most
 * 3 and the scale 2^5, OR_P_SCALE exp(s - r_t) <= 2^8 (no saturation).  l is
 * the sum of the unquantised p = exp(s - M). */
#define OR_P_BLOCK 128
#define OR_P_SCALE 32.0
#define OR_P_LAG_LOG2 3.0

/* Evaluation-error model of an implementation of the P rule, used only to
 * tell which codes and which reference moves are decided at a tie (there
 * either outcome is a correct result of the rule).  u = 2^-24 is the fp32
 * unit roundoff.  The implementation evaluates, in log2 units,
 *     t = s c + (5 - r2),   c = ds_q ds_k scale log2(e),   r2 = m c,
 * where s is an fp32 accumulation of the 128 exact products of decoded
 * codes, m the fp32 maximum of such scores over the reference block, c a
 * product of three fp32 roundings of the scales and the fp32 value of
 * log2(e), r2 and 5 - r2 one fp32 rounding each and t one fused
 * multiply-add, then y = 2^t.  With A_j = scale ds_q ds_k sum_d |q_d k_jd|
 * (so |s_j| <= A_j), A_r the largest A over the block that set r, and
 * t* = (s - r) log2(e) + 5 the exact exponent:
 *   - each score carries at most OR_ACC_ROUNDINGS u A of accumulation error
 *     (in natural units; log2(e) times that in t);
 *   - c is off by at most 4u relative, which reaches t through (s - r) c as
 *     4u |t* - 5| (the same c multiplies s and m);
 *   - the roundings of r2, of 5 - r2 and of the fused multiply-add add
 *     u |r2|, u (5 + |r2|) and u |t|;
 *   - 2^t itself is evaluated to within OR_EXP2_REL relative error.
 * So y carries a relative error of at most
 *     ln2 [log2(e) OR_ACC_ROUNDINGS u (A_j + A_r) + u (4|t* - 5| + 2|r2| + 5 + |t*|)]
 *       + OR_EXP2_REL,
 * doubled here for the second-order terms.  The reference move compares
 * a = m_blk c with r2 + 3 (one fp32 rounding of the sum): a carries
 * log2(e) OR_ACC_ROUNDINGS u A_blk + 5u |a|, r2 + 3 carries
 * log2(e) OR_ACC_ROUNDINGS u A_r + 5u |r2| + u |r2 + 3|, doubled likewise.
 * OR_ACC_ROUNDINGS bounds the tensor cores' fp32 accumulation of one
 * 128-long dot product of E4M3 values (4 MMAs of 32 products): B200's
 * error was measured at up to 7.9 u sum|q_d k_d| over 1.5 M random and
 * adversarial scores (the GPU test of fp8attn_selftest_qk_scores checks
 * the bound), so 16 leaves a factor of two.  OR_EXP2_REL bounds both exp2
 * evaluations the kernel uses: the hardware approximation (measured at
 * 1.45e-7 relative on [-10, 9]) and a degree-5 polynomial (2.13e-7, pinned
 * by a CPU test). */
#define OR_U 5.9604644775390625e-08   /* 2^-24 */
#define OR_ACC_ROUNDINGS 16.0
#define OR_EXP2_REL 4.76837158203125e-07   /* 2^-21 */

static double p_rel_error(double t, double r2, double a_j, double a_r) {
    const double log2e = 1.4426950408889634;
    double dt = log2e * OR_ACC_ROUNDINGS * OR_U * (a_j + a_r)
              + OR_U * (4.0 * fabs(t - 5.0) + 2.0 * fabs(r2) + 5.0 + fabs(t));
    return 2.0 * (0.6931471805599453 * dt + OR_EXP2_REL);
}

/* Largest change of p~ (in units of exp(r - M)) that a code decided at a
 * tie can make: y = 32 exp(s - r) with relative error eps; 0 when
 * y (1 - eps) and y (1 + eps) have the same code. */
static double code_ambiguity(double y, double eps) {
    uint8_t lo = or_e4m3_encode(y * (1.0 - eps));
    uint8_t hi = or_e4m3_encode(y * (1.0 + eps));
    if (lo == hi) return 0.0;
    return fabs(or_e4m3_value(hi) - or_e4m3_value(lo)) / OR_P_SCALE;
}

/* Whether a reference move (block max bm against reference r, natural
 * units) is decided within the implementation's error of the threshold. */
static int move_is_ambiguous(double bm, double a_blk, double r, double a_r) {
    const double log2e = 1.4426950408889634;
    double a = bm * log2e, r2 = r * log2e, b = r2 + OR_P_LAG_LOG2;
    double ea = log2e * OR_ACC_ROUNDINGS * OR_U * a_blk + 5.0 * OR_U * fabs(a);
    double eb = log2e * OR_ACC_ROUNDINGS * OR_U * a_r + 5.0 * OR_U * fabs(r2) + OR_U * fabs(b);
    return fabs(a - b) <= 2.0 * (ea + eb);
}

/* Linear-log P rule: the E4M3 code is 8 t + 56 rounded to the nearest
 * integer (ties to even) and clamped to [0, 128], with t = (s - r) log2(e) + 5
 * the exponent that the exp2 rule would raise 2 to.  In other words the
 * E4M3 bit pattern is read as a fixed-point base-2 logarithm: the exponent
 * field is the integer part of t, the mantissa field its fraction in
 * eighths, so the value is the piecewise-linear interpolation of 2^t
 * between powers of two (Mitchell's approximation) rounded to the E4M3
 * grid.  A NaN score has code 0. */
static uint8_t linear_log_code(double t) {
    double y, n, frac;
    if (isnan(t)) return 0;
    y = 8.0 * t + 56.0;
    if (y <= 0.0) return 0;
    if (y >= 128.0) return 128;
    n = floor(y);
    frac = y - n;
    if (frac > 0.5 || (frac == 0.5 && fmod(n, 2.0) == 1.0)) n += 1.0;
    return (uint8_t)n;
}

/* The linear-log rule's implementation error in t (log2 units): the same
 * score, scale and reference terms as p_rel_error, evaluated as
 * y = sat(s c / 16 + (0.75 - r2 / 16)) = (8 t + 56) / 128: the roundings of
 * r2, of 0.75 - r2/16 and of the fused multiply-add add u |r2|,
 * u |12 - r2| and u |t + 7| (in t units), and no exponential is evaluated.
 * Doubled for second-order terms.  A code is decided at a tie when 8 t + 56
 * lies within 8 times this of a half-integer. */
static double linear_log_t_error(double t, double r2, double a_j, double a_r) {
    const double log2e = 1.4426950408889634;
    double dt = log2e * OR_ACC_ROUNDINGS * OR_U * (a_j + a_r)
              + OR_U * (4.0 * fabs(t - 5.0) + fabs(r2) + fabs(12.0 - r2) + fabs(t + 7.0));
    return 2.0 * dt;
}

/* Largest change of p~ (in units of exp(r - M)) that a linear-log code
 * decided at a tie can make. */
static double linear_log_ambiguity(double t, double dt) {
    uint8_t lo = linear_log_code(t - dt), hi = linear_log_code(t + dt);
    if (lo == hi) return 0.0;
    return fabs(or_e4m3_value(hi) - or_e4m3_value(lo)) / OR_P_SCALE;
}

/* One pass of the P loop over a row's scores (s_buf, a_buf: keys k0..k1-1,
 * M their max).  The reference r follows the rule; a move decided within
 * the implementation's error of the threshold is taken as the fp64 test
 * says, except at block `force_block`, where the opposite is taken.  The
 * block of the first such decision not forced goes to *first_amb.  Writes
 * o (and, with a, the tie allowance) already normalised; returns the number
 * of such decisions not forced. */
static int attend_pass(const att_job* j, int h, int64_t k0, int64_t k1, const double* s_buf,
                       const double* a_buf, double M, int64_t force_block, int64_t* first_amb,
                       double* o, double* a) {
    int d, n_amb = 0;
    int64_t kk;
    double l = 0.0, r = -INFINITY, a_r = 0.0, amb_l = 0.0;
    double dsv = j->kind == 0 ? j->ds_v : 1.0;
    *first_amb = -1;
    for (d = 0; d < j->D; ++d) o[d] = 0.0;
    if (a)
        for (d = 0; d < j->D; ++d) a[d] = 0.0;
    for (kk = k0; kk < k1; ++kk) {
        double s = s_buf[kk - k0];
        double p = exp(s - M);
        double pt = p;
        if ((kk - k0) % OR_P_BLOCK == 0) {
            /* entering a new block: its max, and whether the reference moves */
            int64_t e = kk + OR_P_BLOCK < k1 ? kk + OR_P_BLOCK : k1, x;
            int64_t blk = (kk - k0) / OR_P_BLOCK;
            double bm = -INFINITY, a_blk = 0.0;
            for (x = kk; x < e; ++x) {
                if (s_buf[x - k0] > bm) bm = s_buf[x - k0];
                if (a_buf[x - k0] > a_blk) a_blk = a_buf[x - k0];
            }
            if (r == -INFINITY) {
                r = bm;
                a_r = a_blk;
            } else {
                int move = bm * 1.4426950408889634 > r * 1.4426950408889634 + OR_P_LAG_LOG2;
                if (move_is_ambiguous(bm, a_blk, r, a_r)) {
                    if (blk == force_block) {
                        move = !move;
                    } else {
                        if (*first_amb < 0) *first_amb = blk;
                        ++n_amb;
                    }
                }
                if (move) {
                    r = bm;
                    a_r = a_blk;
                }
            }
        }
        if (j->pquant == 1) {
            double y = OR_P_SCALE * exp(s - r);
            pt = or_e4m3_value(or_e4m3_encode(y)) / OR_P_SCALE * exp(r - M);
            if (a) {
                double tt = (s - r) * 1.4426950408889634 + 5.0;
                double eps = p_rel_error(tt, r * 1.4426950408889634, a_buf[kk - k0], a_r);
                double amb = code_ambiguity(y, eps) * exp(r - M);
                amb_l += amb;
                if (amb > 0.0)
                    for (d = 0; d < j->D; ++d) a[d] += amb * fabs(elem(j, j->v, kk, h, d));
            }
        } else if (j->pquant == 2) {
            double tt = (s - r) * 1.4426950408889634 + 5.0;
            pt = or_e4m3_value(linear_log_code(tt)) / OR_P_SCALE * exp(r - M);
            if (a && !isnan(tt)) {
                double dt = linear_log_t_error(tt, r * 1.4426950408889634, a_buf[kk - k0], a_r);
                double amb = linear_log_ambiguity(tt, dt) * exp(r - M);
                amb_l += amb;
                if (amb > 0.0)
                    for (d = 0; d < j->D; ++d) a[d] += amb * fabs(elem(j, j->v, kk, h, d));
            }
        }
        l += (j->lrule || j->pquant == 2) ? pt : p;
        for (d = 0; d < j->D; ++d) o[d] += pt * elem(j, j->v, kk, h, d);
    }
    if (a && (j->lrule || j->pquant == 2)) {
        /* l = sum p~ moves with the same codes: a flip by D changes the
         * output by ds_v D (v_j - O/l) / (l + D), bounded by
         * ds_v |D| (|v_j| + |O/l|) / (l - sum |D|) */
        double lmin = l - amb_l;
        for (d = 0; d < j->D; ++d)
            a[d] = (amb_l == 0.0) ? 0.0
                 : (lmin > 0.0 ? (a[d] + amb_l * fabs(o[d] / l)) * dsv / lmin : INFINITY);
    } else if (a) {
        for (d = 0; d < j->D; ++d) a[d] = a[d] * dsv / l;
    }
    for (d = 0; d < j->D; ++d) o[d] = o[d] * dsv / l;
    return n_amb;
}

/* One output row (query ri, head h).  When the row's reference moves are all
 * decided away from the threshold there is one result.  When exactly one is
 * decided within the implementation's error of it, both outcomes are
 * correct results of the rule: the row is evaluated both ways and the other
 * outcome goes to alt / alt_amb (NaN there otherwise).  With more than one
 * such decision the row is reported as unverifiable (infinite allowance). */
static void attend_one(const att_job* j, int64_t ri, int h, double* s_buf, double* a_buf,
                       double* tmp) {
    int64_t t = j->rows ? j->rows[ri] : ri;
    int b, d, n_amb;
    int64_t k0, k1, kk, first_amb, first2;
    double M = -INFINITY;
    int64_t base = (ri * j->H + h) * (int64_t)j->D;
    double* o = j->out + base;
    double* a = j->amb ? j->amb + base : NULL;
    double dsq = j->kind == 0 ? j->ds_q : 1.0;
    double dsk = j->kind == 0 ? j->ds_k : 1.0;
    double sc = dsq * dsk * j->scale;
    for (b = 0; b < j->B; ++b)
        if (t >= j->cu[b] && t < j->cu[b + 1]) break;
    k0 = j->cu[b];
    k1 = j->cu[b + 1];
    /* scores: dot of decoded values (exact in fp64 for E4M3), then scales;
     * A_j = the same sum of absolute products (the error model's scale) */
    for (kk = k0; kk < k1; ++kk) {
        double acc = 0.0, aacc = 0.0;
        for (d = 0; d < j->D; ++d) {
            double pr = elem(j, j->q, t, h, d) * elem(j, j->k, kk, h, d);
            acc += pr;
            aacc += fabs(pr);
        }
        s_buf[kk - k0] = acc * sc;
        a_buf[kk - k0] = aacc * fabs(sc);
        if (s_buf[kk - k0] > M) M = s_buf[kk - k0];
    }
    n_amb = attend_pass(j, h, k0, k1, s_buf, a_buf, M, -1, &first_amb, o, a);
    if (j->alt)
        for (d = 0; d < 2 * j->D; ++d) (d < j->D ? j->alt : j->alt_amb)[base + d % j->D] = NAN;
    if (!j->pquant || n_amb == 0 || !a) return;
    if (n_amb == 1 && j->alt) {
        /* the other outcome of the one decision at the threshold */
        if (attend_pass(j, h, k0, k1, s_buf, a_buf, M, first_amb, &first2, tmp, tmp + j->D) == 0) {
            for (d = 0; d < j->D; ++d) {
                j->alt[base + d] = tmp[d];
                j->alt_amb[base + d] = tmp[j->D + d];
            }
            return;
        }
    }
    for (d = 0; d < j->D; ++d) a[d] = INFINITY;
}

static void* att_worker(void* arg) {
    att_job* j = (att_job*)arg;
    int64_t maxlen = 0, total = j->nrows * j->H;
    int b;
    double* s_buf;
    for (b = 0; b < j->B; ++b)
        if (j->cu[b + 1] - j->cu[b] > maxlen) maxlen = j->cu[b + 1] - j->cu[b];
    s_buf = (double*)malloc(sizeof(double) * (2 * (size_t)(maxlen > 0 ? maxlen : 1) +
                                              2 * (size_t)j->D));
    for (;;) {
        int64_t w;
        pthread_mutex_lock(&j->lock);
        w = j->next++;
        pthread_mutex_unlock(&j->lock);
        if (w >= total) break;
        attend_one(j, w / j->H, (int)(w % j->H), s_buf, s_buf + (maxlen > 0 ? maxlen : 1),
                   s_buf + 2 * (maxlen > 0 ? maxlen : 1));
    }
    free(s_buf);
    return NULL;
}

static int run_attention(att_job* j, int nthreads) {
    pthread_t th[256];
    int i;
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (!j->rows) j->nrows = j->cu[j->B];
    pthread_once(&dec_once, fill_dec_table);
    j->next = 0;
    pthread_mutex_init(&j->lock, NULL);
    for (i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, att_worker, j);
    for (i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    pthread_mutex_destroy(&j->lock);
    return nthreads;
}

/* FP8 attention on E4M3 codes [T][H][D] with per-tensor descales.
 * o_i = (sum_j p~_ij dec(v_j)) * ds_v / l_i, l_i = sum_j exp(s_ij - M_i),
 * s_ij = (sum_d dec(q_id) dec(k_jd)) * ds_q * ds_k * scale, and p~ by the
 * block rule above.
 * Returns the number of threads used. */
int or_attention_fp8(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8,
                     const int32_t* cu, int B, int H, int D,
                     double ds_q, double ds_k, double ds_v, double scale,
                     int pquant, int lrule, const int64_t* rows, int64_t nrows,
                     double* out, double* amb, double* alt, double* alt_amb, int nthreads) {
    att_job j;
    memset(&j, 0, sizeof(j));
    j.kind = 0;
    j.q = q8; j.k = k8; j.v = v8;
    j.cu = cu; j.B = B; j.H = H; j.D = D;
    j.ds_q = ds_q; j.ds_k = ds_k; j.ds_v = ds_v; j.scale = scale;
    j.pquant = pquant; j.lrule = lrule;
    j.rows = rows; j.nrows = nrows; j.out = out; j.amb = amb;
    j.alt = amb ? alt : NULL; j.alt_amb = amb ? alt_amb : NULL;
    return run_attention(&j, nthreads);
}

/* Native-dtype attention for skipped layers ([vLLM-Omni] parameters:
 * listed layers keep the native dtype): bf16 inputs, no quantisation. */
int or_attention_bf16(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                      const int32_t* cu, int B, int H, int D, double scale,
                      const int64_t* rows, int64_t nrows, double* out, int nthreads) {
    att_job j;
    memset(&j, 0, sizeof(j));
    j.kind = 1;
    j.q = q; j.k = k; j.v = v;
    j.cu = cu; j.B = B; j.H = H; j.D = D;
    j.ds_q = 1.0; j.ds_k = 1.0; j.ds_v = 1.0; j.scale = scale;
    j.pquant = 0; j.lrule = 0;
    j.rows = rows; j.nrows = nrows; j.out = out;
    return run_attention(&j, nthreads);
}
