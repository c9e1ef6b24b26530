/*
 * pwq_oracle.c -- plain scalar CPU oracle for block-scaled quantisation of
 * BF16 tensors: FP8 block-wise (128x128), MXFP8 (1x32, UE8M0) and NVFP4
 * (1x16, two-level scale), quantise / dequantise / fake-quantise.
 *
 * TEST INFRASTRUCTURE ONLY.  This file defines what the GPU library must
 * compute; it is never part of the product path.  Only the tests, the
 * smoke check and the benchmark's CPU-baseline leg load it.  It shares no
 * code, header, table or constant generator with the CUDA sources.
 *
 * Style: one element at a time, IEEE binary32 ("float") for every step the
 * method states in FP32, and exact comparisons in binary64 ("double") for
 * the codecs.  Built with -O2 -fno-fast-math -ffp-contract=off so that
 * every float operation below is one correctly rounded IEEE operation.
 * Every entry point forces round-to-nearest-even and clears the x86
 * flush-to-zero / denormals-are-zero bits for its duration.
 *
 * Sources (page title, section):
 *   [LPR]  "Low Precision RL" (miles documentation): "Choose a precision"
 *          table (FP8 block-wise 128x128 FP32 scales; MXFP8 1x32 UE8M0;
 *          NVFP4 E2M1 1x16 two-level FP8 + FP32 scales), "Modes" 2 and 3
 *          (E4M3 codes, scales packed as uint8 power-of-two), "Modes" 4.
 *   [LPT]  "低精度训练与 Rollout" (vime documentation): "FP8 训练 + FP8
 *          Rollout" (NVTE_FP8_BLOCK_SCALING_FP32_SCALES=1; dequantise FP8 to
 *          BF16 on weight update).
 *   [QAT]  verl NVFP4 QAT article: section 2.3 (global scale =
 *          amax / (6 * 448), per-16 block scale in E4M3, nearest E2M1 value
 *          on {0, 0.5, 1, 1.5, 2, 3, 4, 6}, multiply back), section 2.4
 *          (q/k/v and gate/up siblings share one global amax), section 3.3
 *          (weight_scale_2 = amax / (6.0 * 448.0)).
 *   [PR503] vime pull request #503, review thread on the NVFP4 QDQ config
 *          (exact round-to-nearest numerics, fast math refused).
 *
 * Readings where the pages are silent:
 *   R1 FP8 tile scale s = fl(amax / 448) is the dequantisation multiplier.
 *   R2 Codes are e4m3(fl(x / s)): IEEE division, then RNE onto E4M3.
 *   R3 A zero scale (all-zero tile/block/group) gives signed-zero codes.
 *   R4 UE8M0 exponent e = min{k : amax <= 448 * 2^k}, clamped to
 *      [-127, 127]; byte = e + 127; amax = 0 gives byte 0.
 *   R5 NVFP4 block scale sb = e4m3(fl(amax_b / fl(6 * gs))), gs = fl(A/2688).
 *   R6 NVFP4 code c = e2m1(fl(x / d)), d = fl(dec(sb) * gs); d = 0 gives ±0.
 *   R7 NVFP4 dequant y = bf16(fl((dec(c) * dec(sb)) * gs)).
 *   R8 Packed nibbles: element 2j in the low nibble, 2j+1 in the high one.
 *   R9 Sign of zero is kept everywhere.
 *   R19-R21 (NVFP4 "4over6", [PR503] NVFP4 QDQ config thread: the flags
 *      NVTE_NVFP4_4OVER6 and NVTE_NVFP4_4OVER6_E4M3_USE_256, which sets the
 *      E4M3 maximum of the global scale to 256 instead of 448; the pages
 *      give no selection rule, so the rule below is a reading and this
 *      part is PARITY UNPINNED against the pages):
 *   R19 gs = fl(A / (6 * E)), E the E4M3 maximum (448 or 256).
 *   R20 Per block, candidate t in {6, 4}: sb_t = e4m3(fl(amax_b /
 *      fl(t * gs))), then codes and values as R6, R7 with sb_t.
 *   R21 err_t = sum over the block's elements, left to right in binary32,
 *      of fl(fl(x - y_t)^2); t = 4 is kept iff err_4 < err_6.
 */
#include <stdint.h>
#include <string.h>
#include <math.h>
#include <fenv.h>
#if defined(__x86_64__) || defined(__i386__)
#include <xmmintrin.h>
#endif

/* ------------------------------------------------------------------ */
/* Floating-point environment guard                                    */
/* ------------------------------------------------------------------ */

typedef struct { int round; unsigned int csr; } fpenv_save;

static fpenv_save env_enter(void) {
    fpenv_save s;
    s.round = fegetround();
    fesetround(FE_TONEAREST);
#if defined(__x86_64__) || defined(__i386__)
    s.csr = _mm_getcsr();
    /* bit 15 = flush-to-zero, bit 6 = denormals-are-zero, bits 13-14 = RC */
    _mm_setcsr(s.csr & ~((1u << 15) | (1u << 6) | (3u << 13)));
#else
    s.csr = 0;
#endif
    return s;
}

static void env_leave(fpenv_save s) {
#if defined(__x86_64__) || defined(__i386__)
    _mm_setcsr(s.csr);
#endif
    fesetround(s.round);
}

/* Returns 1 when this thread's FP state is RN with no FTZ/DAZ after the
 * guard is applied (the tests check this on the host that runs them). */
int or_fp_env_ok(void) {
    fpenv_save s = env_enter();
    int ok = (fegetround() == FE_TONEAREST);
#if defined(__x86_64__) || defined(__i386__)
    unsigned int c = _mm_getcsr();
    ok = ok && !(c & (1u << 15)) && !(c & (1u << 6)) && ((c >> 13) & 3u) == 0;
#endif
    /* a subnormal must survive arithmetic */
    volatile float tiny = 1.0e-40f, two = 2.0f;
    ok = ok && (tiny * two > 0.0f);
    env_leave(s);
    return ok;
}

/* ------------------------------------------------------------------ */
/* BF16                                                                */
/* ------------------------------------------------------------------ */

static float bits_to_float(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t float_to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

float or_bf16_to_f32(uint16_t b) { return bits_to_float((uint32_t)b << 16); }

/* bf16(v): round a finite float to the nearest BF16 value, ties to the
 * even BF16 pattern.  The two BF16 neighbours of |v| are found by
 * truncation (lo) and its successor (hi, which may be +inf); the decision
 * compares |v| with their midpoint, exactly, in double. */
uint16_t or_bf16_round(float v) {
    uint32_t u = float_to_bits(v);
    uint32_t sign = u & 0x80000000u;
    uint32_t mag = u & 0x7fffffffu;
    uint32_t lo = mag & 0xffff0000u;             /* |v| truncated to BF16 */
    if (lo == mag) return (uint16_t)((sign | lo) >> 16);  /* exact */
    uint32_t hi = lo + 0x00010000u;              /* next BF16 magnitude */
    double a = (double)bits_to_float(mag);
    double dlo = (double)bits_to_float(lo);
    double dhi;
    if (hi == 0x7f800000u) {
        /* the BF16 "successor" of the largest finite value is +inf; the
         * rounding midpoint is where the next value would be: lo + ulp/2 */
        dhi = dlo + ldexp(1.0, 127 - 7);          /* ulp of BF16 at 2^127 */
    } else {
        dhi = (double)bits_to_float(hi);
    }
    double mid = (dlo + dhi) / 2.0;              /* exact in double */
    uint32_t pick;
    if (a < mid) pick = lo;
    else if (a > mid) pick = hi;
    else pick = ((lo >> 16) & 1u) ? hi : lo;     /* tie: even BF16 pattern */
    return (uint16_t)((sign | pick) >> 16);
}

/* ------------------------------------------------------------------ */
/* E4M3 (FN variant: no infinities, 0x7F/0xFF are NaN, max 448)         */
/* ------------------------------------------------------------------ */

/* Magnitude of a non-NaN E4M3 code: bias 7, 3 mantissa bits, subnormals
 * m * 2^-9. */
double or_e4m3_decode(uint8_t c) {
    int e = (c >> 3) & 0xf;
    int m = c & 7;
    double mag = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return (c & 0x80) ? -mag : mag;
}

/* The 127 non-negative finite E4M3 values, indexed by code 0x00..0x7E;
 * they increase with the code.  Filled from or_e4m3_decode on first use. */
static double E4M3_VALUES[127];
static int e4m3_table_ready = 0;

static void e4m3_table_init(void) {
    if (e4m3_table_ready) return;
    for (int c = 0; c < 127; c++) E4M3_VALUES[c] = or_e4m3_decode((uint8_t)c);
    e4m3_table_ready = 1;
}

/* e4m3(v): nearest E4M3 value to v, ties to the even code, |v| beyond the
 * largest finite value (448) saturates to it.  A binary search finds the
 * pair of table values that brackets |v|; the choice compares |v| with
 * their midpoint exactly in double.  The sign of v (including -0) is kept. */
uint8_t or_e4m3_encode(double v) {
    e4m3_table_init();
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs(v);
    if (a >= 448.0) return sign | 0x7e;
    /* largest i with E4M3_VALUES[i] <= a (E4M3_VALUES[0] = 0 <= a) */
    int lo_i = 0, hi_i = 126;
    while (lo_i < hi_i) {
        int m = (lo_i + hi_i + 1) / 2;
        if (E4M3_VALUES[m] <= a) lo_i = m; else hi_i = m - 1;
    }
    int i = lo_i;
    double lo = E4M3_VALUES[i];
    if (lo == a) return sign | (uint8_t)i;
    double hi = E4M3_VALUES[i + 1];
    double mid = (lo + hi) / 2.0;
    int code;
    if (a < mid) code = i;
    else if (a > mid) code = i + 1;
    else code = (i % 2 == 0) ? i : i + 1;
    return sign | (uint8_t)code;
}

/* ------------------------------------------------------------------ */
/* E2M1 (values 0, 0.5, 1, 1.5, 2, 3, 4, 6; bit 3 = sign)               */
/* ------------------------------------------------------------------ */

static const double E2M1_VALUES[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double or_e2m1_decode(uint8_t c) {
    double mag = E2M1_VALUES[c & 7];
    return (c & 8) ? -mag : mag;
}

/* e2m1(v): nearest grid value, ties to the even code, saturating at 6. */
uint8_t or_e2m1_encode(double v) {
    uint8_t sign = signbit(v) ? 0x8 : 0x0;
    double a = fabs(v);
    if (a >= 6.0) return sign | 7;
    int i = 0;
    while (i + 1 <= 7 && E2M1_VALUES[i + 1] <= a) i++;
    double lo = E2M1_VALUES[i];
    if (lo == a) return sign | (uint8_t)i;
    double hi = E2M1_VALUES[i + 1];
    double mid = (lo + hi) / 2.0;
    int code;
    if (a < mid) code = i;
    else if (a > mid) code = i + 1;
    else code = (i % 2 == 0) ? i : i + 1;
    return sign | (uint8_t)code;
}

/* ------------------------------------------------------------------ */
/* UE8M0 block exponent (MXFP8)                                         */
/* ------------------------------------------------------------------ */

/* e = min{k integer : amax <= 448 * 2^k}, clamped to [-127, 127]; found by
 * walking k upward and comparing exactly in double.  amax = 0 satisfies
 * every k, so it clamps to -127 (byte 0). */
int or_ue8m0_exponent(float amax) {
    double a = fabs((double)amax);
    int k = -127;
    while (k < 127 && !(a <= ldexp(448.0, k))) k++;
    return k;
}

uint8_t or_ue8m0_byte(float amax) { return (uint8_t)(or_ue8m0_exponent(amax) + 127); }

/* ------------------------------------------------------------------ */
/* Array forms of the codecs (used by the codec tests)                  */
/* ------------------------------------------------------------------ */

void or_bf16_round_array(const float* v, uint16_t* out, int64_t n) {
    fpenv_save s = env_enter();
    for (int64_t i = 0; i < n; i++) out[i] = or_bf16_round(v[i]);
    env_leave(s);
}
void or_e4m3_encode_array(const float* v, uint8_t* out, int64_t n) {
    fpenv_save s = env_enter();
    for (int64_t i = 0; i < n; i++) out[i] = or_e4m3_encode((double)v[i]);
    env_leave(s);
}
void or_e2m1_encode_array(const float* v, uint8_t* out, int64_t n) {
    fpenv_save s = env_enter();
    for (int64_t i = 0; i < n; i++) out[i] = or_e2m1_encode((double)v[i]);
    env_leave(s);
}
void or_ue8m0_byte_array(const float* amax, uint8_t* out, int64_t n) {
    fpenv_save s = env_enter();
    for (int64_t i = 0; i < n; i++) out[i] = or_ue8m0_byte(amax[i]);
    env_leave(s);
}

/* ------------------------------------------------------------------ */
/* FP8 block-wise, 128 x 128 tiles, FP32 scale                          */
/*   [LPR] "Choose a precision" and "Modes" 2; [LPT] FP32 scales.        */
/* Layout: x, q dense [B][M][N]; s dense [B][ceil(M/128)][ceil(N/128)].  */
/* ------------------------------------------------------------------ */

#define FP8_TILE 128

void or_fp8_block_quant(const uint16_t* x, int64_t B, int64_t M, int64_t N,
                        uint8_t* q, float* s) {
    fpenv_save env = env_enter();
    int64_t tm_count = (M + FP8_TILE - 1) / FP8_TILE;
    int64_t tn_count = (N + FP8_TILE - 1) / FP8_TILE;
    for (int64_t b = 0; b < B; b++)
    for (int64_t tm = 0; tm < tm_count; tm++)
    for (int64_t tn = 0; tn < tn_count; tn++) {
        int64_t r0 = tm * FP8_TILE, c0 = tn * FP8_TILE;
        int64_t r1 = r0 + FP8_TILE < M ? r0 + FP8_TILE : M;
        int64_t c1 = c0 + FP8_TILE < N ? c0 + FP8_TILE : N;
        /* tile amax over the valid elements only */
        float amax = 0.0f;
        for (int64_t r = r0; r < r1; r++)
            for (int64_t c = c0; c < c1; c++) {
                float a = fabsf(or_bf16_to_f32(x[(b * M + r) * N + c]));
                if (a > amax) amax = a;
            }
        float scale = amax / 448.0f;                    /* R1: fl(amax/448) */
        s[(b * tm_count + tm) * tn_count + tn] = scale;
        for (int64_t r = r0; r < r1; r++)
            for (int64_t c = c0; c < c1; c++) {
                int64_t i = (b * M + r) * N + c;
                float xv = or_bf16_to_f32(x[i]);
                if (scale == 0.0f) {                   /* R3 */
                    q[i] = signbit(xv) ? 0x80 : 0x00;
                } else {
                    float quot = xv / scale;           /* R2: fl(x/s) */
                    q[i] = or_e4m3_encode((double)quot);
                }
            }
    }
    env_leave(env);
}

void or_fp8_block_dequant(const uint8_t* q, const float* s, int64_t B, int64_t M,
                          int64_t N, uint16_t* y) {
    fpenv_save env = env_enter();
    int64_t tm_count = (M + FP8_TILE - 1) / FP8_TILE;
    int64_t tn_count = (N + FP8_TILE - 1) / FP8_TILE;
    for (int64_t b = 0; b < B; b++)
    for (int64_t r = 0; r < M; r++)
    for (int64_t c = 0; c < N; c++) {
        int64_t i = (b * M + r) * N + c;
        float scale = s[(b * tm_count + r / FP8_TILE) * tn_count + c / FP8_TILE];
        float v = (float)or_e4m3_decode(q[i]) * scale;  /* fl(dec(q) * s) */
        y[i] = or_bf16_round(v);
    }
    env_leave(env);
}

/* ------------------------------------------------------------------ */
/* MXFP8, 1 x 32 blocks along a row, UE8M0 scale byte                   */
/*   [LPR] "Choose a precision" and "Modes" 3.                           */
/* Layout: x, q dense [B][M][N] (N % 32 == 0); e dense [B][M][N/32].     */
/* ------------------------------------------------------------------ */

#define MX_BLOCK 32

void or_mxfp8_quant(const uint16_t* x, int64_t B, int64_t M, int64_t N,
                    uint8_t* q, uint8_t* e) {
    fpenv_save env = env_enter();
    int64_t rows = B * M, nb = N / MX_BLOCK;
    for (int64_t r = 0; r < rows; r++)
    for (int64_t k = 0; k < nb; k++) {
        const uint16_t* xb = x + r * N + k * MX_BLOCK;
        float amax = 0.0f;
        for (int j = 0; j < MX_BLOCK; j++) {
            float a = fabsf(or_bf16_to_f32(xb[j]));
            if (a > amax) amax = a;
        }
        int ex = or_ue8m0_exponent(amax);               /* R4 */
        e[r * nb + k] = (uint8_t)(ex + 127);
        for (int j = 0; j < MX_BLOCK; j++) {
            /* x * 2^-e is exact in double; e4m3 rounds the exact value */
            double v = ldexp((double)or_bf16_to_f32(xb[j]), -ex);
            q[r * N + k * MX_BLOCK + j] = or_e4m3_encode(v);
        }
    }
    env_leave(env);
}

void or_mxfp8_dequant(const uint8_t* q, const uint8_t* e, int64_t B, int64_t M,
                      int64_t N, uint16_t* y) {
    fpenv_save env = env_enter();
    int64_t rows = B * M, nb = N / MX_BLOCK;
    for (int64_t r = 0; r < rows; r++)
    for (int64_t c = 0; c < N; c++) {
        int ex = (int)e[r * nb + c / MX_BLOCK] - 127;
        float p2 = ldexpf(1.0f, ex);                    /* 2^e, exact */
        float v = (float)or_e4m3_decode(q[r * N + c]) * p2;   /* fl(dec(q)*2^e) */
        y[r * N + c] = or_bf16_round(v);
    }
    env_leave(env);
}

/* ------------------------------------------------------------------ */
/* NVFP4, 1 x 16 blocks, E4M3 block scale, FP32 global scale            */
/*   [QAT] 2.3, 2.4, 3.3; [LPR] "Choose a precision" and "Modes" 4.      */
/* Layout: x dense [M][N] (N % 16 == 0); packed [M][N/2]; sb [M][N/16].  */
/* A group (one tensor, or q/k/v or gate/up siblings) shares amax A.     */
/* ------------------------------------------------------------------ */

#define NV_BLOCK 16

/* max |x| over n BF16 values */
float or_amax_bf16(const uint16_t* x, int64_t n) {
    float amax = 0.0f;
    for (int64_t i = 0; i < n; i++) {
        float a = fabsf(or_bf16_to_f32(x[i]));
        if (a > amax) amax = a;
    }
    return amax;
}

/* gs = fl(A / (6 * 448)); 6 * 448 = 2688 exactly. */
float or_nvfp4_global_scale(float group_amax) {
    fpenv_save env = env_enter();
    float gs = group_amax / 2688.0f;
    env_leave(env);
    return gs;
}

/* One 1x16 block whose amax is scaled to t (6 for NVFP4): the E4M3 scale
 * byte and the 16 codes (unpacked). */
static void nvfp4_block_to(const uint16_t* xb, float gs, float t, uint8_t* sb_out, uint8_t codes[NV_BLOCK]) {
    float amax_b = 0.0f;
    for (int j = 0; j < NV_BLOCK; j++) {
        float a = fabsf(or_bf16_to_f32(xb[j]));
        if (a > amax_b) amax_b = a;
    }
    uint8_t sb;
    if (gs == 0.0f) {
        sb = 0x00;                                      /* R3 */
    } else {
        float t_gs = t * gs;                            /* fl(t*gs) */
        float ratio = amax_b / t_gs;                    /* fl(amax_b/fl(t*gs)) */
        sb = or_e4m3_encode((double)ratio);             /* R5 (R20 for t = 4) */
    }
    *sb_out = sb;
    float d = (float)or_e4m3_decode(sb) * gs;          /* fl(dec(sb)*gs) */
    for (int j = 0; j < NV_BLOCK; j++) {
        float xv = or_bf16_to_f32(xb[j]);
        if (d == 0.0f) {
            codes[j] = signbit(xv) ? 0x8 : 0x0;         /* R6, R3 */
        } else {
            float quot = xv / d;                        /* fl(x/d) */
            codes[j] = or_e2m1_encode((double)quot);
        }
    }
}

static void nvfp4_block(const uint16_t* xb, float gs, uint8_t* sb_out, uint8_t codes[NV_BLOCK]) {
    nvfp4_block_to(xb, gs, 6.0f, sb_out, codes);
}

/* y = bf16(fl((dec(c) * dec(sb)) * gs)); the inner product is exact. */
static uint16_t nvfp4_value(uint8_t code, uint8_t sb, float gs) {
    float inner = (float)(or_e2m1_decode(code) * or_e4m3_decode(sb));  /* exact */
    float v = inner * gs;
    return or_bf16_round(v);
}

void or_nvfp4_quant(const uint16_t* x, int64_t M, int64_t N, float group_amax,
                    uint8_t* packed, uint8_t* sb) {
    fpenv_save env = env_enter();
    float gs = group_amax / 2688.0f;
    int64_t nb = N / NV_BLOCK;
    for (int64_t r = 0; r < M; r++)
    for (int64_t k = 0; k < nb; k++) {
        uint8_t codes[NV_BLOCK];
        nvfp4_block(x + r * N + k * NV_BLOCK, gs, &sb[r * nb + k], codes);
        for (int j = 0; j < NV_BLOCK; j += 2)          /* R8 */
            packed[r * (N / 2) + (k * NV_BLOCK + j) / 2] =
                (uint8_t)(codes[j] | (codes[j + 1] << 4));
    }
    env_leave(env);
}

void or_nvfp4_dequant(const uint8_t* packed, const uint8_t* sb, float gs,
                      int64_t M, int64_t N, uint16_t* y) {
    fpenv_save env = env_enter();
    int64_t nb = N / NV_BLOCK;
    for (int64_t r = 0; r < M; r++)
    for (int64_t c = 0; c < N; c++) {
        uint8_t byte = packed[r * (N / 2) + c / 2];
        uint8_t code = (c % 2 == 0) ? (byte & 0xf) : (byte >> 4);
        y[r * N + c] = nvfp4_value(code, sb[r * nb + c / NV_BLOCK], gs);
    }
    env_leave(env);
}

/* Fake-quant (QDQ): the dequantised value of each element's code, BF16. */
void or_nvfp4_fake_quant(const uint16_t* x, int64_t M, int64_t N, float group_amax,
                         uint16_t* y) {
    fpenv_save env = env_enter();
    float gs = group_amax / 2688.0f;
    int64_t nb = N / NV_BLOCK;
    for (int64_t r = 0; r < M; r++)
    for (int64_t k = 0; k < nb; k++) {
        uint8_t codes[NV_BLOCK], sbk;
        nvfp4_block(x + r * N + k * NV_BLOCK, gs, &sbk, codes);
        for (int j = 0; j < NV_BLOCK; j++)
            y[r * N + k * NV_BLOCK + j] = nvfp4_value(codes[j], sbk, gs);
    }
    env_leave(env);
}

/* ------------------------------------------------------------------ */
/* NVFP4 "4over6": each block is scaled so that its amax maps to 6 (the */
/* NVFP4 rule) or to 4, and keeps the one whose dequantised values are   */
/* closer to x; the global scale leaves room for the larger block scale  */
/* by using E = 256 as the E4M3 maximum.                                 */
/*   [PR503] NVFP4 QDQ config thread (NVTE_NVFP4_4OVER6,                  */
/*   NVTE_NVFP4_4OVER6_E4M3_USE_256 -> e4m3_max 256).  Readings R19-R21;  */
/*   PARITY UNPINNED against the pages (no selection rule there).         */
/* The output format is plain NVFP4: or_nvfp4_dequant reads it.          */
/* ------------------------------------------------------------------ */

/* R19: gs = fl(A / (6 * E)); 6 * 448 = 2688 and 6 * 256 = 1536 exactly. */
float or_nvfp4_4over6_global_scale(float group_amax, int e4m3_max) {
    fpenv_save env = env_enter();
    float gs = group_amax / (float)(6 * e4m3_max);
    env_leave(env);
    return gs;
}

/* R21: sum of squared differences of the block's values and its
 * dequantised values, left to right, every step one binary32 operation. */
static float nvfp4_block_err(const uint16_t* xb, const uint8_t codes[NV_BLOCK], uint8_t sb, float gs) {
    float err = 0.0f;
    for (int j = 0; j < NV_BLOCK; j++) {
        float d = or_bf16_to_f32(xb[j]) - or_bf16_to_f32(nvfp4_value(codes[j], sb, gs));
        float sq = d * d;
        err = err + sq;
    }
    return err;
}

/* One block under 4over6: the kept scale byte and codes; *choice = 4 or 6,
 * and the two errors when err6 / err4 are not NULL. */
static void nvfp4_4over6_block(const uint16_t* xb, float gs, uint8_t* sb_out, uint8_t codes[NV_BLOCK],
                               uint8_t* choice, float* err6, float* err4) {
    uint8_t sb6, sb4, c6[NV_BLOCK], c4[NV_BLOCK];
    nvfp4_block_to(xb, gs, 6.0f, &sb6, c6);                                 /* R20, t = 6 */
    nvfp4_block_to(xb, gs, 4.0f, &sb4, c4);                                 /* R20, t = 4 */
    float e6 = nvfp4_block_err(xb, c6, sb6, gs), e4 = nvfp4_block_err(xb, c4, sb4, gs);
    int four = e4 < e6;                                                     /* R21 */
    *sb_out = four ? sb4 : sb6;
    memcpy(codes, four ? c4 : c6, NV_BLOCK);
    if (choice) *choice = four ? 4 : 6;
    if (err6) *err6 = e6;
    if (err4) *err4 = e4;
}

/* x dense [M][N] (N % 16 == 0) with its group's amax A.  choice (optional,
 * [M][N/16]) receives 4 or 6 per block, err (optional, [M][N/16][2]) the
 * two errors (t = 6 first). */
void or_nvfp4_4over6_quant(const uint16_t* x, int64_t M, int64_t N, float group_amax, int e4m3_max,
                           uint8_t* packed, uint8_t* sb, uint8_t* choice, float* err) {
    fpenv_save env = env_enter();
    float gs = group_amax / (float)(6 * e4m3_max);
    int64_t nb = N / NV_BLOCK;
    for (int64_t r = 0; r < M; r++)
    for (int64_t k = 0; k < nb; k++) {
        uint8_t codes[NV_BLOCK];
        int64_t i = r * nb + k;
        nvfp4_4over6_block(x + r * N + k * NV_BLOCK, gs, &sb[i], codes, choice ? &choice[i] : NULL,
                           err ? &err[2 * i] : NULL, err ? &err[2 * i + 1] : NULL);
        for (int j = 0; j < NV_BLOCK; j += 2)          /* R8 */
            packed[r * (N / 2) + (k * NV_BLOCK + j) / 2] =
                (uint8_t)(codes[j] | (codes[j + 1] << 4));
    }
    env_leave(env);
}

void or_nvfp4_4over6_fake_quant(const uint16_t* x, int64_t M, int64_t N, float group_amax, int e4m3_max,
                                uint16_t* y) {
    fpenv_save env = env_enter();
    float gs = group_amax / (float)(6 * e4m3_max);
    int64_t nb = N / NV_BLOCK;
    for (int64_t r = 0; r < M; r++)
    for (int64_t k = 0; k < nb; k++) {
        uint8_t codes[NV_BLOCK], sbk;
        nvfp4_4over6_block(x + r * N + k * NV_BLOCK, gs, &sbk, codes, NULL, NULL, NULL);
        for (int j = 0; j < NV_BLOCK; j++)
            y[r * N + k * NV_BLOCK + j] = nvfp4_value(codes[j], sbk, gs);
    }
    env_leave(env);
}
