/*
 * far_oracle.c -- plain, slow fp64 CPU oracle for the fused
 * "all-reduce + residual-add + RMSNorm (+FP8-e4m3)" epilogue of a
 * row-parallel linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path loads this file:
 * only the test suite, the smoke check and the bench's CPU-baseline /
 * reference legs call it.  It shares no code, header, table or constant
 * generator with the CUDA library; the two meet only through the seeded
 * input generator, which holds none of the method's arithmetic.
 *
 * Sources (web pages, cited by title and section):
 *  [P1] vllm.models.common.ops.fused_allreduce_rms_norm -- docstring of
 *       fused_allreduce_rms_norm: the result is (normed_output, new_residual),
 *       the same as norm(all_reduce(hidden_states), residual); the partials are
 *       the per-rank outputs of a row-parallel linear; the call passes
 *       weight_bias=0.0 for standard RMSNorm ("Gemma would use 1.0"),
 *       fp32_acc=True and rms_eps=norm.variance_epsilon.  With one rank the
 *       call is the plain norm(hidden_states, residual).
 *  [P2] vllm.compilation.sequence_parallelism -- SequenceParallelismPass
 *       docstring: AllReduce -> RMSNorm becomes ReduceScatter -> local RMSNorm
 *       -> AllGather, so the result restricted to a block of rows only depends
 *       on those rows.  "First" patterns have no residual input and return the
 *       all-reduce itself as the next residual.
 *  [P4] vllm.compilation.fusion -- FusedAddRMSNormStaticQuantPattern (static
 *       per-tensor FP8 after fused add+RMSNorm, fp32 scale tensor) and
 *       FusedAddRMSNormDynamicQuantPattern (dynamic per-token FP8, returns
 *       result, residual and one scale per token; scale_ub=None); the QuantKey
 *       constants kFp8StaticTensorSym / kFp8DynamicTokenSym (symmetric).
 *       The same page lists kFp8DynamicTensorSym (dynamic, per-tensor,
 *       symmetric) among the quantisation keys, with no fused op: one scale
 *       for the whole tensor, amax / 448 over every element.
 *  [P3] vllm.distributed.device_communicators.aiter_custom_all_reduce --
 *       build_supports_per_group_quant: a fused all-reduce + RMSNorm +
 *       per-group quantisation exists; the page gives no group shape.
 *  [P5] PR #45307 report -- signature of call_trtllm_fused_allreduce_norm:
 *       norm_out, quant_out, scale_out and scale_factor are all optional.
 *
 * RMSNorm itself is the textbook definition (Zhang & Sennrich, 2019):
 * x / sqrt(mean(x^2) + eps) * weight, the mean taken over the hidden size and
 * eps inside the square root (the pages' "variance_epsilon").
 *
 * Number formats are decoded and encoded from their published definitions:
 * bfloat16 (1-8-7, bias 127), IEEE-754 binary16 (1-5-10, bias 15), and OCP
 * FP8 E4M3 "fn" (1-4-3, bias 7, max finite 448, NaN = S.1111.111, no
 * infinities).  Rounding is to nearest, ties to even, done with nearbyint()
 * in the default rounding mode.
 *
 * Readings where the pages are silent (each one is stated in the project's
 * design notes as well):
 *  - the partial sum is not rounded to the model dtype before the residual
 *    add (fp32_acc=True), and the norm reads that unrounded sum;
 *  - gamma + weight_bias is not rounded to the model dtype;
 *  - the FP8 code is decided in fp32, the precision of the pages' fp32 scale
 *    tensor and fp32 accumulation: the fp64 value o is rounded to fp32, divided
 *    by the fp32 scale with one correct rounding to fp32, then encoded;
 *  - FP8 encoding saturates to +-448 (e4m3fn has no infinity);
 *  - a dynamic row whose fp32 scale is 0 gets scale 0 and all codes 0x00;
 *    NaN elements take no part in a row's amax;
 *  - dynamic per-tensor FP8 takes its amax over the rows of the call
 *    ([row_begin, row_end)) and writes the one scale to scale_out[0];
 *  - per-group FP8: groups of `group` consecutive hidden elements of a row
 *    (group divides H), one scale per (row, group) = amax / 448 at
 *    scale_out[t * (H / group) + h / group].
 */
#include <float.h>
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>

/* Own copies of the enumerations; numbering follows the library's public
 * interface so that callers can pass the same integers to both. */
enum { OR_BF16 = 0, OR_FP16 = 1 };
enum { OR_AR_RESIDUAL_RMSNORM = 0, OR_FP8_STATIC = 1, OR_FP8_TOKEN = 2, OR_FP8_TENSOR = 3,
       OR_FP8_GROUP = 4 };

/* ---------------------------------------------------------------------- */
/* 16-bit floating formats                                                 */
/* ---------------------------------------------------------------------- */

typedef struct {
    int mbits; /* stored fraction bits            */
    int ebits; /* exponent field width            */
    int bias;
    int emin;  /* exponent of the smallest normal */
    int emax;  /* exponent of the largest binade  */
} fmt16;

static fmt16 fmt_of(int dtype)
{
    fmt16 f;
    if (dtype == OR_BF16) {
        f.mbits = 7; f.ebits = 8; f.bias = 127; f.emin = -126; f.emax = 127;
    } else {
        f.mbits = 10; f.ebits = 5; f.bias = 15; f.emin = -14; f.emax = 15;
    }
    return f;
}

/* Value of a 16-bit pattern, exactly, as a double. */
double far_oracle_decode16(uint16_t bits, int dtype)
{
    fmt16 f = fmt_of(dtype);
    int sign = (bits >> 15) & 1;
    int E = (bits >> f.mbits) & ((1 << f.ebits) - 1);
    int M = bits & ((1 << f.mbits) - 1);
    double v;
    if (E == (1 << f.ebits) - 1) {
        v = (M == 0) ? INFINITY : NAN;
    } else if (E == 0) {
        v = ldexp((double)M, f.emin - f.mbits); /* subnormal: M * 2^(emin-mbits) */
    } else {
        v = ldexp(1.0 + ldexp((double)M, -f.mbits), E - f.bias);
    }
    return sign ? -v : v;
}

/* Round a double to the nearest value of the 16-bit format (ties to even),
 * overflowing to infinity, keeping subnormals; return its bit pattern. */
uint16_t far_oracle_round16(double x, int dtype)
{
    fmt16 f = fmt_of(dtype);
    uint16_t sign = signbit(x) ? (uint16_t)0x8000u : (uint16_t)0;
    uint16_t exp_ones = (uint16_t)(((1u << f.ebits) - 1u) << f.mbits);
    if (isnan(x))
        return (uint16_t)(sign | exp_ones | (1u << (f.mbits - 1)));
    double a = fabs(x);
    if (isinf(a))
        return (uint16_t)(sign | exp_ones);
    if (a == 0.0)
        return sign;

    int e;
    frexp(a, &e);          /* a = m * 2^e, m in [0.5, 1): binade exponent e-1 */
    int be = e - 1;
    if (be < f.emin)
        be = f.emin;       /* below the normal range the spacing is fixed */
    double quantum = ldexp(1.0, be - f.mbits);
    double v = nearbyint(a / quantum) * quantum; /* a/quantum is exact */

    double maxfinite = ldexp(2.0 - ldexp(1.0, -f.mbits), f.emax);
    if (v > maxfinite)
        return (uint16_t)(sign | exp_ones);
    if (v == 0.0)
        return sign;

    int ve;
    frexp(v, &ve);
    int vbe = ve - 1;
    if (vbe < f.emin) {
        uint16_t M = (uint16_t)(v / ldexp(1.0, f.emin - f.mbits));
        return (uint16_t)(sign | M);
    }
    uint16_t E = (uint16_t)(vbe + f.bias);
    uint16_t M = (uint16_t)((v / ldexp(1.0, vbe) - 1.0) * ldexp(1.0, f.mbits));
    return (uint16_t)(sign | (uint16_t)(E << f.mbits) | M);
}

/* ---------------------------------------------------------------------- */
/* OCP FP8 E4M3 (fn variant)                                               */
/* ---------------------------------------------------------------------- */

/* Value of an e4m3fn code. */
double far_oracle_e4m3_decode(uint8_t code)
{
    int sign = (code >> 7) & 1;
    int E = (code >> 3) & 0xF;
    int M = code & 0x7;
    double v;
    if (E == 0xF && M == 0x7)
        v = NAN;                              /* the only NaN pattern */
    else if (E == 0)
        v = ldexp((double)M, -9);             /* subnormal: M * 2^-6 / 8 */
    else
        v = ldexp(1.0 + M / 8.0, E - 7);
    return sign ? -v : v;
}

/* Encode a double as e4m3fn: round to nearest, ties to even, saturate to
 * +-448, NaN to 0x7F. */
uint8_t far_oracle_e4m3_encode(double x)
{
    if (isnan(x))
        return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs(x);
    if (a >= 448.0)
        return (uint8_t)(sign | 0x7E);        /* S.1111.110 = 448 */
    if (a == 0.0)
        return sign;

    int e;
    frexp(a, &e);
    int be = e - 1;
    if (be < -6)
        be = -6;                               /* subnormal spacing 2^-9 */
    double quantum = ldexp(1.0, be - 3);
    double v = nearbyint(a / quantum) * quantum;
    if (v > 448.0)
        v = 448.0;                             /* not reachable for a < 448 */
    if (v == 0.0)
        return sign;

    int ve;
    frexp(v, &ve);
    int vbe = ve - 1;
    if (vbe < -6)
        return (uint8_t)(sign | (uint8_t)(v / ldexp(1.0, -9)));
    uint8_t E = (uint8_t)(vbe + 7);
    uint8_t M = (uint8_t)((v / ldexp(1.0, vbe) - 1.0) * 8.0);
    return (uint8_t)(sign | (uint8_t)(E << 3) | M);
}

/* Round to fp32 (C's double -> float conversion: to nearest, ties to even). */
static double to_f32(double x) { return (double)(float)x; }

/* ---------------------------------------------------------------------- */
/* The fused epilogue                                                      */
/* ---------------------------------------------------------------------- */

/* The fp32 accumulation below needs float arithmetic evaluated in float. */
#if !defined(FLT_EVAL_METHOD) || FLT_EVAL_METHOD != 0
#error "the fp32 accumulation mode needs FLT_EVAL_METHOD == 0"
#endif

/* Row t: y = sum of the partials (+ residual) and o = y * rinv * (gamma +
 * weight_bias), both in fp64 into y[H] and o[H]; returns rinv.
 *
 * acc32 = 0: the sum is exact (fp64 holds the sum of these 2-byte values
 * exactly while their exponents span less than 45 binades).
 * acc32 = 1: the pages' fp32_acc=True taken literally [P1]: partial 0, 1,
 * ..., W-1, then the residual, added one after another to an fp32 sum that
 * starts at 0, each addition rounded to fp32 (to nearest, ties to even).
 * The two differ only where a rounded running sum is followed by
 * cancellation; everything after y is fp64 in both. */
static double row_y_o(const uint16_t *const *partials, int W, const uint16_t *residual,
                      const uint16_t *gamma, int64_t t, int64_t H, int dtype,
                      float eps, float weight_bias, int acc32, double *y, double *o)
{
    const int64_t base = t * H;
    /* 1. all-reduce of the partials, then 2. the residual add [P1] */
    for (int64_t h = 0; h < H; ++h) {
        if (acc32) {
            float s = 0.0f; /* 2-byte values convert to float exactly */
            for (int r = 0; r < W; ++r)
                s = s + (float)far_oracle_decode16(partials[r][base + h], dtype);
            if (residual != NULL)
                s = s + (float)far_oracle_decode16(residual[base + h], dtype);
            y[h] = (double)s;
        } else {
            double s = 0.0;
            for (int r = 0; r < W; ++r)
                s += far_oracle_decode16(partials[r][base + h], dtype);
            if (residual != NULL)
                s += far_oracle_decode16(residual[base + h], dtype);
            y[h] = s;
        }
    }
    /* 3. mean of squares over the hidden size, eps inside the root */
    double ss = 0.0;
    for (int64_t h = 0; h < H; ++h)
        ss += y[h] * y[h];
    double ms = ss / (double)H;
    double rinv = 1.0 / sqrt(ms + (double)eps); /* fp32 eps, promoted */
    /* 4. scale by rinv and by (gamma + weight_bias) [P1] */
    for (int64_t h = 0; h < H; ++h) {
        double g = far_oracle_decode16(gamma[h], dtype) + (double)weight_bias;
        o[h] = y[h] * rinv * g;
    }
    return rinv;
}

/*
 * Rows [row_begin, row_end) of a (T, H) problem; all arrays are row-major
 * with row stride H and are indexed by the absolute row.
 *
 *   partials[r]   W arrays of 16-bit patterns (the ranks' partial outputs)
 *   residual      16-bit patterns, or NULL ("First" pattern: no residual)
 *   gamma         H 16-bit patterns
 *   residual_out  receives round(y); may be NULL
 *   norm_out      receives round(o); may be NULL
 *   quant_out     receives e4m3 codes (patterns 1, 2); may be NULL
 *   scale_in      static per-tensor scale (pattern 1)
 *   scale_out     per-row fp32 scale (pattern 2), indexed by absolute row,
 *                 or the one per-tensor scale in scale_out[0] (pattern 3),
 *                 or T x (H / group) per-group scales, row-major (pattern 4)
 *   group         elements per quantisation group (pattern 4)
 *   y_dbg, o_dbg  optional fp64 copies of y and o (T*H each)
 *   rinv_dbg      optional fp64 1/sqrt(ms+eps) per row (T)
 *
 * Returns 0, or -1 for arguments it cannot interpret.
 */
static int fused_impl(const uint16_t *const *partials, int W,
                      const uint16_t *residual, const uint16_t *gamma,
                      int64_t T, int64_t H, int dtype,
                      float eps, float weight_bias, int pattern, int64_t group,
                      int64_t row_begin, int64_t row_end, int acc32,
                      uint16_t *residual_out, uint16_t *norm_out,
                      uint8_t *quant_out, const float *scale_in,
                      float *scale_out,
                      double *y_dbg, double *o_dbg, double *rinv_dbg)
{
    if (W < 1 || H < 1 || T < 0 || row_begin < 0 || row_end > T ||
        row_begin > row_end)
        return -1;
    if (dtype != OR_BF16 && dtype != OR_FP16)
        return -1;
    if (pattern == OR_FP8_STATIC && (quant_out == NULL || scale_in == NULL))
        return -1;
    if ((pattern == OR_FP8_TOKEN || pattern == OR_FP8_TENSOR || pattern == OR_FP8_GROUP) &&
        (quant_out == NULL || scale_out == NULL))
        return -1;
    if (pattern == OR_FP8_GROUP && (group < 1 || H % group != 0))
        return -1;

    /* one row of y and o at a time, in fp64 */
    double *y = (double *)malloc((size_t)H * sizeof(double));
    double *o = (double *)malloc((size_t)H * sizeof(double));
    if (y == NULL || o == NULL) {
        free(y);
        free(o);
        return -1;
    }

    /* dynamic per-tensor FP8: a first pass over the rows for the amax */
    double tensor_scale = 0.0;
    if (pattern == OR_FP8_TENSOR) {
        double amax = 0.0;
        for (int64_t t = row_begin; t < row_end; ++t) {
            row_y_o(partials, W, residual, gamma, t, H, dtype, eps, weight_bias, acc32, y, o);
            for (int64_t h = 0; h < H; ++h) {
                double a = fabs(to_f32(o[h]));
                if (a > amax) /* a NaN element does not take part */
                    amax = a;
            }
        }
        tensor_scale = to_f32(amax / 448.0);
        scale_out[0] = (float)tensor_scale;
    }

    for (int64_t t = row_begin; t < row_end; ++t) {
        const int64_t base = t * H;
        const double rinv = row_y_o(partials, W, residual, gamma, t, H, dtype, eps,
                                    weight_bias, acc32, y, o);

        if (residual_out != NULL)
            for (int64_t h = 0; h < H; ++h)
                residual_out[base + h] = far_oracle_round16(y[h], dtype);
        if (norm_out != NULL)
            for (int64_t h = 0; h < H; ++h)
                norm_out[base + h] = far_oracle_round16(o[h], dtype);

        /* 5a. static per-tensor FP8 [P4 FusedAddRMSNormStaticQuantPattern] */
        if (pattern == OR_FP8_STATIC) {
            double s32 = to_f32((double)scale_in[0]);
            for (int64_t h = 0; h < H; ++h)
                quant_out[base + h] = far_oracle_e4m3_encode(to_f32(to_f32(o[h]) / s32));
        }

        /* 5b. dynamic per-token FP8 [P4 FusedAddRMSNormDynamicQuantPattern]:
         * scale = amax / 448, the largest |o| then maps onto the largest code */
        if (pattern == OR_FP8_TOKEN) {
            double amax = 0.0;
            for (int64_t h = 0; h < H; ++h) {
                double a = fabs(to_f32(o[h]));
                if (a > amax) /* a NaN element does not take part */
                    amax = a;
            }
            double scale = to_f32(amax / 448.0);
            scale_out[t] = (float)scale;
            for (int64_t h = 0; h < H; ++h) {
                if (scale == 0.0)
                    quant_out[base + h] = 0x00;
                else
                    quant_out[base + h] = far_oracle_e4m3_encode(to_f32(to_f32(o[h]) / scale));
            }
        }

        /* 5d. per-group FP8 [P3 per-group quant]: each group of `group`
         * consecutive elements has its own scale, amax / 448 */
        if (pattern == OR_FP8_GROUP) {
            const int64_t ngroups = H / group;
            for (int64_t q = 0; q < ngroups; ++q) {
                double amax = 0.0;
                for (int64_t h = q * group; h < (q + 1) * group; ++h) {
                    double a = fabs(to_f32(o[h]));
                    if (a > amax) /* a NaN element does not take part */
                        amax = a;
                }
                double scale = to_f32(amax / 448.0);
                scale_out[t * ngroups + q] = (float)scale;
                for (int64_t h = q * group; h < (q + 1) * group; ++h) {
                    if (scale == 0.0)
                        quant_out[base + h] = 0x00;
                    else
                        quant_out[base + h] = far_oracle_e4m3_encode(to_f32(to_f32(o[h]) / scale));
                }
            }
        }

        /* 5c. dynamic per-tensor FP8 [P4 kFp8DynamicTensorSym]: the one
         * scale of the first pass */
        if (pattern == OR_FP8_TENSOR) {
            for (int64_t h = 0; h < H; ++h) {
                if (tensor_scale == 0.0)
                    quant_out[base + h] = 0x00;
                else
                    quant_out[base + h] = far_oracle_e4m3_encode(to_f32(to_f32(o[h]) / tensor_scale));
            }
        }

        if (y_dbg != NULL)
            for (int64_t h = 0; h < H; ++h)
                y_dbg[base + h] = y[h];
        if (o_dbg != NULL)
            for (int64_t h = 0; h < H; ++h)
                o_dbg[base + h] = o[h];
        if (rinv_dbg != NULL)
            rinv_dbg[t] = rinv;
    }

    free(y);
    free(o);
    return 0;
}

int far_oracle_fused(const uint16_t *const *partials, int W,
                     const uint16_t *residual, const uint16_t *gamma,
                     int64_t T, int64_t H, int dtype,
                     float eps, float weight_bias, int pattern, int64_t group,
                     int64_t row_begin, int64_t row_end,
                     uint16_t *residual_out, uint16_t *norm_out,
                     uint8_t *quant_out, const float *scale_in,
                     float *scale_out,
                     double *y_dbg, double *o_dbg, double *rinv_dbg)
{
    return fused_impl(partials, W, residual, gamma, T, H, dtype, eps, weight_bias, pattern,
                      group, row_begin, row_end, 0, residual_out, norm_out, quant_out,
                      scale_in, scale_out, y_dbg, o_dbg, rinv_dbg);
}

/* The same with the partials and the residual accumulated in fp32 (acc32,
 * see row_y_o): the reference for the elements where fp32 accumulation,
 * which the pages prescribe, is not exact. */
int far_oracle_fused_acc32(const uint16_t *const *partials, int W,
                           const uint16_t *residual, const uint16_t *gamma,
                           int64_t T, int64_t H, int dtype,
                           float eps, float weight_bias, int pattern, int64_t group,
                           int64_t row_begin, int64_t row_end,
                           uint16_t *residual_out, uint16_t *norm_out,
                           uint8_t *quant_out, const float *scale_in,
                           float *scale_out,
                           double *y_dbg, double *o_dbg, double *rinv_dbg)
{
    return fused_impl(partials, W, residual, gamma, T, H, dtype, eps, weight_bias, pattern,
                      group, row_begin, row_end, 1, residual_out, norm_out, quant_out,
                      scale_in, scale_out, y_dbg, o_dbg, rinv_dbg);
}
