/*
 * sage_oracle.c -- CPU oracle for SageAttention-style quantized attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is a plain, slow, single-threaded
 * restatement of what the quantized attention path computes, written in C
 * with fp64 wherever the method does not fix a precision.  Only the tests,
 * the package's smoke check and the bench's CPU-baseline leg may load it.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * Sources (web pages on the subject; cited by title and section):
 *   [SV2]   "Sage v2 improvements" (xDiT pull request 665): the Hadamard
 *           matrix is built once and reused; inputs need not be contiguous.
 *   [SA3]   "sage_attn3" (FastVideo SageAttention3Impl API page): [B,H,L,D]
 *           inputs, causal flag, softmax_scale.
 *   [PA]    "[FlyDSL] [Misc] pa_decode: key the tile kernel on FlyDSL dtypes
 *           and drop the batch-first plan grid" (AITER pull request 7388):
 *           Changes (FP8_MAX is the finfo max of the format Q/P are
 *           quantized to; the epilogue multiplies by 1/FP8_MAX), PR
 *           Self-Review (FP8_MAX 448 for OCP e4m3), window-family results
 *           (per-token FP8 K/V, sliding window, MTP4).
 *   [DSV4]  "perf(dsv4): qproj wq_b transpose + serving contract;
 *           sparse_attn/indexer tuning" (pypto-lib pull request 676):
 *           sequence diagram -- Hadamard transform, per-head amax,
 *           dequant scale, INT8 rows.
 *   [S2TP]  "Sage2 SM89 Temporal Pair Experiment", section Candidate: the
 *           per-tile sequence QK -> update_mdo -> accumulate_d ->
 *           RS_32_to_8 -> PV with per-row running max m and denominator d.
 *
 * Readings taken where the pages are silent (each one is restated in the
 * function that uses it):
 *   - only K is smoothed (its per-(b,h) mean over the sequence, summed in
 *     fp64 in token order, divided by L in fp64, rounded once to fp32);
 *   - smooth, then rotate by the unnormalised Sylvester Hadamard matrix
 *     (H H^T = D I) with an fp32 butterfly whose stages run h = 1,2,..,D/2;
 *     the 1/D this leaves in Q.K^T is folded into the logit scale;
 *   - INT8 per token block: s = a/127, r = 127/a (two IEEE fp32 divides),
 *     code = clamp(rint_even(x*r), -127, 127); a = 0 gives s = 0, codes 0;
 *   - V per channel: s = a/448, r = 448/a, code = e4m3_rne_satfinite(v*r);
 *   - attention in 128-key tiles, in ascending order, fp64 throughout
 *     except the method's own e4m3 rounding of P*448; the denominator sums
 *     the unquantised probabilities; out = bf16_rne(O*vs/(448*d));
 *   - causal mask is bottom-right aligned: key j is visible to query i iff
 *     j <= i + (Lk - Lq); a row that sees no key outputs zeros.
 *   - the MXFP4 variant ([SV2] changelog: fav3_sage_mxfp4 with a Hadamard
 *     block BLOCK_R = 128, i.e. the whole head for D <= 128; [PA]: MXFP4 is
 *     packed E2M1 with float8_e8m0fnu scales, and Q / P use E4M3 as their
 *     FP8 format): Q and K (K smoothed as above) are rotated, then quantised
 *     per row in blocks of 32 consecutive elements to E2M1 codes with one
 *     power-of-two scale 2^E each, E = floor(log2(amax)) - 2 (the OCP MX
 *     rule: the largest E2M1 value 6 has exponent 2), codes
 *     e2m1_rne_satfinite(x * 2^-E); QK^T over the dequantised values, then
 *     the same per-tile softmax, e4m3 P and FP8 V as above.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_KEY_TILE 128

/* ------------------------------------------------------------------ */
/* Number formats                                                      */
/* ------------------------------------------------------------------ */

/* bf16 is the top half of an IEEE binary32; widening is exact. */
float or_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a double to bf16 (8-bit significand, binary32 exponent range),
 * round-to-nearest-even, overflow to infinity. Computed directly from the
 * double so there is a single rounding. */
uint16_t or_f64_to_bf16(double x)
{
    if (isnan(x)) return 0x7FC0;
    int neg = signbit(x) ? 1 : 0;
    double ax = fabs(x);
    double y;
    if (ax == 0.0) {
        y = 0.0;
    } else if (ax < 0x1p-126) {
        /* bf16 subnormals are multiples of 2^-133 */
        y = nearbyint(ax * 0x1p133) * 0x1p-133;
    } else {
        int e;
        double m = frexp(ax, &e);             /* ax = m * 2^e, m in [0.5, 1) */
        y = ldexp(nearbyint(ldexp(m, 8)), e - 8);
    }
    uint16_t bits;
    if (y > 0x1.FEp127) {
        bits = 0x7F80;                        /* +inf */
    } else {
        float f = (float)y;                   /* exact: y has <= 8 significant bits */
        uint32_t u;
        memcpy(&u, &f, sizeof u);
        bits = (uint16_t)(u >> 16);
    }
    return (uint16_t)(bits | (neg ? 0x8000 : 0));
}

/* OCP FP8 E4M3 (e4m3fn): 1 sign bit, 4 exponent bits with bias 7, 3
 * mantissa bits, no infinities, S.1111.111 is NaN, largest finite 448 (the
 * FP8_MAX the FlyDSL decode page quotes for OCP e4m3). Value of a
 * non-negative code c (0..126): exponent field e = c >> 3, mantissa m = c & 7;
 *   e == 0 : m * 2^-9              (subnormal)
 *   e >  0 : (8 + m) * 2^(e - 10)  (= (1 + m/8) * 2^(e - 7))            */
double or_e4m3_decode(uint8_t code)
{
    int c = code & 0x7F;
    if (c == 0x7F) return NAN;
    int e = c >> 3, m = c & 7;
    double v = (e == 0) ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
    return (code & 0x80) ? -v : v;
}

/* Round to the nearest e4m3 value, ties to the even code, saturating any
 * magnitude at or beyond 448 to 448 (the "satfinite" behaviour); NaN maps
 * to the NaN code. The sign is kept, so tiny negatives become -0 (0x80). */
uint8_t or_e4m3_encode(double x)
{
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double ax = fabs(x);
    if (ax >= 448.0) return (uint8_t)(sign | 0x7E);
    /* largest non-negative code whose value is <= ax (codes are ordered) */
    int lo = 0, hi = 0x7E;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (or_e4m3_decode((uint8_t)mid) <= ax) lo = mid; else hi = mid - 1;
    }
    int c = lo;
    double vc = or_e4m3_decode((uint8_t)c);
    if (vc != ax) {
        double vn = or_e4m3_decode((uint8_t)(c + 1));
        double twice = 2.0 * ax, sum = vc + vn;     /* both exact */
        if (twice > sum) c = c + 1;
        else if (twice == sum && (c & 1)) c = c + 1;
    }
    return (uint8_t)(sign | c);
}

/* ------------------------------------------------------------------ */
/* Hadamard rotation ([SV2]: built once and reused)                    */
/* ------------------------------------------------------------------ */

/* Sylvester construction: H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]].
 * Fills h[D*D] (row-major) with +-1. D must be a power of two. */
int or_hadamard(int D, int32_t* h)
{
    if (D < 1 || (D & (D - 1))) return -1;
    h[0] = 1;
    for (int n = 1; n < D; n *= 2) {
        for (int i = 0; i < n; ++i)
            for (int j = 0; j < n; ++j) {
                int32_t v = h[i * D + j];
                h[i * D + (j + n)] = v;
                h[(i + n) * D + j] = v;
                h[(i + n) * D + (j + n)] = -v;
            }
    }
    return 0;
}

/* In-place fp32 Walsh-Hadamard butterfly: for stages h = 1, 2, ..., D/2 and
 * each pair (j, j+h) inside a 2h-block, (x_j, x_{j+h}) <- (x_j + x_{j+h},
 * x_j - x_{j+h}), each one IEEE binary32 round-to-nearest operation. In
 * exact arithmetic the result is x * H_D (H symmetric), unnormalised. */
void or_fwht_f32(float* x, int D)
{
    for (int h = 1; h < D; h *= 2)
        for (int i = 0; i < D; i += 2 * h)
            for (int j = i; j < i + h; ++j) {
                float a = x[j], b = x[j + h];
                x[j] = a + b;
                x[j + h] = a - b;
            }
}

/* Rows of a matrix, one call per row. */
void or_fwht_rows_f32(float* x, int64_t rows, int D)
{
    for (int64_t r = 0; r < rows; ++r) or_fwht_f32(x + r * D, D);
}

/* OCP MX FP4 E2M1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit,
 * no infinities or NaN. Magnitudes of codes 0..7: 0, 0.5 (subnormal), 1,
 * 1.5, 2, 3, 4, 6; bit 3 is the sign. */
double or_e2m1_decode(uint8_t code)
{
    static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    const double v = mag[code & 7];
    return (code & 8) ? -v : v;
}

/* Round to the nearest E2M1 value, ties to the even code, magnitudes at or
 * beyond 6 saturate to 6 ("satfinite"); the sign is kept (-0 -> 0x8). */
uint8_t or_e2m1_encode(double x)
{
    const uint8_t sign = signbit(x) ? 8 : 0;
    const double ax = fabs(x);
    if (ax >= 6.0) return (uint8_t)(sign | 7);
    int c = 0;                                    /* largest code with value <= ax */
    while (c < 7 && or_e2m1_decode((uint8_t)(c + 1)) <= ax) ++c;
    if (c < 7) {
        const double lo = or_e2m1_decode((uint8_t)c), hi = or_e2m1_decode((uint8_t)(c + 1));
        const double mid = 0.5 * (lo + hi);
        if (ax > mid || (ax == mid && (c & 1))) ++c;
    }
    return (uint8_t)(sign | c);
}

/* ------------------------------------------------------------------ */
/* K smoothing statistic                                               */
/* ------------------------------------------------------------------ */

/* mean[d] = (float)( (sum_{l=0..L-1} (double)k[l][d]) / (double)L ),
 * the fp64 sum taken in token order. k is one (b,h) slice, [L][D]. */
void or_k_mean(const uint16_t* k, int L, int D, float* mean)
{
    for (int d = 0; d < D; ++d) {
        double s = 0.0;
        for (int l = 0; l < L; ++l) s += (double)or_bf16_to_f32(k[(int64_t)l * D + d]);
        mean[d] = (float)(s / (double)L);
    }
}

/* ------------------------------------------------------------------ */
/* INT8 quantisation of Q or K ([DSV4] sequence: rotate, amax, scale)  */
/* ------------------------------------------------------------------ */

/* One (b,h) slice x[L][D] (bf16). If mean is not NULL it is subtracted
 * first (fp32). Each row is rotated with or_fwht_f32. Token blocks of blk
 * rows (the last one short) get one absmax scale each:
 *   a = max |x_hat| over the block, s = a / 127, r = 127 / a,
 *   code = clamp(rint_even(x_hat * r), -127, 127); a == 0 -> s = 0, codes 0.
 * Output codes[Lpad][D] (rows L..Lpad-1 zero), scales[ceil(L/blk)]. */
void or_quant_i8_head(const uint16_t* x, const float* mean, int L, int D, int blk,
                      int Lpad, int8_t* codes, float* scales)
{
    float* rot = (float*)malloc(sizeof(float) * (size_t)L * (size_t)D);
    for (int l = 0; l < L; ++l) {
        float* row = rot + (int64_t)l * D;
        for (int d = 0; d < D; ++d) {
            float v = or_bf16_to_f32(x[(int64_t)l * D + d]);
            if (mean) v = v - mean[d];
            row[d] = v;
        }
        or_fwht_f32(row, D);
    }
    int nb = (L + blk - 1) / blk;
    for (int b = 0; b < nb; ++b) {
        int r0 = b * blk, r1 = r0 + blk < L ? r0 + blk : L;
        float a = 0.0f;
        for (int l = r0; l < r1; ++l)
            for (int d = 0; d < D; ++d) {
                float v = fabsf(rot[(int64_t)l * D + d]);
                if (v > a) a = v;
            }
        if (a == 0.0f) {
            scales[b] = 0.0f;
            for (int l = r0; l < r1; ++l)
                for (int d = 0; d < D; ++d) codes[(int64_t)l * D + d] = 0;
            continue;
        }
        float s = a / 127.0f;
        float r = 127.0f / a;
        scales[b] = s;
        for (int l = r0; l < r1; ++l)
            for (int d = 0; d < D; ++d) {
                float y = rot[(int64_t)l * D + d] * r;
                float q = nearbyintf(y);
                if (q > 127.0f) q = 127.0f;
                if (q < -127.0f) q = -127.0f;
                codes[(int64_t)l * D + d] = (int8_t)q;
            }
    }
    for (int l = L; l < Lpad; ++l)
        for (int d = 0; d < D; ++d) codes[(int64_t)l * D + d] = 0;
    free(rot);
}

/* ------------------------------------------------------------------ */
/* MXFP4 quantisation of Q or K ([SV2] fav3_sage_mxfp4, [PA] MXFP4)    */
/* ------------------------------------------------------------------ */

/* One (b,h) slice x[L][D] (bf16). If mean is not NULL it is subtracted
 * first (fp32); each row is rotated with or_fwht_f32. Per row and block of
 * 32 consecutive elements:
 *   a = max |x_hat| over the block (fp32);
 *   E = floor(log2(a)) - 2, clamped to [-127, 127]; a == 0 gives E = -127;
 *   code = e2m1(x_hat * 2^-E) (a scaling by a power of two: exact);
 *   scale byte = E + 127 (e8m0: the value 2^E).
 * Output codes[Lpad][D/2], element 2i in the low nibble of byte i (rows
 * L..Lpad-1 zero), sf[Lpad][D/32] (rows L..Lpad-1 zero). */
void or_quant_mxfp4_head(const uint16_t* x, const float* mean, int L, int D, int Lpad,
                         uint8_t* codes, uint8_t* sf)
{
    float* row = (float*)malloc(sizeof(float) * (size_t)D);
    const int nb = D / 32;
    memset(codes, 0, (size_t)Lpad * (size_t)(D / 2));
    memset(sf, 0, (size_t)Lpad * (size_t)nb);
    for (int l = 0; l < L; ++l) {
        for (int d = 0; d < D; ++d) {
            float v = or_bf16_to_f32(x[(int64_t)l * D + d]);
            if (mean) v = v - mean[d];
            row[d] = v;
        }
        or_fwht_f32(row, D);
        for (int b = 0; b < nb; ++b) {
            float a = 0.0f;
            for (int e = 0; e < 32; ++e) {
                float v = fabsf(row[32 * b + e]);
                if (v > a) a = v;
            }
            int E = -127;
            if (a > 0.0f) {
                int ex;
                frexp((double)a, &ex);            /* a = f * 2^ex, f in [0.5, 1) */
                E = (ex - 1) - 2;                 /* floor(log2(a)) - 2 */
                if (E < -127) E = -127;
                if (E > 127) E = 127;
            }
            sf[(int64_t)l * nb + b] = (uint8_t)(E + 127);
            for (int e = 0; e < 32; ++e) {
                const int d = 32 * b + e;
                const uint8_t c = (a > 0.0f) ? or_e2m1_encode(ldexp((double)row[d], -E)) : 0;
                codes[(int64_t)l * (D / 2) + d / 2] |= (uint8_t)((d & 1) ? (c << 4) : c);
            }
        }
    }
    free(row);
}

/* ------------------------------------------------------------------ */
/* FP8 quantisation of V (per channel; [S2TP] kernel fuses a V scale)  */
/* ------------------------------------------------------------------ */

/* One (b,h) slice v[L][D] (bf16). Per channel d: a = max_l |v|,
 * s = a / 448, r = 448 / a, code = e4m3(v * r) with the product rounded to
 * fp32 first; a == 0 -> s = 0, codes 0. Output transposed: v8t[D][Lpad]
 * (columns L..Lpad-1 zero), scales[D]. */
void or_quant_v_head(const uint16_t* v, int L, int D, int Lpad, uint8_t* v8t, float* scales)
{
    for (int d = 0; d < D; ++d) {
        float a = 0.0f;
        for (int l = 0; l < L; ++l) {
            float x = fabsf(or_bf16_to_f32(v[(int64_t)l * D + d]));
            if (x > a) a = x;
        }
        uint8_t* dst = v8t + (int64_t)d * Lpad;
        if (a == 0.0f) {
            scales[d] = 0.0f;
            for (int l = 0; l < Lpad; ++l) dst[l] = 0;
            continue;
        }
        float s = a / 448.0f;
        float r = 448.0f / a;
        scales[d] = s;
        for (int l = 0; l < L; ++l) {
            float y = or_bf16_to_f32(v[(int64_t)l * D + d]) * r;
            dst[l] = or_e4m3_encode((double)y);
        }
        for (int l = L; l < Lpad; ++l) dst[l] = 0;
    }
}

/* ------------------------------------------------------------------ */
/* The fp32 rounding margin of P ([S2TP] Candidate: RS_32_to_8)        */
/* ------------------------------------------------------------------ */

/* The scores are converted to FP8 from fp32 ("RS_32_to_8"), so an
 * implementation's 448 p carries fp32 error before the e4m3 rounding, and a
 * code whose exact value lies that close to a rounding midpoint may round
 * the other way. Relative error bound of such an fp32 p = exp(x - m), x and
 * m natural-log logits: the logit is formed with a few fp32 roundings
 * relative to |x| and |m| (2^-24 each, in base-2 units), and the exponential
 * adds a few fp32 ulps; delta = (log2(e) (|x| + |m|) + 16) * 2^-21 bounds
 * both with a margin of about four. */
double or_p_fp32_delta(double x, double m)
{
    return (1.4426950408889634 * (fabs(x) + fabs(m)) + 16.0) * 0x1p-21;   /* log2(e) */
}

/* If a value v >= 0 rounded to e4m3 with a relative perturbation up to
 * delta could land on a neighbouring code of e4m3(v), the distance to that
 * neighbour (the step the code can move by); else 0. */
double or_e4m3_flip_step(double v, double delta)
{
    const uint8_t c = or_e4m3_encode(v);          /* 0 .. 0x7E, v >= 0 */
    const double here = or_e4m3_decode(c);
    double st = 0.0;
    if (c < 0x7E) {                               /* the midpoint above */
        const double up = or_e4m3_decode((uint8_t)(c + 1));
        if (v * (1.0 + delta) >= 0.5 * (here + up)) st = up - here;
    }
    if (c > 0) {                                  /* the midpoint below */
        const double dn = or_e4m3_decode((uint8_t)(c - 1));
        if (v * (1.0 - delta) <= 0.5 * (here + dn) && here - dn > st) st = here - dn;
    }
    return st;
}

/* ------------------------------------------------------------------ */
/* Quantised attention, one (b,h), selected query rows ([S2TP] order)  */
/* ------------------------------------------------------------------ */

/* Inputs for one (b, h): q8[Lq_pad][D], qs[ceil(Lq/blk_q)], k8[Lk_pad][D],
 * ks[ceil(Lk/blk_k)], v8t[D][ldv] (e4m3 codes, keys contiguous), vs[D].
 * For each requested query row i, with c = softmax_scale / D (the 1/D undoes
 * the unnormalised rotation of both Q and K):
 *   x_ij = (double)(sum_d q8[i][d] * k8[j][d]) * qs[i/blk_q] * ks[j/blk_k] * c
 *   masked (causal j > i + Lk - Lq) -> -inf.
 * Key tiles of 128, ascending. Per tile, in the [S2TP] order:
 *   QK:          x_ij for the tile
 *   update_mdo:  m' = max(m, max_j x_ij); alpha = exp(m - m'); O *= alpha
 *   accumulate_d: d = alpha * d + sum_j exp(x_ij - m')   (unquantised)
 *   RS_32_to_8:  P8_ij = e4m3(exp(x_ij - m') * 448)       ([PA] FP8_MAX)
 *   PV:          O[e] += sum_j dec(P8_ij) * dec(v8t[e][j])
 * out[i][e] = bf16_rne(O[e] * vs[e] / (448 * d)) ([PA]: epilogue 1/FP8_MAX);
 * a row with no visible key writes zeros. With quantize_p == 0 the e4m3
 * rounding of P is skipped (P8 = 448 * p exactly), which must then equal
 * exact softmax over the dequantised operands. out_f64 (optional) receives
 * the value before the bf16 rounding. flip_f64 (optional) receives, per
 * output element, how far an fp32 implementation of the same sequence may
 * land from out_f64 through P codes that round the other way: the sum over
 * the keys whose 448 p lies within or_p_fp32_delta of an e4m3 rounding
 * midpoint of step * |V| * vs / (448 d), carried through the rescales like O. */
void or_attn_head(const int8_t* q8, const float* qs, const int8_t* k8, const float* ks,
                  const uint8_t* v8t, int64_t ldv, const float* vs, int Lq, int Lk, int D,
                  int blk_q, int blk_k, double softmax_scale, int causal, int quantize_p,
                  const int32_t* rows, int nrows, uint16_t* out, double* out_f64,
                  double* flip_f64)
{
    const double c = softmax_scale / (double)D;
    double* O = (double*)malloc(sizeof(double) * (size_t)D);
    double* F = (double*)malloc(sizeof(double) * (size_t)D);
    double* x = (double*)malloc(sizeof(double) * OR_KEY_TILE);
    double vdec[256];
    for (int t = 0; t < 256; ++t) vdec[t] = or_e4m3_decode((uint8_t)t);

    for (int r = 0; r < nrows; ++r) {
        const int i = rows[r];
        const int8_t* qi = q8 + (int64_t)i * D;
        const double qscale = (double)qs[i / blk_q];
        double m = -INFINITY, dsum = 0.0;
        for (int e = 0; e < D; ++e) O[e] = F[e] = 0.0;

        for (int t0 = 0; t0 < Lk; t0 += OR_KEY_TILE) {
            int t1 = t0 + OR_KEY_TILE < Lk ? t0 + OR_KEY_TILE : Lk;
            /* QK */
            double mt = -INFINITY;
            for (int j = t0; j < t1; ++j) {
                int visible = !causal || (int64_t)j <= (int64_t)i + (Lk - Lq);
                if (!visible) { x[j - t0] = -INFINITY; continue; }
                const int8_t* kj = k8 + (int64_t)j * D;
                int32_t acc = 0;
                for (int e = 0; e < D; ++e) acc += (int32_t)qi[e] * (int32_t)kj[e];
                double v = (double)acc * qscale * (double)ks[j / blk_k] * c;
                x[j - t0] = v;
                if (v > mt) mt = v;
            }
            /* update_mdo */
            double mnew = m > mt ? m : mt;
            if (mnew == -INFINITY) continue;      /* nothing visible yet */
            double alpha = (m == -INFINITY) ? 0.0 : exp(m - mnew);
            for (int e = 0; e < D; ++e) O[e] *= alpha;
            for (int e = 0; e < D; ++e) F[e] *= alpha;
            /* accumulate_d, RS_32_to_8, PV */
            dsum *= alpha;
            for (int j = t0; j < t1; ++j) {
                if (x[j - t0] == -INFINITY) continue;
                double p = exp(x[j - t0] - mnew);
                dsum += p;
                double p8 = quantize_p ? or_e4m3_decode(or_e4m3_encode(p * 448.0)) : p * 448.0;
                for (int e = 0; e < D; ++e) O[e] += p8 * vdec[v8t[(int64_t)e * ldv + j]];
                if (flip_f64 && quantize_p) {
                    /* the step this P code moves by if an fp32 evaluation of
                       448 p (relative error up to or_p_fp32_delta) rounds it
                       the other way */
                    const double st = or_e4m3_flip_step(p * 448.0, or_p_fp32_delta(x[j - t0], mnew));
                    if (st > 0.0)
                        for (int e = 0; e < D; ++e) F[e] += st * fabs(vdec[v8t[(int64_t)e * ldv + j]]);
                }
            }
            m = mnew;
        }
        for (int e = 0; e < D; ++e) {
            double y = dsum > 0.0 ? O[e] * (double)vs[e] / (448.0 * dsum) : 0.0;
            out[(int64_t)r * D + e] = or_f64_to_bf16(y);
            if (out_f64) out_f64[(int64_t)r * D + e] = y;
            if (flip_f64)
                flip_f64[(int64_t)r * D + e] = dsum > 0.0 ? F[e] * (double)vs[e] / (448.0 * dsum) : 0.0;
        }
    }
    free(x);
    free(O);
    free(F);
}

/* Quantised attention with MXFP4 Q and K, one (b, h), selected query rows.
 * q4[Lq_pad][D/2], qsf[Lq_pad][D/32], k4[Lk_pad][D/2], ksf[Lk_pad][D/32]
 * (layouts of or_quant_mxfp4_head), v8t[D][ldv] and vs[D] as for
 * or_attn_head. For each requested row i, with c = softmax_scale / D:
 *   x_ij = c * sum_b 2^(Eq_ib + Ek_jb) * sum_{d in block b} e2m1(q_id) e2m1(k_jd)
 * (exact in fp64), masked as in or_attn_head; then the same per-tile
 * sequence QK -> update_mdo -> accumulate_d -> RS_32_to_8 -> PV in 128-key
 * tiles, e4m3 P scaled by 448, out = bf16(O * vs / (448 d)). out_f64 and
 * flip_f64 (optional) as for or_attn_head. */
void or_attn_mxfp4_head(const uint8_t* q4, const uint8_t* qsf, const uint8_t* k4, const uint8_t* ksf,
                        const uint8_t* v8t, int64_t ldv, const float* vs, int Lq, int Lk, int D,
                        double softmax_scale, int causal, int quantize_p, const int32_t* rows,
                        int nrows, uint16_t* out, double* out_f64, double* flip_f64)
{
    const double c = softmax_scale / (double)D;
    const int nb = D / 32;
    double* O = (double*)malloc(sizeof(double) * (size_t)D);
    double* F = (double*)malloc(sizeof(double) * (size_t)D);
    double* x = (double*)malloc(sizeof(double) * OR_KEY_TILE);
    double* qd = (double*)malloc(sizeof(double) * (size_t)D);
    double vdec[256];
    for (int t = 0; t < 256; ++t) vdec[t] = or_e4m3_decode((uint8_t)t);

    for (int r = 0; r < nrows; ++r) {
        const int i = rows[r];
        /* the query row's element values without their block scales */
        for (int d = 0; d < D; ++d) {
            const uint8_t byte = q4[(int64_t)i * (D / 2) + d / 2];
            qd[d] = or_e2m1_decode((uint8_t)((d & 1) ? (byte >> 4) : (byte & 15)));
        }
        double m = -INFINITY, dsum = 0.0;
        for (int e = 0; e < D; ++e) O[e] = F[e] = 0.0;

        for (int t0 = 0; t0 < Lk; t0 += OR_KEY_TILE) {
            int t1 = t0 + OR_KEY_TILE < Lk ? t0 + OR_KEY_TILE : Lk;
            double mt = -INFINITY;
            for (int j = t0; j < t1; ++j) {
                int visible = !causal || (int64_t)j <= (int64_t)i + (Lk - Lq);
                if (!visible) { x[j - t0] = -INFINITY; continue; }
                double acc = 0.0;
                for (int b = 0; b < nb; ++b) {
                    double part = 0.0;
                    for (int d = 32 * b; d < 32 * b + 32; ++d) {
                        const uint8_t byte = k4[(int64_t)j * (D / 2) + d / 2];
                        part += qd[d] * or_e2m1_decode((uint8_t)((d & 1) ? (byte >> 4) : (byte & 15)));
                    }
                    const int E = (int)qsf[(int64_t)i * nb + b] - 127 + (int)ksf[(int64_t)j * nb + b] - 127;
                    acc += ldexp(part, E);
                }
                double v = acc * c;
                x[j - t0] = v;
                if (v > mt) mt = v;
            }
            double mnew = m > mt ? m : mt;
            if (mnew == -INFINITY) continue;
            double alpha = (m == -INFINITY) ? 0.0 : exp(m - mnew);
            for (int e = 0; e < D; ++e) O[e] *= alpha;
            for (int e = 0; e < D; ++e) F[e] *= alpha;
            dsum *= alpha;
            for (int j = t0; j < t1; ++j) {
                if (x[j - t0] == -INFINITY) continue;
                double p = exp(x[j - t0] - mnew);
                dsum += p;
                double p8 = quantize_p ? or_e4m3_decode(or_e4m3_encode(p * 448.0)) : p * 448.0;
                for (int e = 0; e < D; ++e) O[e] += p8 * vdec[v8t[(int64_t)e * ldv + j]];
                if (flip_f64 && quantize_p) {
                    const double st = or_e4m3_flip_step(p * 448.0, or_p_fp32_delta(x[j - t0], mnew));
                    if (st > 0.0)
                        for (int e = 0; e < D; ++e) F[e] += st * fabs(vdec[v8t[(int64_t)e * ldv + j]]);
                }
            }
            m = mnew;
        }
        for (int e = 0; e < D; ++e) {
            double y = dsum > 0.0 ? O[e] * (double)vs[e] / (448.0 * dsum) : 0.0;
            out[(int64_t)r * D + e] = or_f64_to_bf16(y);
            if (out_f64) out_f64[(int64_t)r * D + e] = y;
            if (flip_f64)
                flip_f64[(int64_t)r * D + e] = dsum > 0.0 ? F[e] * (double)vs[e] / (448.0 * dsum) : 0.0;
        }
    }
    free(qd);
    free(x);
    free(F);
    free(O);
}

/* Unquantised reference, one (b,h): fp64 softmax(q k^T * softmax_scale) v
 * from the bf16 inputs (no smoothing, rotation or quantisation), same mask
 * convention. q[Lq][D], k[Lk][D], v[Lk][D]; out[nrows][D] in fp64. */
void or_attn_exact_head(const uint16_t* q, const uint16_t* k, const uint16_t* v, int Lq, int Lk,
                        int D, double softmax_scale, int causal, const int32_t* rows, int nrows,
                        double* out)
{
    double* s = (double*)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
    for (int r = 0; r < nrows; ++r) {
        const int i = rows[r];
        double mx = -INFINITY;
        for (int j = 0; j < Lk; ++j) {
            int visible = !causal || (int64_t)j <= (int64_t)i + (Lk - Lq);
            if (!visible) { s[j] = -INFINITY; continue; }
            double acc = 0.0;
            for (int e = 0; e < D; ++e)
                acc += (double)or_bf16_to_f32(q[(int64_t)i * D + e]) *
                       (double)or_bf16_to_f32(k[(int64_t)j * D + e]);
            s[j] = acc * softmax_scale;
            if (s[j] > mx) mx = s[j];
        }
        double* o = out + (int64_t)r * D;
        for (int e = 0; e < D; ++e) o[e] = 0.0;
        if (mx == -INFINITY) continue;
        double den = 0.0;
        for (int j = 0; j < Lk; ++j) {
            if (s[j] == -INFINITY) continue;
            double p = exp(s[j] - mx);
            den += p;
            for (int e = 0; e < D; ++e) o[e] += p * (double)or_bf16_to_f32(v[(int64_t)j * D + e]);
        }
        for (int e = 0; e < D; ++e) o[e] /= den;
    }
    free(s);
}

/* ------------------------------------------------------------------ */
/* Paged FP8 decode, one sequence ([PA] window-family workload)        */
/* ------------------------------------------------------------------ */

/* q[T][H][D] bf16 for one sequence; caches kc, vc: e4m3 codes laid out
 * [num_pages][Hk][page][D]; per-token scales ksc, vsc: [num_pages][Hk][page];
 * ptab[max_pages] maps logical page -> physical page; ctx >= T tokens are
 * cached, the T query tokens being the last T positions (MTP).
 * For query token t at position p = ctx - T + t and head h (kv head
 * h / (H/Hk)):
 *   q_hat = fwht(q) (fp32); a = max |q_hat|; s = a/448; r = 448/a;
 *   q8 = e4m3(q_hat * r)   (a == 0 -> s = 0, q8 = 0).
 *   Keys j in [max(0, p - window + 1), p] (exactly `window` keys once p is
 *   large enough; the T tokens are causal among themselves).
 *   S_j = (sum_e dec(q8_e) dec(k8_je)) * s * ksc_j * softmax_scale / D
 *   (the cached keys are taken as already rotated, so the same 1/D holds).
 *   fp64 softmax over the window (m = max_j S_j, p_j = exp(S_j - m));
 *   PV on bf16 operands ([PA], Changes: PV_BF16): w_j = bf16(fp32(p_j) *
 *   vsc_j), exact bf16 of dec(v8_j); out = sum_j w_j dec(v8_j) / sum_j p_j.
 * out[T][H][D] bf16. */
/* The query side of the decode, one (token, head) row: q_hat = fwht(q)
 * (fp32); a = max |q_hat|; s = a/448, r = 448/a (IEEE fp32 divides);
 * codes[e] = e4m3(fp32(q_hat[e] * r)) ([PA] Changes: Q quantised to the FP8
 * format of the cache, FP8_MAX 448); a == 0 -> s = 0 and codes 0. */
void or_decode_quant_q_row(const uint16_t* q, int D, uint8_t* codes, float* scale)
{
    float* qh = (float*)malloc(sizeof(float) * (size_t)D);
    for (int e = 0; e < D; ++e) qh[e] = or_bf16_to_f32(q[e]);
    or_fwht_f32(qh, D);
    float a = 0.0f;
    for (int e = 0; e < D; ++e) if (fabsf(qh[e]) > a) a = fabsf(qh[e]);
    float s = 0.0f, r = 0.0f;
    if (a != 0.0f) { s = a / 448.0f; r = 448.0f / a; }
    for (int e = 0; e < D; ++e) {
        float y = qh[e] * r;
        codes[e] = (a != 0.0f) ? or_e4m3_encode((double)y) : 0;
    }
    *scale = s;
    free(qh);
}

/* kv_flags (the cache variants of [PA], Performance: "per-tensor and
 * per-token scales"; Window-family results: "transposed V"):
 *   bit 0: per-tensor scales -- ksc[0] and vsc[0] scale every cached token;
 *   bit 1: transposed V -- vc is laid out [num_pages][Hk][D][page]. */
#define OR_KV_PER_TENSOR 1
#define OR_KV_V_TRANSPOSED 2

/* flip_f64 (optional): per output element, how far an implementation may
 * land from out_f64 through the bf16 rounding of the weights: one that keeps
 * a running maximum over key tiles and splits rounds each weight p_j vsc_j
 * at the scale of the maximum it has seen so far and rescales afterwards,
 * not at the window maximum used here. Both roundings are within half a
 * bf16 step of the exact weight: half this rounding's step (known) plus at
 * most 2^-8 of the weight for the other, so the bound is
 * sum_j (ulp(w_j) / 2 + 2^-8 w_j) |v_j| / sum p. */
void or_decode_seq_flags(const uint16_t* q, const uint8_t* kc, const uint8_t* vc, const float* ksc,
                         const float* vsc, const int32_t* ptab, int ctx, int T, int H, int Hk, int D,
                         int page, int window, double softmax_scale, int kv_flags, uint16_t* out,
                         double* out_f64, double* flip_f64)
{
    const int per_tensor = (kv_flags & OR_KV_PER_TENSOR) != 0;
    const int v_trans = (kv_flags & OR_KV_V_TRANSPOSED) != 0;
    uint8_t* qc = (uint8_t*)malloc((size_t)D);
    double* q8 = (double*)malloc(sizeof(double) * (size_t)D);
    double* o = (double*)malloc(sizeof(double) * (size_t)D);
    double* F = (double*)malloc(sizeof(double) * (size_t)D);
    double* sv = (double*)malloc(sizeof(double) * (size_t)(window > 0 ? window : 1));
    const int group = H / Hk;
    for (int t = 0; t < T; ++t)
        for (int h = 0; h < H; ++h) {
            const int hk = h / group;
            const uint16_t* qr = q + ((int64_t)t * H + h) * D;
            float s = 0.0f;
            or_decode_quant_q_row(qr, D, qc, &s);
            for (int e = 0; e < D; ++e) q8[e] = or_e4m3_decode(qc[e]);
            const int p = ctx - T + t;
            int lo = p - window + 1;
            if (lo < 0) lo = 0;
            const int n = p - lo + 1;
            double mx = -INFINITY;
            for (int u = 0; u < n; ++u) {
                const int j = lo + u;
                const int64_t phys = ptab[j / page];
                const int64_t tok = (phys * Hk + hk) * page + (j % page);
                double acc = 0.0;
                for (int e = 0; e < D; ++e) acc += q8[e] * or_e4m3_decode(kc[tok * D + e]);
                sv[u] = acc * (double)s * (double)ksc[per_tensor ? 0 : tok] * (softmax_scale / (double)D);
                if (sv[u] > mx) mx = sv[u];
            }
            for (int e = 0; e < D; ++e) o[e] = F[e] = 0.0;
            double den = 0.0;
            for (int u = 0; u < n; ++u) {
                const int j = lo + u;
                const int64_t phys = ptab[j / page];
                const int64_t tok = (phys * Hk + hk) * page + (j % page);
                double pj = exp(sv[u] - mx);
                den += pj;
                /* PV on bf16 operands: the weight p_j * v_scale_j is formed
                   in fp32 and rounded to bf16 (nearest even) */
                const float wf = (float)pj * vsc[per_tensor ? 0 : tok];
                const uint16_t wb = or_f64_to_bf16((double)wf);
                double w = (double)or_bf16_to_f32(wb);
                const double wmar = flip_f64 ? 0.5 * ((double)or_bf16_to_f32((uint16_t)(wb + 1)) - w) + ldexp(w, -8)
                                             : 0.0;
                for (int e = 0; e < D; ++e) {
                    const int64_t vi = v_trans ? ((phys * Hk + hk) * D + e) * page + (j % page)
                                               : tok * D + e;
                    o[e] += w * or_e4m3_decode(vc[vi]);
                    if (flip_f64) F[e] += wmar * fabs(or_e4m3_decode(vc[vi]));
                }
            }
            for (int e = 0; e < D; ++e) {
                double y = o[e] / den;
                out[((int64_t)t * H + h) * D + e] = or_f64_to_bf16(y);
                if (out_f64) out_f64[((int64_t)t * H + h) * D + e] = y;
                if (flip_f64) flip_f64[((int64_t)t * H + h) * D + e] = F[e] / den;
            }
        }
    free(sv);
    free(F);
    free(o);
    free(q8);
    free(qc);
}

/* Paged decode over an MXFP4 cache ("[FlyDSL] [Misc] pa_decode ...", Changes:
   uint8 KV is MXFP4, packed float4_e2m1fn_x2 with float8_e8m0fnu scales; the
   MXFP4 cache's compute type is bf16; Q is quantised to E4M3). kc, vc:
   [num_pages, Hk, page, D / 2] bytes, element 2i in the low nibble of byte
   i; ksf, vsf: [num_pages, Hk, page, D / 32] e8m0 bytes, one per 32
   consecutive channels of a token (value 2^(E - 127); 255 is NaN). A cached
   element is e2m1(code) * 2^(E - 127), exact. The query is rotated and
   quantised as for the FP8 cache; S_j = (q8 . k_j) * s_q * softmax_scale / D
   (the block scales sit inside k_j, no per-token scale); the PV weight is
   p_j rounded to bf16 (reading: bf16 operands as for the FP8 cache, since the
   split-KV kernel rounds at its own running maxima and an e4m3 P would
   round differently from one split to the next). */
static double or_mx_elem(const uint8_t* codes, const uint8_t* sf, int64_t tok, int D, int e)
{
    const uint8_t byte = codes[tok * (D / 2) + e / 2];
    const uint8_t E = sf[tok * (D / 32) + e / 32];
    if (E == 255) return NAN;
    return or_e2m1_decode((uint8_t)((e & 1) ? (byte >> 4) : (byte & 15))) * ldexp(1.0, (int)E - 127);
}

void or_decode_seq_mxkv(const uint16_t* q, const uint8_t* kc, const uint8_t* vc, const uint8_t* ksf,
                        const uint8_t* vsf, const int32_t* ptab, int ctx, int T, int H, int Hk, int D,
                        int page, int window, double softmax_scale, uint16_t* out, double* out_f64,
                        double* flip_f64)
{
    uint8_t* qc = (uint8_t*)malloc((size_t)D);
    double* q8 = (double*)malloc(sizeof(double) * (size_t)D);
    double* o = (double*)malloc(sizeof(double) * (size_t)D);
    double* F = (double*)malloc(sizeof(double) * (size_t)D);
    double* sv = (double*)malloc(sizeof(double) * (size_t)(window > 0 ? window : 1));
    const int group = H / Hk;
    for (int t = 0; t < T; ++t)
        for (int h = 0; h < H; ++h) {
            const int hk = h / group;
            const uint16_t* qr = q + ((int64_t)t * H + h) * D;
            float s = 0.0f;
            or_decode_quant_q_row(qr, D, qc, &s);
            for (int e = 0; e < D; ++e) q8[e] = or_e4m3_decode(qc[e]);
            const int p = ctx - T + t;
            int lo = p - window + 1;
            if (lo < 0) lo = 0;
            const int n = p - lo + 1;
            double mx = -INFINITY;
            for (int u = 0; u < n; ++u) {
                const int j = lo + u;
                const int64_t tok = ((int64_t)ptab[j / page] * Hk + hk) * page + (j % page);
                double acc = 0.0;
                for (int e = 0; e < D; ++e) acc += q8[e] * or_mx_elem(kc, ksf, tok, D, e);
                sv[u] = acc * (double)s * (softmax_scale / (double)D);
                if (sv[u] > mx) mx = sv[u];
            }
            for (int e = 0; e < D; ++e) o[e] = F[e] = 0.0;
            double den = 0.0;
            for (int u = 0; u < n; ++u) {
                const int j = lo + u;
                const int64_t tok = ((int64_t)ptab[j / page] * Hk + hk) * page + (j % page);
                double pj = exp(sv[u] - mx);
                den += pj;
                const uint16_t wb = or_f64_to_bf16((double)(float)pj);      /* bf16 PV weight */
                double w = (double)or_bf16_to_f32(wb);
                const double wmar = flip_f64 ? 0.5 * ((double)or_bf16_to_f32((uint16_t)(wb + 1)) - w) + ldexp(w, -8)
                                             : 0.0;
                for (int e = 0; e < D; ++e) {
                    const double v = or_mx_elem(vc, vsf, tok, D, e);
                    o[e] += w * v;
                    if (flip_f64) F[e] += wmar * fabs(v);
                }
            }
            for (int e = 0; e < D; ++e) {
                double y = o[e] / den;
                out[((int64_t)t * H + h) * D + e] = or_f64_to_bf16(y);
                if (out_f64) out_f64[((int64_t)t * H + h) * D + e] = y;
                if (flip_f64) flip_f64[((int64_t)t * H + h) * D + e] = F[e] / den;
            }
        }
    free(sv);
    free(F);
    free(o);
    free(q8);
    free(qc);
}

void or_decode_seq(const uint16_t* q, const uint8_t* kc, const uint8_t* vc, const float* ksc,
                   const float* vsc, const int32_t* ptab, int ctx, int T, int H, int Hk, int D,
                   int page, int window, double softmax_scale, uint16_t* out, double* out_f64)
{
    or_decode_seq_flags(q, kc, vc, ksc, vsc, ptab, ctx, T, H, Hk, D, page, window, softmax_scale, 0,
                        out, out_f64, NULL);
}
