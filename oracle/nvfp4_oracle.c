/*
 * nvfp4_oracle.c -- plain, slow, obviously-correct CPU oracle for NVFP4
 * sparse MLA decode.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke entry and
 * the benchmark's CPU-baseline leg may load this file's library.  It shares
 * no code, header, table or helper with the CUDA library, and the CUDA
 * library never calls it.
 *
 * What it follows (page "Prime Intellect Launches Prime Inference, Serving
 * 600B Tokens Daily", section "Four-bit caches make room"):
 *   - the latent MLA cache row shrinks from 576 to 352 bytes under NVFP4, a
 *     4-bit format with one FP8 scale per group of 16 values;
 *   - the native kernel reads only the rows chosen by the sparse indexer and
 *     unpacks them on chip; attention runs on FP16 operands with FP32
 *     accumulation;
 *   - the index list has 2,048 positions and empty entries are zero-filled;
 *   - the staged baseline first unpacks NVFP4 into FP8 buffers.
 * The pages do not define E2M1/E4M3 nor the byte layout, so the standard
 * format definitions are written out below, and the row layout is:
 *   bytes [0,256)   latent dims 0..511 as E2M1 nibbles, byte b holds dim 2b
 *                   in its low nibble and dim 2b+1 in its high nibble;
 *   bytes [256,288) 32 E4M3 group scales, scale g covers dims 16g..16g+15;
 *   bytes [288,352) 64 RoPE dims as E4M3, byte k = RoPE dim k.
 * Readings of points the pages leave open (rounding, zero groups, sign of
 * zero, meaning of an empty entry, the log base of lse) are stated at each
 * function.  Every function here is pinned by a CPU test against something
 * other than itself (value tables, torch's float8 conversion, closed-form
 * bounds, dense attention via numpy, invariances, brute force).
 *
 * Floating point: compile without -ffast-math and with -ffp-contract=off so
 * every float operation below is the IEEE single/double operation written.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_ROW_BYTES 352
#define ORACLE_LATENT 512
#define ORACLE_ROPE 64
#define ORACLE_GROUP 16
#define ORACLE_NGROUPS (ORACLE_LATENT / ORACLE_GROUP)
#define ORACLE_STAGED_ROW 576

/* ---------------------------------------------------------------- formats */

/* E2M1: 1 sign bit (bit 3), 2 exponent bits (bias 1), 1 mantissa bit.
 * Exponent field 0 encodes the subnormal 0.5*m; otherwise the value is
 * 2^(e-1) * (1 + m/2).  The eight magnitudes are 0,0.5,1,1.5,2,3,4,6. */
double oracle_e2m1_value(int code)
{
    int s = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* E4M3 (the "FN" variant): 1 sign bit, 4 exponent bits (bias 7), 3 mantissa
 * bits, no infinities; S.1111.111 is NaN, so the largest finite magnitude is
 * 2^8 * 1.75 = 448.  Exponent field 0 is subnormal: 2^-6 * m/8. */
double oracle_e4m3_value(int code)
{
    int s = (code >> 7) & 1;
    int e = (code >> 3) & 15;
    int m = code & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) mag = ldexp(m / 8.0, -6);
    else mag = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Round |y| to the nearest of the 2^k finite magnitudes of a format listed
 * by oracle_*_value over codes [0, ncodes), ties to the code whose lowest
 * (mantissa) bit is 0, saturating to the largest finite magnitude.  This is
 * round-to-nearest-even with "satfinite", written as a search. */
static int nearest_even_code(double mag, double (*value)(int), int ncodes)
{
    int best = 0;
    double best_err = fabs(mag - value(0));
    for (int c = 1; c < ncodes; ++c) {
        double err = fabs(mag - value(c));
        if (err < best_err || (err == best_err && (c & 1) == 0 && (best & 1) != 0)) {
            best = c;
            best_err = err;
        }
    }
    return best;
}

/* E2M1 encode of an FP32 value: RNE, saturating at 6; the sign bit is the
 * sign of y, so a negative value that rounds to zero gives 0x8 (-0). */
int oracle_e2m1_encode(float y)
{
    int sign = signbit(y) ? 8 : 0;
    double mag = fabs((double)y);
    if (isnan(y)) return 0x7; /* never produced by finite inputs; documented */
    if (mag > 6.0) return sign | 7;
    return sign | nearest_even_code(mag, oracle_e2m1_value, 8);
}

/* E4M3 encode of an FP32 value: RNE, saturating at 448 (never NaN for a
 * finite input); sign bit is the sign of y. */
int oracle_e4m3_encode(float y)
{
    int sign = signbit(y) ? 0x80 : 0;
    double mag = fabs((double)y);
    if (isnan(y)) return 0x7F;
    if (mag > 448.0) return sign | 0x7E;
    return sign | nearest_even_code(mag, oracle_e4m3_value, 0x7F);
}

static float bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* IEEE binary16 -> double, written from the bit fields. */
double oracle_f16_to_double(uint16_t h)
{
    int s = (h >> 15) & 1;
    int e = (h >> 10) & 31;
    int m = h & 1023;
    double mag;
    if (e == 31) return m ? NAN : (s ? -INFINITY : INFINITY);
    if (e == 0) mag = ldexp((double)m, -24);
    else mag = ldexp(1.0 + m / 1024.0, e - 15);
    return s ? -mag : mag;
}

/* ------------------------------------------------------------- quantizer */

/* One group of 16 latent values (BF16 widened exactly to FP32):
 *   a = max_i |x_i|
 *   scale code = E4M3_RNE_sat(a / 6)           (IEEE FP32 divide)
 *   s = value(scale code)
 *   s == 0  -> all 16 nibbles are +0
 *   else    -> nibble_i = E2M1_RNE_sat(x_i / s) (IEEE FP32 divide)
 * 6 is the largest E2M1 magnitude, so a/6 maps the group maximum onto it;
 * a scale rounded down can push |x/s| above 6, which saturates. */
void oracle_quantize_group(const float *x16, uint8_t *nib16, uint8_t *scale_code)
{
    float a = 0.0f;
    for (int i = 0; i < ORACLE_GROUP; ++i) {
        float v = fabsf(x16[i]);
        if (v > a) a = v;
    }
    float q = a / 6.0f;
    int sc = oracle_e4m3_encode(q);
    float s = (float)oracle_e4m3_value(sc);
    *scale_code = (uint8_t)sc;
    for (int i = 0; i < ORACLE_GROUP; ++i) {
        if (s == 0.0f) nib16[i] = 0;
        else nib16[i] = (uint8_t)oracle_e2m1_encode(x16[i] / s);
    }
}

/* Quantize n rows of BF16 latent [n, lat_stride>=512] and RoPE
 * [n, rope_stride>=64] (element strides) into n packed 352-byte rows. */
void oracle_quantize_rows(const uint16_t *latent, int64_t lat_stride,
                          const uint16_t *rope, int64_t rope_stride,
                          int64_t n, uint8_t *rows)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r) {
        uint8_t *row = rows + r * ORACLE_ROW_BYTES;
        memset(row, 0, ORACLE_ROW_BYTES);
        for (int g = 0; g < ORACLE_NGROUPS; ++g) {
            float x[ORACLE_GROUP];
            uint8_t nib[ORACLE_GROUP], sc;
            for (int i = 0; i < ORACLE_GROUP; ++i)
                x[i] = bf16_to_float(latent[r * lat_stride + g * ORACLE_GROUP + i]);
            oracle_quantize_group(x, nib, &sc);
            for (int i = 0; i < ORACLE_GROUP; ++i) {
                int d = g * ORACLE_GROUP + i;
                int byte = d / 2;
                if (d % 2 == 0) row[byte] |= (uint8_t)(nib[i] & 0xF);
                else row[byte] |= (uint8_t)((nib[i] & 0xF) << 4);
            }
            row[256 + g] = sc;
        }
        for (int k = 0; k < ORACLE_ROPE; ++k)
            row[288 + k] = (uint8_t)oracle_e4m3_encode(bf16_to_float(rope[r * rope_stride + k]));
    }
}

/* The pre-NVFP4 cache row (page "Prime Intellect Launches Prime Inference,
 * Serving 600B Tokens Daily", section "Four-bit caches make room": rows were
 * 576 bytes before NVFP4): one E4M3 byte per dim, 512 latent dims then 64
 * RoPE dims, each value E4M3_RNE_sat of the BF16 input with no scale.
 * Quantizes n rows into n 576-byte rows. */
void oracle_quantize_fp8_rows(const uint16_t *latent, int64_t lat_stride,
                              const uint16_t *rope, int64_t rope_stride,
                              int64_t n, uint8_t *rows)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r) {
        uint8_t *row = rows + r * ORACLE_STAGED_ROW;
        for (int d = 0; d < ORACLE_LATENT; ++d)
            row[d] = (uint8_t)oracle_e4m3_encode(bf16_to_float(latent[r * lat_stride + d]));
        for (int k = 0; k < ORACLE_ROPE; ++k)
            row[ORACLE_LATENT + k] = (uint8_t)oracle_e4m3_encode(bf16_to_float(rope[r * rope_stride + k]));
    }
}

/* Dequantize one 352-byte row to 576 values: dims 0..511 are
 * e2m1(nibble) * e4m3(scale of its group), dims 512..575 are e4m3(RoPE).
 * Every such product has at most 6 significant bits and lies in
 * [2^-10, 2688], so it is exact in FP16 (and here in double). */
void oracle_dequant_row(const uint8_t *row, double *out576)
{
    for (int d = 0; d < ORACLE_LATENT; ++d) {
        uint8_t byte = row[d / 2];
        int nib = (d % 2 == 0) ? (byte & 0xF) : (byte >> 4);
        double s = oracle_e4m3_value(row[256 + d / ORACLE_GROUP]);
        out576[d] = oracle_e2m1_value(nib) * s;
    }
    for (int k = 0; k < ORACLE_ROPE; ++k)
        out576[ORACLE_LATENT + k] = oracle_e4m3_value(row[288 + k]);
}

/* Staged baseline row: the dequantized values of one NVFP4 row, each
 * re-encoded E4M3_RNE_sat into a 576-byte row (512 latent then 64 RoPE),
 * the pre-NVFP4 row size.  Page "Prime Intellect Launches Prime Inference",
 * section "Four-bit caches make room": the staged implementation unpacked
 * NVFP4 values into FP8 buffers before attention. */
void oracle_stage_row(const uint8_t *row, uint8_t *out576)
{
    double v[ORACLE_LATENT + ORACLE_ROPE];
    oracle_dequant_row(row, v);
    for (int d = 0; d < ORACLE_LATENT + ORACLE_ROPE; ++d)
        out576[d] = (uint8_t)oracle_e4m3_encode((float)v[d]);
}

/* ------------------------------------------------------------- attention */

/* Sparse MLA decode in FP64 over dequantized rows.
 *
 * For token t and head h, over list positions j with 0 <= idx[t,j] < num_slots
 * (any other entry is empty and contributes nothing -- this is how the
 * pages' treatment of list slots the indexer leaves unfilled is read here;
 * a duplicate index counts once per position):
 *   s_j   = sm_scale * ( sum_{d<512} q_nope[t,h,d] k_j[d]
 *                      + sum_{d<64}  q_rope[t,h,d] k_j[512+d] )
 *   m     = max_j s_j ;  l = sum_j exp(s_j - m)
 *   out   = sum_j exp(s_j - m) * k_j[0:512] / l      (V = the latent part)
 *   lse   = m + ln l                                  (natural log)
 * A token with no valid entry gets out = 0 and lse = -inf.
 * staged == 1 first replaces each key value by its E4M3 re-encoding (the
 * staged FP8 baseline); staged == 2 means the cache holds 576-byte E4M3 rows
 * (oracle_quantize_fp8_rows) and k_j is their decoded values.  q is FP16
 * [T,H,512] and [T,H,64]; out is FP64
 * [T,H,512], lse FP64 [T,H].  Each token's valid rows are dequantized once
 * (the same values for every head); sums run over valid positions in list
 * order; OpenMP only distributes independent rows and heads.
 * Returns 0 on success, nonzero on bad sizes or allocation failure. */
int oracle_sparse_mla(const uint16_t *q_nope, const uint16_t *q_rope,
                      const uint8_t *cache, int64_t num_slots,
                      const int32_t *indices, int topk,
                      int T, int H, float sm_scale, int staged,
                      double *out, double *lse, int nthreads)
{
    const int D = ORACLE_LATENT + ORACLE_ROPE;
    if (T < 0 || H <= 0 || topk < 0) return 1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int64_t *pos = (int64_t *)malloc(sizeof(int64_t) * (topk > 0 ? topk : 1));
    double *K = (double *)malloc(sizeof(double) * (size_t)D * (topk > 0 ? topk : 1));
    if (!pos || !K) { free(pos); free(K); return 2; }
    int failed = 0;
    for (int t = 0; t < T && !failed; ++t) {
        const int32_t *idx = indices + (int64_t)t * topk;
        int nvalid = 0;
        for (int j = 0; j < topk; ++j) {
            int64_t slot = idx[j];
            if (slot >= 0 && slot < num_slots) pos[nvalid++] = slot;
        }
#pragma omp parallel for schedule(static)
        for (int jj = 0; jj < nvalid; ++jj) {
            const uint8_t *row = cache + pos[jj] * (staged == 2 ? ORACLE_STAGED_ROW : ORACLE_ROW_BYTES);
            double *k = K + (size_t)jj * D;
            if (staged == 2) {
                for (int d = 0; d < D; ++d) k[d] = oracle_e4m3_value(row[d]);
            } else if (staged) {
                uint8_t st[ORACLE_STAGED_ROW];
                oracle_stage_row(row, st);
                for (int d = 0; d < D; ++d) k[d] = oracle_e4m3_value(st[d]);
            } else {
                oracle_dequant_row(row, k);
            }
        }
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
        for (int h = 0; h < H; ++h) {
            int64_t th = (int64_t)t * H + h;
            double q[ORACLE_LATENT + ORACLE_ROPE];
            for (int d = 0; d < ORACLE_LATENT; ++d)
                q[d] = oracle_f16_to_double(q_nope[th * ORACLE_LATENT + d]);
            for (int d = 0; d < ORACLE_ROPE; ++d)
                q[ORACLE_LATENT + d] = oracle_f16_to_double(q_rope[th * ORACLE_ROPE + d]);
            double *o = out + th * ORACLE_LATENT;
            for (int d = 0; d < ORACLE_LATENT; ++d) o[d] = 0.0;
            if (nvalid == 0) { lse[th] = -INFINITY; continue; }
            double *s = (double *)malloc(sizeof(double) * nvalid);
            if (!s) { failed |= 1; continue; }
            double m = -INFINITY;
            for (int jj = 0; jj < nvalid; ++jj) {
                const double *k = K + (size_t)jj * D;
                double dot = 0.0;
                for (int d = 0; d < D; ++d) dot += q[d] * k[d];
                s[jj] = (double)sm_scale * dot;
                if (s[jj] > m) m = s[jj];
            }
            double l = 0.0;
            for (int jj = 0; jj < nvalid; ++jj) {
                const double *k = K + (size_t)jj * D;
                double p = exp(s[jj] - m);
                l += p;
                for (int d = 0; d < ORACLE_LATENT; ++d) o[d] += p * k[d];
            }
            for (int d = 0; d < ORACLE_LATENT; ++d) o[d] /= l;
            lse[th] = m + log(l);
            free(s);
        }
    }
    free(pos);
    free(K);
    return failed;
}

/* Number of OpenMP threads the oracle would use (1 without OpenMP). */
int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
