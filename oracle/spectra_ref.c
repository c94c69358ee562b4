/*
 * spectra_ref.c -- plain CPU oracle for the SPECTRA outlier-split INT4 path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark do.  It shares no code, header, table or constant
 * generator with the CUDA library.
 *
 * Source of the method: "SPECTRA: Sparse-Precision Exact Channel Tensor
 * Reconstruction Architecture" (aiwithghost.com re-post of the Dev.to
 * abstract), abstract paragraph:
 *   - channel saliency = fourth-moment kurtosis of each input channel, taken
 *     with the upstream normalisation gain, threshold kappa > 3.0;
 *   - heavy-tailed channels are kept bit-exact in floating point;
 *   - the remaining Gaussian bulk is stored as Group-32 4-bit codes with a
 *     scale and a bit-packed zero point per group.
 * The quantiser is the asymmetric min/max rule: scale = (max-min)/15 stored
 * as FP16, zero = clamp(round(-min/scale), 0, 15), code = clamp(round(w/scale)
 * + zero, 0, 15), rounding half to even.
 *
 * Everything is computed in IEEE double, sequentially, in the order written
 * below.  Build with -O2 -ffp-contract=off (no fused multiply-add), no
 * -ffast-math.  Readings taken where the abstract is silent are listed at the
 * function that takes them.
 *
 * Storage layout of the packed arrays ("RT32", repository-defined; it replaces
 * the Marlin interleave of the abstract, which targets Ampere mma.sync):
 *   N_pad = ceil(N/32)*32, T = N_pad/32 row tiles, G = K/32 groups,
 *   S = ceil(G/8) super-groups of 8 groups, O8 = ceil(n_o/8) outlier octets.
 *   codes   : 16-byte record per (tile t, group g, lane r) at byte
 *             ((t*G + g)*32 + r)*16; record word w (little-endian u32),
 *             nibble j (bits 4j..4j+3) = code of column 32g + 8w + j of row
 *             32t + r.
 *   scales  : FP16 bits, element ((t*S + g/8)*32 + r)*8 + g%8.
 *   zeros   : u32 words, word (t*S + g/8)*32 + r, nibble g%8.
 *   outliers: BF16 bits, element ((t*O8 + j/8)*32 + r)*8 + j%8 = W[32t+r,
 *             idx[j]].
 *   Rows >= N, groups >= G and outlier slots >= n_o are zero.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Status values of the oracle (its own numbering). */
enum {
    REF_OK = 0,
    REF_ERR_INVALID_ARG = 1,
    REF_ERR_SHAPE = 2,
    REF_ERR_NONFINITE = 3,
    REF_ERR_RANGE = 4
};

/* ---------------------------------------------------------------- numbers */

/* BF16 is the upper half of an IEEE binary32 word. */
double spectra_ref_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double spectra_ref_fp16_to_double(uint16_t h)
{
    int sign = h >> 15;
    int e = (h >> 10) & 0x1F;
    int m = h & 0x3FF;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);              /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(m + 1024), e - 25);  /* (1 + m/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/*
 * double -> binary16 with ONE round-to-nearest-even step, subnormals kept,
 * overflow to infinity.  The value is scaled by a power of two (exact) so
 * that the kept bits form an integer, and rint() (default rounding mode:
 * nearest, ties to even) performs the single rounding.
 */
uint16_t spectra_ref_double_to_fp16(double v)
{
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (isnan(v))
        return (uint16_t)(sign | 0x7E00);
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: multiples of 2^-24; q == 1024 encodes 2^-14 */
        double q = rint(ldexp(a, 24));
        return (uint16_t)(sign | (uint16_t)q);
    }
    int e2;
    frexp(a, &e2);            /* a = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1;           /* a in [2^E, 2^(E+1)) */
    if (E > 15)
        return (uint16_t)(sign | 0x7C00);
    double q = rint(ldexp(a, 10 - E)); /* in [1024, 2048] */
    if (q == 2048.0) {
        q = 1024.0;
        E += 1;
    }
    if (E > 15)
        return (uint16_t)(sign | 0x7C00);
    return (uint16_t)(sign | (uint16_t)(((E + 15) << 10) | ((int)q - 1024)));
}

static int is_finite_bf16(uint16_t b) { return ((b >> 7) & 0xFF) != 0xFF; }

/* ---------------------------------------------------------------- saliency */

/*
 * Pearson kurtosis (m4 / m2^2, population moments, not excess) of each
 * column of the gain-scaled matrix a[i][j] = W[i][j] * g[j]
 * (abstract: the channel's fourth-moment kurtosis, computed with the upstream
 * normalisation gain).  gain == NULL means g = 1.
 * Order: S = sum_i a_i (i ascending), mu = S/N; then for i ascending
 * d = a_i - mu, q = d*d, m2 += q, m4 += q*q; m2 /= N, m4 /= N,
 * kappa = m4 / (m2*m2); a column with m2 == 0 gets kappa = 0.
 */
int spectra_ref_kurtosis(const uint16_t *w, const float *gain, int32_t n, int32_t k,
                         double *kappa)
{
    if (!w || !kappa || n < 1 || k < 1)
        return REF_ERR_INVALID_ARG;
    for (int64_t e = 0; e < (int64_t)n * k; ++e)
        if (!is_finite_bf16(w[e]))
            return REF_ERR_NONFINITE;
    if (gain)
        for (int32_t j = 0; j < k; ++j)
            if (!isfinite(gain[j]))
                return REF_ERR_NONFINITE;
    for (int32_t j = 0; j < k; ++j) {
        double g = gain ? (double)gain[j] : 1.0;
        double s = 0.0;
        for (int32_t i = 0; i < n; ++i)
            s = s + spectra_ref_bf16_to_double(w[(int64_t)i * k + j]) * g;
        double mu = s / (double)n;
        double m2 = 0.0, m4 = 0.0;
        for (int32_t i = 0; i < n; ++i) {
            double a = spectra_ref_bf16_to_double(w[(int64_t)i * k + j]) * g;
            double d = a - mu;
            double q = d * d;
            m2 = m2 + q;
            m4 = m4 + q * q;
        }
        m2 = m2 / (double)n;
        m4 = m4 / (double)n;
        kappa[j] = (m2 == 0.0) ? 0.0 : m4 / (m2 * m2);
    }
    return REF_OK;
}

/* Outlier set O = {j : kappa_j > tau} (strict), ascending.  Returns |O|. */
int32_t spectra_ref_split(const double *kappa, int32_t k, double tau, int32_t *idx)
{
    int32_t n_o = 0;
    for (int32_t j = 0; j < k; ++j)
        if (kappa[j] > tau)
            idx[n_o++] = j;
    return n_o;
}

/* ---------------------------------------------------------------- quantiser */

/*
 * Group-32 asymmetric 4-bit quantiser over the bulk matrix B, where B equals
 * W with every outlier column replaced by +0 (the outlier columns live in
 * exact BF16 storage instead).  Canonical outputs (row-major):
 *   codes  [n][k]    one code 0..15 per byte
 *   scales [n][k/32] FP16 bits
 *   zeros  [n][k/32] one zero point 0..15 per byte
 * Per (row i, group g):
 *   values v = (double)B[i][32g..32g+31], with -0 read as +0;
 *   lo = min v, hi = max v (first element, then strict updates);
 *   s  = fp16_rne((hi - lo) / 15.0); infinity -> REF_ERR_RANGE;
 *   S  = (double)s;
 *   S == 0: z = 0 and every code = 0;
 *   else    z = clamp(rint(-lo / S), 0, 15),
 *           c = clamp(rint(v / S) + z, 0, 15).
 */
int spectra_ref_quantize(const uint16_t *w, int32_t n, int32_t k, const int32_t *idx,
                         int32_t n_o, uint8_t *codes, uint16_t *scales, uint8_t *zeros)
{
    if (!w || !codes || !scales || !zeros || n < 1 || k < 1 || n_o < 0 || n_o > k ||
        (n_o > 0 && !idx))
        return REF_ERR_INVALID_ARG;
    if (k % 32 != 0)
        return REF_ERR_SHAPE;
    for (int64_t e = 0; e < (int64_t)n * k; ++e)
        if (!is_finite_bf16(w[e]))
            return REF_ERR_NONFINITE;
    uint8_t *is_out = (uint8_t *)calloc((size_t)k, 1);
    if (!is_out)
        return REF_ERR_INVALID_ARG;
    for (int32_t t = 0; t < n_o; ++t) {
        if (idx[t] < 0 || idx[t] >= k) {
            free(is_out);
            return REF_ERR_INVALID_ARG;
        }
        is_out[idx[t]] = 1;
    }
    const int32_t G = k / 32;
    int status = REF_OK;
    double v[32];
    for (int32_t i = 0; i < n && status == REF_OK; ++i) {
        for (int32_t g = 0; g < G; ++g) {
            for (int kk = 0; kk < 32; ++kk) {
                int32_t j = 32 * g + kk;
                double x = is_out[j] ? 0.0 : spectra_ref_bf16_to_double(w[(int64_t)i * k + j]);
                v[kk] = x + 0.0; /* -0 + +0 = +0 in round-to-nearest */
            }
            double lo = v[0], hi = v[0];
            for (int kk = 1; kk < 32; ++kk) {
                if (v[kk] < lo) lo = v[kk];
                if (v[kk] > hi) hi = v[kk];
            }
            double diff = hi - lo;
            uint16_t sh = spectra_ref_double_to_fp16(diff / 15.0);
            if ((sh & 0x7FFF) == 0x7C00) {
                status = REF_ERR_RANGE;
                break;
            }
            double S = spectra_ref_fp16_to_double(sh);
            scales[(int64_t)i * G + g] = sh;
            uint8_t *crow = codes + (int64_t)i * k + 32 * g;
            if (S == 0.0) {
                zeros[(int64_t)i * G + g] = 0;
                memset(crow, 0, 32);
                continue;
            }
            double zq = rint(-lo / S);
            double z = zq < 0.0 ? 0.0 : (zq > 15.0 ? 15.0 : zq);
            zeros[(int64_t)i * G + g] = (uint8_t)z;
            for (int kk = 0; kk < 32; ++kk) {
                double c = rint(v[kk] / S) + z;
                c = c < 0.0 ? 0.0 : (c > 15.0 ? 15.0 : c);
                crow[kk] = (uint8_t)c;
            }
        }
    }
    free(is_out);
    return status;
}

/* ---------------------------------------------------------------- layout */

static int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

/*
 * Element counts of the packed arrays: out[0] = code bytes, out[1] = FP16
 * scale elements, out[2] = u32 zero words, out[3] = BF16 outlier elements,
 * out[4] = N_pad.
 */
void spectra_ref_layout_sizes(int32_t n, int32_t k, int32_t n_o, int64_t *out)
{
    int64_t np = cdiv(n, 32) * 32, G = k / 32, S = cdiv(G, 8), O8 = cdiv(n_o, 8);
    out[0] = np * k / 2;
    out[1] = np * S * 8;
    out[2] = np * S;
    out[3] = np * O8 * 8;
    out[4] = np;
}

/* canonical -> packed.  w/idx give the outlier columns (exact BF16 copies). */
void spectra_ref_pack_layout(int32_t n, int32_t k, const uint8_t *codes, const uint16_t *scales,
                             const uint8_t *zeros, const uint16_t *w, const int32_t *idx,
                             int32_t n_o, uint8_t *pcodes, uint16_t *pscales, uint32_t *pzeros,
                             uint16_t *poutl)
{
    int64_t sz[5];
    spectra_ref_layout_sizes(n, k, n_o, sz);
    const int64_t np = sz[4], G = k / 32, S = cdiv(G, 8), O8 = cdiv(n_o, 8);
    memset(pcodes, 0, (size_t)sz[0]);
    memset(pscales, 0, (size_t)sz[1] * 2);
    memset(pzeros, 0, (size_t)sz[2] * 4);
    if (sz[3])
        memset(poutl, 0, (size_t)sz[3] * 2);
    for (int64_t i = 0; i < n; ++i) {
        int64_t t = i / 32, r = i % 32;
        for (int64_t kk = 0; kk < k; ++kk) {
            int64_t g = kk / 32, in = kk % 32, word = in / 8, j = in % 8;
            int64_t byte = ((t * G + g) * 32 + r) * 16 + word * 4 + j / 2;
            uint8_t c = codes[i * k + kk] & 0xF;
            pcodes[byte] |= (uint8_t)((j % 2) ? (c << 4) : c);
        }
        for (int64_t g = 0; g < G; ++g) {
            pscales[((t * S + g / 8) * 32 + r) * 8 + g % 8] = scales[i * G + g];
            pzeros[(t * S + g / 8) * 32 + r] |= (uint32_t)(zeros[i * G + g] & 0xF) << (4 * (g % 8));
        }
        for (int64_t o = 0; o < n_o; ++o)
            poutl[((t * O8 + o / 8) * 32 + r) * 8 + o % 8] = w[i * k + idx[o]];
    }
    (void)np;
}

/* packed -> canonical (codes, scales, zeros) for rows 0..n-1. */
void spectra_ref_unpack_layout(int32_t n, int32_t k, const uint8_t *pcodes,
                               const uint16_t *pscales, const uint32_t *pzeros, uint8_t *codes,
                               uint16_t *scales, uint8_t *zeros)
{
    const int64_t G = k / 32, S = cdiv(G, 8);
    for (int64_t i = 0; i < n; ++i) {
        int64_t t = i / 32, r = i % 32;
        for (int64_t kk = 0; kk < k; ++kk) {
            int64_t g = kk / 32, in = kk % 32, word = in / 8, j = in % 8;
            uint8_t b = pcodes[((t * G + g) * 32 + r) * 16 + word * 4 + j / 2];
            codes[i * k + kk] = (uint8_t)((j % 2) ? (b >> 4) : (b & 0xF));
        }
        for (int64_t g = 0; g < G; ++g) {
            scales[i * G + g] = pscales[((t * S + g / 8) * 32 + r) * 8 + g % 8];
            zeros[i * G + g] = (uint8_t)((pzeros[(t * S + g / 8) * 32 + r] >> (4 * (g % 8))) & 0xF);
        }
    }
}

/* ---------------------------------------------------------------- matvec */

/* w_hat[i][k] = (c - z) * S, exact in double. */
void spectra_ref_dequant(int32_t n, int32_t k, const uint8_t *codes, const uint16_t *scales,
                         const uint8_t *zeros, double *w_hat)
{
    const int64_t G = k / 32;
    for (int64_t i = 0; i < n; ++i)
        for (int64_t kk = 0; kk < k; ++kk) {
            double S = spectra_ref_fp16_to_double(scales[i * G + kk / 32]);
            w_hat[i * k + kk] = ((double)codes[i * k + kk] - (double)zeros[i * G + kk / 32]) * S;
        }
}

/*
 * y[m][i] = sum_k w_hat[i][k] * x[m][k]  (k ascending)
 *         + sum_t W[i][idx[t]] * x[m][idx[t]]  (t ascending)
 * in double, with w_hat decoded from the canonical codes on the fly; the
 * bulk holds exact zeros at the outlier columns.  bound[m][i] is the same sum
 * over absolute values, the scale of the acceptance test
 * |y_gpu - y| <= 2e-3 * bound + 1e-5.  bound may be NULL.
 */
void spectra_ref_gemm(int32_t n, int32_t k, const uint8_t *codes, const uint16_t *scales,
                      const uint8_t *zeros, const uint16_t *w, const int32_t *idx, int32_t n_o,
                      const uint16_t *x, int32_t m, double *y, double *bound)
{
    const int64_t G = k / 32;
    for (int64_t mm = 0; mm < m; ++mm) {
        const uint16_t *xr = x + mm * k;
        for (int64_t i = 0; i < n; ++i) {
            double acc = 0.0, b = 0.0;
            for (int64_t kk = 0; kk < k; ++kk) {
                double S = spectra_ref_fp16_to_double(scales[i * G + kk / 32]);
                double wd = ((double)codes[i * k + kk] - (double)zeros[i * G + kk / 32]) * S;
                double xv = spectra_ref_bf16_to_double(xr[kk]);
                acc = acc + wd * xv;
                b = b + fabs(wd) * fabs(xv);
            }
            for (int64_t t = 0; t < n_o; ++t) {
                double wo = spectra_ref_bf16_to_double(w[i * k + idx[t]]);
                double xv = spectra_ref_bf16_to_double(xr[idx[t]]);
                acc = acc + wo * xv;
                b = b + fabs(wo) * fabs(xv);
            }
            y[mm * n + i] = acc;
            if (bound)
                bound[mm * n + i] = b;
        }
    }
}

/* ---------------------------------------------------------------- embedding */

/*
 * double -> bfloat16 (the upper half of an IEEE binary32 word: 8 exponent
 * bits, bias 127, 7 fraction bits) with ONE round-to-nearest-even step,
 * subnormals kept, overflow to infinity.  As for binary16 above, an exact
 * power-of-two scaling makes the kept bits an integer and rint() rounds once.
 */
uint16_t spectra_ref_double_to_bf16(double v)
{
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (isnan(v))
        return (uint16_t)(sign | 0x7FC0);
    if (isinf(v))
        return (uint16_t)(sign | 0x7F80);
    if (a < ldexp(1.0, -126)) {
        /* subnormal range: multiples of 2^-133; q == 128 encodes 2^-126 */
        double q = rint(ldexp(a, 133));
        return (uint16_t)(sign | (uint16_t)q);
    }
    int e2;
    frexp(a, &e2);            /* a = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1;           /* a in [2^E, 2^(E+1)) */
    if (E > 127)
        return (uint16_t)(sign | 0x7F80);
    double q = rint(ldexp(a, 7 - E)); /* in [128, 256] */
    if (q == 256.0) {
        q = 128.0;
        E += 1;
    }
    if (E > 127)
        return (uint16_t)(sign | 0x7F80);
    return (uint16_t)(sign | (uint16_t)(((E + 127) << 7) | ((int)q - 128)));
}

/*
 * Row gather of the reconstructed table (abstract and highlight 5:
 * SpectraFusedEmbedding keeps vocabulary tables in the 4-bit Group-32 format
 * and dequantises the rows it needs while the forward pass runs).  The table
 * E[n][k] (n = vocabulary, k = hidden) is a packed layer like any other; its
 * reconstruction is
 *   E_hat[i][j] = W[i][j]                   for j in O (stored bit-exact),
 *   E_hat[i][j] = (c_ij - z_ig) * S_ig      otherwise (g = j / 32),
 * and out[r][.] = E_hat[ids[r]][.] in double (every value is exact).  The
 * codes, scales and zero points are the canonical arrays of the quantiser.
 * An id outside [0, n) rejects the call before anything is written.
 */
int spectra_ref_embed(int32_t n, int32_t k, const uint8_t *codes, const uint16_t *scales,
                      const uint8_t *zeros, const uint16_t *w, const int32_t *idx, int32_t n_o,
                      const int32_t *ids, int32_t m, double *out)
{
    if (n < 1 || k < 32 || k % 32 != 0 || m < 0 || n_o < 0 || n_o > k)
        return REF_ERR_INVALID_ARG;
    if (m == 0)
        return REF_OK;
    if (!codes || !scales || !zeros || !ids || !out || (n_o > 0 && (!w || !idx)))
        return REF_ERR_INVALID_ARG;
    for (int32_t r = 0; r < m; ++r)
        if (ids[r] < 0 || ids[r] >= n)
            return REF_ERR_INVALID_ARG;
    const int64_t ngroups = k / 32;
    for (int64_t r = 0; r < m; ++r) {
        const int64_t row = ids[r];
        double *dst = out + r * k;
        for (int64_t col = 0; col < k; ++col) {
            const int64_t grp = row * ngroups + col / 32;
            double S = spectra_ref_fp16_to_double(scales[grp]);
            dst[col] = ((double)codes[row * k + col] - (double)zeros[grp]) * S;
        }
        for (int64_t t = 0; t < n_o; ++t)
            dst[idx[t]] = spectra_ref_bf16_to_double(w[row * k + idx[t]]);
    }
    return REF_OK;
}

/* ---------------------------------------------------------------- bulk compaction */

/*
 * Compacted bulk (abstract: the heavy-tailed coordinates are decoupled into
 * bit-exact storage and the residual bulk is quantised; this variant removes
 * the outlier columns from the bulk instead of masking them to +0 in place).
 * The bulk then holds the k - n_o non-outlier columns in ascending order,
 * padded with all-zero columns to a multiple of 32 and to at least one group:
 *   k_bulk = max(32, 32 * ceil((k - n_o) / 32)),
 *   bulk_idx[p] = the p-th non-outlier column for p < k - n_o, -1 after.
 * Returns k_bulk, or -1 when idx is not strictly ascending within [0, k).
 * bulk_idx must hold max(32, k + 31) entries.
 */
int32_t spectra_ref_bulk_columns(int32_t k, const int32_t *idx, int32_t n_o, int32_t *bulk_idx)
{
    if (k < 1 || n_o < 0 || n_o > k || (n_o > 0 && !idx) || !bulk_idx)
        return -1;
    for (int32_t t = 0; t < n_o; ++t)
        if (idx[t] < 0 || idx[t] >= k || (t > 0 && idx[t - 1] >= idx[t]))
            return -1;
    const int32_t nb = k - n_o;
    const int32_t k_bulk = nb <= 32 ? 32 : (int32_t)(cdiv(nb, 32) * 32);
    int32_t p = 0, t = 0;
    for (int32_t j = 0; j < k; ++j) {
        if (t < n_o && idx[t] == j) {
            ++t;
            continue;
        }
        bulk_idx[p++] = j;
    }
    for (; p < k_bulk; ++p)
        bulk_idx[p] = -1;
    return k_bulk;
}

/* W_b[i][p] = W[i][bulk_idx[p]] as BF16 bits, +0 at padding positions. */
void spectra_ref_gather_bulk(const uint16_t *w, int32_t n, int32_t k, const int32_t *bulk_idx,
                             int32_t k_bulk, uint16_t *w_b)
{
    for (int64_t i = 0; i < n; ++i)
        for (int64_t p = 0; p < k_bulk; ++p)
            w_b[i * k_bulk + p] = bulk_idx[p] < 0 ? 0 : w[i * k + bulk_idx[p]];
}

/*
 * Row table: the layout of a table that is only gathered (an untied
 * embedding).  Same canonical arrays as spectra_ref_pack_layout (codes,
 * scales, zeros over k bulk columns; w is the BF16 matrix with kw columns per
 * row); every row's pieces are contiguous:
 *   rcodes   : byte (i*G + g)*16 + 4w + j/2 holds, in its low (j even) or high
 *              (j odd) nibble, the code of bulk column 32g + 8w + j of row i;
 *   rscales  : element i*G + g is the FP16 scale of group g of row i;
 *   rzeros   : word i*S + g/8 holds in nibble g%8 the zero point of group g;
 *   routl    : element i*n_o + o is W[i][idx[o]] (BF16 bits).
 * G = k/32, S = ceil(G/8).  No padding rows.
 */
void spectra_ref_row_table(int32_t n, int32_t k, const uint8_t *codes, const uint16_t *scales,
                           const uint8_t *zeros, const uint16_t *w, int32_t kw, const int32_t *idx,
                           int32_t n_o, uint8_t *rcodes, uint16_t *rscales, uint32_t *rzeros,
                           uint16_t *routl)
{
    const int64_t G = k / 32, S = cdiv(G, 8);
    memset(rcodes, 0, (size_t)(n * G * 16));
    memset(rzeros, 0, (size_t)(n * S) * 4);
    for (int64_t i = 0; i < n; ++i) {
        for (int64_t kk = 0; kk < k; ++kk) {
            int64_t g = kk / 32, in = kk % 32, word = in / 8, j = in % 8;
            uint8_t c = codes[i * k + kk] & 0xF;
            rcodes[(i * G + g) * 16 + word * 4 + j / 2] |= (uint8_t)((j % 2) ? (c << 4) : c);
        }
        for (int64_t g = 0; g < G; ++g) {
            rscales[i * G + g] = scales[i * G + g];
            rzeros[i * S + g / 8] |= (uint32_t)(zeros[i * G + g] & 0xF) << (4 * (g % 8));
        }
        for (int64_t o = 0; o < n_o; ++o)
            routl[i * n_o + o] = w[i * kw + idx[o]];
    }
}

/* The outlier block alone, in the RT32 order of spectra_ref_pack_layout. */
void spectra_ref_pack_outliers(int32_t n, int32_t k, const uint16_t *w, const int32_t *idx,
                               int32_t n_o, uint16_t *poutl)
{
    const int64_t O8 = cdiv(n_o, 8), np = cdiv(n, 32) * 32;
    if (n_o == 0)
        return;
    memset(poutl, 0, (size_t)(np * O8 * 8) * 2);
    for (int64_t i = 0; i < n; ++i) {
        int64_t t = i / 32, r = i % 32;
        for (int64_t slot = 0; slot < n_o; ++slot)
            poutl[((t * O8 + slot / 8) * 32 + r) * 8 + slot % 8] = w[i * k + idx[slot]];
    }
}

/*
 * Matvec over a compacted layer: codes/scales/zeros are the canonical arrays
 * of the bulk [n][k_bulk], w the original BF16 matrix [n][k], x [m][k]:
 *   y[m][i] = sum_p w_hat_b[i][p] * x[m][bulk_idx[p]]   (p ascending, padding skipped)
 *           + sum_t W[i][idx[t]] * x[m][idx[t]]         (t ascending)
 * in double; bound is the same sum over absolute values (may be NULL).
 */
void spectra_ref_gemm_compact(int32_t n, int32_t k, int32_t k_bulk, const uint8_t *codes,
                              const uint16_t *scales, const uint8_t *zeros,
                              const int32_t *bulk_idx, const uint16_t *w, const int32_t *idx,
                              int32_t n_o, const uint16_t *x, int32_t m, double *y, double *bound)
{
    const int64_t Gb = k_bulk / 32;
    for (int64_t mm = 0; mm < m; ++mm) {
        const uint16_t *xr = x + mm * k;
        for (int64_t i = 0; i < n; ++i) {
            double acc = 0.0, b = 0.0;
            for (int64_t p = 0; p < k_bulk; ++p) {
                if (bulk_idx[p] < 0)
                    continue;
                double S = spectra_ref_fp16_to_double(scales[i * Gb + p / 32]);
                double wb = ((double)codes[i * k_bulk + p] - (double)zeros[i * Gb + p / 32]) * S;
                double xb = spectra_ref_bf16_to_double(xr[bulk_idx[p]]);
                acc = acc + wb * xb;
                b = b + fabs(wb) * fabs(xb);
            }
            for (int64_t t = 0; t < n_o; ++t) {
                double wo = spectra_ref_bf16_to_double(w[i * k + idx[t]]);
                double xo = spectra_ref_bf16_to_double(xr[idx[t]]);
                acc = acc + wo * xo;
                b = b + fabs(wo) * fabs(xo);
            }
            y[mm * n + i] = acc;
            if (bound)
                bound[mm * n + i] = b;
        }
    }
}

/*
 * Row gather of a compacted table: out[r][bulk_idx[p]] = (c - z) * S of bulk
 * column p of row ids[r], out[r][idx[t]] = W[ids[r]][idx[t]] (bit-exact); the
 * two sets of columns partition [0, k).  An id outside [0, n) rejects the call.
 */
int spectra_ref_embed_compact(int32_t n, int32_t k, int32_t k_bulk, const uint8_t *codes,
                              const uint16_t *scales, const uint8_t *zeros,
                              const int32_t *bulk_idx, const uint16_t *w, const int32_t *idx,
                              int32_t n_o, const int32_t *ids, int32_t m, double *out)
{
    if (n < 1 || k < 1 || k_bulk < 32 || k_bulk % 32 != 0 || m < 0 || n_o < 0 || n_o > k)
        return REF_ERR_INVALID_ARG;
    for (int32_t r = 0; r < m; ++r)
        if (ids[r] < 0 || ids[r] >= n)
            return REF_ERR_INVALID_ARG;
    const int64_t Gb = k_bulk / 32;
    for (int64_t r = 0; r < m; ++r) {
        const int64_t i = ids[r];
        double *orow = out + r * k;
        for (int64_t p = 0; p < k_bulk; ++p) {
            if (bulk_idx[p] < 0)
                continue;
            double S = spectra_ref_fp16_to_double(scales[i * Gb + p / 32]);
            orow[bulk_idx[p]] = ((double)codes[i * k_bulk + p] - (double)zeros[i * Gb + p / 32]) * S;
        }
        for (int64_t t = 0; t < n_o; ++t)
            orow[idx[t]] = spectra_ref_bf16_to_double(w[i * k + idx[t]]);
    }
    return REF_OK;
}

/* ---------------------------------------------------------------- KV cache */

/*
 * Group-32 4-bit key-value cache (abstract: microscaled Group-32 4-bit KV
 * caching keeps long contexts resident).  Read as the weight quantiser
 * applied to every token's vector of one KV head: the D channels of token t
 * and head h form one row of D/32 groups, each with an FP16 scale and a
 * 4-bit zero point, codes by the same formula (spectra_ref_quantize, no
 * outlier columns).  x is [n_tok][H][D] BF16 (the layout a K or V
 * projection writes); the canonical outputs are indexed by (h, t):
 *   codes  [H][cap][D], scales [H][cap][D/32], zeros [H][cap][D/32],
 * and tokens go to positions pos .. pos + n_tok - 1 of a capacity cap.
 */
int spectra_ref_kv_quantize(const uint16_t *x, int32_t n_tok, int32_t H, int32_t D, int32_t pos,
                            int32_t cap, uint8_t *codes, uint16_t *scales, uint8_t *zeros)
{
    if (!x || n_tok < 1 || H < 1 || D < 32 || D % 32 != 0 || pos < 0 || pos + n_tok > cap)
        return REF_ERR_INVALID_ARG;
    const int64_t G = D / 32;
    uint8_t *c = (uint8_t *)malloc((size_t)D);
    uint16_t *s = (uint16_t *)malloc((size_t)G * 2);
    uint8_t *z = (uint8_t *)malloc((size_t)G);
    if (!c || !s || !z) {
        free(c); free(s); free(z);
        return REF_ERR_INVALID_ARG;
    }
    int st = REF_OK;
    for (int64_t t = 0; t < n_tok && st == REF_OK; ++t)
        for (int64_t h = 0; h < H && st == REF_OK; ++h) {
            st = spectra_ref_quantize(x + (t * H + h) * D, 1, D, NULL, 0, c, s, z);
            if (st != REF_OK)
                break;
            const int64_t slot = h * cap + pos + t;
            memcpy(codes + slot * D, c, (size_t)D);
            memcpy(scales + slot * G, s, (size_t)G * 2);
            memcpy(zeros + slot * G, z, (size_t)G);
        }
    free(c); free(s); free(z);
    return st;
}

/*
 * Decode attention over the 4-bit cache, in double:
 *   k_hat[h][t][d] = (c - z) * S (and v_hat likewise), exact;
 *   for query head i (KV head h = i / (Hq / Hkv)) and tokens t < T:
 *     s_t = scale * sum_d q[i][d] * k_hat[h][t][d]     (d ascending)
 *     p_t = exp(s_t - max_t s_t) / sum_t exp(s_t - max_t s_t)
 *     out[i][d] = sum_t p_t * v_hat[h][t][d]            (t ascending)
 * Also, for the acceptance test: vbound[i][d] = sum_t p_t |v_hat[h][t][d]|
 * and smax[i] = max_t scale * sum_d |q[i][d]| |k_hat[h][t][d]| (either may
 * be NULL).  Caches are canonical arrays of capacity cap (see above).
 */
int spectra_ref_attention(int32_t Hq, int32_t Hkv, int32_t D, int32_t T, int32_t cap,
                          const uint8_t *kc, const uint16_t *ks, const uint8_t *kz,
                          const uint8_t *vc, const uint16_t *vs, const uint8_t *vz,
                          const uint16_t *q, double scale, double *out, double *vbound,
                          double *smax)
{
    if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || D < 32 || D % 32 != 0 || T < 1 || T > cap)
        return REF_ERR_INVALID_ARG;
    const int64_t G = D / 32, grp = Hq / Hkv;
    double *sc = (double *)malloc((size_t)T * sizeof(double));
    double *sa = (double *)malloc((size_t)T * sizeof(double));
    if (!sc || !sa) {
        free(sc); free(sa);
        return REF_ERR_INVALID_ARG;
    }
    for (int64_t i = 0; i < Hq; ++i) {
        const int64_t h = i / grp;
        double m = -INFINITY, sm = 0.0;
        for (int64_t t = 0; t < T; ++t) {
            const int64_t slot = h * cap + t;
            double acc = 0.0, ab = 0.0;
            for (int64_t d = 0; d < D; ++d) {
                double S = spectra_ref_fp16_to_double(ks[slot * G + d / 32]);
                double kv = ((double)kc[slot * D + d] - (double)kz[slot * G + d / 32]) * S;
                double qv = spectra_ref_bf16_to_double(q[i * D + d]);
                acc = acc + qv * kv;
                ab = ab + fabs(qv) * fabs(kv);
            }
            sc[t] = scale * acc;
            sa[t] = fabs(scale) * ab;
            if (sc[t] > m) m = sc[t];
            if (sa[t] > sm) sm = sa[t];
        }
        double l = 0.0;
        for (int64_t t = 0; t < T; ++t) {
            sc[t] = exp(sc[t] - m);
            l = l + sc[t];
        }
        for (int64_t d = 0; d < D; ++d) {
            double o = 0.0, b = 0.0;
            for (int64_t t = 0; t < T; ++t) {
                const int64_t slot = h * cap + t;
                double S = spectra_ref_fp16_to_double(vs[slot * G + d / 32]);
                double vv = ((double)vc[slot * D + d] - (double)vz[slot * G + d / 32]) * S;
                o = o + (sc[t] / l) * vv;
                b = b + (sc[t] / l) * fabs(vv);
            }
            out[i * D + d] = o;
            if (vbound)
                vbound[i * D + d] = b;
        }
        if (smax)
            smax[i] = sm;
    }
    free(sc); free(sa);
    return REF_OK;
}

/*
 * Packed KV cache (repository-defined, like RT32): one slot per (head h,
 * position t), slot = h*cap + t, G = D/32 groups:
 *   codes : 16-byte record per (slot, group g) at byte (slot*G + g)*16; word
 *           w, nibble j holds the code of channel 32g + 8w + j;
 *   scales: FP16 bits, element slot*G + g;
 *   zeros : u32 word slot, nibble g (D <= 256).
 * Slots and nibbles not covered by the canonical arrays stay zero.
 */
void spectra_ref_kv_pack(int32_t H, int32_t cap, int32_t D, const uint8_t *codes,
                         const uint16_t *scales, const uint8_t *zeros, uint8_t *pcodes,
                         uint16_t *pscales, uint32_t *pzeros)
{
    const int64_t G = D / 32, slots = (int64_t)H * cap;
    memset(pcodes, 0, (size_t)(slots * D / 2));
    memset(pscales, 0, (size_t)(slots * G) * 2);
    memset(pzeros, 0, (size_t)slots * 4);
    for (int64_t slot = 0; slot < slots; ++slot)
        for (int64_t ch = 0; ch < D; ++ch) {
            const int64_t grp = ch / 32, in = ch % 32, word = in / 8, nib = in % 8;
            const uint8_t c = codes[slot * D + ch] & 0xF;
            pcodes[(slot * G + grp) * 16 + word * 4 + nib / 2] |= (uint8_t)((nib % 2) ? (c << 4) : c);
            if (in == 0) {
                pscales[slot * G + grp] = scales[slot * G + grp];
                pzeros[slot] |= (uint32_t)(zeros[slot * G + grp] & 0xF) << (4 * grp);
            }
        }
}
