/*
 * oracle.c -- plain, single-threaded CPU oracle for the CSA / HCA hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file: only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or constant with the
 * CUDA library.
 *
 * Every stage is the literal definition, accumulated in double precision.
 * Inputs arrive as float (fp32, and bf16 / e4m3 values widened exactly), or
 * as raw e4m3 codes; outputs are double.  Sources:
 *
 *   [HA] "DeepSeek-V4 混合注意力：从压缩记忆到百万上下文" (brenchcc.github.io notes):
 *        §4.1 two-branch overlapped compression (alpha and C^comp equations),
 *        §4.2 Lightning Indexer score s_{t,i}, §5 HCA (beta and C^hca equations),
 *        §6 SWA window and attention-sink probability p_i, §7 call chain
 *        (compress -> index -> top-k -> gather -> concat with SWA -> one MQA).
 *   [P1] "揭秘DeepSeek-V4-Pro-MXFP4稀疏注意力：哈希索引与DSA如何撑起1M超长上下文？":
 *        window_size 128, index_topk, attn_sink, sparse_attn_kernel gather.
 *   [P2] "解密DeepSeek-V4-Flash-NVFP4的混合注意力机制：压缩稀疏注意力如何提升长文本处理能力":
 *        sparse_attn(q, kv, attn_sink, topk_idxs, softmax_scale) call shape.
 *
 * Readings of points the pages leave open (each is listed in the design notes):
 *   - Compressor rows are 0-based: entry i takes b-rows (i-1)m..im-1 and
 *     a-rows im..(i+1)m-1; softmax position 0..m-1 are the b rows.
 *   - Entry 0 with no previous block has no b positions (logit -inf).
 *   - A trailing partial block yields no entry.
 *   - Index keys are shared by the 64 index heads; no 1/sqrt(d) in the score.
 *   - FP8 (e4m3) inputs are dequantised as code * scale and the score is the
 *     plain definition on the dequantised values.
 *   - Top-k: k largest over i < n_valid, ties to the lower index, output
 *     ascending, padded with -1; -0.0 and +0.0 compare equal.
 *   - Attention: z_j = scale * <q, row_j>; the sink logit is used unscaled;
 *     rows are the gathered entries (idx outside [0, N) contributes nothing)
 *     and the SWA positions max(0, t-127)..t that lie inside the SWA buffer;
 *     no de-duplication between the two sets.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_BAD 1

/* ------------------------------------------------------------------------ */
/* [HA] §4.1: C^comp_{i,j} = sum_r alpha_{i,r,j} C^b_{(i-1)m+r,j}
 *                         + sum_r alpha_{i,m+r,j} C^a_{im+r,j},
 * alpha_{i,:,j} = softmax([Z^b_{(i-1)m:im,j} ; Z^a_{im:(i+1)m,j}]) over 2m.
 * One sequence.  Inputs are [L, c] row-major; prev_Cb / prev_Zb hold the
 * b-branch rows of the block before row 0 ([m, c]) or are NULL.
 * out and mag are [L/m, c]; mag = sum_r alpha |C| (forward-error scale). */
int oracle_compress_csa(const float *Ca, const float *Cb, const float *Za, const float *Zb,
                        const float *prev_Cb, const float *prev_Zb, int64_t L, int c, int m,
                        double *out, double *mag)
{
    if (m <= 0 || c <= 0 || L < 0) return ORC_BAD;
    int64_t n_entries = L / m;
    double *logit = (double *)malloc(sizeof(double) * 2 * m);
    double *value = (double *)malloc(sizeof(double) * 2 * m);
    int *present = (int *)malloc(sizeof(int) * 2 * m);
    if (!logit || !value || !present) { free(logit); free(value); free(present); return ORC_BAD; }
    for (int64_t i = 0; i < n_entries; ++i) {
        for (int j = 0; j < c; ++j) {
            /* the 2m positions: r = 0..m-1 from the previous block's b branch,
             * r = m..2m-1 from this block's a branch */
            for (int r = 0; r < m; ++r) {
                if (i > 0) {
                    int64_t row = (i - 1) * m + r;
                    logit[r] = Zb[row * c + j];
                    value[r] = Cb[row * c + j];
                    present[r] = 1;
                } else if (prev_Zb && prev_Cb) {
                    logit[r] = prev_Zb[(int64_t)r * c + j];
                    value[r] = prev_Cb[(int64_t)r * c + j];
                    present[r] = 1;
                } else {
                    present[r] = 0;
                }
                int64_t arow = i * m + r;
                logit[m + r] = Za[arow * c + j];
                value[m + r] = Ca[arow * c + j];
                present[m + r] = 1;
            }
            double mx = -INFINITY;
            for (int r = 0; r < 2 * m; ++r)
                if (present[r] && logit[r] > mx) mx = logit[r];
            double den = 0.0;
            for (int r = 0; r < 2 * m; ++r)
                if (present[r]) den += exp(logit[r] - mx);
            double acc = 0.0, amag = 0.0;
            for (int r = 0; r < 2 * m; ++r) {
                if (!present[r]) continue;
                double alpha = exp(logit[r] - mx) / den;
                acc += alpha * value[r];
                amag += alpha * fabs(value[r]);
            }
            out[i * c + j] = acc;
            if (mag) mag[i * c + j] = amag;
        }
    }
    free(logit); free(value); free(present);
    return ORC_OK;
}

/* [HA] §5: beta_{i,:,j} = softmax(Z_{im':(i+1)m', j}),
 *          C^hca_{i,j} = sum_r beta_{i,r,j} C_{im'+r, j}.   One sequence. */
int oracle_compress_hca(const float *C, const float *Z, int64_t L, int c, int m,
                        double *out, double *mag)
{
    if (m <= 0 || c <= 0 || L < 0) return ORC_BAD;
    int64_t n_entries = L / m;
    for (int64_t i = 0; i < n_entries; ++i) {
        for (int j = 0; j < c; ++j) {
            double mx = -INFINITY;
            for (int r = 0; r < m; ++r) {
                double z = Z[(i * m + r) * c + j];
                if (z > mx) mx = z;
            }
            double den = 0.0;
            for (int r = 0; r < m; ++r) den += exp((double)Z[(i * m + r) * c + j] - mx);
            double acc = 0.0, amag = 0.0;
            for (int r = 0; r < m; ++r) {
                double beta = exp((double)Z[(i * m + r) * c + j] - mx) / den;
                double v = C[(i * m + r) * c + j];
                acc += beta * v;
                amag += beta * fabs(v);
            }
            out[i * c + j] = acc;
            if (mag) mag[i * c + j] = amag;
        }
    }
    return ORC_OK;
}

/* Causal visibility of compressed entries: entry i (covering raw tokens
 * im..(i+1)m-1) is complete, hence visible to the query at absolute position
 * t, iff (i+1)m <= t+1 ([HA] §6: the SWA branch holds tokens of the block
 * that is not yet full).  Number of visible entries, capped at N. */
int64_t oracle_n_visible(int64_t t, int m, int64_t N)
{
    if (t < 0 || m <= 0) return 0;
    int64_t nv = (t + 1) / m;
    return nv < N ? nv : N;
}

/* [HA] §4.2: s_{t,i} = sum_h w_{t,h} ReLU(<q^I_{t,h}, k^I_i>), i < n_valid(t);
 * s = -inf for n_valid(t) <= i < N.  qI [T, Hi, d], w [T, Hi], kI [N, d],
 * scores and mag [T, N]; mag = sum_h |w| sum_d |q k| (forward-error scale). */
int oracle_index_scores(const float *qI, const float *w, const float *kI, const int32_t *n_valid,
                        int T, int64_t N, int Hi, int d, double *scores, double *mag)
{
    if (T < 0 || N < 0 || Hi <= 0 || d <= 0) return ORC_BAD;
    for (int t = 0; t < T; ++t) {
        int64_t nv = n_valid[t];
        if (nv < 0 || nv > N) return ORC_BAD;
        for (int64_t i = 0; i < N; ++i) {
            if (i >= nv) {
                scores[(int64_t)t * N + i] = -INFINITY;
                if (mag) mag[(int64_t)t * N + i] = 0.0;
                continue;
            }
            double s = 0.0, smag = 0.0;
            for (int h = 0; h < Hi; ++h) {
                const float *q = qI + ((int64_t)t * Hi + h) * d;
                const float *k = kI + i * d;
                double dot = 0.0, dmag = 0.0;
                for (int e = 0; e < d; ++e) {
                    double p = (double)q[e] * (double)k[e];
                    dot += p;
                    dmag += fabs(p);
                }
                double wh = w[(int64_t)t * Hi + h];
                s += wh * (dot > 0.0 ? dot : 0.0);
                smag += fabs(wh) * dmag;
            }
            scores[(int64_t)t * N + i] = s;
            if (mag) mag[(int64_t)t * N + i] = smag;
        }
    }
    return ORC_OK;
}

/* ---- OCP 8-bit floating point, E4M3 variant (bias 7, no infinities,
 * S.1111.111 is NaN, largest finite 448 = 1.75 * 2^8, subnormals 2^-9 * m). */
double oracle_e4m3_decode(uint8_t b)
{
    int s = b >> 7, e = (b >> 3) & 15, mt = b & 7;
    double v;
    if (e == 15 && mt == 7) return NAN;
    if (e == 0) v = ldexp((double)mt, -9);
    else v = ldexp(1.0 + mt / 8.0, e - 7);
    return s ? -v : v;
}

/* Round to the nearest finite e4m3 value, ties to the code with an even
 * mantissa, magnitudes beyond 448 saturate to 448 ("satfinite").  Plain
 * search over the 127 non-negative finite codes, which are increasing. */
uint8_t oracle_e4m3_encode(float x)
{
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a >= 448.0) return sign | 0x7E;
    int lo = 0, hi = 0x7E;               /* decode(lo) <= a < decode(hi) */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (oracle_e4m3_decode((uint8_t)mid) <= a) lo = mid; else hi = mid;
    }
    double dlo = a - oracle_e4m3_decode((uint8_t)lo);
    double dhi = oracle_e4m3_decode((uint8_t)hi) - a;
    int code;
    if (dlo < dhi) code = lo;
    else if (dhi < dlo) code = hi;
    else code = (lo & 1) ? hi : lo;      /* tie: even mantissa */
    return sign | (uint8_t)code;
}

/* Per-row symmetric e4m3 quantisation: scale = amax / 448 (fp32),
 * code = e4m3(x / scale) with the division in fp32; an all-zero row gets
 * scale 1.  x [rows, cols] -> codes [rows, cols], scale [rows]. */
int oracle_quantize_rows_e4m3(const float *x, int64_t rows, int cols, uint8_t *codes, float *scale)
{
    for (int64_t r = 0; r < rows; ++r) {
        float amax = 0.0f;
        for (int j = 0; j < cols; ++j) {
            float a = fabsf(x[r * cols + j]);
            if (a > amax) amax = a;
        }
        volatile float s = amax / 448.0f;
        if (amax == 0.0f) s = 1.0f;
        scale[r] = s;
        for (int j = 0; j < cols; ++j) {
            volatile float y = x[r * cols + j] / s;
            codes[r * cols + j] = oracle_e4m3_encode(y);
        }
    }
    return ORC_OK;
}

/* ---- Hadamard rotation of the index vectors ([P1], the paragraph on the
 * Indexer: the index query passes through RoPE and a Hadamard rotation before
 * its dot products with the compressed keys).  Readings: the rotation is the
 * orthonormal Sylvester-ordered Walsh-Hadamard matrix R = H_n / sqrt(n), with
 * H_1 = [1] and H_2m = [[H_m, H_m], [H_m, -H_m]]; the index keys get the same
 * rotation, so <Rq, Rk> = <q, k> and the scores keep their meaning; it comes
 * before the e4m3 quantisation, as an aid to it.
 * x, y: [rows, n] double, n a power of two <= 1024.  y = R x, summed in
 * double in index order, then multiplied by c = 1 / sqrt(n) (both IEEE
 * double, round to nearest). */
static int orc_is_pow2(int n) { return n > 0 && (n & (n - 1)) == 0; }

int oracle_hadamard_rotate(const double *x, int64_t rows, int n, double *y)
{
    if (!orc_is_pow2(n) || n > 1024 || rows < 0) return ORC_BAD;
    signed char *H = (signed char *)malloc((size_t)n * n);
    if (!H) return ORC_BAD;
    H[0] = 1;
    for (int m = 1; m < n; m *= 2)          /* Sylvester doubling of the m x m block */
        for (int i = 0; i < m; ++i)
            for (int j = 0; j < m; ++j) {
                signed char h = H[(size_t)i * n + j];
                H[(size_t)i * n + (j + m)] = h;
                H[(size_t)(i + m) * n + j] = h;
                H[(size_t)(i + m) * n + (j + m)] = (signed char)-h;
            }
    const double c = 1.0 / sqrt((double)n);
    for (int64_t r = 0; r < rows; ++r)
        for (int i = 0; i < n; ++i) {
            double acc = 0.0;
            for (int j = 0; j < n; ++j) acc += H[(size_t)i * n + j] * x[r * n + j];
            y[r * n + i] = acc * c;
        }
    free(H);
    return ORC_OK;
}

/* Rotated e4m3 quantisation: each row is rotated (oracle_hadamard_rotate on the
 * row widened to double), rounded to fp32, then quantised exactly as in
 * oracle_quantize_rows_e4m3.  x [rows, n] float -> codes [rows, n], scale [rows]. */
int oracle_quantize_rows_e4m3_hadamard(const float *x, int64_t rows, int n, uint8_t *codes, float *scale)
{
    if (!orc_is_pow2(n) || n > 1024 || rows < 0) return ORC_BAD;
    double *xd = (double *)malloc(sizeof(double) * (size_t)n);
    double *yd = (double *)malloc(sizeof(double) * (size_t)n);
    float *yf = (float *)malloc(sizeof(float) * (size_t)n);
    int rc = (xd && yd && yf) ? ORC_OK : ORC_BAD;
    for (int64_t r = 0; r < rows && rc == ORC_OK; ++r) {
        for (int j = 0; j < n; ++j) xd[j] = x[r * n + j];
        rc = oracle_hadamard_rotate(xd, 1, n, yd);
        for (int j = 0; j < n; ++j) yf[j] = (float)yd[j];
        if (rc == ORC_OK) rc = oracle_quantize_rows_e4m3(yf, 1, n, codes + r * n, scale + r);
    }
    free(xd); free(yd); free(yf);
    return rc;
}

/* ---- FP4 index QK ([HA] §2 configuration table and §4.2: the index QK path
 * runs in FP4).  Readings (the pages name no FP4 format for the indexer): OCP
 * MXFP4, i.e. FP4 E2M1 elements (1 sign, 2 exponent bits with bias 1, 1 mantissa
 * bit; no infinities or NaN; largest magnitude 6) with one shared E8M0 scale
 * (2^(c-127)) per block of 32 consecutive dims.  The block scale is
 * X = 2^(floor(log2 amax) - 2), 2 being the exponent of E2M1's largest binade,
 * clamped to 2^-127 .. 2^127; an all-zero block gets X = 1.  Elements are
 * x / X rounded to the nearest E2M1 value, ties to the even mantissa, magnitudes
 * beyond 6 saturating to 6.  The score is the plain definition on the values
 * code * X, as for e4m3. */
double oracle_e2m1_decode(uint8_t c)
{
    static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    return (c & 8) ? -mag[c & 7] : mag[c & 7];
}

/* Nearest E2M1 value by search over the 8 non-negative codes (increasing in
 * magnitude); on a tie the code with mantissa bit 0 (an even code) wins. */
uint8_t oracle_e2m1_encode(double x)
{
    uint8_t sign = signbit(x) ? 8 : 0;
    double a = fabs(x);
    int best = 0;
    for (int c = 1; c < 8; ++c) {
        double d = fabs(oracle_e2m1_decode((uint8_t)c) - a);
        double db = fabs(oracle_e2m1_decode((uint8_t)best) - a);
        if (d < db || (d == db && (c & 1) == 0)) best = c;
    }
    return sign | (uint8_t)best;
}

/* x [rows, n] (n a multiple of 32) -> codes [rows, n] (one E2M1 code per byte,
 * low nibble) and scale [rows, n/32] (E8M0 codes). */
int oracle_quantize_rows_mxfp4(const float *x, int64_t rows, int n, uint8_t *codes, uint8_t *scale)
{
    if (n <= 0 || n % 32 != 0 || rows < 0) return ORC_BAD;
    for (int64_t r = 0; r < rows; ++r)
        for (int b = 0; b < n / 32; ++b) {
            const float *xb = x + r * n + 32 * b;
            double amax = 0.0;
            for (int j = 0; j < 32; ++j)
                if (fabs((double)xb[j]) > amax) amax = fabs((double)xb[j]);
            int e = 0;
            if (amax > 0.0) {
                int E;
                frexp(amax, &E);            /* amax = f 2^E, f in [0.5, 1): floor(log2 amax) = E - 1 */
                e = E - 1 - 2;
                if (e < -127) e = -127;
                if (e > 127) e = 127;
            }
            scale[r * (n / 32) + b] = (uint8_t)(e + 127);
            for (int j = 0; j < 32; ++j)
                codes[r * n + 32 * b + j] = oracle_e2m1_encode(ldexp((double)xb[j], -e));
        }
    return ORC_OK;
}

/* codes / scale as above -> x [rows, n] float (code * 2^(scale-127), exact). */
int oracle_mxfp4_dequantize(const uint8_t *codes, const uint8_t *scale, int64_t rows, int n, float *x)
{
    if (n <= 0 || n % 32 != 0 || rows < 0) return ORC_BAD;
    for (int64_t r = 0; r < rows; ++r)
        for (int j = 0; j < n; ++j) {
            uint8_t s = scale[r * (n / 32) + j / 32];
            if (s == 0xFF) return ORC_BAD;     /* E8M0 NaN */
            x[r * n + j] = (float)ldexp(oracle_e2m1_decode(codes[r * n + j] & 15), (int)s - 127);
        }
    return ORC_OK;
}

/* ---- Partial RoPE ([HA] §6: only the last 64 dims of each head are rotated by
 * position; after the core attention the same dims of the output get the inverse
 * rotation, before the grouped output projection).  Readings (the pages give no
 * pairing, base or position rule for compressed entries): the rotary embedding of
 * the RoFormer paper on dims D-64..D-1, pairs (D-64+2i, D-64+2i+1) for i < 32
 * turned by the angle pos * theta^(-2i/64); theta is a parameter (the MXFP4 page
 * gives compress_rope_theta = 160000 for the compressed layers; its YaRN extension
 * has no stated parameters and is not applied).  inverse != 0 turns by -angle.
 * x [rows, D] double, pos [rows] int64 -> y [rows, D] double; dims below D-64 are
 * copied unchanged.  cos / sin of the angle in double. */
int oracle_rope(const double *x, const int64_t *pos, int64_t rows, int D, double theta, int inverse, double *y)
{
    if (D < 64 || D % 2 != 0 || rows < 0 || !(theta > 1.0)) return ORC_BAD;
    for (int64_t r = 0; r < rows; ++r) {
        const double *xr = x + r * D;
        double *yr = y + r * D;
        for (int j = 0; j < D - 64; ++j) yr[j] = xr[j];
        for (int i = 0; i < 32; ++i) {
            double ang = (double)pos[r] * pow(theta, -2.0 * i / 64.0);
            if (inverse) ang = -ang;
            double c = cos(ang), s = sin(ang);
            double a = xr[D - 64 + 2 * i], b = xr[D - 64 + 2 * i + 1];
            yr[D - 64 + 2 * i] = a * c - b * s;
            yr[D - 64 + 2 * i + 1] = a * s + b * c;
        }
    }
    return ORC_OK;
}

/* ---- Mixed-precision storage of the compressed KV entries ([HA] §4.2, the
 * paragraph on storage precision: the RoPE dims stay BF16, the rest of each
 * compressed entry is FP8).  Readings (the pages give no granularity or layout):
 *   - the RoPE dims are the last 64 of D; the first D-64 dims are e4m3 codes;
 *   - one scale per block of 64 FP8 dims, a power of two s = 2^e with e the
 *     smallest integer such that amax <= 448 * 2^e (an all-zero block: e = 0), so
 *     x / s is exact and code * s is exactly representable in BF16;
 *   - code = e4m3(x / s), nearest value, ties to the even mantissa;
 *   - entry bytes: [D-64 codes][64 BF16 RoPE dims][(D-64)/64 fp32 scales], zero
 *     padding to a multiple of 16 bytes (608 bytes for D = 512).
 * kv holds BF16 values widened exactly to float. */
int64_t oracle_kv8_entry_bytes(int D)
{
    int64_t b = (int64_t)(D - 64) + 128 + 4 * (int64_t)((D - 64) / 64);
    return (b + 15) / 16 * 16;
}

static uint16_t orc_bf16_bits(float x)      /* x is a BF16 value widened exactly */
{
    uint32_t u;
    memcpy(&u, &x, 4);
    return (uint16_t)(u >> 16);
}

int oracle_kv8_quantize(const float *kv, int64_t rows, int D, uint8_t *entries)
{
    if (D < 128 || D % 64 != 0) return ORC_BAD;
    const int nf = D - 64, nb = nf / 64;
    const int64_t eb = oracle_kv8_entry_bytes(D);
    for (int64_t r = 0; r < rows; ++r) {
        const float *x = kv + r * D;
        uint8_t *e = entries + r * eb;
        memset(e, 0, (size_t)eb);
        for (int blk = 0; blk < nb; ++blk) {
            double amax = 0.0;
            for (int j = 0; j < 64; ++j) {
                double a = fabs((double)x[blk * 64 + j]);
                if (a > amax) amax = a;
            }
            int ex = 0;
            if (amax > 0.0) {
                ex = (int)ceil(log2(amax / 448.0));
                while (ldexp(448.0, ex) < amax) ++ex;          /* smallest e with amax <= 448 * 2^e */
                while (ldexp(448.0, ex - 1) >= amax) --ex;
            }
            const double sc = ldexp(1.0, ex);
            for (int j = 0; j < 64; ++j)
                e[blk * 64 + j] = oracle_e4m3_encode((float)((double)x[blk * 64 + j] / sc));
            const float fs = (float)sc;
            memcpy(e + nf + 128 + 4 * blk, &fs, 4);
        }
        for (int j = 0; j < 64; ++j) {
            uint16_t h = orc_bf16_bits(x[nf + j]);
            memcpy(e + nf + 2 * j, &h, 2);
        }
    }
    return ORC_OK;
}

/* Inverse of the storage above: x = code * s for the FP8 dims, the BF16 bits for
 * the RoPE dims.  Every value is exact in float. */
int oracle_kv8_dequantize(const uint8_t *entries, int64_t rows, int D, float *kv)
{
    if (D < 128 || D % 64 != 0) return ORC_BAD;
    const int nf = D - 64;
    const int64_t eb = oracle_kv8_entry_bytes(D);
    for (int64_t r = 0; r < rows; ++r) {
        const uint8_t *e = entries + r * eb;
        float *x = kv + r * D;
        for (int j = 0; j < nf; ++j) {
            float fs;
            memcpy(&fs, e + nf + 128 + 4 * (j / 64), 4);
            x[j] = (float)(oracle_e4m3_decode(e[j]) * (double)fs);
        }
        for (int j = 0; j < 64; ++j) {
            uint16_t h;
            memcpy(&h, e + nf + 2 * j, 2);
            uint32_t u = (uint32_t)h << 16;
            memcpy(&x[nf + j], &u, 4);
        }
    }
    return ORC_OK;
}

/* [HA] §4.2 on dequantised e4m3 inputs: q = code * q_scale[t,h],
 * k = code * k_scale[i]; the score is the plain definition on those values. */
int oracle_index_scores_e4m3(const uint8_t *q8, const float *q_scale, const float *w,
                             const uint8_t *k8, const float *k_scale, const int32_t *n_valid,
                             int T, int64_t N, int Hi, int d, double *scores, double *mag)
{
    double table[256];
    for (int b = 0; b < 256; ++b) table[b] = oracle_e4m3_decode((uint8_t)b);
    double *qd = (double *)malloc(sizeof(double) * (size_t)Hi * d);
    if (!qd) return ORC_BAD;
    for (int t = 0; t < T; ++t) {
        int64_t nv = n_valid[t];
        if (nv < 0 || nv > N) { free(qd); return ORC_BAD; }
        for (int h = 0; h < Hi; ++h)
            for (int e = 0; e < d; ++e)
                qd[h * d + e] = table[q8[((int64_t)t * Hi + h) * d + e]] * (double)q_scale[(int64_t)t * Hi + h];
        for (int64_t i = 0; i < N; ++i) {
            if (i >= nv) {
                scores[(int64_t)t * N + i] = -INFINITY;
                if (mag) mag[(int64_t)t * N + i] = 0.0;
                continue;
            }
            double ks = k_scale[i];
            double s = 0.0, smag = 0.0;
            for (int h = 0; h < Hi; ++h) {
                double dot = 0.0, dmag = 0.0;
                for (int e = 0; e < d; ++e) {
                    double p = qd[h * d + e] * (table[k8[i * d + e]] * ks);
                    dot += p;
                    dmag += fabs(p);
                }
                double wh = w[(int64_t)t * Hi + h];
                s += wh * (dot > 0.0 ? dot : 0.0);
                smag += fabs(wh) * dmag;
            }
            scores[(int64_t)t * N + i] = s;
            if (mag) mag[(int64_t)t * N + i] = smag;
        }
    }
    free(qd);
    return ORC_OK;
}

/* ---- top-k: full sort by (score descending, index ascending) ------------ */
typedef struct { double s; int64_t i; } orc_pair;

static int orc_cmp_desc(const void *a, const void *b)
{
    const orc_pair *x = (const orc_pair *)a, *y = (const orc_pair *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->i < y->i) ? -1 : (x->i > y->i);
}

static int orc_cmp_i32(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/* [HA] §4.2 / §7 topk(scores, k): the k largest s_{t,i} over i < n_valid(t),
 * lower index first among equal scores, returned in ascending index order,
 * padded with -1 when n_valid(t) < k.  scores [T, N] -> idx [T, k]. */
int oracle_topk(const float *scores, const int32_t *n_valid, int T, int64_t N, int k, int32_t *idx)
{
    if (k <= 0 || N < 0) return ORC_BAD;
    orc_pair *buf = (orc_pair *)malloc(sizeof(orc_pair) * (N > 0 ? N : 1));
    if (!buf) return ORC_BAD;
    for (int t = 0; t < T; ++t) {
        int64_t nv = n_valid[t];
        if (nv < 0 || nv > N) { free(buf); return ORC_BAD; }
        for (int64_t i = 0; i < nv; ++i) {
            buf[i].s = (double)scores[(int64_t)t * N + i];   /* -0.0 == +0.0 here */
            buf[i].i = i;
        }
        qsort(buf, (size_t)nv, sizeof(orc_pair), orc_cmp_desc);
        int64_t take = nv < k ? nv : k;
        int32_t *row = idx + (int64_t)t * k;
        for (int64_t j = 0; j < take; ++j) row[j] = (int32_t)buf[j].i;
        qsort(row, (size_t)take, sizeof(int32_t), orc_cmp_i32);
        for (int64_t j = take; j < k; ++j) row[j] = -1;
    }
    free(buf);
    return ORC_OK;
}

/* ---- attention ------------------------------------------------------------
 * [HA] §6: p_j = exp(z_j) / (exp(z_s) + sum_l exp(z_l)), o = sum_j p_j v_j with
 * the shared latent as both key and value ([HA] §4.2 Shared-KV MQA), over
 * memory = concat(SWA rows, selected rows) ([HA] §7).  Two passes: maximum
 * first, then the normalised sum.  One sequence; rows[] lists the memory. */
static void orc_attend(const float *q, int H, int D, double scale, const float *sink,
                       const float **rows, int64_t n_rows, double *out, double *mag, double *z)
{
    for (int h = 0; h < H; ++h) {
        const float *qh = q + (int64_t)h * D;
        double mx = (double)sink[h];
        for (int64_t j = 0; j < n_rows; ++j) {
            double dot = 0.0;
            for (int e = 0; e < D; ++e) dot += (double)qh[e] * (double)rows[j][e];
            z[j] = scale * dot;
            if (z[j] > mx) mx = z[j];
        }
        double den = exp((double)sink[h] - mx);
        for (int64_t j = 0; j < n_rows; ++j) den += exp(z[j] - mx);
        double *oh = out + (int64_t)h * D;
        double *mh = mag ? mag + (int64_t)h * D : NULL;
        for (int e = 0; e < D; ++e) { oh[e] = 0.0; if (mh) mh[e] = 0.0; }
        for (int64_t j = 0; j < n_rows; ++j) {
            double p = exp(z[j] - mx) / den;
            for (int e = 0; e < D; ++e) {
                oh[e] += p * (double)rows[j][e];
                if (mh) mh[e] += p * fabs((double)rows[j][e]);
            }
        }
    }
}

/* SWA rows visible to the query at absolute position t: positions
 * max(0, t-window+1)..t ([P1] window_size 128; [HA] §6), taken from the raw
 * buffer swa[W, D] whose row 0 is absolute position swa_pos0. */
static int64_t orc_swa_rows(const float *swa, int64_t swa_pos0, int W, int D, int64_t t, int window,
                            const float **rows)
{
    int64_t n = 0;
    int64_t p0 = t - window + 1;
    if (p0 < 0) p0 = 0;
    for (int64_t p = p0; p <= t; ++p) {
        int64_t r = p - swa_pos0;
        if (r < 0 || r >= W) continue;
        rows[n++] = swa + r * D;
    }
    return n;
}

/* sparse_attn for one sequence ([P2] sparse_attn(q, kv, attn_sink, topk_idxs,
 * softmax_scale); [HA] §7 gather + concat + shared_kv_mqa).
 * q [T, H, D], kv [N, D], swa [W, D], q_pos [T], sink [H], idx [T, k]
 * -> out, mag [T, H, D]. */
int oracle_sparse_attn(const float *q, const float *kv, const float *swa, int64_t swa_pos0, int W,
                       const int64_t *q_pos, const float *sink, const int32_t *idx, int k,
                       double scale, int window, int T, int H, int D, int64_t N,
                       double *out, double *mag)
{
    int64_t cap = (int64_t)k + window;
    const float **rows = (const float **)malloc(sizeof(float *) * (cap > 0 ? cap : 1));
    double *z = (double *)malloc(sizeof(double) * (cap > 0 ? cap : 1));
    if (!rows || !z) { free(rows); free(z); return ORC_BAD; }
    for (int t = 0; t < T; ++t) {
        int64_t n = orc_swa_rows(swa, swa_pos0, W, D, q_pos[t], window, rows);
        for (int j = 0; j < k; ++j) {
            int64_t i = idx[(int64_t)t * k + j];
            if (i < 0 || i >= N) continue;
            rows[n++] = kv + i * D;
        }
        orc_attend(q + (int64_t)t * H * D, H, D, scale, sink, rows, n,
                   out + (int64_t)t * H * D, mag ? mag + (int64_t)t * H * D : NULL, z);
    }
    free(rows); free(z);
    return ORC_OK;
}

/* hca_attn for one sequence ([HA] §5: dense MQA over every complete summary,
 * concatenated with the SWA rows): entries 0..n_visible(t)-1 of kv. */
int oracle_hca_attn(const float *q, const float *kv, const float *swa, int64_t swa_pos0, int W,
                    const int64_t *q_pos, const float *sink, int ratio, double scale, int window,
                    int T, int H, int D, int64_t N, double *out, double *mag)
{
    int64_t cap = N + window;
    const float **rows = (const float **)malloc(sizeof(float *) * (cap > 0 ? cap : 1));
    double *z = (double *)malloc(sizeof(double) * (cap > 0 ? cap : 1));
    if (!rows || !z) { free(rows); free(z); return ORC_BAD; }
    for (int t = 0; t < T; ++t) {
        int64_t n = orc_swa_rows(swa, swa_pos0, W, D, q_pos[t], window, rows);
        int64_t nv = oracle_n_visible(q_pos[t], ratio, N);
        for (int64_t i = 0; i < nv; ++i) rows[n++] = kv + i * D;
        orc_attend(q + (int64_t)t * H * D, H, D, scale, sink, rows, n,
                   out + (int64_t)t * H * D, mag ? mag + (int64_t)t * H * D : NULL, z);
    }
    free(rows); free(z);
    return ORC_OK;
}

/* ---- Attention over disjoint row sets, put back together.  The [HA] §6 probability
 * p_i = e^{z_i} / (e^{z_s} + sum_j e^{z_j}) over a union of disjoint row sets splits
 * into per-set pieces without the sink: m = max_j z_j (-inf if the set is empty),
 * l = sum_j e^{z_j - m} (0 if empty), o = sum_j e^{z_j - m} row_j / l (0 if empty).
 * sparse_attn's rows for one query restricted to one set: the SWA rows only if W > 0,
 * and the entries kv[idx] with idx in [0, N).  q [T, H, D] -> m, l [T, H], o [T, H, D]. */
int oracle_sparse_attn_partial(const float *q, const float *kv, const float *swa, int64_t swa_pos0, int W,
                               const int64_t *q_pos, const int32_t *idx, int k, double scale, int window,
                               int T, int H, int D, int64_t N, double *m, double *l, double *o)
{
    int64_t cap = (int64_t)k + window;
    const float **rows = (const float **)malloc(sizeof(float *) * (cap > 0 ? cap : 1));
    double *z = (double *)malloc(sizeof(double) * (cap > 0 ? cap : 1));
    if (!rows || !z) { free(rows); free(z); return ORC_BAD; }
    for (int t = 0; t < T; ++t) {
        int64_t n = W > 0 ? orc_swa_rows(swa, swa_pos0, W, D, q_pos[t], window, rows) : 0;
        for (int j = 0; j < k; ++j) {
            int64_t i = idx[(int64_t)t * k + j];
            if (i < 0 || i >= N) continue;
            rows[n++] = kv + i * D;
        }
        for (int h = 0; h < H; ++h) {
            const float *qh = q + ((int64_t)t * H + h) * D;
            double mx = -INFINITY;
            for (int64_t j = 0; j < n; ++j) {
                double dot = 0.0;
                for (int e = 0; e < D; ++e) dot += (double)qh[e] * (double)rows[j][e];
                z[j] = scale * dot;
                if (z[j] > mx) mx = z[j];
            }
            double sum = 0.0;
            for (int64_t j = 0; j < n; ++j) sum += exp(z[j] - mx);
            double *oh = o + ((int64_t)t * H + h) * D;
            for (int e = 0; e < D; ++e) oh[e] = 0.0;
            for (int64_t j = 0; j < n; ++j) {
                double p = exp(z[j] - mx) / sum;
                for (int e = 0; e < D; ++e) oh[e] += p * (double)rows[j][e];
            }
            m[(int64_t)t * H + h] = mx;
            l[(int64_t)t * H + h] = sum;
        }
    }
    free(rows); free(z);
    return ORC_OK;
}

/* The pieces of G disjoint row sets -> the attention output with the sink added once:
 * M = max(z_s, m_g), den = e^{z_s - M} + sum_g l_g e^{m_g - M},
 * out = sum_g l_g e^{m_g - M} o_g / den.  m, l [G, T, H]; o [G, T, H, D]; out [T, H, D]. */
int oracle_attn_combine(int G, int T, int H, int D, const double *m, const double *l, const double *o,
                        const float *sink, double *out)
{
    for (int t = 0; t < T; ++t)
        for (int h = 0; h < H; ++h) {
            double M = (double)sink[h];
            for (int g = 0; g < G; ++g) {
                double mg = m[((int64_t)g * T + t) * H + h];
                if (mg > M) M = mg;
            }
            double den = exp((double)sink[h] - M);
            for (int g = 0; g < G; ++g) {
                int64_t gi = ((int64_t)g * T + t) * H + h;
                if (l[gi] > 0.0) den += l[gi] * exp(m[gi] - M);
            }
            double *oh = out + ((int64_t)t * H + h) * D;
            for (int e = 0; e < D; ++e) oh[e] = 0.0;
            for (int g = 0; g < G; ++g) {
                int64_t gi = ((int64_t)g * T + t) * H + h;
                if (!(l[gi] > 0.0)) continue;
                double wgt = l[gi] * exp(m[gi] - M) / den;
                for (int e = 0; e < D; ++e) oh[e] += wgt * o[gi * D + e];
            }
        }
    return ORC_OK;
}
