/*
 * CPU oracle for the mixed-bitwidth (EXL2-style) quantised matrix multiply.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header or table with the CUDA library.
 *
 * What it computes (plain definitions, slow on purpose):
 *
 *   Format (nightvoyager.top exllamav2 report, "核心价值提炼" and "关键设计决策";
 *   promptquorum "EXL2量化是什么"): the weight matrix W [K x N] (K input rows in
 *   act-order, N output columns) is quantised with a bitwidth b_j in
 *   {2,3,4,5,6,8} per 32-row block j, mixing widths inside one layer, with the
 *   more important rows holding more bits.  Rows are grouped by 128 and each
 *   (group, column) pair has one fp16 scale (GPTQ lineage, "group 128").
 *
 *   Readings taken where the pages are silent:
 *   - Packed layout: for column n and block j, the 32 codes of the block form
 *     a 32*b_j-bit little-endian stream, code r at stream bits [r*b_j, r*b_j+b_j).
 *     Stream bit t is bit (t mod 32) of word row off_j + t/32, where
 *     off_j = sum_{i<j} b_i; words are stored row-major [sum b][N].
 *   - Dequantisation is symmetric around the mid code: w = (q - 2^(b-1)) * s.
 *   - y[m][n] = sum_k x[m][perm[k]] * w[k][n]  (perm[k] is the column of x that
 *     multiplies W row k).
 *
 * Arithmetic: codes are integers, dequantised weights are exact in double
 * (an 8-bit integer times an fp16 value), sums are accumulated in double in
 * natural k order.  fp16 <-> double conversions are written out with integer
 * bit manipulation so no compiler or library rounding is involved.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORC_BLOCK 32
#define ORC_GROUP 128

enum { ORC_OK = 0, ORC_ERR_SHAPE = -2, ORC_ERR_BITS = -3, ORC_ERR_CODE = -9 };

static int width_allowed(int b) {
    return b == 2 || b == 3 || b == 4 || b == 5 || b == 6 || b == 8;
}

/* Sum of block widths = number of packed word rows, or a negative error. */
int64_t oracle_word_rows(const uint8_t *bits, int K) {
    if (K <= 0 || K % ORC_BLOCK) return ORC_ERR_SHAPE;
    int64_t s = 0;
    for (int j = 0; j < K / ORC_BLOCK; ++j) {
        if (!width_allowed(bits[j])) return ORC_ERR_BITS;
        s += bits[j];
    }
    return s;
}

/* Word row where each block starts (off_j), computed here independently. */
static void block_offsets(const uint8_t *bits, int nb, int64_t *off) {
    int64_t s = 0;
    for (int j = 0; j < nb; ++j) { off[j] = s; s += bits[j]; }
}

/* Code of row k, column n, read bit by bit from the packed stream. */
static uint32_t read_code(const uint32_t *qw, int64_t N, int64_t off, int b, int r, int64_t n) {
    uint32_t q = 0;
    for (int t = 0; t < b; ++t) {
        int64_t p = (int64_t)r * b + t;                 /* stream bit */
        uint32_t word = qw[(off + p / 32) * N + n];
        q |= ((word >> (p % 32)) & 1u) << t;
    }
    return q;
}

/* codes [K][N] (uint8, act-order rows) -> qw [sum b][N].  Returns ORC_ERR_CODE
 * if a code does not fit its block width. */
int oracle_pack(const uint8_t *codes, const uint8_t *bits, int K, int N, uint32_t *qw) {
    int64_t rows = oracle_word_rows(bits, K);
    if (rows < 0) return (int)rows;
    if (N <= 0) return ORC_ERR_SHAPE;
    memset(qw, 0, (size_t)rows * (size_t)N * sizeof(uint32_t));
    int nb = K / ORC_BLOCK;
    int64_t off = 0;
    for (int j = 0; j < nb; ++j) {
        int b = bits[j];
        for (int r = 0; r < ORC_BLOCK; ++r) {
            const uint8_t *row = codes + (int64_t)(j * ORC_BLOCK + r) * N;
            for (int64_t n = 0; n < N; ++n) {
                uint32_t q = row[n];
                if (q >> b) return ORC_ERR_CODE;
                for (int t = 0; t < b; ++t) {
                    int64_t p = (int64_t)r * b + t;
                    if ((q >> t) & 1u) qw[(off + p / 32) * N + n] |= 1u << (p % 32);
                }
            }
        }
        off += b;
    }
    return ORC_OK;
}

/* qw -> codes [K][N]: the inverse of oracle_pack. */
int oracle_unpack(const uint32_t *qw, const uint8_t *bits, int K, int N, uint8_t *codes) {
    int64_t rows = oracle_word_rows(bits, K);
    if (rows < 0) return (int)rows;
    int nb = K / ORC_BLOCK;
    int64_t off = 0;
    for (int j = 0; j < nb; ++j) {
        for (int r = 0; r < ORC_BLOCK; ++r)
            for (int64_t n = 0; n < N; ++n)
                codes[(int64_t)(j * ORC_BLOCK + r) * N + n] = (uint8_t)read_code(qw, N, off, bits[j], r, n);
        off += bits[j];
    }
    return ORC_OK;
}

/* IEEE binary16 bit pattern -> exact double. */
double oracle_half_to_double(uint16_t h) {
    int sign = h >> 15, e = (h >> 10) & 0x1f, m = h & 0x3ff;
    double v;
    if (e == 0) v = ldexp((double)m, -24);                    /* zero / subnormal */
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp((double)(1024 + m), e - 25);
    return sign ? -v : v;
}

/* double -> binary16, round to nearest, ties to even, by integer arithmetic on
 * the double's bit pattern (one rounding step). */
uint16_t oracle_double_to_half(double v) {
    uint64_t u;
    memcpy(&u, &v, sizeof u);
    uint16_t sign = (uint16_t)((u >> 48) & 0x8000);
    int e2 = (int)((u >> 52) & 0x7ff);
    uint64_t frac = u & ((1ull << 52) - 1);
    if (e2 == 0x7ff) return frac ? (uint16_t)(sign | 0x7e00) : (uint16_t)(sign | 0x7c00);
    if (e2 == 0 && frac == 0) return sign;
    int e;                 /* value = mant * 2^(e - 52), mant in [2^52, 2^53) */
    uint64_t mant;
    if (e2 == 0) {         /* double subnormal: far below fp16 range */
        return sign;
    }
    e = e2 - 1023;
    mant = frac | (1ull << 52);
    if (e > 15) return (uint16_t)(sign | 0x7c00);
    /* Units of the result's last place: 2^(e-10) for normal fp16, 2^-24 for
     * subnormal fp16.  shift = number of low mantissa bits dropped. */
    int shift = (e >= -14) ? 42 : 28 - e;
    if (shift > 53) return sign;        /* < half of the smallest subnormal */
    uint64_t q = mant >> shift;
    uint64_t rem = mant & ((1ull << shift) - 1);
    uint64_t half = 1ull << (shift - 1);
    if (rem > half || (rem == half && (q & 1))) ++q;
    if (e >= -14) {
        if (q == 2048) { q = 1024; ++e; }
        if (e > 15) return (uint16_t)(sign | 0x7c00);
        return (uint16_t)(sign | ((uint16_t)(e + 15) << 10) | (uint16_t)(q & 0x3ff));
    }
    return (uint16_t)(sign | (uint16_t)q);   /* q == 1024 encodes the smallest normal */
}

/* w[k][n] = (q - 2^(b-1)) * s[k/128][n], exact in double. */
int oracle_dequant_f64(const uint32_t *qw, const uint16_t *scales, const uint8_t *bits,
                       int K, int N, double *w) {
    int64_t rows = oracle_word_rows(bits, K);
    if (rows < 0) return (int)rows;
    int nb = K / ORC_BLOCK;
    int64_t off = 0;
    for (int j = 0; j < nb; ++j) {
        int b = bits[j];
        for (int r = 0; r < ORC_BLOCK; ++r) {
            int k = j * ORC_BLOCK + r;
            for (int64_t n = 0; n < N; ++n) {
                int q = (int)read_code(qw, N, off, b, r, n);
                double s = oracle_half_to_double(scales[(int64_t)(k / ORC_GROUP) * N + n]);
                w[(int64_t)k * N + n] = (double)(q - (1 << (b - 1))) * s;
            }
        }
        off += b;
    }
    return ORC_OK;
}

/* The fp16 dequantised matrix: each exact weight rounded once (RNE). */
int oracle_dequant_f16(const uint32_t *qw, const uint16_t *scales, const uint8_t *bits,
                       int K, int N, uint16_t *w16) {
    int64_t rows = oracle_word_rows(bits, K);
    if (rows < 0) return (int)rows;
    double *w = (double *)malloc((size_t)K * (size_t)N * sizeof(double));
    if (!w) return -100;
    oracle_dequant_f64(qw, scales, bits, K, N, w);
    for (int64_t i = 0; i < (int64_t)K * N; ++i) w16[i] = oracle_double_to_half(w[i]);
    free(w);
    return ORC_OK;
}

/* ---------------------------------------------------------------------------
 * y[m][c] = sum_k x[m][perm[k]] * w[k][col_c], double accumulation in natural
 * k order.  Columns col_c = cols[c] (or c when cols == NULL).  The column list
 * is split across threads; each thread handles whole columns.
 * ------------------------------------------------------------------------- */
typedef struct {
    const double *x; const int32_t *perm; const uint32_t *qw; const uint16_t *scales;
    const uint8_t *bits; const int64_t *off; const int64_t *cols;
    int M, K; int64_t N, ncols, c0, c1; double *y;
} gemm_job;

static void *gemm_worker(void *arg) {
    gemm_job *J = (gemm_job *)arg;
    int nb = J->K / ORC_BLOCK;
    double *acc = (double *)malloc(sizeof(double) * (size_t)J->M);
    for (int64_t c = J->c0; c < J->c1; ++c) {
        int64_t n = J->cols ? J->cols[c] : c;
        for (int m = 0; m < J->M; ++m) acc[m] = 0.0;
        for (int j = 0; j < nb; ++j) {
            int b = J->bits[j];
            for (int r = 0; r < ORC_BLOCK; ++r) {
                int k = j * ORC_BLOCK + r;
                int q = (int)read_code(J->qw, J->N, J->off[j], b, r, n);
                double s = oracle_half_to_double(J->scales[(int64_t)(k / ORC_GROUP) * J->N + n]);
                double w = (double)(q - (1 << (b - 1))) * s;
                int32_t src = J->perm[k];
                for (int m = 0; m < J->M; ++m) acc[m] += J->x[(int64_t)m * J->K + src] * w;
            }
        }
        for (int m = 0; m < J->M; ++m) J->y[(int64_t)m * J->ncols + c] = acc[m];
    }
    free(acc);
    return NULL;
}

/* x: double [M][K]; perm: int32 [K] (a permutation of 0..K-1); qw: [sum b][N];
 * scales: fp16 bits [ceil(K/128)][N]; y: double [M][ncols].
 * nthreads <= 0 uses every online core.  Returns the thread count used, or a
 * negative error. */
int oracle_qgemm_f64(const double *x, const int32_t *perm, const uint32_t *qw,
                     const uint16_t *scales, const uint8_t *bits, int M, int K, int N,
                     const int64_t *cols, int64_t ncols, double *y, int nthreads) {
    int64_t rows = oracle_word_rows(bits, K);
    if (rows < 0) return (int)rows;
    if (M <= 0 || N <= 0) return ORC_ERR_SHAPE;
    for (int k = 0; k < K; ++k)
        if (perm[k] < 0 || perm[k] >= K) return ORC_ERR_SHAPE;
    if (!cols) ncols = N;
    int nb = K / ORC_BLOCK;
    int64_t *off = (int64_t *)malloc(sizeof(int64_t) * (size_t)nb);
    block_offsets(bits, nb, off);
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > ncols) nthreads = (int)ncols;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    gemm_job *jobs = (gemm_job *)malloc(sizeof(gemm_job) * (size_t)nthreads);
    for (int t = 0; t < nthreads; ++t) {
        gemm_job J = {x, perm, qw, scales, bits, off, cols, M, K, N, ncols,
                      ncols * t / nthreads, ncols * (t + 1) / nthreads, y};
        jobs[t] = J;
        pthread_create(&th[t], NULL, gemm_worker, &jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(th); free(jobs); free(off);
    return nthreads;
}

/* Array forms of the two conversions, for the tests. */
void oracle_half_to_double_n(const uint16_t *h, double *v, int64_t n) {
    for (int64_t i = 0; i < n; ++i) v[i] = oracle_half_to_double(h[i]);
}

void oracle_double_to_half_n(const double *v, uint16_t *h, int64_t n) {
    for (int64_t i = 0; i < n; ++i) h[i] = oracle_double_to_half(v[i]);
}

/* ---------------------------------------------------------------------------
 * Quantiser: fp16 weights W [K][N] (act-order rows) and the block widths ->
 * codes [K][N] and fp16 scales [ceil(K/128)][N], the step before pack.
 *
 * The pages (nightvoyager.top exllamav2 report, "关键设计决策", adaptive scale
 * paragraph) name two parts: a 4-bit second-level quantisation of the group
 * scale, qscale = round(sqrt(base_scale / qscale_max) * (scale_maxq + 1)), and
 * a scan of 96 candidate p factors per layer that keeps the one with the
 * lowest quantisation error.  Everything else is this library's reading:
 *
 *   base[g]  = max over the blocks j of group g of max_k |W[k][n]| / 2^(b_j-1)
 *              (the smallest scale at which no weight of the group exceeds
 *              its block's largest code magnitude);
 *   qmax     = max_g base[g] (per column);
 *   qs[g]    = clamp(rint(sqrt(base[g] / qmax) * 16), 1, 16), the 4-bit
 *              second-level scale (scale_maxq = 15);
 *   p_i      = (32 + i) / 96, i = 0..95 (p_64 = 1);
 *   s_i[g]   = fp16(p_i * (qmax * (qs[g]^2 / 256)));
 *   q        = clamp(rint(W * (1 / s)) + 2^(b-1), 0, 2^b - 1), and q = 2^(b-1)
 *              where s is 0 (an all-zero column);
 *   e        = (W - (q - 2^(b-1)) * s)^2;
 *   E(p_i)   = sum over columns n (increasing) of the sum over rows k
 *              (increasing) of e; the layer keeps the smallest E (the lowest
 *              i on ties) and those codes and scales.
 * Arithmetic: single precision, each operation rounded to nearest even (the
 * precision the GPU kernel decides codes in), the error terms and sums in
 * double.  fp16 <-> float conversions go through the exact helpers above.
 * ------------------------------------------------------------------------- */
#define ORC_QCANDS 96

static float cand_factor(int i) { return (float)(32 + i) / 96.0f; }

static float half_to_float(uint16_t h) { return (float)oracle_half_to_double(h); }

/* 4-bit second-level scales qs[g] (as floats 1..16) and qmax of column n. */
static float column_qscales(const uint16_t *w, const uint8_t *bits, int K, int64_t N, int64_t n, float *qs) {
    int G = (K + ORC_GROUP - 1) / ORC_GROUP;
    float qmax = 0.0f;
    for (int g = 0; g < G; ++g) {
        float base = 0.0f;
        for (int k = g * ORC_GROUP; k < K && k < (g + 1) * ORC_GROUP; ++k) {
            float a = fabsf(half_to_float(w[(int64_t)k * N + n]));
            float r = a / (float)(1 << (bits[k / ORC_BLOCK] - 1));  /* exact: a power of two */
            if (r > base) base = r;
        }
        qs[g] = base;  /* base for now */
        if (base > qmax) qmax = base;
    }
    for (int g = 0; g < G; ++g) {
        if (qmax == 0.0f) {
            qs[g] = 16.0f;
            continue;
        }
        float t = rintf(sqrtf(qs[g] / qmax) * 16.0f);
        qs[g] = t < 1.0f ? 1.0f : (t > 16.0f ? 16.0f : t);
    }
    return qmax;
}

static uint16_t cand_scale(float p, float qmax, float qs) {
    float u = qmax * ((qs * qs) / 256.0f);  /* qs^2 exact, /256 exact */
    float v = p * u;
    return oracle_double_to_half((double)v);
}

/* Codes of column n under the given group scales; returns the squared error
 * summed over k in increasing order. */
static double column_codes(const uint16_t *w, const uint8_t *bits, int K, int64_t N, int64_t n,
                           const uint16_t *sc, uint8_t *codes) {
    double err = 0.0;
    int g_cur = -1;
    float s = 0.0f, inv = 0.0f;
    for (int k = 0; k < K; ++k) {
        int g = k / ORC_GROUP;
        if (g != g_cur) {
            g_cur = g;
            s = half_to_float(sc[g]);
            inv = (s == 0.0f) ? 0.0f : 1.0f / s;
        }
        int b = bits[k / ORC_BLOCK], z = 1 << (b - 1);
        float x = half_to_float(w[(int64_t)k * N + n]);
        int q = z;
        if (s != 0.0f) {
            float t = rintf(x * inv);
            if (t != t) t = 0.0f;  /* not a number: the zero point */
            float lo = (float)(-z), hi = (float)((1 << b) - 1 - z);
            t = t < lo ? lo : (t > hi ? hi : t);
            q = (int)t + z;
        }
        if (codes) codes[(int64_t)k * N + n] = (uint8_t)q;
        double d = (double)x - (double)((float)(q - z) * s);
        err += d * d;
    }
    return err;
}

typedef struct {
    const uint16_t *w; const uint8_t *bits; int K; int64_t N, c0, c1; double *colerr;
} quant_job;

static void *quant_worker(void *arg) {
    quant_job *J = (quant_job *)arg;
    int G = (J->K + ORC_GROUP - 1) / ORC_GROUP;
    float *qs = (float *)malloc(sizeof(float) * (size_t)G);
    uint16_t *sc = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)G);
    for (int64_t n = J->c0; n < J->c1; ++n) {
        float qmax = column_qscales(J->w, J->bits, J->K, J->N, n, qs);
        for (int i = 0; i < ORC_QCANDS; ++i) {
            for (int g = 0; g < G; ++g) sc[g] = cand_scale(cand_factor(i), qmax, qs[g]);
            J->colerr[(int64_t)i * J->N + n] = column_codes(J->w, J->bits, J->K, J->N, n, sc, NULL);
        }
    }
    free(qs); free(sc);
    return NULL;
}

/* w: fp16 bits [K][N]; codes: [K][N]; scales: fp16 bits [ceil(K/128)][N];
 * colerr (optional): double [96][N], the error of every column under every
 * candidate; err: double [96], E(p_i).  Returns the chosen candidate index
 * (>= 0) or a negative error.  nthreads <= 0 uses every online core. */
int oracle_quantize(const uint16_t *w, const uint8_t *bits, int K, int N, uint8_t *codes, uint16_t *scales,
                    double *colerr, double *err, int nthreads) {
    int64_t rows = oracle_word_rows(bits, K);
    if (rows < 0) return (int)rows;
    if (N <= 0) return ORC_ERR_SHAPE;
    double *ce = colerr ? colerr : (double *)malloc(sizeof(double) * ORC_QCANDS * (size_t)N);
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > N) nthreads = N;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    quant_job *jobs = (quant_job *)malloc(sizeof(quant_job) * (size_t)nthreads);
    for (int t = 0; t < nthreads; ++t) {
        quant_job J = {w, bits, K, N, (int64_t)N * t / nthreads, (int64_t)N * (t + 1) / nthreads, ce};
        jobs[t] = J;
        pthread_create(&th[t], NULL, quant_worker, &jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(th); free(jobs);
    int best = 0;
    double best_e = 0.0;
    for (int i = 0; i < ORC_QCANDS; ++i) {
        double e = 0.0;
        for (int64_t n = 0; n < N; ++n) e += ce[(int64_t)i * N + n];
        if (err) err[i] = e;
        if (i == 0 || e < best_e) {
            best = i;
            best_e = e;
        }
    }
    int G = (K + ORC_GROUP - 1) / ORC_GROUP;
    float *qs = (float *)malloc(sizeof(float) * (size_t)G);
    uint16_t *sc = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)G);
    for (int64_t n = 0; n < N; ++n) {
        float qmax = column_qscales(w, bits, K, N, n, qs);
        for (int g = 0; g < G; ++g) {
            sc[g] = cand_scale(cand_factor(best), qmax, qs[g]);
            scales[(int64_t)g * N + n] = sc[g];
        }
        column_codes(w, bits, K, N, n, sc, codes);
    }
    free(qs); free(sc);
    if (!colerr) free(ce);
    return best;
}

/* ---------------------------------------------------------------------------
 * KV-cache quantisation with a Hadamard rotation (nightvoyager.top exllamav2
 * report, "创新之处": K/V are rotated by a Sylvester/Paley Hadamard matrix and
 * then quantised to 4 bits; navi2ai ExLlamaV3 page, "核心能力": 2-8 bit caches).
 * Readings taken here (the pages give no more):
 *   - each (token, head) vector v of length D (a power of two, 32..256) is
 *     rotated by the Sylvester matrix H_D (H_1 = [1], H_2n = [[H, H], [H, -H]])
 *     without normalisation: u = H_D v;
 *   - u is cut into groups of 32; each group gets one fp16 scale
 *     s = fp16(max|u| / (2^(b-1) - 1)) and codes
 *     q = clamp(rint(u * (1 / s)) + 2^(b-1), 0, 2^b - 1) (the zero point where
 *     s is 0), packed as the weights' 32-code blocks (b words, code r at bits
 *     [r b, r b + b) of the LSB-first stream);
 *   - dequantisation: u' = (q - 2^(b-1)) s, v' = fp16((H_D u') / D)
 *     (H_D H_D = D I).
 * The rotation runs as the fast Walsh-Hadamard transform in single precision,
 * stage by stage with strides 1, 2, 4, ..., D/2, each stage replacing the pair
 * (a at i, b at i + stride) with (a + b, a - b), every operation rounded to
 * nearest even: the order the GPU kernel uses, so that codes are decided on
 * the same single-precision values.
 * ------------------------------------------------------------------------- */
static int kv_dim_ok(int D) { return D == 32 || D == 64 || D == 128 || D == 256; }

static void fwht_f32(float *a, int D) {
    for (int st = 1; st < D; st <<= 1)
        for (int i = 0; i < D; ++i)
            if (!(i & st)) {
                float x = a[i], y = a[i + st];
                a[i] = x + y;
                a[i + st] = x - y;
            }
}

/* v: fp16 bits [nvec][D]; codes: uint32 [nvec][D/32][b]; scales: fp16 bits
 * [nvec][D/32]. */
int oracle_kv_quantize(const uint16_t *v, int64_t nvec, int D, int b, uint32_t *codes, uint16_t *scales) {
    if (!kv_dim_ok(D) || nvec < 0) return ORC_ERR_SHAPE;
    if (!width_allowed(b)) return ORC_ERR_BITS;
    float u[256];
    const int z = 1 << (b - 1), ng = D / 32;
    for (int64_t t = 0; t < nvec; ++t) {
        for (int i = 0; i < D; ++i) u[i] = half_to_float(v[t * D + i]);
        fwht_f32(u, D);
        for (int g = 0; g < ng; ++g) {
            float amax = 0.0f;
            for (int i = 0; i < 32; ++i) {
                float a = fabsf(u[32 * g + i]);
                if (a > amax) amax = a;
            }
            uint16_t sh = oracle_double_to_half((double)(amax / (float)(z - 1)));
            scales[t * ng + g] = sh;
            float s = half_to_float(sh);
            float inv = (s == 0.0f) ? 0.0f : 1.0f / s;
            uint32_t *w = codes + (t * ng + g) * b;
            for (int k = 0; k < b; ++k) w[k] = 0u;
            for (int i = 0; i < 32; ++i) {
                int q = z;
                if (s != 0.0f) {
                    float r = rintf(u[32 * g + i] * inv);
                    if (r != r) r = 0.0f;
                    float lo = (float)(-z), hi = (float)(z - 1);
                    r = r < lo ? lo : (r > hi ? hi : r);
                    q = (int)r + z;
                }
                for (int k = 0; k < b; ++k)
                    if ((q >> k) & 1) {
                        int p = i * b + k;
                        w[p / 32] |= 1u << (p % 32);
                    }
            }
        }
    }
    return ORC_OK;
}

int oracle_kv_dequantize(const uint32_t *codes, const uint16_t *scales, int64_t nvec, int D, int b, uint16_t *v) {
    if (!kv_dim_ok(D) || nvec < 0) return ORC_ERR_SHAPE;
    if (!width_allowed(b)) return ORC_ERR_BITS;
    float u[256];
    const int z = 1 << (b - 1), ng = D / 32;
    for (int64_t t = 0; t < nvec; ++t) {
        for (int g = 0; g < ng; ++g) {
            const uint32_t *w = codes + (t * ng + g) * b;
            float s = half_to_float(scales[t * ng + g]);
            for (int i = 0; i < 32; ++i) {
                int q = 0;
                for (int k = 0; k < b; ++k) {
                    int p = i * b + k;
                    q |= (int)((w[p / 32] >> (p % 32)) & 1u) << k;
                }
                u[32 * g + i] = (float)(q - z) * s;
            }
        }
        fwht_f32(u, D);
        for (int i = 0; i < D; ++i) v[t * D + i] = oracle_double_to_half((double)(u[i] / (float)D));
    }
    return ORC_OK;
}
