/*
 * tg_oracle.c -- CPU reference for the fused fp16 GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header, table or
 * helper with the CUDA library; it has its own fp16 decoder and encoder and
 * its own loops.
 *
 * What it computes (the plain definition, written out):
 *
 *   ref[i][j] = g( sum_{k<K} a(i,k) * b(k,j)  +  beta(j) )
 *
 *   a(i,k), b(k,j)  the exact values of the fp16 inputs, decoded to double.
 *     Source: "Designing High-Performance GPU Kernels with TileLang"
 *     (thecryptopost.io), the make_matmul kernel: A is an (M,K) float16
 *     tensor, B a (K,N) float16 tensor, C an (M,N) float16 tensor, and the
 *     tile loop accumulates A-tile times B-tile into a "float" fragment.
 *   beta(j) = bias[j] for the BIAS and BIAS_GELU epilogues, else 0.
 *   g = identity for NONE and BIAS; g(v) = v * Phi(v) for BIAS_GELU, where
 *     Phi is the standard normal CDF (the erf form of GELU).
 *     Source: same tutorial (ainovat.com), fused-epilogue section: the bias
 *     add and the GELU are applied to the accumulator before the single
 *     write of the output.
 *   BIAS_GELU_TANH: g(v) = v/2 (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))),
 *     the tanh approximation of GELU (Hendrycks & Gimpel, "Gaussian Error
 *     Linear Units", section 2).
 *   BIAS_SOFTMAX: row-wise softmax of z = A.B + bias over the N columns of
 *     each row, ref[i][j] = exp(z_ij - max_j z_ij) / sum_j exp(z_ij - max_j z_ij).
 *     Source: same tutorial (ainovat.com), the row-wise softmax section (max
 *     and sum reductions per row, normalisation), here as a GEMM epilogue.
 *
 * Attention forward (tgo_attention), for the FlashAttention kernel of the same
 * tutorial (ainovat.com, FlashAttention section: query, key and value tiles,
 * online softmax with running maxima and sums, causal and non-causal, checked
 * against PyTorch's scaled dot-product attention), written as its plain
 * definition rather than the tiled, online algorithm:
 *
 *   s_ij = scale * sum_d q(i,d) k(j,d),   visible(i,j) = j < Sk and (!causal or j <= i)
 *   p_ij = exp(s_ij - max_j' s_ij') / sum_j' exp(s_ij' - max_j' s_ij')  over visible j, j'
 *   O(i,d) = sum_j p_ij v(j,d)   (0 for a row with no visible key)
 *
 *   per (batch, head), Q [Sq, D], K [Sk, D], V [Sk, D], O [Sq, D], all row-major
 *   slices of [B, H, S, D] tensors.  The causal mask keeps key j <= query i
 *   (the lower-triangular mask of scaled dot-product attention, aligned at
 *   the top-left corner when Sq != Sk).
 *
 * Every fp16 x fp16 product is exact in double (11 + 11 significant bits),
 * and a double sum of at most 2^31 such terms keeps an error far below the
 * fp16 resolution of the result, so the double result is the reference;
 * it is NOT rounded to fp16 (except in tgo_gemm_int_exact, which returns
 * the correctly rounded fp16 of an exactly known integer).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - bias is added to the fp32 accumulator before GELU: GELU(acc + bias).
 *   - GELU uses erf (not the tanh approximation); written as
 *     0.5 * v * erfc(-v / sqrt(2)), which equals 0.5 * v * (1 + erf(v/sqrt 2))
 *     exactly in real arithmetic and avoids cancellation for v << 0.
 *   - out-of-range rows/columns contribute nothing; K == 0 gives g(beta(j)).
 *
 * Loop order is i-k-j over a double accumulator row; rows are independent
 * and split across OpenMP threads.  No blocking, no reordering beyond that.
 */
#define _GNU_SOURCE
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define TGO_EPI_NONE 0
#define TGO_EPI_BIAS 1
#define TGO_EPI_BIAS_GELU 2
#define TGO_EPI_BIAS_GELU_TANH 3
#define TGO_EPI_BIAS_SOFTMAX 4

#define TGO_OK 0
#define TGO_ERR_ARG 1
#define TGO_ERR_NOT_INTEGER 2
#define TGO_ERR_RANGE 3

/* fp16 (IEEE 754 binary16) bit pattern -> exact double. */
double tgo_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int exponent = (h >> 10) & 0x1F;
    int mantissa = h & 0x3FF;
    double v;
    if (exponent == 0) {
        v = ldexp((double)mantissa, -24);            /* zero / subnormal */
    } else if (exponent == 31) {
        v = mantissa ? NAN : INFINITY;
    } else {
        v = ldexp((double)(mantissa + 1024), exponent - 25);
    }
    return sign ? -v : v;
}

/* double -> fp16 bit pattern, round to nearest, ties to even. */
uint16_t tgo_double_to_half_rne(double x)
{
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    if (isnan(x)) return 0x7E00;
    double a = fabs(x);
    /* 65504 is the largest finite half; the midpoint to 65536 is 65520 and
     * ties go to the even neighbour 65536, which overflows to infinity. */
    if (a >= 65520.0) return sign | 0x7C00;
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: units of 2^-24; q == 1024 encodes 2^-14 (the
         * smallest normal) with the same bit pattern, so it needs no case. */
        double q = nearbyint(ldexp(a, 24));
        return sign | (uint16_t)q;
    }
    int e2;
    (void)frexp(a, &e2);          /* a = f * 2^e2, f in [0.5, 1) */
    int e = e2 - 1;               /* a in [2^e, 2^(e+1)), e in [-14, 15] */
    double q = nearbyint(ldexp(a, 10 - e));   /* in [1024, 2048] */
    if (q >= 2048.0) { q = 1024.0; e += 1; }
    if (e > 15) return sign | 0x7C00;
    return sign | (uint16_t)(((e + 15) << 10) | ((int)q - 1024));
}

/* GELU, erf form: v * Phi(v), Phi the standard normal CDF. */
double tgo_gelu(double v)
{
    return 0.5 * v * erfc(-v / sqrt(2.0));
}

/* tanh approximation of GELU. */
double tgo_gelu_tanh(double v)
{
    const double c = sqrt(2.0 / M_PI);
    return 0.5 * v * (1.0 + tanh(c * (v + 0.044715 * v * v * v)));
}

/* Elementwise epilogues (all but BIAS_SOFTMAX, which needs the whole row). */
static double apply_epilogue(double acc, double beta, int epilogue)
{
    double v = acc + beta;
    if (epilogue == TGO_EPI_BIAS_GELU) return tgo_gelu(v);
    if (epilogue == TGO_EPI_BIAS_GELU_TANH) return tgo_gelu_tanh(v);
    return v;
}

/* Row softmax in place: z <- exp(z - max z) / sum exp(z - max z). */
static void softmax_row(double *z, int64_t N)
{
    if (N <= 0) return;
    double m = z[0];
    for (int64_t j = 1; j < N; ++j) m = z[j] > m ? z[j] : m;
    double s = 0.0;
    for (int64_t j = 0; j < N; ++j) {
        z[j] = exp(z[j] - m);
        s += z[j];
    }
    for (int64_t j = 0; j < N; ++j) z[j] /= s;
}

static int check_args(const uint16_t *A, const uint16_t *B, const uint16_t *bias,
                      int64_t M, int64_t N, int64_t K, int epilogue)
{
    (void)bias;
    if (M < 0 || N < 0 || K < 0) return TGO_ERR_ARG;
    if (epilogue < TGO_EPI_NONE || epilogue > TGO_EPI_BIAS_SOFTMAX) return TGO_ERR_ARG;
    if ((M > 0 && K > 0 && !A) || (K > 0 && N > 0 && !B)) return TGO_ERR_ARG;
    return TGO_OK;
}

/* Decode an fp16 array into a freshly allocated double array. */
static double *decode_all(const uint16_t *src, int64_t n)
{
    double *dst = (double *)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    if (!dst) return NULL;
    for (int64_t t = 0; t < n; ++t) dst[t] = tgo_half_to_double(src[t]);
    return dst;
}

/* One output row: ref_row[j] = g(sum_k a(i,k) b(k,j) + beta(j)). */
static void one_row(const double *Ad, const double *Bd, const double *biasd,
                    int64_t i, int64_t N, int64_t K, int epilogue, double *ref_row)
{
    for (int64_t j = 0; j < N; ++j) ref_row[j] = 0.0;
    for (int64_t k = 0; k < K; ++k) {
        double a = Ad[i * K + k];
        const double *brow = Bd + k * N;
        for (int64_t j = 0; j < N; ++j) ref_row[j] += a * brow[j];
    }
    for (int64_t j = 0; j < N; ++j) {
        double beta = (epilogue != TGO_EPI_NONE && biasd) ? biasd[j] : 0.0;
        ref_row[j] = apply_epilogue(ref_row[j], beta, epilogue);
    }
    if (epilogue == TGO_EPI_BIAS_SOFTMAX) softmax_row(ref_row, N);
}

/*
 * Reference for the selected rows.  rows[r] in [0, M); out is nrows x N,
 * row-major, double.  rows == NULL means all M rows (nrows ignored).
 * bias may be NULL (treated as zeros).  Returns TGO_OK or an error code.
 */
int tgo_gemm_rows(const uint16_t *A, const uint16_t *B, const uint16_t *bias,
                  int64_t M, int64_t N, int64_t K, int epilogue,
                  const int64_t *rows, int64_t nrows, double *out)
{
    int st = check_args(A, B, bias, M, N, K, epilogue);
    if (st) return st;
    if (!rows) nrows = M;
    if (nrows < 0 || (nrows > 0 && N > 0 && !out)) return TGO_ERR_ARG;
    if (rows)
        for (int64_t r = 0; r < nrows; ++r)
            if (rows[r] < 0 || rows[r] >= M) return TGO_ERR_RANGE;
    if (nrows == 0 || N == 0) return TGO_OK;

    /* Decode only the A rows that are needed. */
    double *Ad = (double *)malloc((size_t)(nrows * (K > 0 ? K : 1)) * sizeof(double));
    double *Bd = decode_all(B, K * N);
    double *biasd = bias ? decode_all(bias, N) : NULL;
    if (!Ad || !Bd || (bias && !biasd)) {
        free(Ad); free(Bd); free(biasd);
        return TGO_ERR_ARG;
    }
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t i = rows ? rows[r] : r;
        for (int64_t k = 0; k < K; ++k) Ad[r * K + k] = tgo_half_to_double(A[i * K + k]);
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r)
        one_row(Ad, Bd, biasd, r, N, K, epilogue, out + r * N);
    free(Ad); free(Bd); free(biasd);
    return TGO_OK;
}

/* Reference for the whole (M, N) output. */
int tgo_gemm(const uint16_t *A, const uint16_t *B, const uint16_t *bias,
             int64_t M, int64_t N, int64_t K, int epilogue, double *out)
{
    return tgo_gemm_rows(A, B, bias, M, N, K, epilogue, NULL, M, out);
}

/*
 * Exact mode for integer-valued inputs: the sum is formed in int64 (exact),
 * the bias (NONE or BIAS only) added as an integer, and the result encoded
 * to fp16 with round-to-nearest-even -- the unique correctly rounded fp16
 * output.  Returns TGO_ERR_NOT_INTEGER if any input is not an integer of
 * magnitude below 2^11 (all such values are exact in fp16), or if the
 * epilogue is BIAS_GELU (whose result is not an integer).
 */
int tgo_gemm_int_exact(const uint16_t *A, const uint16_t *B, const uint16_t *bias,
                       int64_t M, int64_t N, int64_t K, int epilogue, uint16_t *C_bits)
{
    int st = check_args(A, B, bias, M, N, K, epilogue);
    if (st) return st;
    if (epilogue != TGO_EPI_NONE && epilogue != TGO_EPI_BIAS) return TGO_ERR_NOT_INTEGER;
    if (M == 0 || N == 0) return TGO_OK;
    if (!C_bits) return TGO_ERR_ARG;
    int64_t *Ai = (int64_t *)malloc((size_t)(M * (K > 0 ? K : 1)) * sizeof(int64_t));
    int64_t *Bi = (int64_t *)malloc((size_t)((K > 0 ? K : 1) * N) * sizeof(int64_t));
    int64_t *bi = (int64_t *)calloc((size_t)N, sizeof(int64_t));
    if (!Ai || !Bi || !bi) { free(Ai); free(Bi); free(bi); return TGO_ERR_ARG; }
    int bad = 0;
    for (int64_t t = 0; t < M * K && !bad; ++t) {
        double v = tgo_half_to_double(A[t]);
        if (v != floor(v) || fabs(v) >= 2048.0) bad = 1; else Ai[t] = (int64_t)v;
    }
    for (int64_t t = 0; t < K * N && !bad; ++t) {
        double v = tgo_half_to_double(B[t]);
        if (v != floor(v) || fabs(v) >= 2048.0) bad = 1; else Bi[t] = (int64_t)v;
    }
    if (epilogue == TGO_EPI_BIAS && bias)
        for (int64_t j = 0; j < N && !bad; ++j) {
            double v = tgo_half_to_double(bias[j]);
            if (v != floor(v) || fabs(v) >= 2048.0) bad = 1; else bi[j] = (int64_t)v;
        }
    if (bad) { free(Ai); free(Bi); free(bi); return TGO_ERR_NOT_INTEGER; }
    int oom = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < M; ++i) {
        int64_t *acc = (int64_t *)calloc((size_t)N, sizeof(int64_t));
        if (!acc) {
#pragma omp atomic write
            oom = 1;
            continue;
        }
        for (int64_t k = 0; k < K; ++k) {
            int64_t a = Ai[i * K + k];
            for (int64_t j = 0; j < N; ++j) acc[j] += a * Bi[k * N + j];
        }
        for (int64_t j = 0; j < N; ++j)
            C_bits[i * N + j] = tgo_double_to_half_rne((double)(acc[j] + bi[j]));
        free(acc);
    }
    free(Ai); free(Bi); free(bi);
    return oom ? TGO_ERR_ARG : TGO_OK;
}

/* Threads an OpenMP parallel region would use (1 without OpenMP). */
int tgo_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads for the calling thread's later parallel regions (n >= 1; other
 * values change nothing).  Returns the previous count.  Timing only: the
 * results do not depend on it. */
int tgo_set_num_threads(int n)
{
#ifdef _OPENMP
    const int prev = omp_get_max_threads();
    if (n >= 1) omp_set_num_threads(n);
    return prev;
#else
    (void)n;
    return 1;
#endif
}

/* Array versions of the element codecs (for exhaustive tests). */
void tgo_half_to_double_n(const uint16_t *h, int64_t n, double *out)
{
    for (int64_t t = 0; t < n; ++t) out[t] = tgo_half_to_double(h[t]);
}

void tgo_double_to_half_rne_n(const double *x, int64_t n, uint16_t *out)
{
    for (int64_t t = 0; t < n; ++t) out[t] = tgo_double_to_half_rne(x[t]);
}

void tgo_gelu_n(const double *x, int64_t n, double *out)
{
    for (int64_t t = 0; t < n; ++t) out[t] = tgo_gelu(x[t]);
}

void tgo_gelu_tanh_n(const double *x, int64_t n, double *out)
{
    for (int64_t t = 0; t < n; ++t) out[t] = tgo_gelu_tanh(x[t]);
}


/* ---------------------------------------------------------------- attention */

/* One query row r = (b * H + h) * Sq + i of the attention output, from the
 * decoded K and V (double, [B, H, Sk, D]); scores holds Sk doubles. */
static void attention_row(const uint16_t *Q, const double *Kd, const double *Vd, int64_t H,
                          int64_t Sq, int64_t Sk, int64_t D, int causal, double scale, int64_t r,
                          double *scores, double *q, double *out)
{
    const int64_t bh = r / Sq, i = r % Sq;
    const double *K = Kd + bh * Sk * D, *V = Vd + bh * Sk * D;
    (void)H;
    for (int64_t d = 0; d < D; ++d) q[d] = tgo_half_to_double(Q[r * D + d]);
    const int64_t visible = causal ? (i + 1 < Sk ? i + 1 : Sk) : Sk;
    for (int64_t d = 0; d < D; ++d) out[d] = 0.0;
    if (visible <= 0) return;
    double mx = -INFINITY;
    for (int64_t j = 0; j < visible; ++j) {
        double acc = 0.0;
        for (int64_t d = 0; d < D; ++d) acc += q[d] * K[j * D + d];
        scores[j] = scale * acc;
        if (scores[j] > mx) mx = scores[j];
    }
    double sum = 0.0;
    for (int64_t j = 0; j < visible; ++j) {
        scores[j] = exp(scores[j] - mx);
        sum += scores[j];
    }
    for (int64_t j = 0; j < visible; ++j) {
        const double w = scores[j] / sum;
        for (int64_t d = 0; d < D; ++d) out[d] += w * V[j * D + d];
    }
}

/* O for the query rows `rows` (flat indices (b * H + h) * Sq + i; NULL: all
 * B * H * Sq rows in order), each D doubles, into out. */
int tgo_attention(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int64_t B, int64_t H,
                  int64_t Sq, int64_t Sk, int64_t D, int causal, double scale, const int64_t *rows,
                  int64_t nrows, double *out)
{
    if (!Q || !K || !V || !out || B < 0 || H < 0 || Sq < 0 || Sk < 0 || D <= 0) return TGO_ERR_ARG;
    const int64_t total = B * H * Sq;
    const int64_t n = rows ? nrows : total;
    for (int64_t t = 0; rows && t < n; ++t)
        if (rows[t] < 0 || rows[t] >= total) return TGO_ERR_RANGE;
    if (n == 0) return TGO_OK;
    double *Kd = decode_all(K, B * H * Sk * D);
    double *Vd = decode_all(V, B * H * Sk * D);
    if ((!Kd || !Vd) && B * H * Sk * D > 0) {
        free(Kd);
        free(Vd);
        return TGO_ERR_ARG;
    }
    int err = 0;
#pragma omp parallel
    {
        double *scores = malloc(sizeof(double) * (size_t)(Sk > 0 ? Sk : 1));
        double *q = malloc(sizeof(double) * (size_t)D);
        if (!scores || !q) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t t = 0; t < n; ++t)
                attention_row(Q, Kd, Vd, H, Sq, Sk, D, causal, scale, rows ? rows[t] : t, scores, q,
                              out + t * D);
        }
        free(scores);
        free(q);
    }
    free(Kd);
    free(Vd);
    return err ? TGO_ERR_ARG : TGO_OK;
}
