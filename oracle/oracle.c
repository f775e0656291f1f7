/*
 * oracle.c -- plain fp64 CPU oracle of the block-sparse attention forward.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load or call this file's library.  It shares no code,
 * header, table or helper with the CUDA path.
 *
 * What it computes (the plain definition the block-sparse method reaches
 * exactly, up to rounding order):
 *
 *   "Block Sparse Attention with Log-Linear Complexity", section 3.3
 *   (softmax adapted to sparsity): for every query position the softmax
 *   denominator sums exp(score) over the key positions of the key blocks that
 *   the query's block row connects to, and only over those; unconnected
 *   positions carry weight 0.  The SparseFlashAttention article ("SparseFlash
 *   Attention principle") states the attention itself, softmax(Q K^T / sqrt d) V.
 *
 * For batch b, head h and query token q in block row r = q / bs:
 *   K(q)   = union over j in cols(h, r) of the tokens j*bs .. j*bs+bs-1,
 *            minus the tokens k > q when causal is set (absolute positions);
 *   s_k    = scale * sum_c Q[b,h,q,c] * K[b,h,k,c]   (bf16 inputs widened to fp64);
 *   m      = max_k s_k;  w_k = exp(s_k - m) / sum_k' exp(s_k' - m);
 *   O[q]   = sum_k w_k V[b,h,k,:];   LSE[q] = m + ln sum_k exp(s_k - m).
 *   Empty K(q): O[q] = 0 and LSE[q] = -inf.
 *
 * The column set cols(h, r) is a union: a block listed twice counts once and
 * the order of the list does not matter.
 *
 * Parallelism: OpenMP over the query rows; each row is computed by one thread
 * in a fixed order, so the result does not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double widen_bf16(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Attention of one query row.  keys/score/seen are per-thread scratch of
 * sizes N, N and M.  Returns 0 on success, -1 on an out-of-range column. */
static int one_row(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                   const int32_t *row_ptr, const int32_t *col_idx,
                   int64_t b, int64_t h, int64_t q, int H, int N, int d, int bs,
                   double scale, int causal, double *out, double *lse,
                   int64_t *keys, double *score, unsigned char *seen)
{
    const int M = N / bs;
    const int64_t r = q / bs;
    const int64_t head = b * H + h;
    const uint16_t *qrow = Q + (head * N + q) * (int64_t)d;
    const int32_t beg = row_ptr[h * M + r];
    const int32_t end = row_ptr[h * M + r + 1];
    int64_t nk = 0;
    int rc = 0;

    memset(seen, 0, (size_t)M);
    for (int32_t p = beg; p < end; ++p) {
        int32_t j = col_idx[p];
        if (j < 0 || j >= M) { rc = -1; continue; }
        if (seen[j]) continue;
        seen[j] = 1;
        for (int t = 0; t < bs; ++t) {
            int64_t k = (int64_t)j * bs + t;
            if (causal && k > q) continue;
            keys[nk++] = k;
        }
    }

    for (int c = 0; c < d; ++c) out[c] = 0.0;
    if (nk == 0) {
        *lse = -INFINITY;
        return rc;
    }

    double m = -INFINITY;
    for (int64_t i = 0; i < nk; ++i) {
        const uint16_t *krow = K + (head * N + keys[i]) * (int64_t)d;
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += widen_bf16(qrow[c]) * widen_bf16(krow[c]);
        score[i] = scale * dot;
        if (score[i] > m) m = score[i];
    }

    double l = 0.0;
    for (int64_t i = 0; i < nk; ++i) {
        score[i] = exp(score[i] - m);
        l += score[i];
    }
    for (int64_t i = 0; i < nk; ++i) {
        const uint16_t *vrow = V + (head * N + keys[i]) * (int64_t)d;
        const double w = score[i] / l;
        for (int c = 0; c < d; ++c) out[c] += w * widen_bf16(vrow[c]);
    }
    *lse = m + log(l);
    return rc;
}

/*
 * oracle_forward: O and LSE for the rows listed in `rows` (flat index
 * (b*H + h)*N + q), or for every row when rows == NULL (then nrows is ignored
 * and O is [B,H,N,d], LSE is [B,H,N]).  With a row list, O is [nrows, d] and
 * LSE is [nrows].  Q, K, V are bf16 bit patterns, [B,H,N,d] contiguous.
 * row_ptr is [H*M+1], col_idx holds the columns.  nthreads <= 0 uses the
 * OpenMP default.  Returns the number of threads used, or -1 if a column
 * index was out of range (those columns are skipped), or -2 on bad sizes.
 */
int oracle_forward(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                   const int32_t *row_ptr, const int32_t *col_idx,
                   int B, int H, int N, int d, int bs, double scale, int causal,
                   const int64_t *rows, int64_t nrows,
                   double *O, double *LSE, int nthreads)
{
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0 || bs <= 0 || N % bs != 0) return -2;
    const int M = N / bs;
    const int64_t total = rows ? nrows : (int64_t)B * H * N;
    int used = 1;
    int bad = 0;

#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel reduction(| : bad)
#endif
    {
        int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (size_t)N);
        double *score = (double *)malloc(sizeof(double) * (size_t)N);
        unsigned char *seen = (unsigned char *)malloc((size_t)M);
#ifdef _OPENMP
#pragma omp single
        used = omp_get_num_threads();
#pragma omp for schedule(dynamic, 16)
#endif
        for (int64_t i = 0; i < total; ++i) {
            const int64_t flat = rows ? rows[i] : i;
            const int64_t q = flat % N;
            const int64_t bh = flat / N;
            const int64_t h = bh % H;
            const int64_t b = bh / H;
            if (one_row(Q, K, V, row_ptr, col_idx, b, h, q, H, N, d, bs, scale, causal,
                        O + i * (int64_t)d, LSE + i, keys, score, seen) != 0)
                bad = 1;
        }
        free(keys);
        free(score);
        free(seen);
    }
    return bad ? -1 : used;
}
