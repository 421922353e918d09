/*
 * attn_oracle.c -- plain CPU float64 reference for exact scaled-dot-product
 * attention, forward and backward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or load
 * this file; only the tests, the smoke check and the bench's CPU-baseline leg do.
 * It shares no code, header or constant with the CUDA library.
 *
 * What it computes (one (sequence, head) slice of n rows at a time):
 *
 *   S_ij = scale * sum_c Q_ic K_jc                      full n x n matrix
 *   S_ij = -inf  unless (not causal or j <= i) and key_keep[j] != 0
 *                 and block_mask[h][i / block][j / block] != 0
 *   m_i  = max_j S_ij
 *   if m_i == -inf :  O_i = 0,  lse_i = -inf,  P_i. = 0   (fully masked row)
 *   else           :  P_ij = exp(S_ij - m_i) / sum_k exp(S_ik - m_i)
 *                     O_i  = sum_j P_ij V_j
 *                     lse_i = m_i + log sum_j exp(S_ij - m_i)
 *
 * This is the definition the attention pages start from: the five-line
 * PyTorch `standard_attention` (scale, QK^T, masked_fill to -inf, softmax,
 * matmul with V) in "4.5 注意力优化实战：从PyTorch到CUDA的完整流程", 第一步 §1,
 * with the max-subtracted ("safe") softmax of the codechina FlashAttention
 * article §3.1, and the rule that a row whose every score is -inf yields 0
 * instead of 0/0 = NaN, as the math backend's _safe_softmax does in
 * "Profiling in PyTorch (part 3): Attention is all you profile", math-backend
 * section.  The saved per-row quantity for the backward pass is the natural-log
 * logsumexp lse_i.
 *
 * Backward (softmax Jacobian), with dO the upstream gradient:
 *   dV = P^T dO,   dP = dO V^T,   dS_ij = P_ij (dP_ij - sum_k P_ik dP_ik),
 *   dQ = scale * dS K,   dK = scale * dS^T Q.
 * The backward recomputes its own float64 P; it never uses a GPU result.
 *
 * The tile mask is the block-sparse variant named in the codechina FlashAttention
 * article, §7.1 (Block-Sparse FlashAttention: compute only the
 * important pairs, combining a sparsity pattern with the tiling): a pair of a
 * block-row query tile and a block-column key tile either takes part or is left
 * out as a whole; left-out pairs behave exactly like masked scores.
 *
 * FP8 inputs (the mixed-precision direction of the codechina FlashAttention
 * article, §9: FP8 matrix products with higher-precision accumulation) are
 * 8-bit e4m3 codes with one dequantisation factor per tensor.  The attention
 * they define is the one above applied to the decoded values code -> value *
 * factor; oracle_e4m3_decode turns codes into those float64 values (format
 * below), and the forward then runs unchanged.
 *
 * Layouts (element offsets, double precision arrays):
 *   dense   (cu_seqlens == NULL): Q,K,V,O,dO,dQ,dK,dV are [B,H,N,d]; lse is [B,H,N];
 *           key_keep (optional) is [B,N]; block_mask (optional) is [H, nb, nb] with
 *           nb = ceil(N / block), shared by all batch entries.
 *   packed  (cu_seqlens != NULL): tensors are token-major [total,H,d]; lse is
 *           [total,H]; key_keep (optional) is [total]; cu_seqlens has B+1
 *           entries and sequence b owns tokens cu_seqlens[b] .. cu_seqlens[b+1]-1.
 *           Causal indices are local to each sequence.  No block_mask.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    long base;     /* element offset of (row 0, col 0) in Q/K/V/O */
    long rstride;  /* elements between consecutive rows */
    int n;         /* number of rows (queries == keys) */
    long kbase;    /* offset of row 0 in key_keep */
    long lbase;    /* offset of row 0 in lse */
    long lstride;  /* elements between consecutive lse entries */
} slice_t;

static int make_slice(int b, int h, int B, int H, int N, int d, const int *cu, slice_t *s)
{
    if (b < 0 || b >= B || h < 0 || h >= H) return -1;
    if (cu == NULL) {
        s->base = ((long)(b * (long)H + h) * N) * d;
        s->rstride = d;
        s->n = N;
        s->kbase = (long)b * N;
        s->lbase = (long)(b * (long)H + h) * N;
        s->lstride = 1;
    } else {
        long start = cu[b];
        s->n = cu[b + 1] - cu[b];
        if (s->n < 0) return -1;
        s->base = (start * H + h) * (long)d;
        s->rstride = (long)H * d;
        s->kbase = start;
        s->lbase = start * H + h;
        s->lstride = H;
    }
    return 0;
}

/* Fill S (n x n, row-major) with masked scaled scores for one slice.  tiles is
 * this head's [nb x nb] tile mask (or NULL). */
static void scores(const double *q, const double *k, const slice_t *s, int d, double scale,
                   int causal, const unsigned char *keep, const unsigned char *tiles, int block,
                   double *S, int nthreads)
{
    const int n = s->n;
    const int nb = (tiles != NULL) ? (n + block - 1) / block : 0;
#pragma omp parallel for schedule(dynamic, 8) num_threads(nthreads)
    for (int i = 0; i < n; ++i) {
        const double *qi = q + s->base + (long)i * s->rstride;
        for (int j = 0; j < n; ++j) {
            int allowed = (!causal || j <= i) && (keep == NULL || keep[s->kbase + j] != 0) &&
                          (tiles == NULL || tiles[(long)(i / block) * nb + j / block] != 0);
            if (!allowed) {
                S[(long)i * n + j] = -INFINITY;
                continue;
            }
            const double *kj = k + s->base + (long)j * s->rstride;
            double acc = 0.0;
            for (int c = 0; c < d; ++c) acc += qi[c] * kj[c];
            S[(long)i * n + j] = scale * acc;
        }
    }
}

/* Turn S into P in place (row softmax, fully masked rows -> 0); write lse. */
static void softmax_rows(double *S, const slice_t *s, double *lse, int nthreads)
{
    const int n = s->n;
#pragma omp parallel for schedule(static) num_threads(nthreads)
    for (int i = 0; i < n; ++i) {
        double *row = S + (long)i * n;
        double m = -INFINITY;
        for (int j = 0; j < n; ++j)
            if (row[j] > m) m = row[j];
        if (m == -INFINITY) {
            for (int j = 0; j < n; ++j) row[j] = 0.0;
            if (lse) lse[s->lbase + (long)i * s->lstride] = -INFINITY;
            continue;
        }
        double l = 0.0;
        for (int j = 0; j < n; ++j) {
            row[j] = exp(row[j] - m); /* exp(-inf) == 0 exactly */
            l += row[j];
        }
        for (int j = 0; j < n; ++j) row[j] /= l;
        if (lse) lse[s->lbase + (long)i * s->lstride] = m + log(l);
    }
}

static int run_slices(int B, int H, const int *slices, int n_slices, int **out, int *count)
{
    int total = B * H;
    if (slices == NULL) {
        int *all = (int *)malloc(sizeof(int) * (size_t)(total > 0 ? total : 1));
        if (!all) return -1;
        for (int i = 0; i < total; ++i) all[i] = i;
        *out = all;
        *count = total;
        return 0;
    }
    int *sel = (int *)malloc(sizeof(int) * (size_t)(n_slices > 0 ? n_slices : 1));
    if (!sel) return -1;
    for (int i = 0; i < n_slices; ++i) {
        if (slices[i] < 0 || slices[i] >= total) { free(sel); return -1; }
        sel[i] = slices[i];
    }
    *out = sel;
    *count = n_slices;
    return 0;
}

/*
 * Forward.  `slices` (nullable) lists b*H+h indices to compute; others are left
 * untouched in o/lse.  Returns 0, or -1 on a bad argument / allocation failure.
 */
int oracle_attn_fwd(const double *q, const double *k, const double *v, double *o, double *lse,
                    int B, int H, int N, int d, double scale, int is_causal,
                    const int *cu_seqlens, const unsigned char *key_keep,
                    const unsigned char *block_mask, int block,
                    const int *slices, int n_slices, int nthreads)
{
    if (!q || !k || !v || !o || B <= 0 || H <= 0 || N < 0 || d <= 0) return -1;
    if (block_mask && (cu_seqlens || block <= 0)) return -1;
    if (nthreads <= 0) nthreads = 1;
    int *sel = NULL, cnt = 0;
    if (run_slices(B, H, slices, n_slices, &sel, &cnt)) return -1;
    int rc = 0;
    for (int t = 0; t < cnt && rc == 0; ++t) {
        slice_t s;
        int b = sel[t] / H, h = sel[t] % H;
        if (make_slice(b, h, B, H, N, d, cu_seqlens, &s)) { rc = -1; break; }
        const int n = s.n;
        if (n == 0) continue;
        double *S = (double *)malloc(sizeof(double) * (size_t)n * (size_t)n);
        if (!S) { rc = -1; break; }
        const long nb = block_mask ? (N + block - 1) / block : 0;
        scores(q, k, &s, d, scale, is_causal, key_keep, block_mask ? block_mask + (long)h * nb * nb : NULL,
               block, S, nthreads);
        softmax_rows(S, &s, lse, nthreads);
#pragma omp parallel for schedule(static) num_threads(nthreads)
        for (int i = 0; i < n; ++i) {
            double *oi = o + s.base + (long)i * s.rstride;
            const double *pi = S + (long)i * n;
            for (int c = 0; c < d; ++c) oi[c] = 0.0;
            for (int j = 0; j < n; ++j) {
                double p = pi[j];
                if (p == 0.0) continue;
                const double *vj = v + s.base + (long)j * s.rstride;
                for (int c = 0; c < d; ++c) oi[c] += p * vj[c];
            }
        }
        free(S);
    }
    free(sel);
    return rc;
}

/*
 * Backward.  Recomputes P in float64 and writes dq, dk, dv for the selected
 * slices.  Returns 0, or -1 on a bad argument / allocation failure.
 */
int oracle_attn_bwd(const double *q, const double *k, const double *v, const double *dout,
                    double *dq, double *dk, double *dv,
                    int B, int H, int N, int d, double scale, int is_causal,
                    const int *cu_seqlens, const unsigned char *key_keep,
                    const unsigned char *block_mask, int block,
                    const int *slices, int n_slices, int nthreads)
{
    if (!q || !k || !v || !dout || !dq || !dk || !dv || B <= 0 || H <= 0 || N < 0 || d <= 0)
        return -1;
    if (block_mask && (cu_seqlens || block <= 0)) return -1;
    if (nthreads <= 0) nthreads = 1;
    int *sel = NULL, cnt = 0;
    if (run_slices(B, H, slices, n_slices, &sel, &cnt)) return -1;
    int rc = 0;
    for (int t = 0; t < cnt && rc == 0; ++t) {
        slice_t s;
        int b = sel[t] / H, h = sel[t] % H;
        if (make_slice(b, h, B, H, N, d, cu_seqlens, &s)) { rc = -1; break; }
        const int n = s.n;
        if (n == 0) continue;
        double *P = (double *)malloc(sizeof(double) * (size_t)n * (size_t)n);
        double *dS = (double *)malloc(sizeof(double) * (size_t)n * (size_t)n);
        if (!P || !dS) { free(P); free(dS); rc = -1; break; }
        const long nb = block_mask ? (N + block - 1) / block : 0;
        scores(q, k, &s, d, scale, is_causal, key_keep, block_mask ? block_mask + (long)h * nb * nb : NULL,
               block, P, nthreads);
        softmax_rows(P, &s, NULL, nthreads);

        /* dP_ij = dO_i . V_j ; dS_ij = P_ij (dP_ij - sum_k P_ik dP_ik) */
#pragma omp parallel for schedule(dynamic, 8) num_threads(nthreads)
        for (int i = 0; i < n; ++i) {
            const double *doi = dout + s.base + (long)i * s.rstride;
            const double *pi = P + (long)i * n;
            double *dsi = dS + (long)i * n;
            double rowdot = 0.0;
            for (int j = 0; j < n; ++j) {
                if (pi[j] == 0.0) { dsi[j] = 0.0; continue; }
                const double *vj = v + s.base + (long)j * s.rstride;
                double acc = 0.0;
                for (int c = 0; c < d; ++c) acc += doi[c] * vj[c];
                dsi[j] = acc;            /* holds dP_ij for now */
                rowdot += pi[j] * acc;
            }
            for (int j = 0; j < n; ++j) dsi[j] = pi[j] * (dsi[j] - rowdot);
        }

        /* dQ_i = scale * sum_j dS_ij K_j */
#pragma omp parallel for schedule(static) num_threads(nthreads)
        for (int i = 0; i < n; ++i) {
            double *dqi = dq + s.base + (long)i * s.rstride;
            const double *dsi = dS + (long)i * n;
            for (int c = 0; c < d; ++c) dqi[c] = 0.0;
            for (int j = 0; j < n; ++j) {
                double w = dsi[j];
                if (w == 0.0) continue;
                const double *kj = k + s.base + (long)j * s.rstride;
                for (int c = 0; c < d; ++c) dqi[c] += w * kj[c];
            }
            for (int c = 0; c < d; ++c) dqi[c] *= scale;
        }

        /* dK_j = scale * sum_i dS_ij Q_i ;  dV_j = sum_i P_ij dO_i */
#pragma omp parallel for schedule(static) num_threads(nthreads)
        for (int j = 0; j < n; ++j) {
            double *dkj = dk + s.base + (long)j * s.rstride;
            double *dvj = dv + s.base + (long)j * s.rstride;
            for (int c = 0; c < d; ++c) { dkj[c] = 0.0; dvj[c] = 0.0; }
            for (int i = 0; i < n; ++i) {
                double w = dS[(long)i * n + j];
                double p = P[(long)i * n + j];
                if (w == 0.0 && p == 0.0) continue;
                const double *qi = q + s.base + (long)i * s.rstride;
                const double *doi = dout + s.base + (long)i * s.rstride;
                for (int c = 0; c < d; ++c) {
                    dkj[c] += w * qi[c];
                    dvj[c] += p * doi[c];
                }
            }
            for (int c = 0; c < d; ++c) dkj[c] *= scale;
        }
        free(P);
        free(dS);
    }
    free(sel);
    return rc;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * e4m3 (the OCP 8-bit floating-point format's E4M3 encoding): bit 7 sign, bits 3-6
 * a biased exponent e (bias 7), bits 0-2 a mantissa m.
 *   e == 0              : subnormal, (m / 8) * 2^(1 - 7)
 *   e == 15 and m == 7  : NaN (the encoding has no infinities)
 *   otherwise           : (1 + m / 8) * 2^(e - 7)        (largest: 448)
 * out[i] = sign * value(codes[i]) * factor.
 */
void oracle_e4m3_decode(const unsigned char *codes, long n, double factor, double *out)
{
    for (long i = 0; i < n; ++i) {
        const int c = codes[i];
        const int e = (c >> 3) & 15, m = c & 7;
        double v;
        if (e == 15 && m == 7)
            v = NAN;
        else if (e == 0)
            v = ldexp((double)m / 8.0, 1 - 7);
        else
            v = ldexp(1.0 + (double)m / 8.0, e - 7);
        out[i] = ((c & 128) ? -v : v) * factor;
    }
}
