/*
 * halo_oracle.c -- plain, slow, double-precision CPU oracle for HaloNet's
 * blocked local self-attention with haloing.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke() check
 * and the benchmark's CPU-baseline leg may load this library.  It shares no
 * code, header, table or helper with the CUDA path and the CUDA path never
 * calls it.
 *
 * What it computes (HaloNet, "Scaling Local Self-Attention for Parameter
 * Efficient Visual Backbones"):
 *   - Section 2.2 and Figure 1: the H x W map is cut into non-overlapping
 *     b x b query blocks; each block shares one (b+2h) x (b+2h) neighbourhood
 *     made of the block plus an h-pixel halo, padded at the image border.
 *   - Section 2.1: each logit is a content-content term q.k plus a
 *     content-geometry term q.r with r indexed by relative position; the
 *     relative embedding is shared by all heads (footnote 1).
 *   - Appendix A: the relative embedding is factorised along height and
 *     width.  Following the blog page's RelPosEmb module, two full-width
 *     tables rel_h, rel_w of shape [2w-1, d] are summed.
 *   - Blog page, HaloAttention.forward: q is scaled by d^-1/2 before both the
 *     content and the relative logits, keys outside the image are removed from
 *     the softmax, softmax over the window, then the weighted sum of v.
 *   - Section 2.2 and Figure 2: the stride-2 variant subsamples the queries
 *     like a strided convolution and keeps the stride-1 neighbourhood.
 *
 * Readings where the pages are silent or garbled:
 *   relative index  = (key window coordinate) - (query in-block coordinate)
 *                     + w - 1, rows -> rel_h, columns -> rel_w (the blog's
 *                     rel_to_abs recipe, pinned by a test that restates it);
 *   out-of-image keys get weight exactly 0 (the blog's printed mask polarity
 *                     is inverted; the paper pads the border);
 *   stride 2        = queries at even in-block offsets 0,2,..,b-2; the
 *                     relative index uses the pixel's in-block offset.
 *                     The tests pin stride 2 to stride 1 sampled at even
 *                     pixels, but no page fixes the phase or the index
 *                     convention: parity unpinned against the pages for
 *                     this choice.  The absolute table offset is pinned only
 *                     to the blog's rel_to_abs recipe.
 *
 * For each output pixel and head the oracle evaluates the defining formula
 * directly: every window key's logit, the maximum over in-image keys, the
 * exponentials, their sum and the weighted sum of v, all in double precision,
 * from the stored input values (float32, or bf16 widened exactly).
 *
 * SASA-masked variant (section 2.2, the paragraph after Figure 1): the same
 * blocked neighbourhood with h = floor(k/2) and an attention mask that keeps,
 * for each query pixel, only the k x k keys centred on it, so that the op
 * emulates pixel-centred local attention.  Here `kmask` = k (odd, 1 <= k <=
 * 2h + 1); a key is kept when |Y - y| <= k/2 and |X - x| <= k/2 (and it is
 * inside the image).  kmask = 0 means no mask (HaloNet's own, unmasked form).
 *
 * Fused projections (the blog page's HaloAttention: to_q and to_kv are
 * bias-free linear maps of the input feature map x, k and v being the two
 * halves of to_kv's output): q = x Wq^T, [k | v] = x Wkv^T per pixel, exactly
 * (double precision), each rounded to the inputs' dtype as an unfused
 * pipeline would store them, then the operation above.  Pixels outside the
 * image project to zero (no bias), the same as zero-filled keys.
 *
 * Backward (the gradients of a scalar loss L = sum(out * dout) with respect to
 * q, k, v, rel_h and rel_w; the pages train this layer, section 2.2 and
 * Figure 3, but print no gradient): by the chain rule through the defining
 * formula, per output pixel and head with p_j the softmax weights,
 *     dp_j = dout . v_j,   D = sum_j p_j dp_j,   dz_j = p_j (dp_j - D),
 *     dq  = s sum_j dz_j (k_j + rel_h[a_j] + rel_w[b_j]),
 *     dk_j += s dz_j q,  dv_j += p_j dout,
 *     drel_h[a_j] += s dz_j q,  drel_w[b_j] += s dz_j q,
 * where a_j, b_j are the row and column table indices of key j.  The sums
 * run over the kept keys only; dk, dv, drel_h, drel_w collect every query
 * whose window holds the key or uses the table row (the tables are shared by
 * all heads, section 2.1, footnote 1).  Pinned by central finite differences
 * of the forward oracle and by closed-form identities of these sums.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC halo_oracle.c -o liboracle.so -lm
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* dtype codes of the stored inputs */
#define ORACLE_F32 0
#define ORACLE_BF16 1

#define ORACLE_F64 2  /* internal: projected values held in double */

/* Read element i of a float32 or bf16 array as a double (exact widening). */
static double read_elem(const void *base, size_t i, int dtype)
{
    if (dtype == ORACLE_F32) {
        return (double)((const float *)base)[i];
    }
    if (dtype == ORACLE_F64) {
        return ((const double *)base)[i];
    }
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

typedef struct {
    const void *q, *k, *v, *rel_h, *rel_w;
    int N, H, W, heads, d, b, h, S, dtype;
    int kmask;  /* 0: no mask; k: keep the k x k keys centred on the query */
} oracle_args;

/* Whether window key (kr, kc) of query pixel (y, x) takes part in the softmax:
 * inside the image, and, with the SASA mask, inside the k x k square centred
 * on the query. */
static int key_kept(const oracle_args *a, int y, int x, int Y, int X)
{
    if (Y < 0 || Y >= a->H || X < 0 || X >= a->W) return 0;
    if (a->kmask > 0) {
        const int r = a->kmask / 2;
        if (Y - y > r || y - Y > r || X - x > r || x - X > r) return 0;
    }
    return 1;
}

/*
 * One output pixel (n, oy, ox), one head: writes d doubles to out_vec.
 * Scratch z must hold w*w doubles, valid w*w chars.
 */
static void one_pixel_head(const oracle_args *a, int n, int oy, int ox, int head,
                           double *z, char *valid, double *out_vec)
{
    const int w = a->b + 2 * a->h;
    const int C = a->heads * a->d;
    const double s = 1.0 / sqrt((double)a->d);

    /* the query pixel and its block */
    const int y = a->S * oy, x = a->S * ox;
    const int by = y / a->b, bx = x / a->b;
    const int qy = y - by * a->b, qx = x - bx * a->b;
    /* the window's top-left corner in image coordinates */
    const int y0 = by * a->b - a->h, x0 = bx * a->b - a->h;

    const size_t qoff = (((size_t)n * a->H + y) * a->W + x) * C + (size_t)head * a->d;

    /* logits over the whole window; out-of-image keys are marked invalid */
    double m = -INFINITY;
    for (int kr = 0; kr < w; ++kr) {
        for (int kc = 0; kc < w; ++kc) {
            const int Y = y0 + kr, X = x0 + kc;
            const int j = kr * w + kc;
            if (!key_kept(a, y, x, Y, X)) {
                valid[j] = 0;
                z[j] = 0.0;
                continue;
            }
            valid[j] = 1;
            const size_t koff = (((size_t)n * a->H + Y) * a->W + X) * C + (size_t)head * a->d;
            const size_t rh = (size_t)(kr - qy + w - 1) * a->d;
            const size_t rw = (size_t)(kc - qx + w - 1) * a->d;
            double acc = 0.0;
            for (int e = 0; e < a->d; ++e) {
                const double qe = read_elem(a->q, qoff + e, a->dtype);
                const double ke = read_elem(a->k, koff + e, a->dtype);
                const double he = read_elem(a->rel_h, rh + e, a->dtype);
                const double we = read_elem(a->rel_w, rw + e, a->dtype);
                acc += qe * (ke + he + we);
            }
            z[j] = s * acc;
            if (z[j] > m) m = z[j];
        }
    }

    /* softmax over the in-image keys, then the weighted sum of v */
    double Z = 0.0;
    for (int j = 0; j < w * w; ++j) {
        if (valid[j]) {
            z[j] = exp(z[j] - m);
            Z += z[j];
        }
    }
    for (int e = 0; e < a->d; ++e) out_vec[e] = 0.0;
    for (int kr = 0; kr < w; ++kr) {
        for (int kc = 0; kc < w; ++kc) {
            const int j = kr * w + kc;
            if (!valid[j]) continue;
            const int Y = y0 + kr, X = x0 + kc;
            const size_t voff = (((size_t)n * a->H + Y) * a->W + X) * C + (size_t)head * a->d;
            for (int e = 0; e < a->d; ++e) {
                out_vec[e] += z[j] * read_elem(a->v, voff + e, a->dtype);
            }
        }
    }
    for (int e = 0; e < a->d; ++e) out_vec[e] /= Z;
}

static int check_args(const oracle_args *a)
{
    if (!a->q || !a->k || !a->v || !a->rel_h || !a->rel_w) return -1;
    if (a->N <= 0 || a->H <= 0 || a->W <= 0 || a->heads <= 0 || a->d <= 0 || a->b <= 0 || a->h < 0)
        return -2;
    if (a->H % a->b || a->W % a->b) return -3;
    if (a->S != 1 && a->S != 2) return -4;
    if (a->b % a->S) return -3;
    if (a->dtype != ORACLE_F32 && a->dtype != ORACLE_BF16 && a->dtype != ORACLE_F64) return -9;
    if (a->b + 2 * a->h > 4096) return -2;
    if (a->kmask < 0 || (a->kmask > 0 && (a->kmask % 2 == 0 || a->kmask / 2 > a->h))) return -2;
    return 0;
}

/*
 * Full output: out is [N, H/S, W/S, heads*d] doubles.  threads <= 0 uses the
 * OpenMP default.  Returns 0, or a negative code for invalid arguments.
 */
static int full_output(const oracle_args *ap, double *out, int threads)
{
    const oracle_args a = *ap;
    int rc = check_args(&a);
    if (rc) return rc;
    if (!out) return -1;
    const int N = a.N, heads = a.heads, dim_head = a.d, stride = a.S, block = a.b, halo = a.h;
    const int OH = a.H / stride, OW = a.W / stride, C = heads * dim_head;
    const int w = block + 2 * halo;
    const long total = (long)N * heads * OH * OW;
#ifdef _OPENMP
    const int nt_call = threads > 0 ? threads : omp_get_max_threads();
#else
    (void)threads;
    const int nt_call = 1;
#endif
#pragma omp parallel num_threads(nt_call)
    {
        double *z = (double *)__builtin_alloca(sizeof(double) * (size_t)w * w);
        char *valid = (char *)__builtin_alloca((size_t)w * w);
        double *vec = (double *)__builtin_alloca(sizeof(double) * (size_t)dim_head);
#pragma omp for schedule(static)
        for (long u = 0; u < total; ++u) {
            /* unit u = (n, head, oy, ox) */
            long t = u;
            const int ox = (int)(t % OW); t /= OW;
            const int oy = (int)(t % OH); t /= OH;
            const int head = (int)(t % heads); t /= heads;
            const int n = (int)t;
            one_pixel_head(&a, n, oy, ox, head, z, valid, vec);
            double *dst = out + (((size_t)n * OH + oy) * OW + ox) * C + (size_t)head * dim_head;
            for (int e = 0; e < dim_head; ++e) dst[e] = vec[e];
        }
    }
    return 0;
}

int halo_oracle_f64(const void *q, const void *k, const void *v,
                    const void *rel_h, const void *rel_w, double *out,
                    int N, int H, int W, int heads, int dim_head,
                    int block, int halo, int stride, int dtype, int threads)
{
    oracle_args a = {q, k, v, rel_h, rel_w, N, H, W, heads, dim_head, block, halo, stride, dtype, 0};
    return full_output(&a, out, threads);
}

/*
 * SASA-masked variant: as halo_oracle_f64, each query keeping only the
 * kmask x kmask keys centred on it (kmask odd, kmask/2 <= halo).
 */
int halo_oracle_masked_f64(const void *q, const void *k, const void *v,
                           const void *rel_h, const void *rel_w, double *out,
                           int N, int H, int W, int heads, int dim_head,
                           int block, int halo, int stride, int kmask, int dtype, int threads)
{
    oracle_args a = {q, k, v, rel_h, rel_w, N, H, W, heads, dim_head, block, halo, stride, dtype, kmask};
    if (kmask <= 0) return -2;
    return full_output(&a, out, threads);
}

/*
 * Backward of one output pixel and head: recomputes the softmax weights of
 * the kept keys (as one_pixel_head does), then adds this query's terms to
 * dq (written), dk, dv (accumulated, [N, H, W, C] doubles) and to the
 * caller's table accumulators drh, drw ([2w-1, d] doubles each).
 * Scratch: z, p hold w*w doubles, valid w*w chars, dov d doubles.
 */
static void one_pixel_head_bwd(const oracle_args *a, const void *dout, int n, int oy, int ox, int head,
                               double *z, char *valid, double *dov,
                               double *dq, double *dk, double *dv, double *drh, double *drw)
{
    const int w = a->b + 2 * a->h;
    const int C = a->heads * a->d;
    const int OH = a->H / a->S, OW = a->W / a->S;
    const double s = 1.0 / sqrt((double)a->d);
    const int y = a->S * oy, x = a->S * ox;
    const int by = y / a->b, bx = x / a->b;
    const int qy = y - by * a->b, qx = x - bx * a->b;
    const int y0 = by * a->b - a->h, x0 = bx * a->b - a->h;
    const size_t qoff = (((size_t)n * a->H + y) * a->W + x) * C + (size_t)head * a->d;
    const size_t ooff = (((size_t)n * OH + oy) * OW + ox) * C + (size_t)head * a->d;

    /* forward: logits of the kept keys, maximum, softmax weights p_j */
    double m = -INFINITY;
    for (int kr = 0; kr < w; ++kr) {
        for (int kc = 0; kc < w; ++kc) {
            const int Y = y0 + kr, X = x0 + kc, j = kr * w + kc;
            valid[j] = (char)key_kept(a, y, x, Y, X);
            z[j] = 0.0;
            if (!valid[j]) continue;
            const size_t koff = (((size_t)n * a->H + Y) * a->W + X) * C + (size_t)head * a->d;
            const size_t rh = (size_t)(kr - qy + w - 1) * a->d, rw = (size_t)(kc - qx + w - 1) * a->d;
            double acc = 0.0;
            for (int e = 0; e < a->d; ++e)
                acc += read_elem(a->q, qoff + e, a->dtype) *
                       (read_elem(a->k, koff + e, a->dtype) + read_elem(a->rel_h, rh + e, a->dtype) +
                        read_elem(a->rel_w, rw + e, a->dtype));
            z[j] = s * acc;
            if (z[j] > m) m = z[j];
        }
    }
    double Z = 0.0;
    for (int j = 0; j < w * w; ++j)
        if (valid[j]) { z[j] = exp(z[j] - m); Z += z[j]; }
    for (int j = 0; j < w * w; ++j) z[j] = valid[j] ? z[j] / Z : 0.0;  /* z now holds p_j */

    /* dp_j = dout . v_j and D = sum_j p_j dp_j */
    for (int e = 0; e < a->d; ++e) dov[e] = read_elem(dout, ooff + e, a->dtype);
    double D = 0.0;
    for (int kr = 0; kr < w; ++kr) {
        for (int kc = 0; kc < w; ++kc) {
            const int j = kr * w + kc;
            if (!valid[j]) continue;
            const size_t voff = (((size_t)n * a->H + (y0 + kr)) * a->W + (x0 + kc)) * C + (size_t)head * a->d;
            double dp = 0.0;
            for (int e = 0; e < a->d; ++e) dp += dov[e] * read_elem(a->v, voff + e, a->dtype);
            D += z[j] * dp;
        }
    }
    /* second sweep: dz_j and every gradient term */
    double *dqv = dq + qoff;
    for (int e = 0; e < a->d; ++e) dqv[e] = 0.0;
    for (int kr = 0; kr < w; ++kr) {
        for (int kc = 0; kc < w; ++kc) {
            const int j = kr * w + kc;
            if (!valid[j]) continue;
            const size_t koff = (((size_t)n * a->H + (y0 + kr)) * a->W + (x0 + kc)) * C + (size_t)head * a->d;
            const size_t rh = (size_t)(kr - qy + w - 1) * a->d, rw = (size_t)(kc - qx + w - 1) * a->d;
            double dp = 0.0;
            for (int e = 0; e < a->d; ++e) dp += dov[e] * read_elem(a->v, koff + e, a->dtype);
            const double dz = z[j] * (dp - D);
            for (int e = 0; e < a->d; ++e) {
                const double qe = read_elem(a->q, qoff + e, a->dtype);
                dqv[e] += s * dz * (read_elem(a->k, koff + e, a->dtype) + read_elem(a->rel_h, rh + e, a->dtype) +
                                    read_elem(a->rel_w, rw + e, a->dtype));
                dk[koff + e] += s * dz * qe;
                dv[koff + e] += z[j] * dov[e];
                drh[rh + e] += s * dz * qe;
                drw[rw + e] += s * dz * qe;
            }
        }
    }
}

/*
 * Gradients of L = sum(out * dout): dout is [N, H/S, W/S, C] in the inputs'
 * dtype; dq, dk, dv are [N, H, W, C] doubles (dq is zero at the pixels that
 * are not queries at stride 2), drel_h, drel_w [2w-1, d] doubles.  kmask as
 * in halo_oracle_masked_f64 (0: no mask).  Parallel over (image, head): those
 * write disjoint parts of dq, dk, dv; the tables' sums are kept per thread
 * and added in thread order at the end.
 */
int halo_oracle_bwd_f64(const void *q, const void *k, const void *v,
                        const void *rel_h, const void *rel_w, const void *dout,
                        double *dq, double *dk, double *dv, double *drel_h, double *drel_w,
                        int N, int H, int W, int heads, int dim_head,
                        int block, int halo, int stride, int kmask, int dtype, int threads)
{
    oracle_args a = {q, k, v, rel_h, rel_w, N, H, W, heads, dim_head, block, halo, stride, dtype, kmask};
    int rc = check_args(&a);
    if (rc) return rc;
    if (!dout || !dq || !dk || !dv || !drel_h || !drel_w) return -1;
    const int OH = H / stride, OW = W / stride, C = heads * dim_head;
    const int w = block + 2 * halo, R = 2 * w - 1;
    const size_t nin = (size_t)N * H * W * C, ntab = (size_t)R * dim_head;
    memset(dq, 0, nin * sizeof(double));
    memset(dk, 0, nin * sizeof(double));
    memset(dv, 0, nin * sizeof(double));
#ifdef _OPENMP
    const int nt_call = threads > 0 ? threads : omp_get_max_threads();
    const int nt = nt_call;
#else
    (void)threads;
    const int nt_call = 1;
    const int nt = 1;
#endif
    double *part = (double *)calloc((size_t)nt * 2 * ntab, sizeof(double));
    if (!part) return -2;
    const long units = (long)N * heads;
#pragma omp parallel num_threads(nt_call)
    {
#ifdef _OPENMP
        const int tid = omp_get_thread_num();
#else
        const int tid = 0;
#endif
        double *z = (double *)malloc(sizeof(double) * (size_t)w * w);
        char *valid = (char *)malloc((size_t)w * w);
        double *dov = (double *)malloc(sizeof(double) * (size_t)dim_head);
        double *drh = part + (size_t)tid * 2 * ntab, *drw = drh + ntab;
#pragma omp for schedule(static)
        for (long u = 0; u < units; ++u) {
            const int n = (int)(u / heads), head = (int)(u % heads);
            for (int oy = 0; oy < OH; ++oy)
                for (int ox = 0; ox < OW; ++ox)
                    one_pixel_head_bwd(&a, dout, n, oy, ox, head, z, valid, dov, dq, dk, dv, drh, drw);
        }
        free(z);
        free(valid);
        free(dov);
    }
    for (size_t i = 0; i < ntab; ++i) {
        double sh = 0.0, sw = 0.0;
        for (int t = 0; t < nt; ++t) {
            sh += part[(size_t)t * 2 * ntab + i];
            sw += part[(size_t)t * 2 * ntab + ntab + i];
        }
        drel_h[i] = sh;
        drel_w[i] = sw;
    }
    free(part);
    return 0;
}

/* A double rounded to the stored dtype (float32, or bf16 by round to nearest
 * even of the float32 value), returned as a double. */
static double round_to_dtype(double x, int dtype)
{
    float f = (float)x;
    if (dtype == ORACLE_F32) return (double)f;
    uint32_t bits;
    memcpy(&bits, &f, sizeof bits);
    bits = (bits + 0x7FFFu + ((bits >> 16) & 1u)) & 0xFFFF0000u;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/*
 * Fused projections: x [N, H, W, c_in] and the weights wq [heads*d, c_in],
 * wkv [2*heads*d, c_in] (the linear layers' [out, in] layout) in `dtype`;
 * out [N, H/S, W/S, heads*d] doubles.  q, k, v are formed exactly, rounded
 * to `dtype`, then the operation.
 */
int halo_oracle_fused_f64(const void *x, const void *wq, const void *wkv,
                          const void *rel_h, const void *rel_w, double *out,
                          int N, int H, int W, int c_in, int heads, int dim_head,
                          int block, int halo, int stride, int dtype, int threads)
{
    if (!x || !wq || !wkv || !rel_h || !rel_w || !out) return -1;
    if (c_in <= 0) return -2;
    if (dtype != ORACLE_F32 && dtype != ORACLE_BF16) return -9;
    const int C = heads * dim_head;
    const size_t npix = (size_t)N * H * W;
    double *q = (double *)malloc(npix * C * sizeof(double));
    double *k = (double *)malloc(npix * C * sizeof(double));
    double *v = (double *)malloc(npix * C * sizeof(double));
    double *rh = (double *)malloc((size_t)(2 * (block + 2 * halo) - 1) * dim_head * sizeof(double));
    double *rw = (double *)malloc((size_t)(2 * (block + 2 * halo) - 1) * dim_head * sizeof(double));
    if (!q || !k || !v || !rh || !rw) {
        free(q); free(k); free(v); free(rh); free(rw);
        return -2;
    }
#ifdef _OPENMP
    const int nt_call = threads > 0 ? threads : omp_get_max_threads();
#endif
#pragma omp parallel for num_threads(nt_call) schedule(static)
    for (long pix = 0; pix < (long)npix; ++pix) {
        for (int o = 0; o < C; ++o) {
            double aq = 0.0, ak = 0.0, av = 0.0;
            for (int ci = 0; ci < c_in; ++ci) {
                const double xe = read_elem(x, (size_t)pix * c_in + ci, dtype);
                aq += xe * read_elem(wq, (size_t)o * c_in + ci, dtype);
                ak += xe * read_elem(wkv, (size_t)o * c_in + ci, dtype);
                av += xe * read_elem(wkv, (size_t)(C + o) * c_in + ci, dtype);
            }
            q[(size_t)pix * C + o] = round_to_dtype(aq, dtype);
            k[(size_t)pix * C + o] = round_to_dtype(ak, dtype);
            v[(size_t)pix * C + o] = round_to_dtype(av, dtype);
        }
    }
    const size_t ntab = (size_t)(2 * (block + 2 * halo) - 1) * dim_head;
    for (size_t i = 0; i < ntab; ++i) {
        rh[i] = read_elem(rel_h, i, dtype);
        rw[i] = read_elem(rel_w, i, dtype);
    }
    oracle_args a = {q, k, v, rh, rw, N, H, W, heads, dim_head, block, halo, stride, ORACLE_F64, 0};
    const int rc = full_output(&a, out, threads);
    free(q); free(k); free(v); free(rh); free(rw);
    return rc;
}

/*
 * Sampled output pixels: samples holds nsamples (n, oy, ox) triples; out is
 * [nsamples, heads*d] doubles.  Used for parity at full sizes, where the whole
 * output would take the oracle too long.
 */
int halo_oracle_samples_f64(const void *q, const void *k, const void *v,
                            const void *rel_h, const void *rel_w,
                            const int *samples, int nsamples, double *out,
                            int N, int H, int W, int heads, int dim_head,
                            int block, int halo, int stride, int dtype, int threads)
{
    oracle_args a = {q, k, v, rel_h, rel_w, N, H, W, heads, dim_head, block, halo, stride, dtype, 0};
    int rc = check_args(&a);
    if (rc) return rc;
    if (!samples || !out) return -1;
    const int OH = H / stride, OW = W / stride, C = heads * dim_head;
    const int w = block + 2 * halo;
    for (int i = 0; i < nsamples; ++i) {
        const int n = samples[3 * i], oy = samples[3 * i + 1], ox = samples[3 * i + 2];
        if (n < 0 || n >= N || oy < 0 || oy >= OH || ox < 0 || ox >= OW) return -2;
    }
    const long total = (long)nsamples * heads;
#ifdef _OPENMP
    const int nt_call = threads > 0 ? threads : omp_get_max_threads();
#else
    (void)threads;
    const int nt_call = 1;
#endif
#pragma omp parallel num_threads(nt_call)
    {
        double *z = (double *)__builtin_alloca(sizeof(double) * (size_t)w * w);
        char *valid = (char *)__builtin_alloca((size_t)w * w);
        double *vec = (double *)__builtin_alloca(sizeof(double) * (size_t)dim_head);
#pragma omp for schedule(static)
        for (long u = 0; u < total; ++u) {
            const int i = (int)(u / heads), head = (int)(u % heads);
            one_pixel_head(&a, samples[3 * i], samples[3 * i + 1], samples[3 * i + 2], head, z, valid, vec);
            double *dst = out + (size_t)i * C + (size_t)head * dim_head;
            for (int e = 0; e < dim_head; ++e) dst[e] = vec[e];
        }
    }
    return 0;
}

/* Number of OpenMP threads a parallel region would use (for reporting). */
int halo_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
