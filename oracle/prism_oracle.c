/*
 * prism_oracle.c -- plain, slow, fp64 CPU oracle of Prism's dynamic sparse
 * video self-attention hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, import or
 * call this file: only the tests, the package's smoke check and the benchmark's
 * CPU-baseline / reference arm use it.  It shares no code, header, table or
 * helper with the CUDA library; both sides only read the same seeded inputs.
 *
 * Source of every definition: the paper guide "Prism: Dynamic Sparse Attention
 * cho Huan luyen Mo hinh Tao Video-Am thanh Dong thoi Do phan giai Goc 2K"
 * (xyznot.com, paper 2610.05416), cited below as [Prism guide, <section>]:
 *   - "Cac y tuong cot loi" (core ideas): 8x8x8 macro-zones, 16 candidate
 *     shapes of volume 64/128/256, hybrid Top-k / Top-p.
 *   - Method section 1 (variation indicator): sigma^2_{v,d}, r_{v,d}, g_d.
 *   - Method section 2 (block volume and shape): tau_128, tau_256, l*_d,
 *     nearest candidate in log2 space.
 *   - Method section 3 (hybrid Top-k / Top-p attention): pooled key blocks,
 *     block probabilities P_i, S_i = Top-k(P_i,k) U Top-p(P_i,p), online
 *     softmax attention restricted to S_i.
 * Where the guide leaves a step open, the reading taken is stated at the
 * function that implements it.
 *
 * Arithmetic: every value is fp64.  bf16 inputs are widened exactly.  Loops
 * follow the definitions in the order the guide writes them; there is no
 * blocking, fusion or reordering beyond that.  OpenMP only splits independent
 * outer iterations (zones, rows, requested outputs).
 *
 * Parity status per function (see the tests that pin them):
 *   orc_shape_table, orc_lstar, orc_pick_shape     pinned (enumeration, closed
 *                                                  form vs numeric minimum,
 *                                                  brute-force argmin)
 *   orc_zone_stats                                 pinned (separable fields with
 *                                                  closed-form variances)
 *   orc_zone_decide (rho, B)                       pinned on special cases only
 *                                                  (the density formula is a
 *                                                  reading, not printed)
 *   orc_blocks, orc_perm, orc_pool                 pinned (tiling invariants,
 *                                                  linear-field closed form)
 *   orc_select_row / orc_select                    pinned (hand-worked rows,
 *                                                  Top-k / Top-p invariants)
 *   orc_attn_*                                     pinned (dense reduction vs
 *                                                  library SDPA, masked dense,
 *                                                  finite differences)
 *   orc_attn_fwd_taylor_rows                       pinned (exact when every block
 *                                                  is constant; uniform scores give
 *                                                  the global mean of V; error of
 *                                                  second order in a zero-mean key
 *                                                  perturbation)
 *   orc_hilbert_index, orc_hilbert_perm            pinned (a bijection of the cube
 *                                                  whose consecutive points are unit
 *                                                  steps and whose aligned sub-cubes
 *                                                  are index intervals; the grid's
 *                                                  order is by increasing index)
 *   orc_pool_blocks                                pinned (block constants, index
 *                                                  means, equal to orc_pool on boxes)
 *   orc_audio_norms                                pinned (closed forms: constant
 *                                                  rows, one-hot rows, integer
 *                                                  norms; an exact rational sum
 *                                                  on random rows)
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ZONE 8 /* Z_T = Z_H = Z_W = 8 [Prism guide, core ideas, bullet 1] */
#define ZVOL (ZONE * ZONE * ZONE)

static double widen_bf16(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------ */
/* Candidate shapes [Prism guide, core ideas bullet 3; Method section 2].    */
/* Edges are powers of two in {2,4,8}; a shape of volume B = 2^S has edge    */
/* exponents (eT,eH,eW) in {1,2,3}^3 with eT+eH+eW = S.  The table lists the */
/* volumes 64, 128, 256 in that order, each in lexicographic (eT,eH,eW)      */
/* order; that fixed order is also the tie-break (lowest index wins).        */
/* ------------------------------------------------------------------------ */
int orc_shape_table(int *exps /* [16][3] */)
{
    int n = 0;
    for (int S = 6; S <= 8; ++S)
        for (int eT = 1; eT <= 3; ++eT)
            for (int eH = 1; eH <= 3; ++eH)
                for (int eW = 1; eW <= 3; ++eW)
                    if (eT + eH + eW == S) {
                        if (exps) {
                            exps[3 * n + 0] = eT;
                            exps[3 * n + 1] = eH;
                            exps[3 * n + 2] = eW;
                        }
                        ++n;
                    }
    return n;
}

/* Continuous optimum in log2 space [Prism guide, Method section 2, l* eq.]:
 *   l*_d = -1/2 log2 g_d + 1/3 (S + 1/2 log2 g_T + 1/2 log2 g_H + 1/2 log2 g_W). */
void orc_lstar(const double *g, int S, double *l)
{
    double sum_half_log = 0.5 * log2(g[0]) + 0.5 * log2(g[1]) + 0.5 * log2(g[2]);
    for (int d = 0; d < 3; ++d)
        l[d] = -0.5 * log2(g[d]) + (1.0 / 3.0) * ((double)S + sum_half_log);
}

/* Nearest candidate of volume 2^S to l* in Euclidean log2 distance
 * [Prism guide, Method section 2, last sentence].  Returns the table index;
 * *gap = (second-best squared distance) - (best squared distance). */
int orc_pick_shape(const double *l, int S, double *gap)
{
    int exps[16 * 3];
    int n = orc_shape_table(exps);
    int best = -1;
    double bd = INFINITY, second = INFINITY;
    for (int c = 0; c < n; ++c) {
        if (exps[3 * c] + exps[3 * c + 1] + exps[3 * c + 2] != S)
            continue;
        double dist = 0.0;
        for (int d = 0; d < 3; ++d) {
            double diff = l[d] - (double)exps[3 * c + d];
            dist += diff * diff;
        }
        if (dist < bd) {
            second = bd;
            bd = dist;
            best = c;
        } else if (dist < second) {
            second = dist;
        }
    }
    if (gap)
        *gap = second - bd;
    return best;
}

/* ------------------------------------------------------------------------ */
/* Zone statistics [Prism guide, Method section 1, first eq.].               */
/* For zone m and axis d, the slice means Vbar^{(d)}_{m,i,c} average the 64  */
/* tokens of the zone whose d-coordinate is the i-th of the zone; mu_{m,c}   */
/* is their mean (= the zone mean);                                          */
/*   sigma^2_{v,d}(m) = 1/C sum_c 1/8 sum_i (Vbar^{(d)}_{m,i,c} - mu_{m,c})^2 */
/* Reading: the channel set is all heads x head_dim of V (one shape per      */
/* zone, shared by every head), because the audio norms carry no head index. */
/* The audio statistics sigma^2_{a,d}(m) are the same construction on the    */
/* one-channel field a_{t,h,w}; a_mean is the zone mean of a; a_max the grid */
/* maximum.  V is [T*H*W][C] bf16 bits in raster token order, a is [T*H*W].  */
/* ------------------------------------------------------------------------ */
static void slice_variances(const double *cube /* [8][8][8] */, double *var3)
{
    /* Writes the three directional variances of slice means of one channel. */
    double mean = 0.0;
    for (int i = 0; i < ZVOL; ++i)
        mean += cube[i];
    mean /= (double)ZVOL;
    for (int d = 0; d < 3; ++d) {
        double acc = 0.0;
        for (int i = 0; i < ZONE; ++i) {
            double s = 0.0;
            for (int u = 0; u < ZONE; ++u)
                for (int v = 0; v < ZONE; ++v) {
                    int t, h, w;
                    if (d == 0) { t = i; h = u; w = v; }
                    else if (d == 1) { t = u; h = i; w = v; }
                    else { t = u; h = v; w = i; }
                    s += cube[(t * ZONE + h) * ZONE + w];
                }
            double slice_mean = s / (double)(ZONE * ZONE);
            acc += (slice_mean - mean) * (slice_mean - mean);
        }
        var3[d] = acc / (double)ZONE;
    }
}

void orc_zone_stats(const uint16_t *V, const float *a, int T, int H, int W, int C,
                    double *sig_v /* [M][3] */, double *sig_a /* [M][3] */,
                    double *a_mean /* [M] */, double *a_max /* [1] */)
{
    int MT = T / ZONE, MH = H / ZONE, MW = W / ZONE, M = MT * MH * MW;
#pragma omp parallel for schedule(dynamic)
    for (int m = 0; m < M; ++m) {
        int zt = m / (MH * MW), zh = (m / MW) % MH, zw = m % MW;
        double cube[ZVOL], var3[3], acc3[3] = {0.0, 0.0, 0.0};
        for (int c = 0; c < C; ++c) {
            for (int t = 0; t < ZONE; ++t)
                for (int h = 0; h < ZONE; ++h)
                    for (int w = 0; w < ZONE; ++w) {
                        size_t tok = ((size_t)(zt * ZONE + t) * H + (zh * ZONE + h)) * W + (zw * ZONE + w);
                        cube[(t * ZONE + h) * ZONE + w] = widen_bf16(V[tok * (size_t)C + c]);
                    }
            slice_variances(cube, var3);
            for (int d = 0; d < 3; ++d)
                acc3[d] += var3[d];
        }
        for (int d = 0; d < 3; ++d)
            sig_v[3 * m + d] = acc3[d] / (double)C;

        double mean = 0.0;
        for (int t = 0; t < ZONE; ++t)
            for (int h = 0; h < ZONE; ++h)
                for (int w = 0; w < ZONE; ++w) {
                    size_t tok = ((size_t)(zt * ZONE + t) * H + (zh * ZONE + h)) * W + (zw * ZONE + w);
                    cube[(t * ZONE + h) * ZONE + w] = (double)a[tok];
                    mean += (double)a[tok];
                }
        slice_variances(cube, var3);
        for (int d = 0; d < 3; ++d)
            sig_a[3 * m + d] = var3[d];
        a_mean[m] = mean / (double)ZVOL;
    }
    double mx = -INFINITY;
    for (size_t n = 0; n < (size_t)T * H * W; ++n)
        if ((double)a[n] > mx)
            mx = (double)a[n];
    *a_max = mx;
}

/* ------------------------------------------------------------------------ */
/* Indicator, density, volume and shape.                                     */
/*  r_{v,d} = sigma^2_{v,d} / sum_d' sigma^2_{v,d'}   [Method section 1]     */
/*  vhat_{a,d} = sigma^2_{a,d} / sum_d' sigma^2_{a,d'} (reading: the same     */
/*      normalisation applied to a; scale-free)                              */
/*  abar(m) = mean over the zone of a / max over the grid of a, in [0,1]     */
/*      (reading: plainest map of a non-negative norm into [0,1])            */
/*  g_d = r_{v,d} + abar * vhat_{a,d} + eps            [Method section 1]     */
/*  A zero denominator (a constant zone) gives 1/3 on each axis (reading).  */
/*  rho(m) = min(1, max(s(m)/max_m' s(m'), abar(m))) with s = sum_d sigma^2_v */
/*      (reading: fine blocks where the video changes fast OR the audio      */
/*      coupling is strong)                                                  */
/*  B = 64 if rho >= tau_128 = 0.5; 128 if rho >= tau_256 = 0.25; else 256  */
/*      [Method section 2, first sentence; direction is a reading]           */
/*  shape = nearest candidate of volume B to l*(g)     [Method section 2]     */
/* fixed >= 0 forces that table index for every zone (fixed-shape configs). */
/* Diagnostics: gap_shape = distance^2 margin of the chosen shape, gap_rho = */
/* min |rho - tau|.                                                          */
/* ------------------------------------------------------------------------ */
void orc_zone_decide(int M, const double *sig_v, const double *sig_a, const double *a_mean,
                     double a_max, double eps, int fixed,
                     double *g, double *rho, double *lstar, int *zB, int *zshape,
                     double *gap_shape, double *gap_rho)
{
    double s_max = 0.0;
    for (int m = 0; m < M; ++m) {
        double s = sig_v[3 * m] + sig_v[3 * m + 1] + sig_v[3 * m + 2];
        if (s > s_max)
            s_max = s;
    }
    int exps[16 * 3];
    orc_shape_table(exps);
    for (int m = 0; m < M; ++m) {
        double sv = sig_v[3 * m] + sig_v[3 * m + 1] + sig_v[3 * m + 2];
        double sa = sig_a[3 * m] + sig_a[3 * m + 1] + sig_a[3 * m + 2];
        double abar = (a_max > 0.0) ? a_mean[m] / a_max : 0.0;
        for (int d = 0; d < 3; ++d) {
            double r = (sv < 1e-30) ? (1.0 / 3.0) : sig_v[3 * m + d] / sv;
            double vh = (sa < 1e-30) ? (1.0 / 3.0) : sig_a[3 * m + d] / sa;
            g[3 * m + d] = r + abar * vh + eps;
        }
        double rv = (s_max > 0.0) ? sv / s_max : 0.0;
        double r = rv > abar ? rv : abar;
        if (r > 1.0)
            r = 1.0;
        rho[m] = r;
        double g1 = fabs(r - 0.5), g2 = fabs(r - 0.25);
        gap_rho[m] = g1 < g2 ? g1 : g2;
        if (fixed >= 0) {
            int S = exps[3 * fixed] + exps[3 * fixed + 1] + exps[3 * fixed + 2];
            zB[m] = 1 << S;
            zshape[m] = fixed;
            orc_lstar(&g[3 * m], S, &lstar[3 * m]);
            gap_shape[m] = INFINITY;
            continue;
        }
        int B = (r >= 0.5) ? 64 : ((r >= 0.25) ? 128 : 256);
        int S = (B == 64) ? 6 : ((B == 128) ? 7 : 8);
        zB[m] = B;
        orc_lstar(&g[3 * m], S, &lstar[3 * m]);
        zshape[m] = orc_pick_shape(&lstar[3 * m], S, &gap_shape[m]);
    }
}

/* ------------------------------------------------------------------------ */
/* Blocks.  Each zone is tiled by its shape (bT,bH,bW); blocks are numbered  */
/* zone by zone in raster order of the zone grid, and inside a zone in       */
/* raster order of its (8/bT)x(8/bH)x(8/bW) sub-grid (reading: the guide     */
/* fixes no order).  box[j] = {t0,h0,w0,bT,bH,bW} in token coordinates.     */
/* ------------------------------------------------------------------------ */
int orc_blocks(int T, int H, int W, const int *zshape, int *box /* [N/64][6] or NULL */)
{
    int exps[16 * 3];
    orc_shape_table(exps);
    int MT = T / ZONE, MH = H / ZONE, MW = W / ZONE;
    int nb = 0;
    for (int m = 0; m < MT * MH * MW; ++m) {
        int zt = m / (MH * MW), zh = (m / MW) % MH, zw = m % MW;
        int bT = 1 << exps[3 * zshape[m]], bH = 1 << exps[3 * zshape[m] + 1],
            bW = 1 << exps[3 * zshape[m] + 2];
        for (int it = 0; it < ZONE / bT; ++it)
            for (int ih = 0; ih < ZONE / bH; ++ih)
                for (int iw = 0; iw < ZONE / bW; ++iw) {
                    if (box) {
                        int *b = &box[6 * nb];
                        b[0] = zt * ZONE + it * bT;
                        b[1] = zh * ZONE + ih * bH;
                        b[2] = zw * ZONE + iw * bW;
                        b[3] = bT;
                        b[4] = bH;
                        b[5] = bW;
                    }
                    ++nb;
                }
    }
    return nb;
}

/* Block-contiguous order: blocks in order, tokens of a block in raster
 * (t,h,w) order.  perm[new] = old raster token index. */
void orc_perm(int T, int H, int W, int nb, const int *box, int *perm)
{
    (void)T;
    size_t n = 0;
    for (int j = 0; j < nb; ++j) {
        const int *b = &box[6 * j];
        for (int t = b[0]; t < b[0] + b[3]; ++t)
            for (int h = b[1]; h < b[1] + b[4]; ++h)
                for (int w = b[2]; w < b[2] + b[5]; ++w)
                    perm[n++] = (t * H + h) * W + w;
    }
}

/* Mean-pooling of X = Q or K over each block, per head
 * [Prism guide, Method section 3: key blocks mean-pooled to Kbar_j; the
 * query blocks are pooled the same way (reading)].  X is [T*H*W][heads][D]
 * bf16 bits; Xbar is [heads][nb][D]. */
void orc_pool(const uint16_t *X, int T, int H, int W, int heads, int D, int nb,
              const int *box, double *Xbar)
{
    (void)T;
#pragma omp parallel for schedule(dynamic)
    for (int j = 0; j < nb; ++j) {
        const int *b = &box[6 * j];
        double cnt = (double)(b[3] * b[4] * b[5]);
        for (int hd = 0; hd < heads; ++hd)
            for (int c = 0; c < D; ++c) {
                double s = 0.0;
                for (int t = b[0]; t < b[0] + b[3]; ++t)
                    for (int h = b[1]; h < b[1] + b[4]; ++h)
                        for (int w = b[2]; w < b[2] + b[5]; ++w) {
                            size_t tok = ((size_t)t * H + h) * W + w;
                            s += widen_bf16(X[(tok * heads + hd) * D + c]);
                        }
                Xbar[((size_t)hd * nb + j) * D + c] = s / cnt;
            }
    }
}

/* Block means over blocks given as runs of a permutation: block j holds
 * the tokens perm[blk_off[j]] ... perm[blk_off[j+1]-1].  X is [N][heads][D]
 * bf16 bits; Xbar is [heads][nb][D].  The sum runs in block order. */
void orc_pool_blocks(const uint16_t *X, int heads, int D, int nb, const int *perm,
                     const int *blk_off, double *Xbar)
{
#pragma omp parallel for schedule(dynamic)
    for (int j = 0; j < nb; ++j) {
        double cnt = (double)(blk_off[j + 1] - blk_off[j]);
        for (int hd = 0; hd < heads; ++hd)
            for (int c = 0; c < D; ++c) {
                double s = 0.0;
                for (int m = blk_off[j]; m < blk_off[j + 1]; ++m)
                    s += widen_bf16(X[((size_t)perm[m] * heads + hd) * D + c]);
                Xbar[((size_t)hd * nb + j) * D + c] = s / cnt;
            }
    }
}

/* ------------------------------------------------------------------------ */
/* Hilbert-order fixed blocks [DFSAttn page, first component: tokens are     */
/* reordered along a 3D Hilbert curve, so that tokens next to each other in  */
/* the order are neighbours in space and time, and grouped into blocks].     */
/*                                                                           */
/* The curve is the one of the 2^k cube, k the smallest with 2^k >= T, H, W, */
/* with the index of Skilling's method ("Programming the Hilbert curve",     */
/* AIP Conf. Proc. 707, 2004): the coordinates (x0, x1, x2) = (t, h, w) go   */
/* through the method's two passes -- for each bit level from the top, the   */
/* lower bits of x0 are inverted (where x_i has that bit) or exchanged with  */
/* those of x_i (where it does not); then a Gray encoding across the three   */
/* coordinates -- and the index is read off the transformed coordinates bit  */
/* level by bit level from the top, x0's bit first.  Reading: a grid that is */
/* not a cube takes the cube's curve restricted to its tokens (the pages do  */
/* not say how the curve meets a non-cube grid).                             */
/* ------------------------------------------------------------------------ */
uint64_t orc_hilbert_index(int t, int h, int w, int k)
{
    unsigned x[3] = {(unsigned)t, (unsigned)h, (unsigned)w};
    if (k < 1)
        return 0;
    unsigned top = 1u << (k - 1);
    /* pass 1: from the top bit level down to level 1 */
    for (unsigned q = top; q > 1; q >>= 1) {
        unsigned low = q - 1;
        for (int i = 0; i < 3; ++i) {
            if (x[i] & q) {
                x[0] ^= low;
            } else {
                unsigned diff = (x[0] ^ x[i]) & low;
                x[0] ^= diff;
                x[i] ^= diff;
            }
        }
    }
    /* pass 2: Gray encoding */
    x[1] ^= x[0];
    x[2] ^= x[1];
    unsigned flip = 0;
    for (unsigned q = top; q > 1; q >>= 1)
        if (x[2] & q)
            flip ^= q - 1;
    for (int i = 0; i < 3; ++i)
        x[i] ^= flip;
    /* interleave: bit levels from the top, x0 before x1 before x2 */
    uint64_t idx = 0;
    for (int b = k - 1; b >= 0; --b)
        for (int i = 0; i < 3; ++i)
            idx = (idx << 1) | ((x[i] >> b) & 1u);
    return idx;
}

void orc_hilbert_indices(const int *pts /* [n][3] (t,h,w) */, long long n, int k, uint64_t *out)
{
#pragma omp parallel for schedule(static)
    for (long long r = 0; r < n; ++r)
        out[r] = orc_hilbert_index(pts[3 * r], pts[3 * r + 1], pts[3 * r + 2], k);
}

typedef struct {
    uint64_t key;
    int tok;
} hkey_t;

static int cmp_hkey(const void *pa, const void *pb)
{
    const hkey_t *a = (const hkey_t *)pa, *b = (const hkey_t *)pb;
    return (a->key > b->key) - (a->key < b->key);
}

/* perm[n] = raster index of the n-th grid token along the curve. */
void orc_hilbert_perm(int T, int H, int W, int *perm)
{
    int k = 0;
    while ((1 << k) < T || (1 << k) < H || (1 << k) < W)
        ++k;
    size_t N = (size_t)T * H * W;
    hkey_t *a = (hkey_t *)malloc(sizeof(hkey_t) * N);
    for (int t = 0; t < T; ++t)
        for (int h = 0; h < H; ++h)
            for (int w = 0; w < W; ++w) {
                size_t n = ((size_t)t * H + h) * W + w;
                a[n].key = orc_hilbert_index(t, h, w, k);
                a[n].tok = (int)n;
            }
    qsort(a, N, sizeof(hkey_t), cmp_hkey);
    for (size_t n = 0; n < N; ++n)
        perm[n] = a[n].tok;
    free(a);
}

/* ------------------------------------------------------------------------ */
/* Hybrid selection for one query block [Prism guide, Method section 3]:    */
/*   P = softmax_j(z_j);  S = Top-k(P,k) U Top-p(P,p).                       */
/* Order: descending z (equivalently descending P), equal z by ascending j.  */
/* Top-k = first min(k,nb) of that order.  Top-p = the shortest prefix whose */
/* cumulative mass reaches p (the CDF cutoff; nb if rounding never reaches   */
/* p).  Both are prefixes of one order, so the union is the longer prefix.   */
/* The per-row cap (a workload parameter, not on the pages) truncates the    */
/* union to its first `cap` entries.  sel receives the chosen j ascending.  */
/* diag[0] = z margin at the cut (last kept minus first dropped, +inf if all */
/* kept); diag[1] = distance of the cumulative mass to p around the Top-p    */
/* cut; diag[2] = 1 if the cap shortened the union.  Returns the count.     */
/* ------------------------------------------------------------------------ */
typedef struct {
    double z;
    int j;
} zj_t;

static int cmp_zj(const void *pa, const void *pb)
{
    const zj_t *a = (const zj_t *)pa, *b = (const zj_t *)pb;
    if (a->z > b->z) return -1;
    if (a->z < b->z) return 1;
    return (a->j > b->j) - (a->j < b->j);
}

static int cmp_int(const void *pa, const void *pb)
{
    int a = *(const int *)pa, b = *(const int *)pb;
    return (a > b) - (a < b);
}

int orc_select_row(const double *z, int nb, int k, double p, int cap, int *sel, double *diag)
{
    zj_t *ord = (zj_t *)malloc(sizeof(zj_t) * (size_t)nb);
    double zmax = -INFINITY;
    for (int j = 0; j < nb; ++j) {
        ord[j].z = z[j];
        ord[j].j = j;
        if (z[j] > zmax)
            zmax = z[j];
    }
    double denom = 0.0;
    for (int j = 0; j < nb; ++j)
        denom += exp(z[j] - zmax);
    qsort(ord, (size_t)nb, sizeof(zj_t), cmp_zj);

    int n_k = k < nb ? k : nb;
    int n_p = nb;
    double cum = 0.0, prev = 0.0, mass_gap = INFINITY;
    for (int n = 0; n < nb; ++n) {
        prev = cum;
        cum += exp(ord[n].z - zmax) / denom;
        if (cum >= p) {
            n_p = n + 1;
            mass_gap = cum - p;
            if (n > 0 && p - prev < mass_gap)
                mass_gap = p - prev;
            break;
        }
    }
    int want = n_k > n_p ? n_k : n_p;
    int n = want < cap ? want : cap;
    if (n > nb)
        n = nb;
    for (int q = 0; q < n; ++q)
        sel[q] = ord[q].j;
    qsort(sel, (size_t)n, sizeof(int), cmp_int);
    if (diag) {
        diag[0] = (n < nb) ? ord[n - 1].z - ord[n].z : INFINITY;
        diag[1] = mass_gap;
        diag[2] = (want > n) ? 1.0 : 0.0;
    }
    free(ord);
    return n;
}

/* Selection for every (head, query block): z_ij = Qbar_i . Kbar_j / sqrt(D)
 * [Method section 3: pooled queries scored against pooled keys; no
 * block-size correction (reading)].  cap = max(k, floor(max_frac*nb)) when
 * max_frac > 0, else nb.  cols is [heads][nb][stride], cnt [heads][nb],
 * diag [heads][nb][3]. */
int orc_cap(int nb, int k, double max_frac)
{
    if (!(max_frac > 0.0))
        return nb;
    int c = (int)floor(max_frac * (double)nb);
    if (c < k)
        c = k;
    if (c > nb)
        c = nb;
    return c;
}

void orc_select(const double *Qbar, const double *Kbar, int heads, int nb, int D, int k,
                double p, double max_frac, int stride, int *cnt, int *cols, double *diag)
{
    int cap = orc_cap(nb, k, max_frac);
    double sq = sqrt((double)D);
#pragma omp parallel
    {
        double *z = (double *)malloc(sizeof(double) * (size_t)nb);
#pragma omp for schedule(dynamic, 4)
        for (long long r = 0; r < (long long)heads * nb; ++r) {
            int hd = (int)(r / nb), i = (int)(r % nb);
            const double *q = &Qbar[((size_t)hd * nb + i) * D];
            for (int j = 0; j < nb; ++j) {
                const double *kk = &Kbar[((size_t)hd * nb + j) * D];
                double dot = 0.0;
                for (int c = 0; c < D; ++c)
                    dot += q[c] * kk[c];
                z[j] = dot / sq;
            }
            cnt[r] = orc_select_row(z, nb, k, p, cap, &cols[(size_t)r * stride],
                                    diag ? &diag[3 * (size_t)r] : NULL);
        }
        free(z);
    }
}

/* ------------------------------------------------------------------------ */
/* Sparse attention [Prism guide, Method section 3, last sentence]: each     */
/* query token of block i attends, under one softmax, to every token of     */
/* every key block in S_i:                                                   */
/*   s_qt = q.k_t / sqrt(D);  O_q = sum_t softmax_t(s_qt) v_t;               */
/*   LSE_q = log sum_t exp(s_qt).                                            */
/* Backward of L = sum_q dO_q . O_q (the standard softmax-attention          */
/* gradient, restricted to the same pairs):                                  */
/*   P_qt = exp(s_qt - LSE_q),  dP_qt = dO_q . v_t,                          */
/*   Delta_q = sum_t P_qt dP_qt,  dS_qt = P_qt (dP_qt - Delta_q),            */
/*   dQ_q = sum_t dS_qt k_t / sqrt(D),  dK_t = sum_q dS_qt q_q / sqrt(D),    */
/*   dV_t = sum_q P_qt dO_q.                                                 */
/* Tokens are raster indices; Q,K,V,dO are [N][heads][D] bf16 bits.  The    */
/* selection is (cnt, cols, stride) as written by orc_select; the blocks    */
/* are given as perm / blk_off: block j holds the tokens perm[blk_off[j]],  */
/* ..., perm[blk_off[j+1]-1], in that order (for zone blocks, raster order  */
/* inside the box).  Only requested outputs are computed.                   */
/* ------------------------------------------------------------------------ */
typedef struct {
    const uint16_t *Q, *K, *V, *dO;
    int heads, D, nb, stride;
    const int *perm, *blk_off, *cnt, *cols;
    int *tok2blk;
} attn_ctx;

static void ctx_init(attn_ctx *cx, int T, int H, int W)
{
    size_t N = (size_t)T * H * W;
    cx->tok2blk = (int *)malloc(sizeof(int) * N);
    for (int j = 0; j < cx->nb; ++j)
        for (int n = cx->blk_off[j]; n < cx->blk_off[j + 1]; ++n)
            cx->tok2blk[cx->perm[n]] = j;
}

/* Scores of query token q (head hd) against every selected key token, in
 * the order: selected blocks ascending, tokens of a block in block order.
 * Returns the count; toks/s receive the key tokens and their scores. */
static int row_scores(const attn_ctx *cx, int hd, int q, int *toks, double *s)
{
    int i = cx->tok2blk[q];
    size_t r = (size_t)hd * cx->nb + i;
    const int *cl = &cx->cols[r * cx->stride];
    double sq = sqrt((double)cx->D);
    int n = 0;
    for (int u = 0; u < cx->cnt[r]; ++u) {
        for (int m = cx->blk_off[cl[u]]; m < cx->blk_off[cl[u] + 1]; ++m) {
            int kt = cx->perm[m];
            double dot = 0.0;
            for (int c = 0; c < cx->D; ++c)
                dot += widen_bf16(cx->Q[((size_t)q * cx->heads + hd) * cx->D + c]) *
                       widen_bf16(cx->K[((size_t)kt * cx->heads + hd) * cx->D + c]);
            toks[n] = kt;
            s[n] = dot / sq;
            ++n;
        }
    }
    return n;
}

static double row_lse(const double *s, int n)
{
    double mx = -INFINITY;
    for (int u = 0; u < n; ++u)
        if (s[u] > mx)
            mx = s[u];
    double l = 0.0;
    for (int u = 0; u < n; ++u)
        l += exp(s[u] - mx);
    return mx + log(l);
}

void orc_attn_fwd_rows(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                       int T, int H, int W, int heads, int D, int nb, const int *perm,
                       const int *blk_off, const int *cnt, const int *cols, int stride,
                       int nreq, const int *req_h, const int *req_tok,
                       double *O /* [nreq][D] */, double *lse /* [nreq] */)
{
    attn_ctx cx = {Q, K, V, NULL, heads, D, nb, stride, perm, blk_off, cnt, cols, NULL};
    ctx_init(&cx, T, H, W);
    size_t N = (size_t)T * H * W;
#pragma omp parallel
    {
        int *toks = (int *)malloc(sizeof(int) * N);
        double *s = (double *)malloc(sizeof(double) * N);
#pragma omp for schedule(dynamic, 4)
        for (int r = 0; r < nreq; ++r) {
            int hd = req_h[r], q = req_tok[r];
            int n = row_scores(&cx, hd, q, toks, s);
            double L = row_lse(s, n);
            for (int c = 0; c < D; ++c)
                O[(size_t)r * D + c] = 0.0;
            for (int u = 0; u < n; ++u) {
                double pr = exp(s[u] - L);
                for (int c = 0; c < D; ++c)
                    O[(size_t)r * D + c] += pr * widen_bf16(V[((size_t)toks[u] * heads + hd) * D + c]);
            }
            lse[r] = L;
        }
        free(toks);
        free(s);
    }
    free(cx.tok2blk);
}

/* ------------------------------------------------------------------------ */
/* Forward with a zeroth-order Taylor term for the key blocks outside S_i.   */
/* [In-Context Sparse Attention article, the grouped-computation paragraphs: */
/* the flat path replaces the tokens of a key block by the block's mean and  */
/* keeps only the zeroth-order term of the exponential's expansion.]         */
/* Reading, for the blocks Prism's selection leaves out: for a token t of a  */
/* key block j not in S_i, exp(q.k_t/sqrt(D)) is expanded around the block's */
/* mean key kbar_j (mean of its bf16 keys, fp64) and cut after the constant  */
/* term, exp(q.kbar_j/sqrt(D)).  Summed over the |B_j| tokens of the block:  */
/*   normaliser  += |B_j| exp(q.kbar_j/sqrt(D))                              */
/*   numerator   += exp(q.kbar_j/sqrt(D)) sum_t v_t                          */
/*                = |B_j| exp(q.kbar_j/sqrt(D)) vbar_j.                      */
/* The tokens of the blocks in S_i enter exactly, as in orc_attn_fwd_rows;   */
/* one softmax normalises both parts.  LSE is log of the whole normaliser.  */
/* ------------------------------------------------------------------------ */
void orc_attn_fwd_taylor_rows(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                              int T, int H, int W, int heads, int D, int nb, const int *perm,
                              const int *blk_off, const int *cnt, const int *cols, int stride,
                              int nreq, const int *req_h, const int *req_tok,
                              double *O /* [nreq][D] */, double *lse /* [nreq] */)
{
    attn_ctx cx = {Q, K, V, NULL, heads, D, nb, stride, perm, blk_off, cnt, cols, NULL};
    ctx_init(&cx, T, H, W);
    size_t N = (size_t)T * H * W;
    double *Kbar = (double *)malloc(sizeof(double) * (size_t)heads * nb * D);
    double *Vbar = (double *)malloc(sizeof(double) * (size_t)heads * nb * D);
    orc_pool_blocks(K, heads, D, nb, perm, blk_off, Kbar);
    orc_pool_blocks(V, heads, D, nb, perm, blk_off, Vbar);
    double sq = sqrt((double)D);
#pragma omp parallel
    {
        int *toks = (int *)malloc(sizeof(int) * N);
        double *s = (double *)malloc(sizeof(double) * N);
        double *z = (double *)malloc(sizeof(double) * nb);
        char *in_s = (char *)malloc((size_t)nb);
#pragma omp for schedule(dynamic, 4)
        for (int r = 0; r < nreq; ++r) {
            int hd = req_h[r], q = req_tok[r];
            int i = cx.tok2blk[q];
            size_t row = (size_t)hd * nb + i;
            memset(in_s, 0, (size_t)nb);
            for (int u = 0; u < cnt[row]; ++u)
                in_s[cols[row * stride + u]] = 1;
            /* exact part: every token of the selected blocks */
            int n = row_scores(&cx, hd, q, toks, s);
            /* Taylor part: one pooled term per block outside S_i */
            double mx = -INFINITY;
            for (int u = 0; u < n; ++u)
                if (s[u] > mx)
                    mx = s[u];
            for (int j = 0; j < nb; ++j) {
                if (in_s[j])
                    continue;
                double dot = 0.0;
                for (int c = 0; c < D; ++c)
                    dot += widen_bf16(Q[((size_t)q * heads + hd) * D + c]) * Kbar[((size_t)hd * nb + j) * D + c];
                z[j] = dot / sq;
                if (z[j] > mx)
                    mx = z[j];
            }
            double l = 0.0;
            for (int u = 0; u < n; ++u)
                l += exp(s[u] - mx);
            for (int j = 0; j < nb; ++j)
                if (!in_s[j])
                    l += (double)(blk_off[j + 1] - blk_off[j]) * exp(z[j] - mx);
            double L = mx + log(l);
            for (int c = 0; c < D; ++c)
                O[(size_t)r * D + c] = 0.0;
            for (int u = 0; u < n; ++u) {
                double pr = exp(s[u] - L);
                for (int c = 0; c < D; ++c)
                    O[(size_t)r * D + c] += pr * widen_bf16(V[((size_t)toks[u] * heads + hd) * D + c]);
            }
            for (int j = 0; j < nb; ++j) {
                if (in_s[j])
                    continue;
                double wt = (double)(blk_off[j + 1] - blk_off[j]) * exp(z[j] - L);
                for (int c = 0; c < D; ++c)
                    O[(size_t)r * D + c] += wt * Vbar[((size_t)hd * nb + j) * D + c];
            }
            lse[r] = L;
        }
        free(toks);
        free(s);
        free(z);
        free(in_s);
    }
    free(Kbar);
    free(Vbar);
    free(cx.tok2blk);
}

void orc_attn_bwd_dq_rows(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                          const uint16_t *dO, int T, int H, int W, int heads, int D, int nb,
                          const int *perm, const int *blk_off, const int *cnt, const int *cols, int stride,
                          int nreq, const int *req_h, const int *req_tok,
                          double *dQ /* [nreq][D] */)
{
    attn_ctx cx = {Q, K, V, dO, heads, D, nb, stride, perm, blk_off, cnt, cols, NULL};
    ctx_init(&cx, T, H, W);
    size_t N = (size_t)T * H * W;
    double sq = sqrt((double)D);
#pragma omp parallel
    {
        int *toks = (int *)malloc(sizeof(int) * N);
        double *s = (double *)malloc(sizeof(double) * N);
        double *dp = (double *)malloc(sizeof(double) * N);
#pragma omp for schedule(dynamic, 4)
        for (int r = 0; r < nreq; ++r) {
            int hd = req_h[r], q = req_tok[r];
            int n = row_scores(&cx, hd, q, toks, s);
            double L = row_lse(s, n);
            double delta = 0.0;
            for (int u = 0; u < n; ++u) {
                double d = 0.0;
                for (int c = 0; c < D; ++c)
                    d += widen_bf16(dO[((size_t)q * heads + hd) * D + c]) *
                         widen_bf16(V[((size_t)toks[u] * heads + hd) * D + c]);
                dp[u] = d;
                delta += exp(s[u] - L) * d;
            }
            for (int c = 0; c < D; ++c)
                dQ[(size_t)r * D + c] = 0.0;
            for (int u = 0; u < n; ++u) {
                double ds = exp(s[u] - L) * (dp[u] - delta);
                for (int c = 0; c < D; ++c)
                    dQ[(size_t)r * D + c] += ds * widen_bf16(K[((size_t)toks[u] * heads + hd) * D + c]) / sq;
            }
        }
        free(toks);
        free(s);
        free(dp);
    }
    free(cx.tok2blk);
}

static int row_has(const int *cl, int n, int j)
{
    int lo = 0, hi = n - 1;
    while (lo <= hi) {
        int mid = (lo + hi) / 2;
        if (cl[mid] == j)
            return 1;
        if (cl[mid] < j)
            lo = mid + 1;
        else
            hi = mid - 1;
    }
    return 0;
}

void orc_attn_bwd_dkv_rows(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                           const uint16_t *dO, int T, int H, int W, int heads, int D, int nb,
                           const int *perm, const int *blk_off, const int *cnt, const int *cols, int stride,
                           int nreq, const int *req_h, const int *req_tok,
                           double *dK /* [nreq][D] */, double *dV /* [nreq][D] */)
{
    attn_ctx cx = {Q, K, V, dO, heads, D, nb, stride, perm, blk_off, cnt, cols, NULL};
    ctx_init(&cx, T, H, W);
    size_t N = (size_t)T * H * W;
    double sq = sqrt((double)D);
    /* Query blocks whose selection holds a requested key token's block. */
    char *need = (char *)calloc((size_t)heads * nb, 1);
    for (int r = 0; r < nreq; ++r) {
        int hd = req_h[r], j = cx.tok2blk[req_tok[r]];
        for (int i = 0; i < nb; ++i) {
            size_t row = (size_t)hd * nb + i;
            if (row_has(&cols[row * stride], cnt[row], j))
                need[row] = 1;
        }
    }
    /* LSE_q and Delta_q of every query token of those blocks. */
    double *L = (double *)malloc(sizeof(double) * (size_t)heads * N);
    double *Dl = (double *)malloc(sizeof(double) * (size_t)heads * N);
#pragma omp parallel
    {
        int *toks = (int *)malloc(sizeof(int) * N);
        double *s = (double *)malloc(sizeof(double) * N);
#pragma omp for schedule(dynamic, 16)
        for (long long qq = 0; qq < (long long)heads * N; ++qq) {
            int hd = (int)(qq / (long long)N);
            int q = (int)(qq % (long long)N);
            if (!need[(size_t)hd * nb + cx.tok2blk[q]])
                continue;
            int n = row_scores(&cx, hd, q, toks, s);
            double lq = row_lse(s, n);
            double delta = 0.0;
            for (int u = 0; u < n; ++u) {
                double d = 0.0;
                for (int c = 0; c < D; ++c)
                    d += widen_bf16(dO[((size_t)q * heads + hd) * D + c]) *
                         widen_bf16(V[((size_t)toks[u] * heads + hd) * D + c]);
                delta += exp(s[u] - lq) * d;
            }
            L[qq] = lq;
            Dl[qq] = delta;
        }
        free(toks);
        free(s);
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nreq; ++r) {
        int hd = req_h[r], kt = req_tok[r], j = cx.tok2blk[kt];
        double *dk = &dK[(size_t)r * D], *dv = &dV[(size_t)r * D];
        for (int c = 0; c < D; ++c)
            dk[c] = dv[c] = 0.0;
        for (int i = 0; i < nb; ++i) {
            size_t row = (size_t)hd * nb + i;
            if (!row_has(&cols[row * stride], cnt[row], j))
                continue;
            for (int m = blk_off[i]; m < blk_off[i + 1]; ++m) {
                int q = perm[m];
                double dot = 0.0, dpq = 0.0;
                for (int c = 0; c < D; ++c) {
                    dot += widen_bf16(Q[((size_t)q * heads + hd) * D + c]) *
                           widen_bf16(K[((size_t)kt * heads + hd) * D + c]);
                    dpq += widen_bf16(dO[((size_t)q * heads + hd) * D + c]) *
                           widen_bf16(V[((size_t)kt * heads + hd) * D + c]);
                }
                double pr = exp(dot / sq - L[(size_t)hd * N + q]);
                double ds = pr * (dpq - Dl[(size_t)hd * N + q]);
                for (int c = 0; c < D; ++c) {
                    dv[c] += pr * widen_bf16(dO[((size_t)q * heads + hd) * D + c]);
                    dk[c] += ds * widen_bf16(Q[((size_t)q * heads + hd) * D + c]) / sq;
                }
            }
        }
    }
    free(need);
    free(L);
    free(Dl);
    free(cx.tok2blk);
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Audio guidance a_{t,h,w} = || h^_{t,h,w} ||_2 [Prism guide, Method section
 * 1, the sentence before the g_d equation]: the L2 norm, over the channels,
 * of the audio-to-video cross-attention output of each video token, which the
 * layer caches for the next layer's plan.  h is [rows][C] bf16 bits, a is
 * [rows] (rows = batch * T * H * W in raster order).  The squares are summed
 * in channel order.                                                        */
void orc_audio_norms(const uint16_t *h, double *a, long long rows, int C)
{
#pragma omp parallel for schedule(static)
    for (long long r = 0; r < rows; ++r) {
        double s = 0.0;
        for (int c = 0; c < C; ++c) {
            const double x = widen_bf16(h[r * (long long)C + c]);
            s += x * x;
        }
        a[r] = sqrt(s);
    }
}
