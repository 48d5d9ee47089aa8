/*
 * mta_oracle.c -- plain fp64 CPU reference of the Multi-Token Attention (MTA)
 * forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke entry
 * and the CPU-baseline leg of the benchmark may load this library.  The CUDA
 * library never links, includes or calls it, and it includes nothing from the
 * CUDA side.
 *
 * Sources (page titles, sections, equations):
 *   [MHA]  "Multi-Token Attention -- Paper Graph", section 3.4, "Standard
 *          Multi-Head Attention": A^ = Q K^T / sqrt(d), causal Mask_-inf,
 *          softmax over keys, output A V per head.
 *   [KQ4]  same page, "Key-Query Convolution", Eq. (4): the kernel indices run
 *          over i' in [0, c_q) (queries looking back) and
 *          j' in [-floor(c_k/2), ceil(c_k/2) - 1] (keys both ways); the tap
 *          (i', j') multiplies q_{i-i'} k_{j-j'}^T / sqrt(d).
 *   [KQ5]  same section, Eq. (5), the two-pass masking the page calls the
 *          default: Softmax(Mask_-inf(Conv2d_theta(Mask_0(A^)))).
 *   [HM7]  same page, "Head Mixing Convolution", Eq. (7): heads split into
 *          non-overlapping groups of c_h; A^h_new = sum_h' w_{h h'} A^h',
 *          applied after the softmax ("Putting Everything Together",
 *          "Mixed (key-query pre-softmax, head post-softmax)").
 *   [GN]   same page, "Group Normalization with Sigmoid Gating": GroupNorm
 *          over the concatenation of the heads, one group per head (each
 *          head's d-vector is normalised on its own);
 *          "Article Overview: Multi-Token Attention", section 2, "Group
 *          Normalization with Depth Scaling": the scale is a depth scaling.
 *   [GATE] "Multi-Token Attention -- Paper Graph", "Group Normalization with
 *          Sigmoid Gating": the pages' default scale, one learned scalar g_h
 *          per head, output = GroupNorm(concat) * sigmoid(g_h) on head h.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - taps that fall outside [0,T) x [0,T) read zero (zero padding);
 *   - w_head is stored [group][out head][in head];
 *   - GroupNorm uses the biased variance and eps inside the square root,
 *     with a per-channel affine (gamma, beta) over the H*d concatenation;
 *   - depth scaling is a caller-supplied scalar multiplying the GN output;
 *   - the sigmoid gate multiplies the GN output (after its affine) in place
 *     of the depth scale.
 *
 * Layouts: q, k, v are [B][H][T][d]; w_kq is [H][c_q][c_k] with the tap
 * (i', j') at [h][i'][j' + floor(c_k/2)]; w_head is [H/c_h][c_h][c_h];
 * gn_weight, gn_bias are [H*d]; out is [B][T][H*d].
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int B, H, T, d, c_q, c_k, c_h;
    double gn_eps;
} mta_oracle_shape;

typedef struct {
    const double *q, *k, *v, *w_kq, *w_head, *gn_weight, *gn_bias;
    double depth_scale;
    const double *gate;   /* [H] gate logits g_h, or NULL for the depth scale */
} mta_oracle_args;

static int shape_ok(const mta_oracle_shape *s)
{
    if (!s) return 0;
    if (s->B < 1 || s->H < 1 || s->T < 1 || s->d < 1) return 0;
    if (s->c_q < 1 || s->c_k < 1 || s->c_h < 1) return 0;
    if (s->H % s->c_h != 0) return 0;
    return 1;
}

static const double *row_of(const double *x, const mta_oracle_shape *s,
                            int b, int h, int t)
{
    return x + (((size_t)b * s->H + h) * s->T + t) * s->d;
}

/* [MHA] then the first mask of [KQ5]: the scaled logit q_r . k_c / sqrt(d)
 * when key c is not in the future of query r, zero otherwise; rows or
 * columns outside [0,T) are zero padding.  Fills out[0..T). */
static void masked0_logit_row(const mta_oracle_shape *s, const mta_oracle_args *a,
                              int b, int h, int r, double *out)
{
    const int T = s->T, d = s->d;
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    for (int c = 0; c < T; ++c) out[c] = 0.0;
    if (r < 0 || r >= T) return;
    const double *qr = row_of(a->q, s, b, h, r);
    for (int c = 0; c <= r; ++c) {
        const double *kc = row_of(a->k, s, b, h, c);
        double dot = 0.0;
        for (int e = 0; e < d; ++e) dot += qr[e] * kc[e];
        out[c] = dot * inv_sqrt_d;
    }
}

/* [KQ4]/[KQ5]: C[i][j] = sum_{i'} sum_{j'} theta[i'][j'] A0[i-i'][j-j'] for
 * j in [0, i]; then the second mask of [KQ5] sets C[i][j] = -inf for j > i.
 * rows[i'] holds the masked logit row A0[i - i'][*]. */
static void conv_row(const mta_oracle_shape *s, const mta_oracle_args *a, int h,
                     int i, double *const *rows, double *C)
{
    const int T = s->T, c_q = s->c_q, c_k = s->c_k;
    const int jlo = -(c_k / 2);               /* -floor(c_k/2)    */
    const int jhi = (c_k + 1) / 2 - 1;        /*  ceil(c_k/2) - 1 */
    const double *theta = a->w_kq + (size_t)h * c_q * c_k;
    for (int j = 0; j < T; ++j) {
        if (j > i) { C[j] = -INFINITY; continue; }
        double acc = 0.0;
        for (int ip = 0; ip < c_q; ++ip) {
            if (i - ip < 0) continue;          /* zero row above the sequence */
            for (int jp = jlo; jp <= jhi; ++jp) {
                int c = j - jp;
                if (c < 0 || c >= T) continue; /* zero padding */
                acc += theta[ip * c_k + (jp - jlo)] * rows[ip][c];
            }
        }
        C[j] = acc;
    }
}

/* [MHA] softmax over keys of a row whose masked entries are -inf. */
static void softmax_row(int T, const double *C, double *P)
{
    double m = -INFINITY;
    for (int j = 0; j < T; ++j) if (C[j] > m) m = C[j];
    double sum = 0.0;
    for (int j = 0; j < T; ++j) {
        P[j] = (C[j] == -INFINITY) ? 0.0 : exp(C[j] - m);
        sum += P[j];
    }
    for (int j = 0; j < T; ++j) P[j] /= sum;
}

/* Work buffers for one (batch, head group) unit. */
typedef struct {
    double *ring;   /* [c_h][c_q][T] masked logit rows, ring over the query index */
    double *C;      /* [T] */
    double *P;      /* [c_h][T] pre-mix probabilities of the group's heads */
    double *A;      /* [T] mixed attention row of one output head */
    double *O;      /* [d] */
} unit_buffers;

static int alloc_unit(const mta_oracle_shape *s, unit_buffers *u)
{
    size_t T = (size_t)s->T;
    u->ring = (double *)calloc((size_t)s->c_h * s->c_q * T, sizeof(double));
    u->C = (double *)malloc(T * sizeof(double));
    u->P = (double *)malloc((size_t)s->c_h * T * sizeof(double));
    u->A = (double *)malloc(T * sizeof(double));
    u->O = (double *)malloc((size_t)s->d * sizeof(double));
    return u->ring && u->C && u->P && u->A && u->O;
}

static void free_unit(unit_buffers *u)
{
    free(u->ring); free(u->C); free(u->P); free(u->A); free(u->O);
}

/* Optional per-row intermediates (each [c_h][T] or [c_h][d]); any may be NULL. */
typedef struct {
    double *C;      /* conv logits after both masks, per head of the group */
    double *P;      /* pre-mix softmax rows */
    double *A;      /* post-mix attention rows */
    double *O;      /* pre-normalisation head outputs A^h V^h, [c_h][d] */
} row_taps;

/* One query row i of one (batch b, group g), given the masked logit rows:
 * rows_per_head[hh * c_q + ip] is A0[i - ip] of head g*c_h + hh.
 * Writes out_row[h*d + e] (the [H*d] output row of (b, i)) for the group's
 * heads when out_row != NULL, and the intermediates asked for in taps. */
static void group_row(const mta_oracle_shape *s, const mta_oracle_args *a,
                      int b, int g, int i, unit_buffers *u,
                      double *const *rows_per_head, double *out_row, row_taps *taps)
{
    const int T = s->T, d = s->d, c_h = s->c_h;
    /* [KQ5] per head: conv, masks, softmax. */
    for (int hh = 0; hh < c_h; ++hh) {
        int h = g * c_h + hh;
        conv_row(s, a, h, i, rows_per_head + (size_t)hh * s->c_q, u->C);
        if (taps && taps->C) memcpy(taps->C + (size_t)hh * T, u->C, T * sizeof(double));
        softmax_row(T, u->C, u->P + (size_t)hh * T);
        if (taps && taps->P) memcpy(taps->P + (size_t)hh * T, u->P + (size_t)hh * T, T * sizeof(double));
    }
    /* [HM7] post-softmax head mixing, then A^h V^h of the output head [MHA]. */
    const double *wg = a->w_head + (size_t)g * c_h * c_h;
    for (int ho = 0; ho < c_h; ++ho) {
        int h = g * c_h + ho;
        for (int j = 0; j < T; ++j) {
            double acc = 0.0;
            for (int hi = 0; hi < c_h; ++hi) acc += wg[ho * c_h + hi] * u->P[(size_t)hi * T + j];
            u->A[j] = acc;
        }
        if (taps && taps->A) memcpy(taps->A + (size_t)ho * T, u->A, T * sizeof(double));
        for (int e = 0; e < d; ++e) u->O[e] = 0.0;
        for (int j = 0; j <= i; ++j) {
            const double *vj = row_of(a->v, s, b, h, j);
            for (int e = 0; e < d; ++e) u->O[e] += u->A[j] * vj[e];
        }
        if (taps && taps->O) memcpy(taps->O + (size_t)ho * d, u->O, d * sizeof(double));
        if (!out_row) continue;
        /* [GN]: the head's d-vector is one group; biased variance. */
        double mean = 0.0;
        for (int e = 0; e < d; ++e) mean += u->O[e];
        mean /= d;
        double var = 0.0;
        for (int e = 0; e < d; ++e) var += (u->O[e] - mean) * (u->O[e] - mean);
        var /= d;
        double inv = 1.0 / sqrt(var + s->gn_eps);
        /* [GATE] sigmoid(g_h), or the depth scale */
        double scale = a->gate ? 1.0 / (1.0 + exp(-a->gate[h])) : a->depth_scale;
        for (int e = 0; e < d; ++e) {
            size_t chn = (size_t)h * d + e;
            double y = (u->O[e] - mean) * inv * a->gn_weight[chn] + a->gn_bias[chn];
            out_row[chn] = scale * y;
        }
    }
}

/* Points rows[hh*c_q + ip] at A0[i - ip] of each head of group g, computing
 * every row afresh into the unit's buffer (rows above the sequence are the
 * zero row). */
static void fresh_rows(const mta_oracle_shape *s, const mta_oracle_args *a, int b, int g,
                       int i, unit_buffers *u, const double *zero_row, double **rows)
{
    for (int hh = 0; hh < s->c_h; ++hh) {
        double *base = u->ring + (size_t)hh * s->c_q * s->T;
        for (int ip = 0; ip < s->c_q; ++ip) {
            if (i - ip < 0) { rows[(size_t)hh * s->c_q + ip] = (double *)zero_row; continue; }
            masked0_logit_row(s, a, b, g * s->c_h + hh, i - ip, base + (size_t)ip * s->T);
            rows[(size_t)hh * s->c_q + ip] = base + (size_t)ip * s->T;
        }
    }
}

/* Full forward: out[B][T][H*d].  Units (b, g) are independent and spread over
 * threads; inside a unit the query rows run in order, keeping the last c_q
 * masked logit rows of each head in a ring.  Returns 0 on success. */
static int forward_args(const mta_oracle_shape *s, const mta_oracle_args *pa, double *out,
                        int nthreads)
{
    if (!shape_ok(s) || !pa->q || !pa->k || !pa->v || !pa->w_kq || !pa->w_head ||
        !pa->gn_weight || !pa->gn_bias || !out)
        return -1;
    const mta_oracle_args a = *pa;
    const int G = s->H / s->c_h;
    const int units = s->B * G;
    const size_t HD = (size_t)s->H * s->d;
    int failed = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1) reduction(|:failed)
#endif
    for (int un = 0; un < units; ++un) {
        int b = un / G, g = un % G;
        unit_buffers u;
        double **rows = (double **)malloc((size_t)s->c_h * s->c_q * sizeof(double *));
        double *zero_row = (double *)calloc((size_t)s->T, sizeof(double));
        if (!alloc_unit(s, &u) || !rows || !zero_row) {
            failed |= 1; free_unit(&u); free(rows); free(zero_row); continue;
        }
        for (int i = 0; i < s->T; ++i) {
            for (int hh = 0; hh < s->c_h; ++hh) {
                double *base = u.ring + (size_t)hh * s->c_q * s->T;
                /* the new row i takes the ring slot of row i - c_q */
                masked0_logit_row(s, &a, b, g * s->c_h + hh, i, base + (size_t)(i % s->c_q) * s->T);
                for (int ip = 0; ip < s->c_q; ++ip) {
                    int r = i - ip;
                    rows[(size_t)hh * s->c_q + ip] =
                        (r < 0) ? zero_row : base + (size_t)(r % s->c_q) * s->T;
                }
            }
            group_row(s, &a, b, g, i, &u, rows, out + ((size_t)b * s->T + i) * HD, NULL);
        }
        free_unit(&u);
        free(rows);
        free(zero_row);
    }
    return failed ? -2 : 0;
}

/* Output rows of one batch entry, each computed from scratch: for every
 * requested query row rows_idx[n], out_rows[n][H*d] receives out[b][i][*].
 * Used to check large problems at sampled positions. */
static int rows_args(const mta_oracle_shape *s, const mta_oracle_args *pa, int b,
                     const int *rows_idx, int nrows, double *out_rows, int nthreads)
{
    if (!shape_ok(s) || !pa->q || !pa->k || !pa->v || !pa->w_kq || !pa->w_head ||
        !pa->gn_weight || !pa->gn_bias || !out_rows || !rows_idx || b < 0 || b >= s->B ||
        nrows < 0)
        return -1;
    for (int n = 0; n < nrows; ++n)
        if (rows_idx[n] < 0 || rows_idx[n] >= s->T) return -1;
    const mta_oracle_args a = *pa;
    const int G = s->H / s->c_h;
    const size_t HD = (size_t)s->H * s->d;
    const int tasks = nrows * G;
    int failed = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1) reduction(|:failed)
#endif
    for (int t = 0; t < tasks; ++t) {
        int n = t / G, g = t % G;
        unit_buffers u;
        double **rows = (double **)malloc((size_t)s->c_h * s->c_q * sizeof(double *));
        double *zero_row = (double *)calloc((size_t)s->T, sizeof(double));
        if (!alloc_unit(s, &u) || !rows || !zero_row) {
            failed |= 1; free_unit(&u); free(rows); free(zero_row); continue;
        }
        fresh_rows(s, &a, b, g, rows_idx[n], &u, zero_row, rows);
        group_row(s, &a, b, g, rows_idx[n], &u, rows, out_rows + (size_t)n * HD, NULL);
        free_unit(&u);
        free(rows);
        free(zero_row);
    }
    return failed ? -2 : 0;
}

int mta_oracle_forward(const mta_oracle_shape *s, const double *q, const double *k,
                       const double *v, const double *w_kq, const double *w_head,
                       const double *gn_weight, const double *gn_bias,
                       double depth_scale, double *out, int nthreads)
{
    mta_oracle_args a = {q, k, v, w_kq, w_head, gn_weight, gn_bias, depth_scale, NULL};
    return forward_args(s, &a, out, nthreads);
}

/* The same forward with the [GATE] scale: out head h is multiplied by
 * sigmoid(gate[h]) instead of a depth scale. */
int mta_oracle_forward_gated(const mta_oracle_shape *s, const double *q, const double *k,
                             const double *v, const double *w_kq, const double *w_head,
                             const double *gn_weight, const double *gn_bias,
                             const double *gate, double *out, int nthreads)
{
    if (!gate) return -1;
    mta_oracle_args a = {q, k, v, w_kq, w_head, gn_weight, gn_bias, 0.0, gate};
    return forward_args(s, &a, out, nthreads);
}

int mta_oracle_rows(const mta_oracle_shape *s, const double *q, const double *k,
                    const double *v, const double *w_kq, const double *w_head,
                    const double *gn_weight, const double *gn_bias,
                    double depth_scale, int b, const int *rows_idx, int nrows,
                    double *out_rows, int nthreads)
{
    mta_oracle_args a = {q, k, v, w_kq, w_head, gn_weight, gn_bias, depth_scale, NULL};
    return rows_args(s, &a, b, rows_idx, nrows, out_rows, nthreads);
}

int mta_oracle_rows_gated(const mta_oracle_shape *s, const double *q, const double *k,
                          const double *v, const double *w_kq, const double *w_head,
                          const double *gn_weight, const double *gn_bias,
                          const double *gate, int b, const int *rows_idx, int nrows,
                          double *out_rows, int nthreads)
{
    if (!gate) return -1;
    mta_oracle_args a = {q, k, v, w_kq, w_head, gn_weight, gn_bias, 0.0, gate};
    return rows_args(s, &a, b, rows_idx, nrows, out_rows, nthreads);
}

/* Intermediates of one batch entry for small T; any output may be NULL:
 *   C   [H][T][T]  conv logits after both masks of [KQ5] (-inf above the diagonal)
 *   P   [H][T][T]  pre-mix softmax probabilities
 *   A   [H][T][T]  post-mix attention [HM7]
 *   O   [H][T][d]  pre-normalisation head outputs A^h V^h
 *   out [T][H*d]   final output of this batch entry */
int mta_oracle_stages(const mta_oracle_shape *s, const double *q, const double *k,
                      const double *v, const double *w_kq, const double *w_head,
                      const double *gn_weight, const double *gn_bias,
                      double depth_scale, int b, double *C, double *P, double *A,
                      double *O, double *out)
{
    if (!shape_ok(s) || !q || !k || !v || !w_kq || !w_head || !gn_weight || !gn_bias ||
        b < 0 || b >= s->B)
        return -1;
    mta_oracle_args a = {q, k, v, w_kq, w_head, gn_weight, gn_bias, depth_scale, NULL};
    const int T = s->T, d = s->d, c_h = s->c_h, c_q = s->c_q, H = s->H;
    const int G = H / c_h;
    const size_t HD = (size_t)H * d;
    unit_buffers u;
    double **rows = (double **)malloc((size_t)c_h * c_q * sizeof(double *));
    double *zero_row = (double *)calloc((size_t)T, sizeof(double));
    double *tC = (double *)malloc((size_t)c_h * T * sizeof(double));
    double *tP = (double *)malloc((size_t)c_h * T * sizeof(double));
    double *tA = (double *)malloc((size_t)c_h * T * sizeof(double));
    double *tO = (double *)malloc((size_t)c_h * d * sizeof(double));
    int ok = alloc_unit(s, &u) && rows && zero_row && tC && tP && tA && tO;
    if (ok) {
        for (int g = 0; g < G; ++g) {
            for (int i = 0; i < T; ++i) {
                fresh_rows(s, &a, b, g, i, &u, zero_row, rows);
                row_taps taps = {tC, tP, tA, tO};
                group_row(s, &a, b, g, i, &u, rows, out ? out + (size_t)i * HD : NULL, &taps);
                for (int hh = 0; hh < c_h; ++hh) {
                    int h = g * c_h + hh;
                    size_t off = ((size_t)h * T + i) * T;
                    if (C) memcpy(C + off, tC + (size_t)hh * T, T * sizeof(double));
                    if (P) memcpy(P + off, tP + (size_t)hh * T, T * sizeof(double));
                    if (A) memcpy(A + off, tA + (size_t)hh * T, T * sizeof(double));
                    if (O) memcpy(O + ((size_t)h * T + i) * d, tO + (size_t)hh * d, d * sizeof(double));
                }
            }
        }
    }
    free_unit(&u); free(rows); free(zero_row); free(tC); free(tP); free(tA); free(tO);
    return ok ? 0 : -2;
}

int mta_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
