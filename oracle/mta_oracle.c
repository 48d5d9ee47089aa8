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
 *   [POST] "Multi-Token Attention -- Paper Graph", "Key-Query Convolution",
 *          the post-softmax variant: Mask_0(Conv2d_theta(Softmax(
 *          Mask_-inf(A^)))), the same convolution (index ranges of Eq. (4))
 *          applied to the attention probabilities, future entries zeroed.
 *   [FULL] same page, "Putting Everything Together: The Full MTA Module":
 *          the compositions of the two convolutions around the softmax and
 *          the repeat of the MTA convolution (key-query, then head) after it;
 *          "both pre-softmax" is the key-query conv followed by [HMPRE], the
 *          separable case of the 3-D convolution over (query, key, head).
 *   [HMPRE] same page, "Head Mixing Convolution", pre-softmax version: the
 *          logits of a group's heads are mixed, A^h_new = sum_h' w A^h'.
 *   [CONV3D] same page, "Putting Everything Together", "Both pre-softmax
 *          (3D convolution view)": one kernel over (query, key, head) per
 *          group, C^h[i][j] = sum_{h' in group} sum_{i',j'}
 *          theta3[h][h'][i'][j'] A0^{h'}[i-i'][j-j'].
 *   [EXACT] same page, Eq. (4): the tap (i', j') of output (i, j) adds
 *          theta q_{i-i'} k_{j-j'}^T / sqrt(d) whenever key j - j' <= i (the
 *          indicator 1_{i >= j-j'}), which Eq. (5)'s two-pass masking
 *          narrows to j - j' <= i - i'.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - taps that fall outside [0,T) x [0,T) read zero (zero padding);
 *   - w_head is stored [group][out head][in head];
 *   - GroupNorm uses the biased variance and eps inside the square root,
 *     with a per-channel affine (gamma, beta) over the H*d concatenation;
 *   - depth scaling is a caller-supplied scalar multiplying the GN output;
 *   - the sigmoid gate multiplies the GN output (after its affine) in place
 *     of the depth scale.
 *   - a composition runs the steps in one fixed order, each bracketed step
 *     optional: Mask_0 -> [key-query conv] -> [head mix of the logits] ->
 *     Mask_-inf -> softmax -> [head mix] -> [key-query conv -> Mask_0] ->
 *     [head mix] -> A V -> GN; with [EXACT] the first conv reads the
 *     unmasked logits under the indicator instead of Mask_0's zeros;
 *     the pages' default has the first two, the repeat all four, and "both
 *     post-softmax" the last two; both key-query kernels are c_q x c_k.
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
    const double *q, *k, *v;
    const double *w_kq;        /* key-query kernel before the softmax, or NULL */
    const double *w_head_pre;  /* head mix of the logits before the softmax, or NULL */
    int exact;                 /* [EXACT] masking of the first conv instead of [KQ5] */
    const double *w_kq_3d;     /* [CONV3D] kernel in place of w_kq, or NULL */
    const double *w_head;      /* head mix right after the softmax, or NULL */
    const double *w_kq_post;   /* key-query kernel on the probabilities, or NULL */
    const double *w_head_post; /* head mix after w_kq_post, or NULL */
    const double *gn_weight, *gn_bias;
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
 * columns outside [0,T) are zero padding.  Fills out[0..T).  Under [EXACT]
 * the row also keeps the logits of the c_q - 1 keys after r, which the taps
 * of the next queries may use (every later key is left out by the
 * indicator). */
static void masked0_logit_row(const mta_oracle_shape *s, const mta_oracle_args *a,
                              int b, int h, int r, double *out)
{
    const int T = s->T, d = s->d;
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    for (int c = 0; c < T; ++c) out[c] = 0.0;
    if (r < 0 || r >= T) return;
    const double *qr = row_of(a->q, s, b, h, r);
    const int last = a->exact ? r + s->c_q - 1 : r;
    for (int c = 0; c <= last && c < T; ++c) {
        const double *kc = row_of(a->k, s, b, h, c);
        double dot = 0.0;
        for (int e = 0; e < d; ++e) dot += qr[e] * kc[e];
        out[c] = dot * inv_sqrt_d;
    }
}

/* [KQ4]: out[j] = sum_{i'} sum_{j'} theta[i'][j'] X[i-i'][j-j'] for j in
 * [0, i], and out[j] = fill for j > i: -inf is the second mask of [KQ5]
 * (ahead of a softmax), 0 the Mask_0 of [POST] (after one).  rows[i'] holds
 * the row X[i - i'][*]; X is zero outside [0,T) x [0,T) (zero padding).
 * With exact != 0 a tap reading key c > i is left out ([EXACT]). */
static void conv2d_row(const mta_oracle_shape *s, const double *theta, int i,
                       double *const *rows, int exact, double fill, double *out)
{
    const int T = s->T, c_q = s->c_q, c_k = s->c_k;
    const int jlo = -(c_k / 2);               /* -floor(c_k/2)    */
    const int jhi = (c_k + 1) / 2 - 1;        /*  ceil(c_k/2) - 1 */
    for (int j = 0; j < T; ++j) {
        if (j > i) { out[j] = fill; continue; }
        double acc = 0.0;
        for (int ip = 0; ip < c_q; ++ip) {
            if (i - ip < 0) continue;          /* zero row above the sequence */
            for (int jp = jlo; jp <= jhi; ++jp) {
                int c = j - jp;
                if (c < 0 || c >= T) continue; /* zero padding */
                if (exact && c > i) continue;  /* the indicator 1_{i >= j - j'} */
                acc += theta[ip * c_k + (jp - jlo)] * rows[ip][c];
            }
        }
        out[j] = acc;
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

/* [HM7] over the c_h heads of one group: out[ho][j] = sum_{hi} wg[ho][hi]
 * in[hi][j], in and out [c_h][T]; wg == NULL means no mixing (a copy). */
static void head_mix(int c_h, int T, const double *wg, const double *in, double *out)
{
    for (int ho = 0; ho < c_h; ++ho)
        for (int j = 0; j < T; ++j) {
            if (!wg) { out[(size_t)ho * T + j] = in[(size_t)ho * T + j]; continue; }
            double acc = 0.0;
            for (int hi = 0; hi < c_h; ++hi) acc += wg[ho * c_h + hi] * in[(size_t)hi * T + j];
            out[(size_t)ho * T + j] = acc;
        }
}

/* [HMPRE] on the logits of query row r: out[ho][j] = sum_{hi} wg[ho][hi]
 * in[hi][j] for the keys j <= r; later keys stay -inf (the second mask of
 * [KQ5]).  in and out are [c_h][T]. */
static void logit_mix(int c_h, int T, int r, const double *wg, const double *in, double *out)
{
    for (int ho = 0; ho < c_h; ++ho) {
        const double *wrow = wg + (size_t)ho * c_h;   /* output head ho's weights */
        for (int j = 0; j < T; ++j) {
            if (j > r) { out[(size_t)ho * T + j] = -INFINITY; continue; }
            double acc = 0.0;
            for (int hi = 0; hi < c_h; ++hi) acc += wrow[hi] * in[(size_t)hi * T + j];
            out[(size_t)ho * T + j] = acc;
        }
    }
}

/* [MHA] O = A V over the keys j <= i of head h (A is zero on later keys),
 * then [GN] on O with the [GATE] or depth scale into out_row[h*d ..
 * h*d + d) when out_row != NULL. */
static void pv_groupnorm_row(const mta_oracle_shape *s, const mta_oracle_args *a, int b,
                             int h, int i, const double *A, double *O, double *out_row)
{
    const int d = s->d;
    for (int e = 0; e < d; ++e) O[e] = 0.0;
    for (int j = 0; j <= i; ++j) {
        const double *vj = row_of(a->v, s, b, h, j);
        for (int e = 0; e < d; ++e) O[e] += A[j] * vj[e];
    }
    if (!out_row) return;
    /* [GN]: the head's d-vector is one group; biased variance. */
    double mean = 0.0;
    for (int e = 0; e < d; ++e) mean += O[e];
    mean /= d;
    double var = 0.0;
    for (int e = 0; e < d; ++e) var += (O[e] - mean) * (O[e] - mean);
    var /= d;
    double inv = 1.0 / sqrt(var + s->gn_eps);
    /* [GATE] sigmoid(g_h), or the depth scale */
    double scale = a->gate ? 1.0 / (1.0 + exp(-a->gate[h])) : a->depth_scale;
    for (int e = 0; e < d; ++e) {
        size_t chn = (size_t)h * d + e;
        double y = (O[e] - mean) * inv * a->gn_weight[chn] + a->gn_bias[chn];
        out_row[chn] = scale * y;
    }
}

/* Work buffers for one (batch, head group) unit. */
typedef struct {
    double *ring0;  /* [c_h][c_q][T] masked logit rows A0, a ring over the query index */
    double *ring1;  /* [c_h][c_q][T] first-stage attention rows A1, the same ring */
    double *C;      /* [c_h][T] softmax inputs before the logit mix */
    double *Cm;     /* [c_h][T] after the logit mix [HMPRE] */
    double *Ct;     /* [T] one input head's conv under [CONV3D] */
    double *P;      /* [c_h][T] softmax rows of the group's heads */
    double *A1;     /* [c_h][T] first-stage rows (after the first head mix) */
    double *A2;     /* [c_h][T] after the post-softmax key-query conv */
    double *A3;     /* [c_h][T] after the second head mix: the rows that meet V */
    double *O;      /* [d] */
    double *zero;   /* [T] the zero row above the sequence */
    double **rows0; /* [c_h * c_q] row pointers into ring0 */
    double **rows1; /* [c_h * c_q] row pointers into ring1 */
} unit_buffers;

static int alloc_unit(const mta_oracle_shape *s, unit_buffers *u)
{
    size_t T = (size_t)s->T, hq = (size_t)s->c_h * s->c_q, hT = (size_t)s->c_h * T;
    u->ring0 = (double *)calloc(hq * T, sizeof(double));
    u->ring1 = (double *)calloc(hq * T, sizeof(double));
    u->C = (double *)malloc(hT * sizeof(double));
    u->Cm = (double *)malloc(hT * sizeof(double));
    u->Ct = (double *)malloc(T * sizeof(double));
    u->P = (double *)malloc(hT * sizeof(double));
    u->A1 = (double *)malloc(hT * sizeof(double));
    u->A2 = (double *)malloc(hT * sizeof(double));
    u->A3 = (double *)malloc(hT * sizeof(double));
    u->O = (double *)malloc((size_t)s->d * sizeof(double));
    u->zero = (double *)calloc(T, sizeof(double));
    u->rows0 = (double **)malloc(hq * sizeof(double *));
    u->rows1 = (double **)malloc(hq * sizeof(double *));
    return u->ring0 && u->ring1 && u->C && u->Cm && u->Ct && u->P && u->A1 && u->A2 && u->A3 && u->O &&
           u->zero && u->rows0 && u->rows1;
}

static void free_unit(unit_buffers *u)
{
    free(u->ring0); free(u->ring1); free(u->C); free(u->Cm); free(u->Ct); free(u->P); free(u->A1); free(u->A2);
    free(u->A3); free(u->O); free(u->zero); free(u->rows0); free(u->rows1);
}

/* Optional per-row intermediates of one group (each [c_h][T] or [c_h][d]);
 * any may be NULL. */
typedef struct {
    double *C;      /* logits that enter the softmax, both masks applied */
    double *P;      /* softmax rows */
    double *A1;     /* first-stage rows, after the first head mix */
    double *A;      /* the attention rows that meet V */
    double *O;      /* pre-normalisation head outputs A^h V^h, [c_h][d] */
} row_taps;

/* Query row r of group g up to the first head mix.  rows0[hh*c_q + ip] is
 * A0[r - ip] of head g*c_h + hh.  [KQ5] per head: the key-query conv with
 * w_kq, or the [CONV3D] kernel over the group's heads, when given (else
 * A0[r] itself) and Mask_-inf; [HMPRE] with
 * w_head_pre when given; softmax; then [HM7] with w_head when given.
 * Leaves the group's rows in u->A1. */
static void first_stage(const mta_oracle_shape *s, const mta_oracle_args *a, int g, int r,
                        unit_buffers *u, double *const *rows0, row_taps *taps)
{
    const int T = s->T, c_h = s->c_h, c_q = s->c_q, c_k = s->c_k;
    for (int hh = 0; hh < c_h; ++hh) {
        int h = g * c_h + hh;
        double *const *rows = rows0 + (size_t)hh * c_q;
        double *C = u->C + (size_t)hh * T;
        if (a->w_kq_3d) {
            for (int j = 0; j < T; ++j) C[j] = (j <= r) ? 0.0 : -INFINITY;
            for (int hi = 0; hi < c_h; ++hi) {      /* every input head of the group */
                const double *th3 = a->w_kq_3d + ((size_t)h * c_h + hi) * c_q * c_k;
                conv2d_row(s, th3, r, rows0 + (size_t)hi * c_q, a->exact, -INFINITY, u->Ct);
                for (int j = 0; j <= r && j < T; ++j) C[j] += u->Ct[j];
            }
        } else if (a->w_kq)
            conv2d_row(s, a->w_kq + (size_t)h * c_q * c_k, r, rows, a->exact, -INFINITY, C);
        else
            for (int j = 0; j < T; ++j) C[j] = (j <= r) ? rows[0][j] : -INFINITY;
    }
    const double *logits = u->C;
    if (a->w_head_pre) {
        logit_mix(c_h, T, r, a->w_head_pre + (size_t)g * c_h * c_h, u->C, u->Cm);
        logits = u->Cm;
    }
    for (int hh = 0; hh < c_h; ++hh)
        softmax_row(T, logits + (size_t)hh * T, u->P + (size_t)hh * T);
    if (taps && taps->C) memcpy(taps->C, logits, (size_t)c_h * T * sizeof(double));
    head_mix(c_h, T, a->w_head ? a->w_head + (size_t)g * c_h * c_h : NULL, u->P, u->A1);
    if (taps && taps->P) memcpy(taps->P, u->P, (size_t)c_h * T * sizeof(double));
    if (taps && taps->A1) memcpy(taps->A1, u->A1, (size_t)c_h * T * sizeof(double));
}

/* Query row i of group g of batch entry b from the first-stage rows on:
 * rows1[hh*c_q + ip] is A1[i - ip] of head g*c_h + hh.  [POST] per head:
 * the key-query conv with w_kq_post when given, future keys zero (else
 * A1[i] itself); [HM7] with w_head_post when given; then per output head
 * A V and [GN] into out_row (the [H*d] output row of (b, i)) when given. */
static void second_stage(const mta_oracle_shape *s, const mta_oracle_args *a, int b, int g,
                         int i, unit_buffers *u, double *const *rows1, double *out_row,
                         row_taps *taps)
{
    const int T = s->T, d = s->d, c_h = s->c_h, c_q = s->c_q, c_k = s->c_k;
    for (int hh = 0; hh < c_h; ++hh) {
        int h = g * c_h + hh;
        double *const *rows = rows1 + (size_t)hh * c_q;
        if (a->w_kq_post)
            conv2d_row(s, a->w_kq_post + (size_t)h * c_q * c_k, i, rows, 0, 0.0,
                       u->A2 + (size_t)hh * T);
        else
            memcpy(u->A2 + (size_t)hh * T, rows[0], T * sizeof(double));
    }
    head_mix(c_h, T, a->w_head_post ? a->w_head_post + (size_t)g * c_h * c_h : NULL, u->A2,
             u->A3);
    for (int ho = 0; ho < c_h; ++ho) {
        int h = g * c_h + ho;
        pv_groupnorm_row(s, a, b, h, i, u->A3 + (size_t)ho * T, u->O, out_row);
        if (taps && taps->A) memcpy(taps->A + (size_t)ho * T, u->A3 + (size_t)ho * T, T * sizeof(double));
        if (taps && taps->O) memcpy(taps->O + (size_t)ho * d, u->O, d * sizeof(double));
    }
}

/* rows[hh*c_q + ip] = row i - ip of head hh in a [c_h][c_q][T] ring indexed
 * by the row number modulo c_q, or the zero row above the sequence. */
static void point_rows(const mta_oracle_shape *s, double *ring, int i, double *zero,
                       double **rows)
{
    for (int hh = 0; hh < s->c_h; ++hh)
        for (int ip = 0; ip < s->c_q; ++ip) {
            int r = i - ip;
            rows[(size_t)hh * s->c_q + ip] =
                (r < 0) ? zero : ring + ((size_t)hh * s->c_q + (r % s->c_q)) * s->T;
        }
}

/* Query row i of (b, g) from scratch: the first-stage rows A1[i - ip] for
 * ip < c_q (only ip = 0 without a post-softmax conv), each from freshly
 * computed masked logit rows; then the second stage.  Taps are those of
 * row i. */
static void fresh_row(const mta_oracle_shape *s, const mta_oracle_args *a, int b, int g, int i,
                      unit_buffers *u, double *out_row, row_taps *taps)
{
    const int T = s->T, c_h = s->c_h, c_q = s->c_q;
    const int needed = a->w_kq_post ? c_q : 1;
    for (int ip = 0; ip < c_q; ++ip) {
        const int r = i - ip;
        for (int hh = 0; hh < c_h; ++hh) u->rows1[(size_t)hh * c_q + ip] = u->zero;
        if (ip >= needed || r < 0) continue;
        for (int hh = 0; hh < c_h; ++hh)
            for (int ip2 = 0; ip2 < c_q; ++ip2) {
                double *slot = u->ring0 + ((size_t)hh * c_q + ip2) * T;
                masked0_logit_row(s, a, b, g * c_h + hh, r - ip2, slot);
                u->rows0[(size_t)hh * c_q + ip2] = slot;
            }
        first_stage(s, a, g, r, u, u->rows0, ip == 0 ? taps : NULL);
        for (int hh = 0; hh < c_h; ++hh) {
            double *slot = u->ring1 + ((size_t)hh * c_q + ip) * T;
            memcpy(slot, u->A1 + (size_t)hh * T, T * sizeof(double));
            u->rows1[(size_t)hh * c_q + ip] = slot;
        }
    }
    second_stage(s, a, b, g, i, u, u->rows1, out_row, taps);
}

static int args_ok(const mta_oracle_shape *s, const mta_oracle_args *a)
{
    return shape_ok(s) && a->q && a->k && a->v && a->gn_weight && a->gn_bias;
}

/* Rows per task of the full forward: 0 picks a size from the thread count;
 * a positive value forces it (the tests use that to show that the split does
 * not change a single bit). */
static int g_row_chunk = 0;

/* Full forward: out[B][T][H*d].  Units (b, g) are independent; inside a unit
 * the query rows run in order, keeping the last c_q masked logit rows and
 * first-stage rows of each head in rings.  When there are fewer units than
 * threads, each unit's rows are also split into chunks run as separate
 * tasks: a chunk first recomputes the 2 (c_q - 1) rows before it, which
 * refills both rings with exactly the values the unsplit loop would hold
 * (every masked logit row is computed on its own from q and k), and writes
 * output only from its first row on.  Returns 0 on success. */
static int forward_args(const mta_oracle_shape *s, const mta_oracle_args *pa, double *out,
                        int nthreads)
{
    if (!args_ok(s, pa) || !out) return -1;
    const mta_oracle_args a = *pa;
    const int G = s->H / s->c_h;
    const int units = s->B * G;
    const size_t HD = (size_t)s->H * s->d;
    int threads = 1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
    threads = omp_get_max_threads();
#endif
    int chunk = s->T;
    if (g_row_chunk > 0)
        chunk = g_row_chunk;
    else if (units < 4 * threads) {
        const int per_unit = (4 * threads + units - 1) / units;
        chunk = (s->T + per_unit - 1) / per_unit;
        if (chunk < 256) chunk = 256;
    }
    const int nchunks = (s->T + chunk - 1) / chunk;
    const int warm = 2 * (s->c_q - 1);
    int failed = 0;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) reduction(|:failed)
#endif
    for (int task = 0; task < units * nchunks; ++task) {
        /* later chunks cost more (causal rows grow): start with them */
        const int un = task % units, ch = nchunks - 1 - task / units;
        const int b = un / G, g = un % G;
        const int first = ch * chunk;
        const int last = first + chunk < s->T ? first + chunk : s->T;
        unit_buffers u;
        if (!alloc_unit(s, &u)) { failed |= 1; free_unit(&u); continue; }
        const size_t T = (size_t)s->T;
        for (int i = first - warm > 0 ? first - warm : 0; i < last; ++i) {
            /* the new rows i take the ring slots of rows i - c_q */
            const size_t slot = (size_t)(i % s->c_q);
            for (int hh = 0; hh < s->c_h; ++hh)
                masked0_logit_row(s, &a, b, g * s->c_h + hh, i,
                                  u.ring0 + ((size_t)hh * s->c_q + slot) * T);
            point_rows(s, u.ring0, i, u.zero, u.rows0);
            first_stage(s, &a, g, i, &u, u.rows0, NULL);
            for (int hh = 0; hh < s->c_h; ++hh)
                memcpy(u.ring1 + ((size_t)hh * s->c_q + slot) * T, u.A1 + (size_t)hh * T,
                       T * sizeof(double));
            if (i < first) continue;   /* warm-up row: rings only */
            point_rows(s, u.ring1, i, u.zero, u.rows1);
            second_stage(s, &a, b, g, i, &u, u.rows1, out + ((size_t)b * s->T + i) * HD, NULL);
        }
        free_unit(&u);
    }
    return failed ? -2 : 0;
}

/* Output rows of one batch entry, each computed from scratch: for every
 * requested query row rows_idx[n], out_rows[n][H*d] receives out[b][i][*].
 * Used to check large problems at sampled positions. */
static int rows_args(const mta_oracle_shape *s, const mta_oracle_args *pa, int b,
                     const int *rows_idx, int nrows, double *out_rows, int nthreads)
{
    if (!args_ok(s, pa) || !out_rows || !rows_idx || b < 0 || b >= s->B || nrows < 0)
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
        if (!alloc_unit(s, &u)) { failed |= 1; free_unit(&u); continue; }
        fresh_row(s, &a, b, g, rows_idx[n], &u, out_rows + (size_t)n * HD, NULL);
        free_unit(&u);
    }
    return failed ? -2 : 0;
}

/* Intermediates of batch entry b (small T), any output may be NULL; each
 * map is [H][T][T], O is [H][T][d], out is [T][H*d] (see row_taps). */
static int stages_args(const mta_oracle_shape *s, const mta_oracle_args *pa, int b, double *C,
                       double *P, double *A1, double *A, double *O, double *out)
{
    if (!args_ok(s, pa) || b < 0 || b >= s->B) return -1;
    const int T = s->T, d = s->d, c_h = s->c_h, H = s->H;
    const int G = H / c_h;
    const size_t HD = (size_t)H * d;
    unit_buffers u;
    double *tC = (double *)malloc((size_t)c_h * T * sizeof(double));
    double *tP = (double *)malloc((size_t)c_h * T * sizeof(double));
    double *tA1 = (double *)malloc((size_t)c_h * T * sizeof(double));
    double *tA = (double *)malloc((size_t)c_h * T * sizeof(double));
    double *tO = (double *)malloc((size_t)c_h * d * sizeof(double));
    int ok = alloc_unit(s, &u) && tC && tP && tA1 && tA && tO;
    if (ok) {
        for (int g = 0; g < G; ++g) {
            for (int i = 0; i < T; ++i) {
                row_taps taps = {tC, tP, tA1, tA, tO};
                fresh_row(s, pa, b, g, i, &u, out ? out + (size_t)i * HD : NULL, &taps);
                for (int hh = 0; hh < c_h; ++hh) {
                    int h = g * c_h + hh;
                    size_t off = ((size_t)h * T + i) * T, src = (size_t)hh * T;
                    if (C) memcpy(C + off, tC + src, T * sizeof(double));
                    if (P) memcpy(P + off, tP + src, T * sizeof(double));
                    if (A1) memcpy(A1 + off, tA1 + src, T * sizeof(double));
                    if (A) memcpy(A + off, tA + src, T * sizeof(double));
                    if (O) memcpy(O + ((size_t)h * T + i) * d, tO + (size_t)hh * d, d * sizeof(double));
                }
            }
        }
    }
    free_unit(&u); free(tC); free(tP); free(tA1); free(tA); free(tO);
    return ok ? 0 : -2;
}

/* The pages' default composition ([KQ5] then [HM7]). */
static mta_oracle_args default_args(const double *q, const double *k, const double *v,
                                    const double *w_kq, const double *w_head,
                                    const double *gn_weight, const double *gn_bias,
                                    double depth_scale, const double *gate)
{
    mta_oracle_args a = {0};
    a.q = q; a.k = k; a.v = v; a.w_kq = w_kq; a.w_head = w_head;
    a.gn_weight = gn_weight; a.gn_bias = gn_bias; a.depth_scale = depth_scale; a.gate = gate;
    return a;
}

/* A composition of [FULL]: each weight may be NULL (that step is left out). */
typedef struct {
    const double *w_kq;        /* [H][c_q][c_k] key-query conv before the softmax */
    const double *w_head_pre;  /* [H/c_h][c_h][c_h] [HMPRE] mix of the logits */
    const double *w_head;      /* [H/c_h][c_h][c_h] [HM7] mix after the softmax */
    const double *w_kq_post;   /* [H][c_q][c_k] [POST] conv of the probabilities */
    const double *w_head_post; /* [H/c_h][c_h][c_h] [HM7] mix after w_kq_post */
    int exact_mask;            /* nonzero: [EXACT] masking of the w_kq conv */
    const double *w_kq_3d;     /* [H/c_h][c_h][c_h][c_q][c_k] [CONV3D] kernel, in place
                                  of w_kq (giving both is an error) */
} mta_oracle_composition;

static mta_oracle_args composed_args(const double *q, const double *k, const double *v,
                                     const mta_oracle_composition *c,
                                     const double *gn_weight, const double *gn_bias,
                                     double depth_scale, const double *gate)
{
    mta_oracle_args a = default_args(q, k, v, c->w_kq, c->w_head, gn_weight, gn_bias,
                                     depth_scale, gate);
    a.w_head_pre = c->w_head_pre;
    a.exact = c->exact_mask != 0;
    a.w_kq_post = c->w_kq_post;
    a.w_head_post = c->w_head_post;
    a.w_kq_3d = c->w_kq_3d;
    return a;
}

int mta_oracle_forward(const mta_oracle_shape *s, const double *q, const double *k,
                       const double *v, const double *w_kq, const double *w_head,
                       const double *gn_weight, const double *gn_bias,
                       double depth_scale, double *out, int nthreads)
{
    if (!w_kq || !w_head) return -1;
    mta_oracle_args a = default_args(q, k, v, w_kq, w_head, gn_weight, gn_bias, depth_scale, NULL);
    return forward_args(s, &a, out, nthreads);
}

/* The same forward with the [GATE] scale: out head h is multiplied by
 * sigmoid(gate[h]) instead of a depth scale. */
int mta_oracle_forward_gated(const mta_oracle_shape *s, const double *q, const double *k,
                             const double *v, const double *w_kq, const double *w_head,
                             const double *gn_weight, const double *gn_bias,
                             const double *gate, double *out, int nthreads)
{
    if (!w_kq || !w_head || !gate) return -1;
    mta_oracle_args a = default_args(q, k, v, w_kq, w_head, gn_weight, gn_bias, 0.0, gate);
    return forward_args(s, &a, out, nthreads);
}

/* [FULL]: the composition *c; gate may be NULL (depth scale). */
int mta_oracle_forward_composed(const mta_oracle_shape *s, const double *q, const double *k,
                                const double *v, const mta_oracle_composition *c,
                                const double *gn_weight, const double *gn_bias,
                                double depth_scale, const double *gate, double *out,
                                int nthreads)
{
    if (!c || (c->w_kq && c->w_kq_3d)) return -1;
    mta_oracle_args a = composed_args(q, k, v, c, gn_weight, gn_bias, depth_scale, gate);
    return forward_args(s, &a, out, nthreads);
}

int mta_oracle_rows(const mta_oracle_shape *s, const double *q, const double *k,
                    const double *v, const double *w_kq, const double *w_head,
                    const double *gn_weight, const double *gn_bias,
                    double depth_scale, int b, const int *rows_idx, int nrows,
                    double *out_rows, int nthreads)
{
    if (!w_kq || !w_head) return -1;
    mta_oracle_args a = default_args(q, k, v, w_kq, w_head, gn_weight, gn_bias, depth_scale, NULL);
    return rows_args(s, &a, b, rows_idx, nrows, out_rows, nthreads);
}

int mta_oracle_rows_gated(const mta_oracle_shape *s, const double *q, const double *k,
                          const double *v, const double *w_kq, const double *w_head,
                          const double *gn_weight, const double *gn_bias,
                          const double *gate, int b, const int *rows_idx, int nrows,
                          double *out_rows, int nthreads)
{
    if (!w_kq || !w_head || !gate) return -1;
    mta_oracle_args a = default_args(q, k, v, w_kq, w_head, gn_weight, gn_bias, 0.0, gate);
    return rows_args(s, &a, b, rows_idx, nrows, out_rows, nthreads);
}

int mta_oracle_rows_composed(const mta_oracle_shape *s, const double *q, const double *k,
                             const double *v, const mta_oracle_composition *c,
                             const double *gn_weight, const double *gn_bias,
                             double depth_scale, const double *gate, int b,
                             const int *rows_idx, int nrows, double *out_rows, int nthreads)
{
    if (!c || (c->w_kq && c->w_kq_3d)) return -1;
    mta_oracle_args a = composed_args(q, k, v, c, gn_weight, gn_bias, depth_scale, gate);
    return rows_args(s, &a, b, rows_idx, nrows, out_rows, nthreads);
}

/* Intermediates of one batch entry of the default composition for small T;
 * any output may be NULL:
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
    if (!w_kq || !w_head) return -1;
    mta_oracle_args a = default_args(q, k, v, w_kq, w_head, gn_weight, gn_bias, depth_scale, NULL);
    return stages_args(s, &a, b, C, P, NULL, A, O, out);
}

/* Intermediates of one batch entry of any composition (small T): as
 * mta_oracle_stages (C is the softmax input, after the logit mix), plus A1
 * [H][T][T] (the rows after the first head mix); A is then the attention
 * that meets V. */
int mta_oracle_stages_composed(const mta_oracle_shape *s, const double *q, const double *k,
                               const double *v, const mta_oracle_composition *c,
                               const double *gn_weight, const double *gn_bias,
                               double depth_scale, const double *gate, int b, double *C,
                               double *P, double *A1, double *A, double *O, double *out)
{
    if (!c || (c->w_kq && c->w_kq_3d)) return -1;
    mta_oracle_args a = composed_args(q, k, v, c, gn_weight, gn_bias, depth_scale, gate);
    return stages_args(s, &a, b, C, P, A1, A, O, out);
}

/* Rows per task of the full forward (0: chosen from the thread count). */
void mta_oracle_set_row_chunk(int rows) { g_row_chunk = rows > 0 ? rows : 0; }

int mta_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
