/*
 * dgrad_oracle.c -- plain, slow fp64 CPU oracle for convolution backward-data.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the checker, not the product: only
 * the test suite, the smoke check and the benchmark's CPU-baseline leg may
 * load it.  It shares no code, header, table or helper with the CUDA library
 * in convolution_backward_b200/csrc, and it includes nothing from there.
 *
 * What it computes.  The pages ("add the pointwise fast path dgrad was
 * missing", Technical Details; "channel-packed and large-filter depthwise
 * dgrad", Technical Details) never write dgrad as a formula; they treat it as
 * the backward-data pass of the forward convolution.  We take the textbook
 * reading: for a forward convolution with dilation 1, stride S, per-axis
 * padding (ph, pw) and g groups (K = g*Kg output channels, C = g*Cg input
 * channels)
 *
 *   y[n,ho,wo,k] = sum_{r<KH, s<KW, cg<Cg} x[n, ho*S-ph+r, wo*S-pw+s, g(k)*Cg+cg]
 *                                          * Wt(k, r, s, cg)        (x = 0 off-image)
 *
 * dgrad is the exact adjoint of that map in x:
 *
 *   dX[n,h,w,c] = sum over (ho,wo,k,r,s) with h = ho*S-ph+r, w = wo*S-pw+s,
 *                 g(k) = c/Cg, cg = c - g(k)*Cg  of  dY[n,ho,wo,k] * Wt(k,r,s,cg).
 *
 * Ho = floor((H + 2*ph - KH)/S) + 1 and Wo = floor((W + 2*pw - KW)/S) + 1, the
 * column count using the column padding ("channel-packed and large-filter
 * depthwise dgrad", Technical Details, per-axis padding: Wo uses PAD_W).
 *
 * The filter is addressed through four strides (k, r, s, cg) so one routine
 * covers both filter layouts of the two cases on the pages:
 *   pointwise  W[K][C]        : Wt(k,0,0,c) = W[k*C + c]   (pointwise page: W offset k*C + c)
 *   depthwise  W[KH][KW][C]   : Wt(c,r,s,0) = W[(r*KW+s)*C + c]  (groups = C = K, Cg = Kg = 1)
 * dY is addressed through four strides (n, ho, wo, k) as well; the tests use a
 * wrong dY pixel stride (K+1 instead of K) to plant a mistake and check that
 * the pins catch it, the same mutation the pointwise page used.
 *
 * Functions (each a separate formulation; the tests pin them to each other and
 * to mathematics, never to the CUDA path):
 *   oracle_dgrad          scatter loop from the adjoint definition above
 *   oracle_dgrad_points   the same definition evaluated per output element (gather form)
 *   oracle_conv_fwd       forward convolution, gather form (for the adjoint identity)
 *   oracle_dw_rotated     stride-1 depthwise dgrad as a forward correlation of dY with
 *                         the 180-degree rotated filter at padding KH-1-ph, KW-1-pw
 *                         (depthwise page, Technical Details, rotated-filter dgrad)
 *   oracle_dw_rowstream   depthwise dgrad by the row-streaming schedule: dY rows stream
 *                         into circular accumulator rows, finished rows are flushed, and a
 *                         tail flushes the rows past the last dY row (depthwise page,
 *                         Technical Details, channel-packed row-streaming dgrad)
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int64_t N, H, W, C, K;       /* x / dX: N,H,W,C ; y / dY: N,Ho,Wo,K */
    int64_t KH, KW, S, ph, pw;   /* filter extents, stride, per-axis padding */
    int64_t groups;              /* g: K = g*Kg, C = g*Cg */
} oracle_geom_t;

enum { ORACLE_OK = 0, ORACLE_BAD = 1 };

static int64_t extent_out(int64_t in, int64_t pad, int64_t k, int64_t s)
{
    int64_t num = in + 2 * pad - k;
    if (num < 0) return 0;
    return num / s + 1;
}

static int check_geom(const oracle_geom_t* g)
{
    if (!g) return ORACLE_BAD;
    if (g->N < 0 || g->H < 1 || g->W < 1 || g->C < 1 || g->K < 1) return ORACLE_BAD;
    if (g->KH < 1 || g->KW < 1 || g->S < 1 || g->ph < 0 || g->pw < 0) return ORACLE_BAD;
    if (g->groups < 1 || g->C % g->groups || g->K % g->groups) return ORACLE_BAD;
    if (extent_out(g->H, g->ph, g->KH, g->S) < 1) return ORACLE_BAD;
    if (extent_out(g->W, g->pw, g->KW, g->S) < 1) return ORACLE_BAD;
    return ORACLE_OK;
}

int oracle_out_dims(const oracle_geom_t* g, int64_t* Ho, int64_t* Wo)
{
    if (check_geom(g)) return ORACLE_BAD;
    *Ho = extent_out(g->H, g->ph, g->KH, g->S);
    *Wo = extent_out(g->W, g->pw, g->KW, g->S);
    return ORACLE_OK;
}

static int g_threads = 0;

void oracle_set_threads(int n) { g_threads = n; }

int oracle_get_threads(void)
{
#ifdef _OPENMP
    return g_threads > 0 ? g_threads : omp_get_max_threads();
#else
    return 1;
#endif
}

/* Scatter form of the adjoint definition: walk every (n, ho, wo, k, r, s, cg)
 * term once and add it into a zeroed fp64 dX.  Parallel over n only: each batch
 * item owns a disjoint slice of dX, so the per-item order is the plain loop
 * order. */
int oracle_dgrad(const oracle_geom_t* g,
                 const double* dy, const int64_t ystr[4],
                 const double* wt, const int64_t wstr[4],
                 double* dx)
{
    if (check_geom(g) || !dy || !wt || !dx || !ystr || !wstr) return ORACLE_BAD;
    const int64_t Ho = extent_out(g->H, g->ph, g->KH, g->S);
    const int64_t Wo = extent_out(g->W, g->pw, g->KW, g->S);
    const int64_t Kg = g->K / g->groups, Cg = g->C / g->groups;
    const int64_t H = g->H, W = g->W, C = g->C;
    memset(dx, 0, sizeof(double) * (size_t)(g->N * H * W * C));
    int nt = oracle_get_threads();
    (void)nt;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (int64_t n = 0; n < g->N; ++n) {
        double* dxn = dx + n * H * W * C;
        for (int64_t ho = 0; ho < Ho; ++ho)
        for (int64_t wo = 0; wo < Wo; ++wo)
        for (int64_t k = 0; k < g->K; ++k) {
            const double v = dy[n * ystr[0] + ho * ystr[1] + wo * ystr[2] + k * ystr[3]];
            const int64_t grp = k / Kg;
            for (int64_t r = 0; r < g->KH; ++r) {
                const int64_t h = ho * g->S - g->ph + r;
                if (h < 0 || h >= H) continue;
                for (int64_t s = 0; s < g->KW; ++s) {
                    const int64_t w = wo * g->S - g->pw + s;
                    if (w < 0 || w >= W) continue;
                    for (int64_t cg = 0; cg < Cg; ++cg) {
                        const double f = wt[k * wstr[0] + r * wstr[1] + s * wstr[2] + cg * wstr[3]];
                        dxn[(h * W + w) * C + grp * Cg + cg] += v * f;
                    }
                }
            }
        }
    }
    return ORACLE_OK;
}

/* Gather form of the same definition, one output element at a time:
 *   dX[n,h,w,c] = sum_{k in group(c)} sum_{r,s : (h+ph-r) = ho*S, (w+pw-s) = wo*S,
 *                 0<=ho<Ho, 0<=wo<Wo} dY[n,ho,wo,k] * Wt(k,r,s,c-g(c)*Cg).
 * pts holds npts quadruples (n,h,w,c). */
int oracle_dgrad_points(const oracle_geom_t* g,
                        const double* dy, const int64_t ystr[4],
                        const double* wt, const int64_t wstr[4],
                        const int64_t* pts, int64_t npts, double* out)
{
    if (check_geom(g) || !dy || !wt || !pts || !out || !ystr || !wstr) return ORACLE_BAD;
    const int64_t Ho = extent_out(g->H, g->ph, g->KH, g->S);
    const int64_t Wo = extent_out(g->W, g->pw, g->KW, g->S);
    const int64_t Kg = g->K / g->groups, Cg = g->C / g->groups;
    for (int64_t i = 0; i < npts; ++i) {
        const int64_t n = pts[4 * i], h = pts[4 * i + 1], w = pts[4 * i + 2], c = pts[4 * i + 3];
        if (n < 0 || n >= g->N || h < 0 || h >= g->H || w < 0 || w >= g->W || c < 0 || c >= g->C)
            return ORACLE_BAD;
    }
    int nt = oracle_get_threads();
    (void)nt;
#pragma omp parallel for schedule(static) num_threads(nt)
    for (int64_t i = 0; i < npts; ++i) {
        const int64_t n = pts[4 * i], h = pts[4 * i + 1], w = pts[4 * i + 2], c = pts[4 * i + 3];
        const int64_t grp = c / Cg, cg = c - grp * Cg;
        double acc = 0.0;
        for (int64_t k = grp * Kg; k < (grp + 1) * Kg; ++k)
        for (int64_t r = 0; r < g->KH; ++r) {
            const int64_t th = h + g->ph - r;
            if (th < 0 || th % g->S) continue;
            const int64_t ho = th / g->S;
            if (ho >= Ho) continue;
            for (int64_t s = 0; s < g->KW; ++s) {
                const int64_t tw = w + g->pw - s;
                if (tw < 0 || tw % g->S) continue;
                const int64_t wo = tw / g->S;
                if (wo >= Wo) continue;
                acc += dy[n * ystr[0] + ho * ystr[1] + wo * ystr[2] + k * ystr[3]]
                     * wt[k * wstr[0] + r * wstr[1] + s * wstr[2] + cg * wstr[3]];
            }
        }
        out[i] = acc;
    }
    return ORACLE_OK;
}

/* Forward convolution, gather form (the map whose adjoint dgrad is):
 *   y[n,ho,wo,k] = sum_{r,s,cg} x[n, ho*S-ph+r, wo*S-pw+s, g(k)*Cg+cg] * Wt(k,r,s,cg).
 * x is dense NHWC, y is dense N,Ho,Wo,K. */
int oracle_conv_fwd(const oracle_geom_t* g, const double* x,
                    const double* wt, const int64_t wstr[4], double* y)
{
    if (check_geom(g) || !x || !wt || !y || !wstr) return ORACLE_BAD;
    const int64_t Ho = extent_out(g->H, g->ph, g->KH, g->S);
    const int64_t Wo = extent_out(g->W, g->pw, g->KW, g->S);
    const int64_t Kg = g->K / g->groups, Cg = g->C / g->groups;
    int nt = oracle_get_threads();
    (void)nt;
#pragma omp parallel for schedule(static) num_threads(nt)
    for (int64_t n = 0; n < g->N; ++n)
    for (int64_t ho = 0; ho < Ho; ++ho)
    for (int64_t wo = 0; wo < Wo; ++wo)
    for (int64_t k = 0; k < g->K; ++k) {
        const int64_t grp = k / Kg;
        double acc = 0.0;
        for (int64_t r = 0; r < g->KH; ++r) {
            const int64_t h = ho * g->S - g->ph + r;
            if (h < 0 || h >= g->H) continue;
            for (int64_t s = 0; s < g->KW; ++s) {
                const int64_t w = wo * g->S - g->pw + s;
                if (w < 0 || w >= g->W) continue;
                for (int64_t cg = 0; cg < Cg; ++cg)
                    acc += x[((n * g->H + h) * g->W + w) * g->C + grp * Cg + cg]
                         * wt[k * wstr[0] + r * wstr[1] + s * wstr[2] + cg * wstr[3]];
            }
        }
        y[((n * Ho + ho) * Wo + wo) * g->K + k] = acc;
    }
    return ORACLE_OK;
}

/* Stride-1 depthwise dgrad written as the pages' rotated-filter correlation:
 * pad dY by P'h = KH-1-ph rows and P'w = KW-1-pw columns, then correlate it
 * with the filter rotated by 180 degrees (row r' of the rotated filter is row
 * KH-1-r' of W, read back to front):
 *   dX[n,h,w,c] = sum_{r'<KH, s'<KW} dYpad[n, h+r', w+s', c] * W[KH-1-r'][KW-1-s'][c]
 * where dYpad[n, i, j, c] = dY[n, i-P'h, j-P'w, c] inside dY and 0 outside.
 * Requires groups = C = K, S = 1 and ph <= KH-1, pw <= KW-1 (non-negative
 * rotated padding).  dY dense (N,Ho,Wo,C), W dense [KH][KW][C]. */
int oracle_dw_rotated(const oracle_geom_t* g, const double* dy, const double* w, double* dx)
{
    if (check_geom(g) || !dy || !w || !dx) return ORACLE_BAD;
    if (g->S != 1 || g->groups != g->C || g->K != g->C) return ORACLE_BAD;
    if (g->ph > g->KH - 1 || g->pw > g->KW - 1) return ORACLE_BAD;
    const int64_t Ho = extent_out(g->H, g->ph, g->KH, 1);
    const int64_t Wo = extent_out(g->W, g->pw, g->KW, 1);
    const int64_t Prh = g->KH - 1 - g->ph, Prw = g->KW - 1 - g->pw, C = g->C;
    int nt = oracle_get_threads();
    (void)nt;
#pragma omp parallel for schedule(static) num_threads(nt)
    for (int64_t n = 0; n < g->N; ++n)
    for (int64_t h = 0; h < g->H; ++h)
    for (int64_t x = 0; x < g->W; ++x)
    for (int64_t c = 0; c < C; ++c) {
        double acc = 0.0;
        for (int64_t rr = 0; rr < g->KH; ++rr) {
            const int64_t i = h + rr - Prh;        /* row of dY under tap rr */
            if (i < 0 || i >= Ho) continue;
            for (int64_t ss = 0; ss < g->KW; ++ss) {
                const int64_t j = x + ss - Prw;    /* column of dY under tap ss */
                if (j < 0 || j >= Wo) continue;
                acc += dy[((n * Ho + i) * Wo + j) * C + c]
                     * w[((g->KH - 1 - rr) * g->KW + (g->KW - 1 - ss)) * C + c];
            }
        }
        dx[((n * g->H + h) * g->W + x) * C + c] = acc;
    }
    return ORACLE_OK;
}

/* Depthwise dgrad by the row-streaming schedule (any stride):
 *  - dY rows ho = 0..Ho-1 are streamed in order;
 *  - row ho adds into the accumulator rows h = ho*S - ph + r (r < KH) that lie
 *    on the image; accumulator row h lives in circular slot h mod R;
 *  - after row ho every dX row below (ho+1)*S - ph is final: it is written out
 *    and its slot cleared;
 *  - after the last dY row a tail flushes every row still open, up to H-1,
 *    including rows no dY row reached (they come out zero).
 * R = max(KH, S) slots suffice: while row ho is applied the rows touched span
 * KH consecutive rows, and the rows flushed after it span at most S.
 * dY dense (N,Ho,Wo,C), W dense [KH][KW][C], groups = C = K. */
int oracle_dw_rowstream(const oracle_geom_t* g, const double* dy, const double* w, double* dx)
{
    if (check_geom(g) || !dy || !w || !dx) return ORACLE_BAD;
    if (g->groups != g->C || g->K != g->C) return ORACLE_BAD;
    const int64_t Ho = extent_out(g->H, g->ph, g->KH, g->S);
    const int64_t Wo = extent_out(g->W, g->pw, g->KW, g->S);
    const int64_t H = g->H, W = g->W, C = g->C, S = g->S;
    const int64_t R = g->KH > S ? g->KH : S;
    int nt = oracle_get_threads();
    (void)nt;
    int bad = 0;
#pragma omp parallel for schedule(static) num_threads(nt) reduction(| : bad)
    for (int64_t n = 0; n < g->N; ++n) {
        double* ring = (double*)calloc((size_t)(R * W * C), sizeof(double));
        if (!ring) { bad = 1; continue; }
        int64_t next_flush = 0;                      /* first dX row not yet written */
        for (int64_t ho = 0; ho < Ho; ++ho) {
            for (int64_t r = 0; r < g->KH; ++r) {
                const int64_t h = ho * S - g->ph + r;
                if (h < 0 || h >= H) continue;
                double* acc = ring + (h % R) * W * C;
                for (int64_t wo = 0; wo < Wo; ++wo)
                for (int64_t s = 0; s < g->KW; ++s) {
                    const int64_t x = wo * S - g->pw + s;
                    if (x < 0 || x >= W) continue;
                    for (int64_t c = 0; c < C; ++c)
                        acc[x * C + c] += dy[((n * Ho + ho) * Wo + wo) * C + c]
                                        * w[(r * g->KW + s) * C + c];
                }
            }
            int64_t done = (ho + 1) * S - g->ph;    /* rows below this are final */
            if (done > H) done = H;
            for (; next_flush < done; ++next_flush) {
                double* acc = ring + (next_flush % R) * W * C;
                memcpy(dx + (n * H + next_flush) * W * C, acc, sizeof(double) * (size_t)(W * C));
                memset(acc, 0, sizeof(double) * (size_t)(W * C));
            }
        }
        for (; next_flush < H; ++next_flush) {         /* tail */
            double* acc = ring + (next_flush % R) * W * C;
            memcpy(dx + (n * H + next_flush) * W * C, acc, sizeof(double) * (size_t)(W * C));
            memset(acc, 0, sizeof(double) * (size_t)(W * C));
        }
        free(ring);
    }
    return bad ? ORACLE_BAD : ORACLE_OK;
}
