/*
 * schnet_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, float64 CPU statement of what the SchNet continuous-filter
 * convolution (CFConv) energy/force path and its Langevin / velocity-Verlet
 * update compute.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this file's shared library.  It shares no code,
 * header, table or constant generator with the CUDA library.
 *
 * Sources (the pages give the steps by name, not their formulas):
 *   - "FlashSchNet: Fast and Accurate Coarse-Grained Neural Network Molecular
 *     Dynamics" (paper-curation summary), section How: the step order
 *     pairwise distance -> Gaussian basis -> cosine envelope (flash radial
 *     basis), cutoff masking -> neighbour gather -> filter multiply ->
 *     reduction (flash message passing), CSR segment reduce in forward and
 *     backward (flash aggregation), forces from the backward pass.
 *   - Same work, OpenAlex record, abstract: the four techniques (1)-(4).
 *   - "Ab Initio Accuracy Beyond the Cutoff" (Tessera, aiqbench item),
 *     abstract: conservative neighbour skin, topology fixed between rebuilds.
 * Where the pages are silent the plain textbook SchNet reading is taken:
 *   Gaussian e_k(d) = exp(-(d-mu_k)^2 / (2 sigma^2)), mu_k = linspace;
 *   cosine cutoff f_c(d) = (cos(pi d / r_c) + 1) / 2 for d < r_c, else 0;
 *   shifted softplus ssp(x) = ln(1 + e^x) - ln 2;
 *   filter W(d) = f_c(d) * (ssp(e(d) W1 + b1) W2 + b2), one filter per
 *   interaction; interaction: h = x W_in, m_i = sum_j h_j (.) W(d_ij),
 *   x += ssp(m Wo1 + bo1) Wo2 + bo2; readout eps_i = ssp(x R1 + c1) R2 + c2,
 *   E = sum_i eps_i; F = -dE/dr, derived by hand below.
 * All dense weights are row-major [in][out]; x W means sum over "in".
 *
 * Aggregation is a CSR segment sum over destination rows (rows hold the
 * neighbours j of atom i in ascending j), as the flash-aggregation step
 * states; the backward pass of each interaction is also done row by row
 * over the same (symmetric) list, so no scatter is needed.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef M_PI
#define M_PI 3.14159265358979323846
#endif
#define OR_LN2 0.69314718055994530942

/* ------------------------------------------------------------------ */
/* Scalar building blocks                                              */
/* ------------------------------------------------------------------ */

/* shifted softplus ln(1+e^x) - ln 2, written in the overflow-free form
 * max(x,0) + ln(1 + e^-|x|) - ln 2. */
double or_ssp(double x)
{
    double pos = x > 0.0 ? x : 0.0;
    return pos + log1p(exp(-fabs(x))) - OR_LN2;
}

/* d ssp / dx = e^x / (1 + e^x), the logistic function. */
double or_dssp(double x)
{
    if (x >= 0.0) return 1.0 / (1.0 + exp(-x));
    double t = exp(x);
    return t / (1.0 + t);
}

/* cosine envelope (flash radial basis step "cosine envelope"). */
double or_fc(double d, double rc)
{
    return d < rc ? 0.5 * (cos(M_PI * d / rc) + 1.0) : 0.0;
}

double or_dfc(double d, double rc)
{
    return d < rc ? -0.5 * (M_PI / rc) * sin(M_PI * d / rc) : 0.0;
}

/* Centre of the k-th Gaussian: K centres spread evenly over
 * [rbf_min, rbf_max], both ends included. */
double or_rbf_center(int k, int K, double rmin, double rmax)
{
    if (K <= 1) return rmin;
    return rmin + (double)k * (rmax - rmin) / (double)(K - 1);
}

/* Gaussian expansion of one distance and its d-derivative. */
void or_rbf(double d, int K, double rmin, double rmax, double sigma,
            double *e, double *de)
{
    double inv2s2 = 1.0 / (2.0 * sigma * sigma);
    for (int k = 0; k < K; ++k) {
        double t = d - or_rbf_center(k, K, rmin, rmax);
        e[k] = exp(-t * t * inv2s2);
        if (de) de[k] = -t / (sigma * sigma) * e[k];
    }
}

/* ------------------------------------------------------------------ */
/* Model description                                                   */
/* ------------------------------------------------------------------ */

typedef struct {
    int T, F, K, L;            /* types, features, Gaussians, interactions */
    double rbf_min, rbf_max, rbf_sigma, cutoff;
    int periodic;              /* 1: minimum image in an orthorhombic box */
    double box[3];
} or_model;

typedef struct {
    const double *emb;   /* [T][F]   */
    const double *W_in;  /* [L][F][F] */
    const double *W1;    /* [L][K][F] */
    const double *b1;    /* [L][F]   */
    const double *W2;    /* [L][F][F] */
    const double *b2;    /* [L][F]   */
    const double *Wo1;   /* [L][F][F] */
    const double *bo1;   /* [L][F]   */
    const double *Wo2;   /* [L][F][F] */
    const double *bo2;   /* [L][F]   */
    const double *R1;    /* [F][H], H = F/2 */
    const double *c1;    /* [H]      */
    const double *R2;    /* [H]      */
    double c2;
} or_weights;

/* v = r_j - r_i, minimum image when periodic. */
static void pair_vec(const or_model *m, const double *ri, const double *rj,
                     double *v)
{
    for (int c = 0; c < 3; ++c) {
        double t = rj[c] - ri[c];
        if (m->periodic) t -= m->box[c] * nearbyint(t / m->box[c]);
        v[c] = t;
    }
}

/* Filter of interaction l at distance d (< cutoff) and its d-derivative:
 *   p = e(d) W1 + b1,  a = ssp(p),  z = a W2 + b2,  W = f_c(d) z,
 *   dW/dd = f_c'(d) z + f_c(d) ((ssp'(p) (.) (e'(d) W1)) W2).
 * work must hold 2K + 4F doubles.  dW may be NULL. */
void or_filter(const or_model *m, const or_weights *w, int l, double d,
               double *W, double *dW, double *work)
{
    const int K = m->K, F = m->F;
    double *e = work, *de = work + K;
    double *p = de + K, *dp = p + F, *a = dp + F, *da = a + F;
    const double *W1 = w->W1 + (size_t)l * K * F;
    const double *b1 = w->b1 + (size_t)l * F;
    const double *W2 = w->W2 + (size_t)l * F * F;
    const double *b2 = w->b2 + (size_t)l * F;

    or_rbf(d, K, m->rbf_min, m->rbf_max, m->rbf_sigma, e, de);
    double fc = or_fc(d, m->cutoff), dfc = or_dfc(d, m->cutoff);

    for (int f = 0; f < F; ++f) {
        double s = b1[f], ds = 0.0;
        for (int k = 0; k < K; ++k) {
            s += e[k] * W1[(size_t)k * F + f];
            ds += de[k] * W1[(size_t)k * F + f];
        }
        p[f] = s;
        dp[f] = ds;
    }
    for (int f = 0; f < F; ++f) {
        a[f] = or_ssp(p[f]);
        da[f] = or_dssp(p[f]) * dp[f];
    }
    for (int f = 0; f < F; ++f) {
        double z = b2[f], dz = 0.0;
        for (int g = 0; g < F; ++g) {
            z += a[g] * W2[(size_t)g * F + f];
            dz += da[g] * W2[(size_t)g * F + f];
        }
        W[f] = fc * z;
        if (dW) dW[f] = dfc * z + fc * dz;
    }
}

/* ------------------------------------------------------------------ */
/* Neighbour list with skin (what the GPU list must reproduce exactly)  */
/* ------------------------------------------------------------------ */

/* All ordered pairs (i, j), i != j, of the same replica with
 * d^2 < (cutoff + skin)^2.  Coordinates are float32 values; the test is
 * done in float64 as
 *   dx = x_j - x_i;  periodic: dx = dx - L * nearbyint(dx / L)
 *   d2 = (dx*dx + dy*dy) + dz*dz
 * with every operation rounded on its own (no fused multiply-add), so the
 * inclusion decision is a well-defined bit-exact function of the inputs.
 * Rows are ascending in i, and each row lists j ascending.
 * Returns the number of edges; if that exceeds cap, col is left partial
 * and the (true) count is still returned. */
int64_t or_neighbors(int n, const float *pos, int R, const int *rep_off,
                     float cutoff, float skin, int periodic, const float *box,
                     int64_t cap, int32_t *row_ptr, int32_t *col)
{
    const double rl = (double)cutoff + (double)skin;
    const double rl2 = rl * rl;
    int64_t e = 0;
    for (int r = 0; r < R; ++r) {
        int a = rep_off[r], b = rep_off[r + 1];
        for (int i = a; i < b; ++i) {
            row_ptr[i] = (int32_t)e;
            for (int j = a; j < b; ++j) {
                if (j == i) continue;
                double v[3];
                for (int c = 0; c < 3; ++c) {
                    double t = (double)pos[3 * j + c] - (double)pos[3 * i + c];
                    if (periodic) {
                        double L = (double)box[c];
                        double k = nearbyint(t / L);
                        double s = L * k;
                        t = t - s;
                    }
                    v[c] = t;
                }
                double xx = v[0] * v[0];
                double yy = v[1] * v[1];
                double zz = v[2] * v[2];
                double d2 = xx + yy;
                d2 = d2 + zz;
                if (d2 < rl2) {
                    if (e < cap) col[e] = j;
                    ++e;
                }
            }
        }
    }
    if (n > 0) row_ptr[n] = (int32_t)e;
    return e;
}

/* ------------------------------------------------------------------ */
/* Exact-cutoff CSR used by the energy evaluation                       */
/* ------------------------------------------------------------------ */

typedef struct {
    int n;
    int64_t *ptr;   /* [n+1] */
    int *col;       /* [E]   */
    double *dist;   /* [E]   */
    double *vec;    /* [E][3], r_j - r_i */
} or_csr;

static void csr_free(or_csr *c)
{
    free(c->ptr); free(c->col); free(c->dist); free(c->vec);
    memset(c, 0, sizeof(*c));
}

/* Pairs (i, j) of one replica with 0 < d_ij < cutoff, rows ascending. */
static int csr_build(const or_model *m, int n, const double *pos, int R,
                     const int *rep_off, or_csr *c)
{
    c->n = n;
    c->ptr = (int64_t *)calloc((size_t)n + 1, sizeof(int64_t));
    if (!c->ptr) return -1;
    int *rep_of = (int *)malloc(sizeof(int) * (size_t)(n > 0 ? n : 1));
    if (!rep_of) return -1;
    for (int r = 0; r < R; ++r)
        for (int i = rep_off[r]; i < rep_off[r + 1]; ++i) rep_of[i] = r;

    #pragma omp parallel for schedule(dynamic, 16)
    for (int i = 0; i < n; ++i) {
        int r = rep_of[i];
        int64_t cnt = 0;
        for (int j = rep_off[r]; j < rep_off[r + 1]; ++j) {
            if (j == i) continue;
            double v[3];
            pair_vec(m, pos + 3 * i, pos + 3 * j, v);
            double d = sqrt(v[0] * v[0] + v[1] * v[1] + v[2] * v[2]);
            if (d > 0.0 && d < m->cutoff) ++cnt;
        }
        c->ptr[i + 1] = cnt;
    }
    for (int i = 0; i < n; ++i) c->ptr[i + 1] += c->ptr[i];
    int64_t E = c->ptr[n];
    size_t Ea = (size_t)(E > 0 ? E : 1);
    c->col = (int *)malloc(sizeof(int) * Ea);
    c->dist = (double *)malloc(sizeof(double) * Ea);
    c->vec = (double *)malloc(sizeof(double) * 3 * Ea);
    if (!c->col || !c->dist || !c->vec) { free(rep_of); return -1; }

    #pragma omp parallel for schedule(dynamic, 16)
    for (int i = 0; i < n; ++i) {
        int r = rep_of[i];
        int64_t e = c->ptr[i];
        for (int j = rep_off[r]; j < rep_off[r + 1]; ++j) {
            if (j == i) continue;
            double v[3];
            pair_vec(m, pos + 3 * i, pos + 3 * j, v);
            double d = sqrt(v[0] * v[0] + v[1] * v[1] + v[2] * v[2]);
            if (d > 0.0 && d < m->cutoff) {
                c->col[e] = j;
                c->dist[e] = d;
                c->vec[3 * e + 0] = v[0];
                c->vec[3 * e + 1] = v[1];
                c->vec[3 * e + 2] = v[2];
                ++e;
            }
        }
    }
    free(rep_of);
    return 0;
}

/* ------------------------------------------------------------------ */
/* CFConv aggregation as a CSR segment sum                             */
/* ------------------------------------------------------------------ */

/* m_i = sum over row i of h_j (.) W(d_ij), interaction l. */
static void cfconv_rows(const or_model *m, const or_weights *w, int l,
                        const or_csr *c, const double *h, double *out)
{
    const int F = m->F, K = m->K;
    #pragma omp parallel
    {
        double *Wf = (double *)malloc(sizeof(double) * (size_t)(F + 2 * K + 4 * F));
        double *work = Wf + F;
        #pragma omp for schedule(dynamic, 8)
        for (int i = 0; i < c->n; ++i) {
            double *mi = out + (size_t)i * F;
            for (int f = 0; f < F; ++f) mi[f] = 0.0;
            for (int64_t e = c->ptr[i]; e < c->ptr[i + 1]; ++e) {
                or_filter(m, w, l, c->dist[e], Wf, NULL, work);
                const double *hj = h + (size_t)c->col[e] * F;
                for (int f = 0; f < F; ++f) mi[f] += hj[f] * Wf[f];
            }
        }
        free(Wf);
    }
}

/* Public tap used by the aggregation pin: segment sum over the exact-cutoff
 * rows of the given positions, for interaction l and given h [n][F]. */
int or_cfconv(const or_model *m, const or_weights *w, int l, int n,
              const double *pos, int R, const int *rep_off, const double *h,
              double *out)
{
    or_csr c = {0};
    if (csr_build(m, n, pos, R, rep_off, &c)) { csr_free(&c); return -1; }
    cfconv_rows(m, w, l, &c, h, out);
    csr_free(&c);
    return 0;
}

/* Public tap: the exact-cutoff edge list (row, col, d) in CSR order.
 * Call with cap = 0 to get the count. */
int64_t or_cut_edges(const or_model *m, int n, const double *pos, int R,
                     const int *rep_off, int64_t cap, int32_t *row,
                     int32_t *col, double *dist)
{
    or_csr c = {0};
    if (csr_build(m, n, pos, R, rep_off, &c)) { csr_free(&c); return -1; }
    int64_t E = c.ptr[n];
    if (E <= cap) {
        for (int i = 0; i < n; ++i)
            for (int64_t e = c.ptr[i]; e < c.ptr[i + 1]; ++e) {
                row[e] = i; col[e] = c.col[e]; dist[e] = c.dist[e];
            }
    }
    csr_free(&c);
    return E;
}

/* ------------------------------------------------------------------ */
/* Energy and forces                                                   */
/* ------------------------------------------------------------------ */

static void dense(const double *x, const double *W, const double *b,
                  int nin, int nout, double *y)
{
    for (int o = 0; o < nout; ++o) y[o] = b ? b[o] : 0.0;
    for (int i = 0; i < nin; ++i) {
        double xi = x[i];
        const double *Wi = W + (size_t)i * nout;
        for (int o = 0; o < nout; ++o) y[o] += xi * Wi[o];
    }
}

/* y[i] = sum_o g[o] W[i][o]   (product with the transpose) */
static void dense_t(const double *g, const double *W, int nin, int nout,
                    double *y)
{
    for (int i = 0; i < nin; ++i) {
        const double *Wi = W + (size_t)i * nout;
        double s = 0.0;
        for (int o = 0; o < nout; ++o) s += g[o] * Wi[o];
        y[i] = s;
    }
}

/* Energy per replica E[R], energy per atom eps[n] (may be NULL) and
 * forces F[n][3] = -dE/dr (may be NULL), all float64.
 * Returns 0, -1 on allocation failure, -2 on a type outside [0, T). */
int or_energy_forces(const or_model *m, const or_weights *w, int n,
                     const double *pos, const int *types, int R,
                     const int *rep_off, double *E, double *eps,
                     double *forces)
{
    const int F = m->F, L = m->L, H = m->F / 2;
    for (int i = 0; i < n; ++i)
        if (types[i] < 0 || types[i] >= m->T) return -2;

    or_csr c = {0};
    if (csr_build(m, n, pos, R, rep_off, &c)) { csr_free(&c); return -1; }

    size_t nF = (size_t)n * F;
    double *x = (double *)malloc(sizeof(double) * (nF ? nF : 1));
    double *hs = (double *)malloc(sizeof(double) * (nF * L ? nF * L : 1));
    double *qs = (double *)malloc(sizeof(double) * (nF * L ? nF * L : 1));
    double *mm = (double *)malloc(sizeof(double) * (nF ? nF : 1));
    double *pr = (double *)malloc(sizeof(double) * ((size_t)n * H + 1));
    double *ea = (double *)malloc(sizeof(double) * ((size_t)n + 1));
    if (!x || !hs || !qs || !mm || !pr || !ea) {
        free(x); free(hs); free(qs); free(mm); free(pr); free(ea);
        csr_free(&c);
        return -1;
    }

    /* ---- forward ---- */
    for (int i = 0; i < n; ++i)
        memcpy(x + (size_t)i * F, w->emb + (size_t)types[i] * F,
               sizeof(double) * F);

    for (int l = 0; l < L; ++l) {
        const double *Win = w->W_in + (size_t)l * F * F;
        double *h = hs + (size_t)l * nF;
        double *q = qs + (size_t)l * nF;
        #pragma omp parallel for schedule(static)
        for (int i = 0; i < n; ++i)
            dense(x + (size_t)i * F, Win, NULL, F, F, h + (size_t)i * F);

        cfconv_rows(m, w, l, &c, h, mm);

        const double *Wo1 = w->Wo1 + (size_t)l * F * F, *bo1 = w->bo1 + (size_t)l * F;
        const double *Wo2 = w->Wo2 + (size_t)l * F * F, *bo2 = w->bo2 + (size_t)l * F;
        #pragma omp parallel
        {
            double *a = (double *)malloc(sizeof(double) * F * 2);
            double *v = a + F;
            #pragma omp for schedule(static)
            for (int i = 0; i < n; ++i) {
                double *qi = q + (size_t)i * F;
                dense(mm + (size_t)i * F, Wo1, bo1, F, F, qi);
                for (int f = 0; f < F; ++f) a[f] = or_ssp(qi[f]);
                dense(a, Wo2, bo2, F, F, v);
                for (int f = 0; f < F; ++f) x[(size_t)i * F + f] += v[f];
            }
            free(a);
        }
    }

    /* readout: eps_i = ssp(x R1 + c1) R2 + c2 */
    #pragma omp parallel for schedule(static)
    for (int i = 0; i < n; ++i) {
        double *p = pr + (size_t)i * H;
        dense(x + (size_t)i * F, w->R1, w->c1, F, H, p);
        double s = w->c2;
        for (int k = 0; k < H; ++k) s += or_ssp(p[k]) * w->R2[k];
        ea[i] = s;
    }
    for (int r = 0; r < R; ++r) {
        double s = 0.0;
        for (int i = rep_off[r]; i < rep_off[r + 1]; ++i) s += ea[i];
        E[r] = s;
    }
    if (eps) memcpy(eps, ea, sizeof(double) * (size_t)n);

    if (!forces) {
        free(x); free(hs); free(qs); free(mm); free(pr); free(ea);
        csr_free(&c);
        return 0;
    }

    /* ---- backward ---- */
    double *g = x;   /* dE/dx, reuses x */
    double *u = mm;  /* dE/dm */
    double *dh = (double *)malloc(sizeof(double) * (nF ? nF : 1));
    if (!dh) {
        free(x); free(hs); free(qs); free(mm); free(pr); free(ea);
        csr_free(&c);
        return -1;
    }
    for (size_t t = 0; t < (size_t)n * 3; ++t) forces[t] = 0.0;

    /* dE/dx^L from the readout: g_f = sum_k R1[f][k] ssp'(pr_k) R2[k] */
    #pragma omp parallel
    {
        double *t = (double *)malloc(sizeof(double) * (H + 1));
        #pragma omp for schedule(static)
        for (int i = 0; i < n; ++i) {
            for (int k = 0; k < H; ++k)
                t[k] = or_dssp(pr[(size_t)i * H + k]) * w->R2[k];
            dense_t(t, w->R1, F, H, g + (size_t)i * F);
        }
        free(t);
    }

    for (int l = L - 1; l >= 0; --l) {
        const double *h = hs + (size_t)l * nF;
        const double *q = qs + (size_t)l * nF;
        const double *Wo1 = w->Wo1 + (size_t)l * F * F;
        const double *Wo2 = w->Wo2 + (size_t)l * F * F;
        const double *Win = w->W_in + (size_t)l * F * F;

        /* u = ((g Wo2^T) (.) ssp'(q)) Wo1^T */
        #pragma omp parallel
        {
            double *t = (double *)malloc(sizeof(double) * F);
            #pragma omp for schedule(static)
            for (int i = 0; i < n; ++i) {
                dense_t(g + (size_t)i * F, Wo2, F, F, t);
                for (int o = 0; o < F; ++o) t[o] *= or_dssp(q[(size_t)i * F + o]);
                dense_t(t, Wo1, F, F, u + (size_t)i * F);
            }
            free(t);
        }

        /* Row j of the symmetric list:
         *   dE/dh_j = sum_{i in row j} u_i (.) W(d_ji)
         *   D_ji    = sum_f W'(d_ji)_f (u_j,f h_i,f + u_i,f h_j,f)
         *             (both directed edges of the pair: dE/dd for the pair)
         *   F_j    -= sum_i D_ji (r_j - r_i) / d_ji                          */
        #pragma omp parallel
        {
            const int K = m->K;
            double *Wf = (double *)malloc(sizeof(double) * (size_t)(2 * F + 2 * K + 4 * F));
            double *dWf = Wf + F, *work = dWf + F;
            #pragma omp for schedule(dynamic, 8)
            for (int j = 0; j < n; ++j) {
                double *dhj = dh + (size_t)j * F;
                const double *uj = u + (size_t)j * F, *hj = h + (size_t)j * F;
                double fx = 0.0, fy = 0.0, fz = 0.0;
                for (int f = 0; f < F; ++f) dhj[f] = 0.0;
                for (int64_t e = c.ptr[j]; e < c.ptr[j + 1]; ++e) {
                    int i = c.col[e];
                    double d = c.dist[e];
                    or_filter(m, w, l, d, Wf, dWf, work);
                    const double *ui = u + (size_t)i * F, *hi = h + (size_t)i * F;
                    double D = 0.0;
                    for (int f = 0; f < F; ++f) {
                        dhj[f] += ui[f] * Wf[f];
                        D += dWf[f] * (uj[f] * hi[f] + ui[f] * hj[f]);
                    }
                    /* vec = r_i - r_j here (row j, column i), so
                     * (r_j - r_i)/d = -vec/d and F_j -= D (r_j - r_i)/d. */
                    fx += D * c.vec[3 * e + 0] / d;
                    fy += D * c.vec[3 * e + 1] / d;
                    fz += D * c.vec[3 * e + 2] / d;
                }
                forces[3 * j + 0] += fx;
                forces[3 * j + 1] += fy;
                forces[3 * j + 2] += fz;
            }
            free(Wf);
        }

        /* g <- g + dh W_in^T  (residual path plus the h = x W_in path) */
        #pragma omp parallel
        {
            double *t = (double *)malloc(sizeof(double) * F);
            #pragma omp for schedule(static)
            for (int i = 0; i < n; ++i) {
                dense_t(dh + (size_t)i * F, Win, F, F, t);
                for (int f = 0; f < F; ++f) g[(size_t)i * F + f] += t[f];
            }
            free(t);
        }
    }

    free(dh);
    free(x); free(hs); free(qs); free(mm); free(pr); free(ea);
    csr_free(&c);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers:  */
/* as easy as 1, 2, 3", SC'11) and Box-Muller normals                   */
/* ------------------------------------------------------------------ */

void or_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2],
                      uint32_t out[4])
{
    const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
    const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) { k0 += W0; k1 += W1; }
        uint64_t p0 = (uint64_t)M0 * c0;
        uint64_t p1 = (uint64_t)M1 * c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        uint32_t n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* Three standard normals per atom for step `step`:
 * key = (seed low, seed high), counter = (atom, step low, step high, 0);
 * the four 32-bit outputs x_a map to u_a = (x_a + 1) / 2^32 in (0, 1];
 * Box-Muller: xi_0 = r0 cos(2 pi u1), xi_1 = r0 sin(2 pi u1),
 * xi_2 = r1 cos(2 pi u3) with r = sqrt(-2 ln u0), r1 = sqrt(-2 ln u2). */
void or_noise(uint64_t seed, uint64_t step, int n, double *xi)
{
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    for (int i = 0; i < n; ++i) {
        uint32_t ctr[4] = {(uint32_t)i, (uint32_t)step, (uint32_t)(step >> 32), 0u};
        uint32_t o[4];
        or_philox4x32_10(ctr, key, o);
        double u[4];
        for (int a = 0; a < 4; ++a) u[a] = ((double)o[a] + 1.0) / 4294967296.0;
        double r0 = sqrt(-2.0 * log(u[0])), r1 = sqrt(-2.0 * log(u[2]));
        xi[3 * i + 0] = r0 * cos(2.0 * M_PI * u[1]);
        xi[3 * i + 1] = r0 * sin(2.0 * M_PI * u[1]);
        xi[3 * i + 2] = r1 * cos(2.0 * M_PI * u[3]);
    }
}

/* ------------------------------------------------------------------ */
/* BAOAB Langevin (Leimkuhler-Matthews splitting); gamma = 0 is         */
/* velocity Verlet.  Units: A, fs, amu, kcal/mol, K.                     */
/* ------------------------------------------------------------------ */

#define OR_ACC 4.184e-4          /* (kcal/mol/A)/amu -> A/fs^2 */
#define OR_KB  0.0019872041      /* kcal/mol/K */

/* B (half kick with forces F), A (half drift), O (friction + noise),
 * A (half drift).  xi: [n][3] standard normals (ignored if gamma == 0). */
void or_baoa(int n, double *pos, double *vel, const double *F,
             const double *mass, double dt, double gamma_per_ps,
             double temperature, const double *xi)
{
    double c1 = exp(-gamma_per_ps * 1e-3 * dt);
    double kT = OR_KB * temperature;
    for (int i = 0; i < n; ++i) {
        double inv_m = 1.0 / mass[i];
        double sv = sqrt((1.0 - c1 * c1) * kT * OR_ACC * inv_m);
        for (int c = 0; c < 3; ++c) {
            double v = vel[3 * i + c] + 0.5 * dt * OR_ACC * F[3 * i + c] * inv_m;
            double r = pos[3 * i + c] + 0.5 * dt * v;
            if (gamma_per_ps != 0.0) v = c1 * v + sv * xi[3 * i + c];
            r = r + 0.5 * dt * v;
            vel[3 * i + c] = v;
            pos[3 * i + c] = r;
        }
    }
}

/* Closing half kick with the forces at the new positions. */
void or_b(int n, double *vel, const double *F, const double *mass, double dt)
{
    for (int i = 0; i < n; ++i)
        for (int c = 0; c < 3; ++c)
            vel[3 * i + c] += 0.5 * dt * OR_ACC * F[3 * i + c] / mass[i];
}

/* Kinetic energy per replica, kcal/mol. */
void or_kinetic(int n, const double *vel, const double *mass, int R,
                const int *rep_off, double *ekin)
{
    for (int r = 0; r < R; ++r) {
        double s = 0.0;
        for (int i = rep_off[r]; i < rep_off[r + 1]; ++i)
            s += 0.5 * mass[i] *
                 (vel[3 * i] * vel[3 * i] + vel[3 * i + 1] * vel[3 * i + 1] +
                  vel[3 * i + 2] * vel[3 * i + 2]);
        ekin[r] = s / OR_ACC;
    }
}

/* One full MD step: BAOA with F (forces at pos, updated in place to the
 * forces at the new positions), then the closing B.  noise: [n][3] normals,
 * or NULL to draw them from or_noise(seed, step).  epot/ekin: [R]. */
int or_md_step(const or_model *m, const or_weights *w, int n, double *pos,
               double *vel, const int *types, const double *mass, int R,
               const int *rep_off, double dt, double gamma_per_ps,
               double temperature, uint64_t seed, uint64_t step,
               const double *noise, double *F, double *epot, double *ekin)
{
    double *xi = NULL;
    if (gamma_per_ps != 0.0 && !noise) {
        xi = (double *)malloc(sizeof(double) * 3 * (size_t)(n > 0 ? n : 1));
        if (!xi) return -1;
        or_noise(seed, step, n, xi);
        noise = xi;
    }
    or_baoa(n, pos, vel, F, mass, dt, gamma_per_ps, temperature, noise);
    free(xi);
    int rc = or_energy_forces(m, w, n, pos, types, R, rep_off, epot, NULL, F);
    if (rc) return rc;
    or_b(n, vel, F, mass, dt);
    or_kinetic(n, vel, mass, R, rep_off, ekin);
    return 0;
}
