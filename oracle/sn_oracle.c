/*
 * sn_oracle.c -- plain double-precision CPU oracle of the SchNet energy/force hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's CPU-baseline
 * leg may load this library.  It shares no code with the CUDA path; both read the same
 * seeded inputs and nothing else.
 *
 * What it computes (FlashSchNet, arXiv 2602.13140):
 *   - neighbour list: directed edges j -> i for every pair of the same replica closer than
 *     r_cut, as CSR grouped by destination (§3.2 "Building the neighbor list"; §4.3 "Index
 *     construction under dynamic neighbor lists").  Membership is decided by an fp32 test
 *     (see pair_within) so that any fp32 implementation can reproduce the list bit for bit;
 *   - u_e = r_dst - r_src, d_e = |u_e| (§3.2 "Distances and radial basis");
 *   - b~_e = RBF(d_e) * C(d_e) with Gaussians exp(-gamma (d - mu_k)^2), mu_k = k r_cut/(K-1),
 *     and the cosine envelope C(d) = (cos(pi d / r_cut) + 1) / 2 (§4.2 "Fused forward
 *     operator": the envelope multiplies the basis, the filter network reads the product);
 *   - w_e = MLP_filter(b~_e) = W2 ssp(W1 b~_e + b1) + b2  (§3.2 "Filter network");
 *   - h_i = sum_{e: dst[e]=i} x_src[e] (.) w_e  (§3.2 "CFConv message passing and
 *     aggregation"; §4 "Computation targeted by FlashSchNet");
 *   - x^{t+1}_i = x^t_i + U2 ssp(U1 h_i + c1) + c2  (§3.2: point-wise update network with a
 *     residual connection), repeated for T blocks;
 *   - eps_i = MLP_out(x^T_i) = R2 ssp(R1 x^T_i + e1) + e2, E_r = sum of eps_i over replica r
 *     (§3.2 "Energy readout");
 *   - F_i = -dE/dr_i (§3.1, §3.2 "Forces via autodiff"), by hand-written reverse mode.  The
 *     backward aggregation is the source-grouped segmented reduction of §4.3 ("Source grouped
 *     segmented reduction in backward pass"), over an index built by bucket sort on src.
 *   - velocity Verlet integration of the resulting forces.
 * ssp(x) = ln(e^x/2 + 1/2) is the shifted softplus of SchNet (Schutt et al., 2017).
 *
 * Everything is double except the fp32 neighbour test.  Reductions run in a fixed order
 * (rows and source groups in ascending edge order), so results do not depend on the number
 * of OpenMP threads.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC (no FMA contraction:
 * the fp32 neighbour test must round exactly as written).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { SNO_OK = 0, SNO_ERR_ARG = 1, SNO_ERR_CAPACITY = 2, SNO_ERR_NOMEM = 3 };

static const double SNO_PI = 3.14159265358979323846;
static const double SNO_LN2 = 0.69314718055994530942;
static const double SNO_KAPPA = 4.184e-4; /* A^2 fs^-2 per (kcal/mol)/amu */

/* ------------------------------------------------------------------------------------------
 * Neighbour list
 * ---------------------------------------------------------------------------------------- */

/* fp32 edge test: dx = x_j - x_i per axis; for a periodic axis dx -= L * rint(dx / L);
 * r2 = (dx*dx + dy*dy) + dz*dz; edge iff r2 < r_cut*r_cut (all in float, each operation
 * rounded on its own). */
int sno_pair_within(const float *pi, const float *pj, const float *box, float r_cut)
{
    float rc2 = r_cut * r_cut;
    float d[3];
    for (int a = 0; a < 3; ++a) {
        float dx = pj[a] - pi[a];
        if (box[a] > 0.0f) {
            float q = rintf(dx / box[a]);
            float shift = box[a] * q;
            dx = dx - shift;
        }
        d[a] = dx;
    }
    float r2 = d[0] * d[0];
    float yy = d[1] * d[1];
    float zz = d[2] * d[2];
    r2 = r2 + yy;
    r2 = r2 + zz;
    return r2 < rc2;
}

static int check_box(const float *box, float r_cut)
{
    int n_per = 0;
    for (int a = 0; a < 3; ++a) {
        if (box[a] < 0.0f) return SNO_ERR_ARG;
        if (box[a] > 0.0f) {
            ++n_per;
            if (!(r_cut < 0.5f * box[a])) return SNO_ERR_ARG;
        }
    }
    (void)n_per;
    return SNO_OK;
}

/* O(N^2) brute force within each replica.  Rows by destination i ascending, sources j
 * ascending inside a row.  On overflow returns SNO_ERR_CAPACITY with *n_edges = needed. */
int sno_neighbors_brute(int n_per, int n_rep, const float *box, float r_cut, const float *pos,
                        int64_t cap, int32_t *row_ptr, int32_t *col, int64_t *n_edges)
{
    if (n_per < 0 || n_rep < 0 || !(r_cut > 0.0f) || check_box(box, r_cut)) return SNO_ERR_ARG;
    int64_t N = (int64_t)n_per * n_rep;
    int32_t *cnt = (int32_t *)calloc((size_t)N + 1, sizeof(int32_t));
    if (!cnt) return SNO_ERR_NOMEM;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < N; ++i) {
        int64_t r0 = (i / n_per) * n_per;
        int32_t c = 0;
        for (int64_t j = r0; j < r0 + n_per; ++j)
            if (j != i && sno_pair_within(pos + 3 * i, pos + 3 * j, box, r_cut)) ++c;
        cnt[i] = c;
    }
    int64_t total = 0;
    for (int64_t i = 0; i < N; ++i) total += cnt[i];
    *n_edges = total;
    if (total > cap || total > INT32_MAX) { free(cnt); return SNO_ERR_CAPACITY; }
    row_ptr[0] = 0;
    for (int64_t i = 0; i < N; ++i) row_ptr[i + 1] = row_ptr[i] + cnt[i];
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < N; ++i) {
        int64_t r0 = (i / n_per) * n_per;
        int32_t p = row_ptr[i];
        for (int64_t j = r0; j < r0 + n_per; ++j)
            if (j != i && sno_pair_within(pos + 3 * i, pos + 3 * j, box, r_cut)) col[p++] = (int32_t)j;
    }
    free(cnt);
    return SNO_OK;
}

static int cmp_i32(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/* Cell list for a fully periodic box with at least 3 cells per axis (otherwise falls back
 * to the brute force).  Cells have side L/n >= r_cut * (1 + 1e-4); atoms are binned by
 * their coordinate wrapped into [0, L) in double.  Candidates from the 27 surrounding
 * cells go through the same fp32 test; each row is then sorted by source. */
int sno_neighbors_cells(int n_per, int n_rep, const float *box, float r_cut, const float *pos,
                        int64_t cap, int32_t *row_ptr, int32_t *col, int64_t *n_edges)
{
    if (n_per < 0 || n_rep < 0 || !(r_cut > 0.0f) || check_box(box, r_cut)) return SNO_ERR_ARG;
    int nc[3];
    for (int a = 0; a < 3; ++a) {
        if (!(box[a] > 0.0f))
            return sno_neighbors_brute(n_per, n_rep, box, r_cut, pos, cap, row_ptr, col, n_edges);
        nc[a] = (int)floor((double)box[a] / ((double)r_cut * 1.0001));
        if (nc[a] < 3)
            return sno_neighbors_brute(n_per, n_rep, box, r_cut, pos, cap, row_ptr, col, n_edges);
    }
    int64_t N = (int64_t)n_per * n_rep;
    int64_t ncell1 = (int64_t)nc[0] * nc[1] * nc[2];
    int64_t ncell = ncell1 * n_rep;
    int32_t *cell_of = (int32_t *)malloc(sizeof(int32_t) * (size_t)(N ? N : 1));
    int32_t *cstart = (int32_t *)calloc((size_t)ncell + 1, sizeof(int32_t));
    int32_t *catoms = (int32_t *)malloc(sizeof(int32_t) * (size_t)(N ? N : 1));
    int32_t *cnt = (int32_t *)calloc((size_t)N + 1, sizeof(int32_t));
    if (!cell_of || !cstart || !catoms || !cnt) {
        free(cell_of); free(cstart); free(catoms); free(cnt);
        return SNO_ERR_NOMEM;
    }
    for (int64_t i = 0; i < N; ++i) {
        int c3[3];
        for (int a = 0; a < 3; ++a) {
            double L = box[a];
            double x = fmod((double)pos[3 * i + a], L);
            if (x < 0) x += L;
            int c = (int)floor(x / (L / nc[a]));
            if (c >= nc[a]) c = nc[a] - 1;
            if (c < 0) c = 0;
            c3[a] = c;
        }
        cell_of[i] = (int32_t)((i / n_per) * ncell1 + ((int64_t)c3[0] * nc[1] + c3[1]) * nc[2] + c3[2]);
        cstart[cell_of[i] + 1]++;
    }
    for (int64_t c = 0; c < ncell; ++c) cstart[c + 1] += cstart[c];
    {
        int32_t *fill = (int32_t *)malloc(sizeof(int32_t) * (size_t)(ncell ? ncell : 1));
        memcpy(fill, cstart, sizeof(int32_t) * (size_t)ncell);
        for (int64_t i = 0; i < N; ++i) catoms[fill[cell_of[i]]++] = (int32_t)i;
        free(fill);
    }
    /* pass 1: count, pass 2: fill + sort */
    for (int pass = 0; pass < 2; ++pass) {
        if (pass == 1) {
            int64_t total = 0;
            for (int64_t i = 0; i < N; ++i) total += cnt[i];
            *n_edges = total;
            if (total > cap || total > INT32_MAX) {
                free(cell_of); free(cstart); free(catoms); free(cnt);
                return SNO_ERR_CAPACITY;
            }
            row_ptr[0] = 0;
            for (int64_t i = 0; i < N; ++i) row_ptr[i + 1] = row_ptr[i] + cnt[i];
        }
#pragma omp parallel for schedule(dynamic, 16)
        for (int64_t i = 0; i < N; ++i) {
            int64_t rep = i / n_per;
            int64_t lc = cell_of[i] - rep * ncell1;
            int cz = (int)(lc % nc[2]), cy = (int)((lc / nc[2]) % nc[1]), cx = (int)(lc / ((int64_t)nc[1] * nc[2]));
            int32_t c = 0;
            int32_t p = pass ? row_ptr[i] : 0;
            for (int ox = -1; ox <= 1; ++ox)
                for (int oy = -1; oy <= 1; ++oy)
                    for (int oz = -1; oz <= 1; ++oz) {
                        int x = (cx + ox + nc[0]) % nc[0], y = (cy + oy + nc[1]) % nc[1], z = (cz + oz + nc[2]) % nc[2];
                        int64_t cc = rep * ncell1 + ((int64_t)x * nc[1] + y) * nc[2] + z;
                        for (int32_t q = cstart[cc]; q < cstart[cc + 1]; ++q) {
                            int32_t j = catoms[q];
                            if (j == i) continue;
                            if (sno_pair_within(pos + 3 * i, pos + 3 * j, box, r_cut)) {
                                if (pass) col[p++] = j; else ++c;
                            }
                        }
                    }
            if (pass) qsort(col + row_ptr[i], (size_t)(row_ptr[i + 1] - row_ptr[i]), sizeof(int32_t), cmp_i32);
            else cnt[i] = c;
        }
    }
    free(cell_of); free(cstart); free(catoms); free(cnt);
    return SNO_OK;
}

/* ------------------------------------------------------------------------------------------
 * Model
 * ---------------------------------------------------------------------------------------- */

typedef struct {
    const double *W1, *b1, *W2, *b2, *U1, *c1, *U2, *c2;
} block_w;

typedef struct {
    int F, K, T, n_types, H;
    double r_cut, gamma;
    double *buf;
    const double *emb;
    block_w *blk;
    const double *R1, *e1, *R2, *e2;
} model;

/* Blob layout: Emb[n_types][F]; per block W1[F][K] b1[F] W2[F][F] b2[F] U1[F][F] c1[F]
 * U2[F][F] c2[F]; R1[H][F] e1[H] R2[1][H] e2[1]; H = F/2.  Linear: y = W x + b. */
static int64_t blob_size(int F, int K, int T, int n_types)
{
    int64_t H = F / 2;
    int64_t per = (int64_t)F * K + F + 3 * ((int64_t)F * F + F);
    return (int64_t)n_types * F + T * per + H * F + H + H + 1;
}

static int model_load(model *m, const int32_t *dims, double r_cut, double gamma,
                      const float *weights, int64_t n_weights)
{
    m->F = dims[0]; m->K = dims[1]; m->T = dims[2]; m->n_types = dims[3];
    m->H = m->F / 2;
    m->r_cut = r_cut; m->gamma = gamma;
    if (m->F < 2 || m->F % 2 || m->K < 2 || m->T < 0 || m->n_types < 1 || !(r_cut > 0)) return SNO_ERR_ARG;
    if (n_weights != blob_size(m->F, m->K, m->T, m->n_types)) return SNO_ERR_ARG;
    m->buf = (double *)malloc(sizeof(double) * (size_t)n_weights);
    m->blk = (block_w *)malloc(sizeof(block_w) * (size_t)(m->T ? m->T : 1));
    if (!m->buf || !m->blk) { free(m->buf); free(m->blk); return SNO_ERR_NOMEM; }
    for (int64_t q = 0; q < n_weights; ++q) m->buf[q] = (double)weights[q];
    const double *p = m->buf;
    int F = m->F, K = m->K, H = m->H;
    m->emb = p; p += (int64_t)m->n_types * F;
    for (int t = 0; t < m->T; ++t) {
        block_w *b = &m->blk[t];
        b->W1 = p; p += (int64_t)F * K; b->b1 = p; p += F;
        b->W2 = p; p += (int64_t)F * F; b->b2 = p; p += F;
        b->U1 = p; p += (int64_t)F * F; b->c1 = p; p += F;
        b->U2 = p; p += (int64_t)F * F; b->c2 = p; p += F;
    }
    m->R1 = p; p += (int64_t)H * F; m->e1 = p; p += H;
    m->R2 = p; p += H; m->e2 = p; p += 1;
    return SNO_OK;
}

static void model_free(model *m)
{
    free(m->buf);
    free(m->blk);
}

/* shifted softplus ssp(x) = ln(1 + e^x) - ln 2, and its derivative sigma(x) */
static double ssp(double x) { return (x > 0 ? x + log1p(exp(-x)) : log1p(exp(x))) - SNO_LN2; }
static double sigm(double x) { return x >= 0 ? 1.0 / (1.0 + exp(-x)) : exp(x) / (1.0 + exp(x)); }

/* y[n_out] = W[n_out][n_in] x + b */
static void linear(const double *W, const double *b, const double *x, double *y, int n_out, int n_in)
{
    for (int o = 0; o < n_out; ++o) {
        double acc = b ? b[o] : 0.0;
        for (int k = 0; k < n_in; ++k) acc += W[(int64_t)o * n_in + k] * x[k];
        y[o] = acc;
    }
}

/* y[n_in] = W^T[n_in][n_out] x   (W stored [n_out][n_in]) */
static void linear_t(const double *W, const double *x, double *y, int n_out, int n_in)
{
    for (int k = 0; k < n_in; ++k) y[k] = 0.0;
    for (int o = 0; o < n_out; ++o)
        for (int k = 0; k < n_in; ++k) y[k] += W[(int64_t)o * n_in + k] * x[o];
}

/* pair vector u = r_i - r_j (minimum image on periodic axes) and its length */
static double pair_vec(const double *pos, const float *box, int64_t i, int64_t j, double *u)
{
    double r2 = 0.0;
    for (int a = 0; a < 3; ++a) {
        double dx = pos[3 * j + a] - pos[3 * i + a];
        if (box[a] > 0.0f) dx -= (double)box[a] * rint(dx / (double)box[a]);
        u[a] = -dx;
        r2 += dx * dx;
    }
    return sqrt(r2);
}

/* Radial basis with cosine envelope: bt_k = phi_k(d) C(d) and dbt_k = d(bt_k)/dd. */
static void radial_basis(const model *m, double d, double *bt, double *dbt)
{
    double C = 0.5 * (cos(SNO_PI * d / m->r_cut) + 1.0);
    double dC = -0.5 * (SNO_PI / m->r_cut) * sin(SNO_PI * d / m->r_cut);
    for (int k = 0; k < m->K; ++k) {
        double mu = (double)k * m->r_cut / (double)(m->K - 1);
        double phi = exp(-m->gamma * (d - mu) * (d - mu));
        double dphi = -2.0 * m->gamma * (d - mu) * phi;
        bt[k] = phi * C;
        if (dbt) dbt[k] = dphi * C + phi * dC;
    }
}

/* Filter network on one edge: a = W1 bt + b1, s = ssp(a), w = W2 s + b2. */
static void filter_fwd(const model *m, const block_w *bw, const double *bt, double *a, double *s, double *w)
{
    linear(bw->W1, bw->b1, bt, a, m->F, m->K);
    for (int f = 0; f < m->F; ++f) s[f] = ssp(a[f]);
    linear(bw->W2, bw->b2, s, w, m->F, m->F);
}

/* Per-thread scratch for one edge. */
typedef struct {
    double *bt, *dbt, *a, *s, *w, *wbar, *sbar, *abar, *btbar, *hvec, *tmp;
} scratch;

static scratch scratch_new(const model *m)
{
    scratch s;
    int F = m->F, K = m->K;
    double *p = (double *)calloc((size_t)(4 * K + 9 * F), sizeof(double));
    s.bt = p; p += K; s.dbt = p; p += K; s.btbar = p; p += K; p += K;
    s.a = p; p += F; s.s = p; p += F; s.w = p; p += F; s.wbar = p; p += F;
    s.sbar = p; p += F; s.abar = p; p += F; s.hvec = p; p += F; s.tmp = p; p += 2 * F;
    return s;
}

static void scratch_free(scratch *s) { free(s->bt); }

/*
 * Energy and forces at double positions pos[N][3] over a given edge list.
 * energy[n_rep] (kcal/mol), forces[N][3] (kcal/mol/A), eps[N] per-atom energies (optional).
 */
int sno_energy_forces_f64(const int32_t *dims, double r_cut, double gamma,
                          const float *weights, int64_t n_weights,
                          int n_per, int n_rep, const float *box, const double *pos,
                          const int32_t *types, const int32_t *row_ptr, const int32_t *col,
                          int64_t n_edges, double *energy, double *forces, double *eps)
{
    model m;
    int st = model_load(&m, dims, r_cut, gamma, weights, n_weights);
    if (st) return st;
    const int F = m.F, T = m.T, H = m.H;
    const int64_t N = (int64_t)n_per * n_rep, E = n_edges;
    if (N > 0 && row_ptr[N] != E) { model_free(&m); return SNO_ERR_ARG; }
    for (int64_t i = 0; i < N; ++i)
        if (types[i] < 0 || types[i] >= m.n_types) { model_free(&m); return SNO_ERR_ARG; }
    for (int64_t e = 0; e < E; ++e)
        if (col[e] < 0 || col[e] >= N) { model_free(&m); return SNO_ERR_ARG; }

    /* destination of each edge */
    int32_t *dst = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E ? E : 1));
    for (int64_t i = 0; i < N; ++i)
        for (int64_t e = row_ptr[i]; e < row_ptr[i + 1]; ++e) dst[e] = (int32_t)i;
    /* source-grouped index: bucket sort of the edges on src, stable in e */
    int32_t *sptr = (int32_t *)calloc((size_t)N + 1, sizeof(int32_t));
    int32_t *sedge = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E ? E : 1));
    for (int64_t e = 0; e < E; ++e) sptr[col[e] + 1]++;
    for (int64_t i = 0; i < N; ++i) sptr[i + 1] += sptr[i];
    {
        int32_t *fill = (int32_t *)malloc(sizeof(int32_t) * (size_t)(N ? N : 1));
        if (N) memcpy(fill, sptr, sizeof(int32_t) * (size_t)N);
        for (int64_t e = 0; e < E; ++e) sedge[fill[col[e]]++] = (int32_t)e;
        free(fill);
    }

    double *x = (double *)malloc(sizeof(double) * (size_t)((T + 1) * N * F + 1));   /* x^t, t=0..T */
    double *pp = (double *)malloc(sizeof(double) * (size_t)(T * N * F + 1));        /* p^t = U1 h + c1 */
    double *o = (double *)malloc(sizeof(double) * (size_t)(N * H + 1));            /* readout hidden */
    double *xbar = (double *)calloc((size_t)(N * F + 1), sizeof(double));
    double *xbar2 = (double *)calloc((size_t)(N * F + 1), sizeof(double));
    double *hbar = (double *)calloc((size_t)(N * F + 1), sizeof(double));
    double *dbar = (double *)calloc((size_t)(E + 1), sizeof(double));
    double *epsv = (double *)malloc(sizeof(double) * (size_t)(N + 1));

    /* embedding */
    for (int64_t i = 0; i < N; ++i)
        memcpy(x + i * F, m.emb + (int64_t)types[i] * F, sizeof(double) * F);

    /* ---- forward: T interaction blocks ---- */
    for (int t = 0; t < T; ++t) {
        const block_w *bw = &m.blk[t];
        const double *xt = x + (int64_t)t * N * F;
        double *xn = x + (int64_t)(t + 1) * N * F;
        double *pt = pp + (int64_t)t * N * F;
#pragma omp parallel
        {
            scratch sc = scratch_new(&m);
#pragma omp for schedule(dynamic, 8)
            for (int64_t i = 0; i < N; ++i) {
                double *h = sc.hvec;
                for (int f = 0; f < F; ++f) h[f] = 0.0;
                for (int64_t e = row_ptr[i]; e < row_ptr[i + 1]; ++e) {
                    int64_t j = col[e];
                    double u[3];
                    double d = pair_vec(pos, box, i, j, u);
                    radial_basis(&m, d, sc.bt, NULL);
                    filter_fwd(&m, bw, sc.bt, sc.a, sc.s, sc.w);
                    for (int f = 0; f < F; ++f) h[f] += xt[j * F + f] * sc.w[f];
                }
                linear(bw->U1, bw->c1, h, pt + i * F, F, F);
                for (int f = 0; f < F; ++f) sc.tmp[f] = ssp(pt[i * F + f]);
                linear(bw->U2, bw->c2, sc.tmp, sc.tmp + F, F, F);
                for (int f = 0; f < F; ++f) xn[i * F + f] = xt[i * F + f] + sc.tmp[F + f];
            }
            scratch_free(&sc);
        }
    }

    /* ---- readout ---- */
    const double *xT = x + (int64_t)T * N * F;
    for (int64_t i = 0; i < N; ++i) {
        linear(m.R1, m.e1, xT + i * F, o + i * H, H, F);
        double acc = m.e2[0];
        for (int k = 0; k < H; ++k) acc += m.R2[k] * ssp(o[i * H + k]);
        epsv[i] = acc;
    }
    for (int r = 0; r < n_rep; ++r) {
        double acc = 0.0;
        for (int64_t i = (int64_t)r * n_per; i < (int64_t)(r + 1) * n_per; ++i) acc += epsv[i];
        energy[r] = acc;
    }
    if (eps) memcpy(eps, epsv, sizeof(double) * (size_t)N);

    /* ---- backward ---- */
    /* readout: obar = R2 (.) sigma(o), xbar^T = R1^T obar */
    double *ob = (double *)malloc(sizeof(double) * (size_t)H);
    for (int64_t i = 0; i < N; ++i) {
        for (int k = 0; k < H; ++k) ob[k] = m.R2[k] * sigm(o[i * H + k]);
        linear_t(m.R1, ob, xbar + i * F, H, F);
    }
    free(ob);
    for (int t = T - 1; t >= 0; --t) {
        const block_w *bw = &m.blk[t];
        const double *xt = x + (int64_t)t * N * F;
        const double *pt = pp + (int64_t)t * N * F;
        /* update network: qbar = U2^T xbar, pbar = qbar (.) sigma(p), hbar = U1^T pbar */
#pragma omp parallel
        {
            scratch sc = scratch_new(&m);
#pragma omp for schedule(static)
            for (int64_t i = 0; i < N; ++i) {
                linear_t(bw->U2, xbar + i * F, sc.tmp, F, F);
                for (int f = 0; f < F; ++f) sc.tmp[f] *= sigm(pt[i * F + f]);
                linear_t(bw->U1, sc.tmp, hbar + i * F, F, F);
            }
            scratch_free(&sc);
        }
        /* edges, grouped by source j: xbar^t_j = xbar^{t+1}_j + sum_{e: src=j} hbar_dst (.) w_e,
         * and per edge: wbar = hbar_dst (.) x_src, sbar = W2^T wbar, abar = sbar (.) sigma(a),
         * btbar = W1^T abar, dbar_e += sum_k btbar_k d(bt_k)/dd */
#pragma omp parallel
        {
            scratch sc = scratch_new(&m);
#pragma omp for schedule(dynamic, 8)
            for (int64_t j = 0; j < N; ++j) {
                double *acc = xbar2 + j * F;
                for (int f = 0; f < F; ++f) acc[f] = xbar[j * F + f];
                for (int64_t q = sptr[j]; q < sptr[j + 1]; ++q) {
                    int64_t e = sedge[q];
                    int64_t i = dst[e];
                    double u[3];
                    double d = pair_vec(pos, box, i, j, u);
                    radial_basis(&m, d, sc.bt, sc.dbt);
                    filter_fwd(&m, bw, sc.bt, sc.a, sc.s, sc.w);
                    for (int f = 0; f < F; ++f) acc[f] += hbar[i * F + f] * sc.w[f];
                    for (int f = 0; f < F; ++f) sc.wbar[f] = hbar[i * F + f] * xt[j * F + f];
                    linear_t(bw->W2, sc.wbar, sc.sbar, F, F);
                    for (int f = 0; f < F; ++f) sc.abar[f] = sc.sbar[f] * sigm(sc.a[f]);
                    linear_t(bw->W1, sc.abar, sc.btbar, F, m.K);
                    double db = 0.0;
                    for (int k = 0; k < m.K; ++k) db += sc.btbar[k] * sc.dbt[k];
                    dbar[e] += db;
                }
            }
            scratch_free(&sc);
        }
        double *tmpp = xbar; xbar = xbar2; xbar2 = tmpp;
    }

    /* forces: dE/dr_i = sum_{e: dst=i} dbar_e u_e/d_e - sum_{e: src=i} dbar_e u_e/d_e */
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i) {
        double g[3] = {0.0, 0.0, 0.0};
        for (int64_t e = row_ptr[i]; e < row_ptr[i + 1]; ++e) {
            double u[3];
            double d = pair_vec(pos, box, i, col[e], u);
            for (int a = 0; a < 3; ++a) g[a] += dbar[e] * u[a] / d;
        }
        for (int64_t q = sptr[i]; q < sptr[i + 1]; ++q) {
            int64_t e = sedge[q];
            double u[3];
            double d = pair_vec(pos, box, dst[e], i, u);
            for (int a = 0; a < 3; ++a) g[a] -= dbar[e] * u[a] / d;
        }
        for (int a = 0; a < 3; ++a) forces[3 * i + a] = -g[a];
    }

    free(dst); free(sptr); free(sedge); free(x); free(pp); free(o);
    free(xbar); free(xbar2); free(hbar); free(dbar); free(epsv);
    model_free(&m);
    return SNO_OK;
}

/* Same with float positions (the hot path's input type), promoted to double. */
int sno_energy_forces(const int32_t *dims, double r_cut, double gamma,
                      const float *weights, int64_t n_weights,
                      int n_per, int n_rep, const float *box, const float *pos,
                      const int32_t *types, const int32_t *row_ptr, const int32_t *col,
                      int64_t n_edges, double *energy, double *forces, double *eps)
{
    int64_t N = (int64_t)n_per * n_rep;
    double *p = (double *)malloc(sizeof(double) * (size_t)(3 * N + 1));
    if (!p) return SNO_ERR_NOMEM;
    for (int64_t q = 0; q < 3 * N; ++q) p[q] = (double)pos[q];
    int st = sno_energy_forces_f64(dims, r_cut, gamma, weights, n_weights, n_per, n_rep, box, p,
                                   types, row_ptr, col, n_edges, energy, forces, eps);
    free(p);
    return st;
}

/* ------------------------------------------------------------------------------------------
 * Velocity Verlet (NVE):  v += dt/2 kappa F/m;  r += dt v;  rebuild list;  F = F(r);
 * v += dt/2 kappa F/m.  State in double; the list is built from the positions rounded to
 * float (the list's own test is fp32).  forces: in F(t0), out F(t_end).
 * epot[n_steps][n_rep], ekin[n_steps][n_rep] after each step (kcal/mol), optional.
 * ---------------------------------------------------------------------------------------- */
int sno_md_vv(const int32_t *dims, double r_cut, double gamma, const float *weights, int64_t n_weights,
              int n_per, int n_rep, const float *box, double *pos, double *vel, double *forces,
              const int32_t *types, double mass, double dt, int n_steps,
              double *epot, double *ekin, int64_t *n_edges_last)
{
    int64_t N = (int64_t)n_per * n_rep;
    if (!(mass > 0) || n_steps < 0) return SNO_ERR_ARG;
    int64_t cap = 64 * N + 64;
    int32_t *row_ptr = (int32_t *)malloc(sizeof(int32_t) * (size_t)(N + 1));
    int32_t *col = (int32_t *)malloc(sizeof(int32_t) * (size_t)cap);
    float *pf = (float *)malloc(sizeof(float) * (size_t)(3 * N + 1));
    double *en = (double *)malloc(sizeof(double) * (size_t)(n_rep + 1));
    const double c = 0.5 * dt * SNO_KAPPA / mass;
    int st = SNO_OK;
    for (int s = 0; s < n_steps && st == SNO_OK; ++s) {
        for (int64_t q = 0; q < 3 * N; ++q) {
            vel[q] += c * forces[q];
            pos[q] += dt * vel[q];
        }
        for (int64_t q = 0; q < 3 * N; ++q) pf[q] = (float)pos[q];
        int64_t E = 0;
        for (;;) {
            int periodic = box[0] > 0 && box[1] > 0 && box[2] > 0;
            st = periodic ? sno_neighbors_cells(n_per, n_rep, box, (float)r_cut, pf, cap, row_ptr, col, &E)
                          : sno_neighbors_brute(n_per, n_rep, box, (float)r_cut, pf, cap, row_ptr, col, &E);
            if (st != SNO_ERR_CAPACITY) break;
            cap = E + E / 2 + 64;
            free(col);
            col = (int32_t *)malloc(sizeof(int32_t) * (size_t)cap);
        }
        if (st) break;
        if (n_edges_last) *n_edges_last = E;
        st = sno_energy_forces_f64(dims, r_cut, gamma, weights, n_weights, n_per, n_rep, box, pos,
                                   types, row_ptr, col, E, en, forces, NULL);
        if (st) break;
        for (int64_t q = 0; q < 3 * N; ++q) vel[q] += c * forces[q];
        for (int r = 0; r < n_rep; ++r) {
            double ke = 0.0;
            for (int64_t q = (int64_t)r * n_per * 3; q < (int64_t)(r + 1) * n_per * 3; ++q)
                ke += 0.5 * mass * vel[q] * vel[q] / SNO_KAPPA;
            if (epot) epot[(int64_t)s * n_rep + r] = en[r];
            if (ekin) ekin[(int64_t)s * n_rep + r] = ke;
        }
    }
    free(row_ptr); free(col); free(pf); free(en);
    return st;
}

int sno_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------------------------
 * Langevin dynamics (FlashSchNet §5.1 "Experimental setting": Langevin dynamics at 300 K,
 * 4 fs steps), integrated with the BAOAB splitting (Leimkuhler and Matthews, 2013):
 *   B: v += dt/2 kappa F/m;  A: r += dt/2 v;
 *   O: v = a v + b xi,  a = exp(-friction dt),  b = sqrt((1 - a^2) kB T kappa / m);
 *   A: r += dt/2 v;  rebuild the list;  F = F(r);  B: v += dt/2 kappa F/m.
 * xi for (step s, atom i) comes from Philox4x32-10 (Salmon, Moraes, Dror and Shaw, 2011) with
 * counter (s mod 2^32, s / 2^32, i, 0) and key (seed mod 2^32, seed / 2^32): its four 32-bit
 * words u_q = (r_q + 1/2) / 2^32 give xi_x, xi_y = sqrt(-2 ln u0) (cos, sin)(2 pi u1) and
 * xi_z = sqrt(-2 ln u2) cos(2 pi u3) (Box-Muller).
 * ---------------------------------------------------------------------------------------- */

/* Philox4x32 with 10 rounds: each round multiplies words 0 and 2 by the two round constants
 * (64-bit products), recombines the halves with words 1 and 3 and the key, and the key is
 * advanced by the two Weyl constants between rounds. */
void sno_philox4x32_10(const uint32_t *ctr, const uint32_t *key, uint32_t *out)
{
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        const uint64_t p0 = (uint64_t)0xD2511F53u * c0;
        const uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
        const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
        const uint32_t n1 = (uint32_t)p1;
        const uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
        const uint32_t n3 = (uint32_t)p0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* the three standard normal deviates of (step, atom) */
void sno_langevin_noise(uint64_t seed, int64_t step, int64_t atom, double *xi)
{
    const uint32_t ctr[4] = {(uint32_t)step, (uint32_t)((uint64_t)step >> 32), (uint32_t)atom, 0u};
    const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t r[4];
    sno_philox4x32_10(ctr, key, r);
    double u[4];
    for (int q = 0; q < 4; ++q) u[q] = ((double)r[q] + 0.5) / 4294967296.0;
    const double rad0 = sqrt(-2.0 * log(u[0])), rad2 = sqrt(-2.0 * log(u[2]));
    xi[0] = rad0 * cos(2.0 * SNO_PI * u[1]);
    xi[1] = rad0 * sin(2.0 * SNO_PI * u[1]);
    xi[2] = rad2 * cos(2.0 * SNO_PI * u[3]);
}

int sno_md_langevin(const int32_t *dims, double r_cut, double gamma, const float *weights, int64_t n_weights,
                    int n_per, int n_rep, const float *box, double *pos, double *vel, double *forces,
                    const int32_t *types, double mass, double dt, int n_steps, double temperature,
                    double friction, uint64_t seed, int64_t step0, double *epot, double *ekin)
{
    int64_t N = (int64_t)n_per * n_rep;
    if (!(mass > 0) || n_steps < 0 || !(temperature >= 0) || !(friction >= 0)) return SNO_ERR_ARG;
    int64_t cap = 64 * N + 64;
    int32_t *row_ptr = (int32_t *)malloc(sizeof(int32_t) * (size_t)(N + 1));
    int32_t *col = (int32_t *)malloc(sizeof(int32_t) * (size_t)cap);
    float *pf = (float *)malloc(sizeof(float) * (size_t)(3 * N + 1));
    double *en = (double *)malloc(sizeof(double) * (size_t)(n_rep + 1));
    const double c = 0.5 * dt * SNO_KAPPA / mass;
    const double kB = 0.0019872041;
    const double a = exp(-friction * dt);
    const double b = sqrt((1.0 - a * a) * kB * temperature * SNO_KAPPA / mass);
    int st = SNO_OK;
    for (int s = 0; s < n_steps && st == SNO_OK; ++s) {
        for (int64_t i = 0; i < N; ++i) {
            double xi[3];
            sno_langevin_noise(seed, step0 + s, i, xi);
            for (int d = 0; d < 3; ++d) {
                const int64_t q = 3 * i + d;
                vel[q] += c * forces[q];
                pos[q] += 0.5 * dt * vel[q];
                vel[q] = a * vel[q] + b * xi[d];
                pos[q] += 0.5 * dt * vel[q];
            }
        }
        for (int64_t q = 0; q < 3 * N; ++q) pf[q] = (float)pos[q];
        int64_t E = 0;
        for (;;) {
            int periodic = box[0] > 0 && box[1] > 0 && box[2] > 0;
            st = periodic ? sno_neighbors_cells(n_per, n_rep, box, (float)r_cut, pf, cap, row_ptr, col, &E)
                          : sno_neighbors_brute(n_per, n_rep, box, (float)r_cut, pf, cap, row_ptr, col, &E);
            if (st != SNO_ERR_CAPACITY) break;
            cap = E + E / 2 + 64;
            free(col);
            col = (int32_t *)malloc(sizeof(int32_t) * (size_t)cap);
        }
        if (st) break;
        st = sno_energy_forces_f64(dims, r_cut, gamma, weights, n_weights, n_per, n_rep, box, pos,
                                   types, row_ptr, col, E, en, forces, NULL);
        if (st) break;
        for (int64_t q = 0; q < 3 * N; ++q) vel[q] += c * forces[q];
        for (int r = 0; r < n_rep; ++r) {
            double ke = 0.0;
            for (int64_t q = (int64_t)r * n_per * 3; q < (int64_t)(r + 1) * n_per * 3; ++q)
                ke += 0.5 * mass * vel[q] * vel[q] / SNO_KAPPA;
            if (epot) epot[(int64_t)s * n_rep + r] = en[r];
            if (ekin) ekin[(int64_t)s * n_rep + r] = ke;
        }
    }
    free(row_ptr); free(col); free(pf); free(en);
    return st;
}
