/*
 * mlg_oracle.c -- plain, slow, obviously correct CPU oracle of the
 * neighbour-graph hot path.  TEST INFRASTRUCTURE ONLY: only the tests, the
 * smoke check and the benchmark's CPU-baseline leg may load this library.  It
 * shares no code, header, table or constant with the CUDA path.
 *
 * What it computes, and where the pages define it:
 *
 *  - Destination-sorted CSR of all periodic neighbour images within rcut
 *    (deepmd-kit issue "DPA4 .pt2 LAMMPS (C++ AOTI) inference 3-6x slower than
 *    Python (ASE)", Root cause analysis, bottleneck 1: createEdgeTensors()
 *    builds edge indices and edge vectors for every neighbour pair; issue
 *    "NeighborGraph attention is 4-9x slower than dense", Proposed fix: the
 *    destination CSR destination_order / destination_row_ptr).
 *    Brute force: every (destination i, source j) pair, every lattice image S
 *    that can be within rcut, exact fp64 test r^2 < rcut^2.
 *  - Per-centre cap sel / nnei_max (DPA4 issue, Reproduction: sel=181;
 *    NeighborGraph issue, Measurements: repinit nsel 120 / rcut 6, repformer
 *    nsel 40 / rcut 4): when a centre has more in-cutoff neighbours than the
 *    cap, the nearest nnei_max are kept, ties broken by (source, shift).
 *  - Canonical order inside a centre: (source, shift x, shift y, shift z).
 *  - Smooth switch s(r): cosine from r_on to rcut (the "smooth" attention of
 *    the NeighborGraph issue, Measurements: graph smooth / dense smooth).
 *    cos(pi u) is evaluated by this file's own Taylor series of sin, so that
 *    the value is reproducible bit for bit.
 *  - Block-dense per-centre multi-head attention (NeighborGraph issue,
 *    Proposed fix: dense attention math per centre with per-row masks for the
 *    ragged tails, scattered back to the edge axis): Q = G Wq, K = G Wk,
 *    V = G Wv; per head l_ab = s_a s_b (q_a . k_b) / sqrt(d); softmax over
 *    the centre's real edges b; O_a = sum_b P_ab V_b.
 *  - Slot-occupancy ("smooth") attention (NeighborGraph issue, Numerics note and
 *    "Graph-native alternatives": phantom slots counted in a denominator that
 *    depends on slot occupancy; the weights factor as
 *    w_b = softmax_b * (sum_b e_b / D~)).
 *    Reading: the dense route pads every centre to nnei_max slots with zero
 *    features and zero switch, so a padded slot's logit is exactly 0 and,
 *    unmasked, it enters the softmax denominator; it adds nothing to the
 *    numerator (its value row is 0).  With phi = nnei_max - n phantoms:
 *    m = max(max_b l_ab, 0 if phi > 0), D~ = sum_b e^(l_ab - m) + phi e^(-m),
 *    O_a = sum_b e^(l_ab - m) V_b / D~.
 *  - Verlet-list reuse (DPA4 issue, Proposed optimizations: device tensors
 *    cached across the MD steps in which the neighbour list is unchanged; the
 *    MD engine decides when it changes, by the usual skin criterion, which the
 *    pages leave to the engine): from a candidate list built at rcut + skin
 *    without a cap, each step recomputes every candidate's vector from the
 *    current coordinates, keeps r < rcut, and then applies the cap and the
 *    canonical order, as the full build does.
 *    While no atom has moved skin/2 or more since the list was built, every
 *    pair within rcut is a candidate, so the result equals the full build.
 *  - Local attention, one query per centre (NeighborGraph issue, "Graph-native
 *    alternatives", item 2: LocalAtten maps onto the per-centre CSR segment
 *    with queries = centres and keys = edges): q_i = H_i Wq from the centre's
 *    own feature row, K = G_i Wk, V = G_i Wv from its edges; per head
 *    l_b = s_b (q_i . k_b) / sqrt(d); softmax over b; out_i = sum_b P_b V_b.
 *
 * Build: gcc -std=c11 -O2 -ffp-contract=off -fopenmp -shared -fPIC.
 * No -ffast-math, no contraction: every product and sum below is rounded
 * separately, in the order written.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_ARG (-1)
#define ORC_ERR_MEM (-2)
#define ORC_ERR_ROWPTR (-3)

/* ------------------------------------------------------------------ */
/* Switch function                                                     */
/* ------------------------------------------------------------------ */

/* cos(pi u) written as -sin(pi (u - 1/2)); sin by its Taylor series through
 * x^23, Horner form in x^2.  Coefficient k is (-1)^k / (2k+1)!, obtained by
 * the recurrence c_0 = 1, c_k = -c_{k-1} / ((2k)(2k+1)) with each division
 * rounded to double.  On |x| <= pi/2 the first omitted term is below 1e-20. */
#define ORC_NTAYLOR 12

static void orc_taylor_coeffs(double c[ORC_NTAYLOR]) {
    c[0] = 1.0;
    for (int k = 1; k < ORC_NTAYLOR; ++k) {
        double div = (double)((2 * k) * (2 * k + 1));
        c[k] = -c[k - 1] / div;
    }
}

double oracle_cos_pi(double u) {
    double c[ORC_NTAYLOR];
    orc_taylor_coeffs(c);
    const double pi = 3.141592653589793; /* the double nearest pi */
    double t = u - 0.5;
    double x = pi * t;
    double x2 = x * x;
    double p = c[ORC_NTAYLOR - 1];
    for (int k = ORC_NTAYLOR - 2; k >= 0; --k) {
        double q = x2 * p;
        p = c[k] + q;
    }
    double sinx = x * p;
    return -sinx;
}

/* s(r) = 1 for r < r_on; 0 for r >= rcut; otherwise 0.5 (1 + cos(pi u)) with
 * u = (r - r_on) / (rcut - r_on).  Written as 0.5 * (1 - sin(pi (u - 1/2))). */
double oracle_switch_one(double r, double rcut, double r_on) {
    if (r < r_on) return 1.0;
    if (r >= rcut) return 0.0;
    double num = r - r_on;
    double den = rcut - r_on;
    double u = num / den;
    double c = oracle_cos_pi(u);   /* = -sin(...) */
    double one_plus = 1.0 + c;
    return 0.5 * one_plus;
}

void oracle_switch(int64_t m, const double* r, double rcut, double r_on, double* s) {
    for (int64_t k = 0; k < m; ++k) s[k] = oracle_switch_one(r[k], rcut, r_on);
}

/* ------------------------------------------------------------------ */
/* Geometry                                                            */
/* ------------------------------------------------------------------ */

typedef struct {
    double a[3][3];      /* box rows a1, a2, a3 */
    int pbc[3];
    int any_periodic;
    double recip[3][3];  /* recip[k] = (a_l x a_m) / V, so f_k = x . recip[k] */
    double reach[3];     /* rcut / h_k, h_k = perpendicular height of the cell */
    double rcut, rc2;
} orc_geom;

static void cross3(const double* u, const double* v, double* w) {
    w[0] = u[1] * v[2] - u[2] * v[1];
    w[1] = u[2] * v[0] - u[0] * v[2];
    w[2] = u[0] * v[1] - u[1] * v[0];
}

static int geom_init(orc_geom* g, const double* box, const uint8_t* pbc, double rcut) {
    if (!(rcut > 0.0) || !isfinite(rcut)) return ORC_ERR_ARG;
    g->any_periodic = 0;
    for (int k = 0; k < 3; ++k) {
        g->pbc[k] = pbc[k] ? 1 : 0;
        g->any_periodic |= g->pbc[k];
        for (int c = 0; c < 3; ++c) {
            g->a[k][c] = box[3 * k + c];
            if (!isfinite(g->a[k][c])) return ORC_ERR_ARG;
        }
    }
    g->rcut = rcut;
    g->rc2 = rcut * rcut;
    for (int k = 0; k < 3; ++k) g->reach[k] = 0.0;
    if (!g->any_periodic) return ORC_OK;
    double c12[3], c20[3], c01[3];
    cross3(g->a[1], g->a[2], c12);
    cross3(g->a[2], g->a[0], c20);
    cross3(g->a[0], g->a[1], c01);
    double vol = g->a[0][0] * c12[0] + g->a[0][1] * c12[1] + g->a[0][2] * c12[2];
    if (!(fabs(vol) > 0.0)) return ORC_ERR_ARG;
    const double* cr[3] = {c12, c20, c01};
    for (int k = 0; k < 3; ++k) {
        double nrm = sqrt(cr[k][0] * cr[k][0] + cr[k][1] * cr[k][1] + cr[k][2] * cr[k][2]);
        for (int c = 0; c < 3; ++c) g->recip[k][c] = cr[k][c] / vol;
        double h = fabs(vol) / nrm;
        g->reach[k] = rcut / h;
    }
    return ORC_OK;
}

/* The edge vector of destination i, source j, integer image S:
 *   sh_c = (S_0 a1_c + S_1 a2_c) + S_2 a3_c,   v_c = (x_j,c + sh_c) - x_i,c
 *   r^2  = (v_0 v_0 + v_1 v_1) + v_2 v_2
 * Every product and sum rounded separately, in this order. */
static double edge_vec(const orc_geom* g, const double* xi, const double* xj,
                       const int* S, double* v) {
    double s0 = (double)S[0], s1 = (double)S[1], s2 = (double)S[2];
    for (int c = 0; c < 3; ++c) {
        double p0 = s0 * g->a[0][c];
        double p1 = s1 * g->a[1][c];
        double p2 = s2 * g->a[2][c];
        double sh = p0 + p1;
        sh = sh + p2;
        double xs = xj[c] + sh;
        v[c] = xs - xi[c];
    }
    double r2 = v[0] * v[0];
    double t1 = v[1] * v[1];
    double t2 = v[2] * v[2];
    r2 = r2 + t1;
    r2 = r2 + t2;
    return r2;
}

typedef struct {
    double r2;
    int32_t j;
    int32_t S[3];
} orc_cand;

typedef struct {
    orc_cand* buf;
    int64_t len, cap;
} orc_vec;

static int vec_push(orc_vec* v, orc_cand c) {
    if (v->len == v->cap) {
        int64_t nc = v->cap ? 2 * v->cap : 256;
        orc_cand* nb = (orc_cand*)realloc(v->buf, (size_t)nc * sizeof(orc_cand));
        if (!nb) return ORC_ERR_MEM;
        v->buf = nb;
        v->cap = nc;
    }
    v->buf[v->len++] = c;
    return ORC_OK;
}

/* total order used for truncation: (r^2, j, S_x, S_y, S_z) ascending */
static int cmp_dist(const void* pa, const void* pb) {
    const orc_cand* a = (const orc_cand*)pa;
    const orc_cand* b = (const orc_cand*)pb;
    if (a->r2 < b->r2) return -1;
    if (a->r2 > b->r2) return 1;
    if (a->j != b->j) return a->j < b->j ? -1 : 1;
    for (int k = 0; k < 3; ++k)
        if (a->S[k] != b->S[k]) return a->S[k] < b->S[k] ? -1 : 1;
    return 0;
}

/* canonical order inside a centre: (j, S_x, S_y, S_z) ascending */
static int cmp_canon(const void* pa, const void* pb) {
    const orc_cand* a = (const orc_cand*)pa;
    const orc_cand* b = (const orc_cand*)pb;
    if (a->j != b->j) return a->j < b->j ? -1 : 1;
    for (int k = 0; k < 3; ++k)
        if (a->S[k] != b->S[k]) return a->S[k] < b->S[k] ? -1 : 1;
    return 0;
}

/* Fractional coordinates f_k = x . recip[k] (periodic systems only). */
static double* make_frac(const orc_geom* g, int64_t n, const double* x) {
    double* f = (double*)malloc((size_t)(3 * (n > 0 ? n : 1)) * sizeof(double));
    if (!f) return NULL;
    for (int64_t j = 0; j < n; ++j)
        for (int k = 0; k < 3; ++k)
            f[3 * j + k] = g->any_periodic
                ? x[3 * j] * g->recip[k][0] + x[3 * j + 1] * g->recip[k][1] + x[3 * j + 2] * g->recip[k][2]
                : 0.0;
    return f;
}

/* All in-cutoff (j, S) of destination i, by brute force over every j and
 * every image S whose fractional offset can reach within rcut.  For a
 * periodic axis k, |v . n_k| = h_k |f_k(v)| <= |v|, so an accepted image has
 * |f_k(x_j) - f_k(x_i) + S_k| < rcut / h_k; the range below adds a margin of
 * 1e-6 (fractional units) for rounding and is then checked exactly. */
static int centre_all(const orc_geom* g, int64_t n, const double* x, const double* frac,
                      int64_t i, orc_vec* out) {
    out->len = 0;
    const double* xi = x + 3 * i;
    for (int64_t j = 0; j < n; ++j) {
        const double* xj = x + 3 * j;
        int lo[3] = {0, 0, 0}, hi[3] = {0, 0, 0};
        int skip = 0;
        for (int k = 0; k < 3; ++k) {
            if (!g->pbc[k]) continue;
            double df = frac[3 * j + k] - frac[3 * i + k];
            if (!isfinite(df) || fabs(df) > 1e12) { skip = 1; break; }
            lo[k] = (int)ceil(-df - g->reach[k] - 1e-6);
            hi[k] = (int)floor(-df + g->reach[k] + 1e-6);
            if (lo[k] > hi[k]) { skip = 1; break; }
        }
        if (skip) continue;
        int S[3];
        for (S[0] = lo[0]; S[0] <= hi[0]; ++S[0])
            for (S[1] = lo[1]; S[1] <= hi[1]; ++S[1])
                for (S[2] = lo[2]; S[2] <= hi[2]; ++S[2]) {
                    if (j == i && S[0] == 0 && S[1] == 0 && S[2] == 0) continue;
                    double v[3];
                    double r2 = edge_vec(g, xi, xj, S, v);
                    if (r2 < g->rc2) {
                        orc_cand c;
                        c.r2 = r2;
                        c.j = (int32_t)j;
                        c.S[0] = S[0]; c.S[1] = S[1]; c.S[2] = S[2];
                        if (vec_push(out, c) != ORC_OK) return ORC_ERR_MEM;
                    }
                }
    }
    return ORC_OK;
}

/* The cap and the order of a centre's in-cutoff edges: when there are more
 * than nnei_max, the nnei_max smallest by (r^2, source, shift) are kept; the
 * row is then put in canonical order. */
static void keep_nearest_canonical(orc_vec* buf, int32_t nnei_max) {
    if (buf->len > nnei_max) {
        qsort(buf->buf, (size_t)buf->len, sizeof(orc_cand), cmp_dist);
        buf->len = nnei_max;
    }
    qsort(buf->buf, (size_t)buf->len, sizeof(orc_cand), cmp_canon);
}

/* The kept edges of centre i in canonical order; returns raw count in *raw. */
static int centre_edges(const orc_geom* g, int64_t n, const double* x, const double* frac,
                        int64_t i, int32_t nnei_max, orc_vec* buf, int64_t* raw) {
    int rc = centre_all(g, n, x, frac, i, buf);
    if (rc != ORC_OK) return rc;
    *raw = buf->len;
    keep_nearest_canonical(buf, nnei_max);
    return ORC_OK;
}

static void write_edge(const orc_geom* g, const double* x, int64_t i, const orc_cand* c,
                       double r_on, int32_t* src, int32_t* shift, double* vec,
                       double* dist, double* sw) {
    double v[3];
    double r2 = edge_vec(g, x + 3 * i, x + 3 * (int64_t)c->j, c->S, v);
    double r = sqrt(r2);
    *src = c->j;
    shift[0] = c->S[0]; shift[1] = c->S[1]; shift[2] = c->S[2];
    vec[0] = v[0]; vec[1] = v[1]; vec[2] = v[2];
    *dist = r;
    *sw = oracle_switch_one(r, g->rcut, r_on);
}

static void set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

/* Per-centre kept and raw neighbour counts. */
int oracle_count(int64_t n, const double* coords, const double* box, const uint8_t* pbc,
                 double rcut, int32_t nnei_max, int32_t* n_kept, int64_t* n_raw,
                 int nthreads) {
    orc_geom g;
    if (n < 0 || nnei_max <= 0) return ORC_ERR_ARG;
    int rc = geom_init(&g, box, pbc, rcut);
    if (rc != ORC_OK) return rc;
    double* frac = make_frac(&g, n, coords);
    if (!frac) return ORC_ERR_MEM;
    set_threads(nthreads);
    int err = ORC_OK;
#pragma omp parallel
    {
        orc_vec buf = {0, 0, 0};
#pragma omp for schedule(dynamic, 16)
        for (int64_t i = 0; i < n; ++i) {
            int64_t raw = 0;
            int e = centre_edges(&g, n, coords, frac, i, nnei_max, &buf, &raw);
            if (e != ORC_OK) {
#pragma omp atomic write
                err = e;
            }
            n_kept[i] = (int32_t)buf.len;
            n_raw[i] = raw;
        }
        free(buf.buf);
    }
    free(frac);
    return err;
}

/* Fill the CSR arrays; row_ptr must be the exclusive prefix sum of n_kept. */
int oracle_fill(int64_t n, const double* coords, const double* box, const uint8_t* pbc,
                double rcut, double r_on, int32_t nnei_max, const int64_t* row_ptr,
                int32_t* src, int32_t* shift, double* vec, double* dist, double* sw,
                int nthreads) {
    orc_geom g;
    if (n < 0 || nnei_max <= 0) return ORC_ERR_ARG;
    int rc = geom_init(&g, box, pbc, rcut);
    if (rc != ORC_OK) return rc;
    double* frac = make_frac(&g, n, coords);
    if (!frac) return ORC_ERR_MEM;
    set_threads(nthreads);
    int err = ORC_OK;
#pragma omp parallel
    {
        orc_vec buf = {0, 0, 0};
#pragma omp for schedule(dynamic, 16)
        for (int64_t i = 0; i < n; ++i) {
            int64_t raw = 0;
            int e = centre_edges(&g, n, coords, frac, i, nnei_max, &buf, &raw);
            if (e == ORC_OK && row_ptr[i + 1] - row_ptr[i] != buf.len) e = ORC_ERR_ROWPTR;
            if (e != ORC_OK) {
#pragma omp atomic write
                err = e;
                continue;
            }
            for (int64_t a = 0; a < buf.len; ++a) {
                int64_t p = row_ptr[i] + a;
                write_edge(&g, coords, i, &buf.buf[a], r_on, src + p, shift + 3 * p,
                           vec + 3 * p, dist + p, sw + p);
            }
        }
        free(buf.buf);
    }
    free(frac);
    return err;
}

/* One centre only (for sampled checks of very large systems).  Writes up to
 * `cap` kept edges; returns the kept count (or a negative error), raw count
 * in *n_raw. */
int64_t oracle_centre(int64_t n, const double* coords, const double* box, const uint8_t* pbc,
                      double rcut, double r_on, int32_t nnei_max, int64_t i, int64_t cap,
                      int32_t* src, int32_t* shift, double* vec, double* dist, double* sw,
                      int64_t* n_raw) {
    orc_geom g;
    if (n < 0 || nnei_max <= 0 || i < 0 || i >= n) return ORC_ERR_ARG;
    int rc = geom_init(&g, box, pbc, rcut);
    if (rc != ORC_OK) return rc;
    double* frac = make_frac(&g, n, coords);
    if (!frac) return ORC_ERR_MEM;
    orc_vec buf = {0, 0, 0};
    int64_t raw = 0;
    rc = centre_edges(&g, n, coords, frac, i, nnei_max, &buf, &raw);
    free(frac);
    if (rc != ORC_OK) { free(buf.buf); return rc; }
    *n_raw = raw;
    int64_t m = buf.len < cap ? buf.len : cap;
    for (int64_t a = 0; a < m; ++a)
        write_edge(&g, coords, i, &buf.buf[a], r_on, src + a, shift + 3 * a, vec + 3 * a,
                   dist + a, sw + a);
    int64_t kept = buf.len;
    free(buf.buf);
    return kept;
}

/* ------------------------------------------------------------------ */
/* Verlet-list reuse                                                   */
/* ------------------------------------------------------------------ */

/* The kept edges of centre i chosen from a stored candidate row (source,
 * shift) instead of from every source and image: each candidate's vector is
 * recomputed from the current coordinates by edge_vec, kept if r^2 < rcut^2,
 * the nearest nnei_max kept by (r^2, source, shift), and the row put in
 * canonical order.  Returns the raw count in *raw. */
static int centre_refine(const orc_geom* g, const double* x, int64_t i, const int64_t* cand_ptr,
                         const int32_t* cand_src, const int32_t* cand_shift, int32_t nnei_max,
                         orc_vec* buf, int64_t* raw) {
    buf->len = 0;
    for (int64_t p = cand_ptr[i]; p < cand_ptr[i + 1]; ++p) {
        orc_cand c;
        c.j = cand_src[p];
        c.S[0] = cand_shift[3 * p];
        c.S[1] = cand_shift[3 * p + 1];
        c.S[2] = cand_shift[3 * p + 2];
        double v[3];
        c.r2 = edge_vec(g, x + 3 * i, x + 3 * (int64_t)c.j, c.S, v);
        if (c.r2 < g->rc2)
            if (vec_push(buf, c) != ORC_OK) return ORC_ERR_MEM;
    }
    *raw = buf->len;
    keep_nearest_canonical(buf, nnei_max);
    return ORC_OK;
}

/* Per-centre kept and raw counts from a candidate list (cand_ptr [n+1],
 * cand_src [C], cand_shift [C][3]: the list built at a larger cutoff). */
int oracle_refine_count(int64_t n, const double* coords, const double* box, const uint8_t* pbc,
                        double rcut, int32_t nnei_max, const int64_t* cand_ptr,
                        const int32_t* cand_src, const int32_t* cand_shift, int32_t* n_kept,
                        int64_t* n_raw) {
    orc_geom g;
    if (n < 0 || nnei_max <= 0) return ORC_ERR_ARG;
    int rc = geom_init(&g, box, pbc, rcut);
    if (rc != ORC_OK) return rc;
    orc_vec buf = {0, 0, 0};
    for (int64_t i = 0; i < n && rc == ORC_OK; ++i) {
        int64_t raw = 0;
        rc = centre_refine(&g, coords, i, cand_ptr, cand_src, cand_shift, nnei_max, &buf, &raw);
        n_kept[i] = (int32_t)buf.len;
        n_raw[i] = raw;
    }
    free(buf.buf);
    return rc;
}

/* The CSR arrays from a candidate list; row_ptr must be the exclusive prefix
 * sum of the kept counts. */
int oracle_refine_fill(int64_t n, const double* coords, const double* box, const uint8_t* pbc,
                       double rcut, double r_on, int32_t nnei_max, const int64_t* cand_ptr,
                       const int32_t* cand_src, const int32_t* cand_shift,
                       const int64_t* row_ptr, int32_t* src, int32_t* shift, double* vec,
                       double* dist, double* sw) {
    orc_geom g;
    if (n < 0 || nnei_max <= 0) return ORC_ERR_ARG;
    int rc = geom_init(&g, box, pbc, rcut);
    if (rc != ORC_OK) return rc;
    orc_vec buf = {0, 0, 0};
    for (int64_t i = 0; i < n && rc == ORC_OK; ++i) {
        int64_t raw = 0;
        rc = centre_refine(&g, coords, i, cand_ptr, cand_src, cand_shift, nnei_max, &buf, &raw);
        if (rc == ORC_OK && row_ptr[i + 1] - row_ptr[i] != buf.len) rc = ORC_ERR_ROWPTR;
        for (int64_t a = 0; rc == ORC_OK && a < buf.len; ++a) {
            int64_t p = row_ptr[i] + a;
            write_edge(&g, coords, i, &buf.buf[a], r_on, src + p, shift + 3 * p, vec + 3 * p,
                       dist + p, sw + p);
        }
    }
    free(buf.buf);
    return rc;
}

/* ------------------------------------------------------------------ */
/* Block-dense per-centre attention                                    */
/* ------------------------------------------------------------------ */

/* y = x W for the n rows of one centre: out[a][m] = sum_k x[a][k] W[k][m],
 * summed over k in ascending order. */
static void project(int64_t n, int c, const double* x, const double* W, double* out) {
    for (int64_t a = 0; a < n; ++a)
        for (int m = 0; m < c; ++m) {
            double acc = 0.0;
            for (int k = 0; k < c; ++k) acc = acc + x[a * c + k] * W[(int64_t)k * c + m];
            out[a * c + m] = acc;
        }
}

/* Attention map of one head for one centre: P[a][b], a, b < n. */
static void head_map(int64_t n, int c, int d, int h, const double* s, const double* Q,
                     const double* K, double* P) {
    double rsd = sqrt((double)d);
    for (int64_t a = 0; a < n; ++a) {
        double m = -INFINITY;
        for (int64_t b = 0; b < n; ++b) {
            double dot = 0.0;
            for (int t = 0; t < d; ++t) dot = dot + Q[a * c + h * d + t] * K[b * c + h * d + t];
            double l = ((s[a] * s[b]) * dot) / rsd;
            P[a * n + b] = l;
            if (l > m) m = l;
        }
        double z = 0.0;
        for (int64_t b = 0; b < n; ++b) {
            double e = exp(P[a * n + b] - m);
            P[a * n + b] = e;
            z = z + e;
        }
        for (int64_t b = 0; b < n; ++b) P[a * n + b] = P[a * n + b] / z;
    }
}

/* One attention layer over every centre of the CSR.  G and out are [E][c]
 * row-major in CSR order; W* are [c][c] row-major (y = x W); sw is s(r) per
 * edge.  Rows outside [0, row_ptr[n_centres]) are not touched. */
int oracle_attention(int64_t n_centres, const int64_t* row_ptr, const double* sw, int32_t c,
                     int32_t heads, const double* G, const double* Wq, const double* Wk,
                     const double* Wv, double* out, int nthreads) {
    if (n_centres < 0 || c <= 0 || heads <= 0 || c % heads != 0) return ORC_ERR_ARG;
    int d = c / heads;
    set_threads(nthreads);
    int err = ORC_OK;
#pragma omp parallel
    {
        double *Q = NULL, *K = NULL, *V = NULL, *P = NULL;
        int64_t have = 0;
#pragma omp for schedule(dynamic, 4)
        for (int64_t i = 0; i < n_centres; ++i) {
            int64_t base = row_ptr[i];
            int64_t n = row_ptr[i + 1] - base;
            if (n <= 0) continue;
            if (n > have) {
                free(Q); free(K); free(V); free(P);
                Q = (double*)malloc((size_t)(n * c) * sizeof(double));
                K = (double*)malloc((size_t)(n * c) * sizeof(double));
                V = (double*)malloc((size_t)(n * c) * sizeof(double));
                P = (double*)malloc((size_t)(n * n) * sizeof(double));
                have = n;
                if (!Q || !K || !V || !P) {
#pragma omp atomic write
                    err = ORC_ERR_MEM;
                    have = 0;
                    continue;
                }
            }
            const double* x = G + base * c;
            project(n, c, x, Wq, Q);
            project(n, c, x, Wk, K);
            project(n, c, x, Wv, V);
            for (int h = 0; h < heads; ++h) {
                head_map(n, c, d, h, sw + base, Q, K, P);
                for (int64_t a = 0; a < n; ++a)
                    for (int t = 0; t < d; ++t) {
                        double acc = 0.0;
                        for (int64_t b = 0; b < n; ++b)
                            acc = acc + P[a * n + b] * V[b * c + h * d + t];
                        out[(base + a) * c + h * d + t] = acc;
                    }
            }
        }
        free(Q); free(K); free(V); free(P);
    }
    return err;
}

/* Attention map P[a][b] of centre i, head h (for row-sum and masking pins). */
int oracle_attention_map(const int64_t* row_ptr, const double* sw, int32_t c, int32_t heads,
                         const double* G, const double* Wq, const double* Wk, int64_t i,
                         int32_t h, double* P) {
    if (c <= 0 || heads <= 0 || c % heads != 0 || h < 0 || h >= heads) return ORC_ERR_ARG;
    int d = c / heads;
    int64_t base = row_ptr[i];
    int64_t n = row_ptr[i + 1] - base;
    if (n <= 0) return ORC_OK;
    double* Q = (double*)malloc((size_t)(n * c) * sizeof(double));
    double* K = (double*)malloc((size_t)(n * c) * sizeof(double));
    if (!Q || !K) { free(Q); free(K); return ORC_ERR_MEM; }
    project(n, c, G + base * c, Wq, Q);
    project(n, c, G + base * c, Wk, K);
    head_map(n, c, d, h, sw + base, Q, K, P);
    free(Q); free(K);
    return ORC_OK;
}

/* Local attention over every centre: one query per centre from its own
 * feature row H_i (q_i = H_i Wq), keys and values from its edges (K = G_i Wk,
 * V = G_i Wv); per head h, l_b = s_b (q_i . k_b) / sqrt(d), P = softmax over
 * the centre's edges b, out_i = sum_b P_b V_b, heads concatenated.  The
 * centre has no distance of its own, so only the key's switch s_b weighs the
 * logit.  A centre without edges gets a zero row.  H and out are
 * [n_centres][c], G is [E][c] in CSR order. */
int oracle_local_attention(int64_t n_centres, const int64_t* row_ptr, const double* sw,
                           int32_t c, int32_t heads, const double* H, const double* G,
                           const double* Wq, const double* Wk, const double* Wv, double* out,
                           int nthreads) {
    if (n_centres < 0 || c <= 0 || heads <= 0 || c % heads != 0) return ORC_ERR_ARG;
    int d = c / heads;
    double rsd = sqrt((double)d);
    set_threads(nthreads);
    int err = ORC_OK;
#pragma omp parallel
    {
        double *q = (double*)malloc((size_t)c * sizeof(double));
        double *K = NULL, *V = NULL, *P = NULL;
        int64_t have = 0;
#pragma omp for schedule(dynamic, 16)
        for (int64_t i = 0; i < n_centres; ++i) {
            int64_t base = row_ptr[i];
            int64_t n = row_ptr[i + 1] - base;
            for (int m = 0; m < c; ++m) out[i * c + m] = 0.0;
            if (n <= 0) continue;
            if (n > have) {
                free(K); free(V); free(P);
                K = (double*)malloc((size_t)(n * c) * sizeof(double));
                V = (double*)malloc((size_t)(n * c) * sizeof(double));
                P = (double*)malloc((size_t)n * sizeof(double));
                have = n;
            }
            if (!q || !K || !V || !P) {
#pragma omp atomic write
                err = ORC_ERR_MEM;
                have = 0;
                continue;
            }
            project(1, c, H + i * c, Wq, q);
            project(n, c, G + base * c, Wk, K);
            project(n, c, G + base * c, Wv, V);
            for (int h = 0; h < heads; ++h) {
                double m = -INFINITY;
                for (int64_t b = 0; b < n; ++b) {
                    double dot = 0.0;
                    for (int t = 0; t < d; ++t) dot = dot + q[h * d + t] * K[b * c + h * d + t];
                    double l = (sw[base + b] * dot) / rsd;
                    P[b] = l;
                    if (l > m) m = l;
                }
                double z = 0.0;
                for (int64_t b = 0; b < n; ++b) {
                    double e = exp(P[b] - m);
                    P[b] = e;
                    z = z + e;
                }
                for (int t = 0; t < d; ++t) {
                    double acc = 0.0;
                    for (int64_t b = 0; b < n; ++b) acc = acc + (P[b] / z) * V[b * c + h * d + t];
                    out[i * c + h * d + t] = acc;
                }
            }
        }
        free(q); free(K); free(V); free(P);
    }
    return err;
}

/* Slot-occupancy ("smooth") attention over every centre: as oracle_attention,
 * plus phi = nnei_max - n phantom slots of logit exactly 0 and value 0 in the
 * softmax of every row (the dense route's zero-padded, unmasked slots):
 * m = max(max_b l_ab, 0 if phi > 0), D~ = sum_b e^(l_ab - m) + phi e^(-m),
 * O_a = sum_b e^(l_ab - m) V_b / D~.  Centres with n > nnei_max are an error
 * (phi would be negative). */
int oracle_attention_smooth(int64_t n_centres, const int64_t* row_ptr, const double* sw,
                            int32_t c, int32_t heads, int32_t nnei_max, const double* G,
                            const double* Wq, const double* Wk, const double* Wv, double* out,
                            int nthreads) {
    if (n_centres < 0 || c <= 0 || heads <= 0 || c % heads != 0 || nnei_max < 1)
        return ORC_ERR_ARG;
    for (int64_t i = 0; i < n_centres; ++i)
        if (row_ptr[i + 1] - row_ptr[i] > nnei_max) return ORC_ERR_ARG;
    int d = c / heads;
    double rsd = sqrt((double)d);
    set_threads(nthreads);
    int err = ORC_OK;
#pragma omp parallel
    {
        double *Q = NULL, *K = NULL, *V = NULL, *E = NULL;
        int64_t have = 0;
#pragma omp for schedule(dynamic, 4)
        for (int64_t i = 0; i < n_centres; ++i) {
            int64_t base = row_ptr[i];
            int64_t n = row_ptr[i + 1] - base;
            if (n <= 0) continue;
            if (n > have) {
                free(Q); free(K); free(V); free(E);
                Q = (double*)malloc((size_t)(n * c) * sizeof(double));
                K = (double*)malloc((size_t)(n * c) * sizeof(double));
                V = (double*)malloc((size_t)(n * c) * sizeof(double));
                E = (double*)malloc((size_t)n * sizeof(double));
                have = n;
                if (!Q || !K || !V || !E) {
#pragma omp atomic write
                    err = ORC_ERR_MEM;
                    have = 0;
                    continue;
                }
            }
            const double* x = G + base * c;
            const double* s = sw + base;
            int64_t phi = nnei_max - n;
            project(n, c, x, Wq, Q);
            project(n, c, x, Wk, K);
            project(n, c, x, Wv, V);
            for (int h = 0; h < heads; ++h)
                for (int64_t a = 0; a < n; ++a) {
                    double m = phi > 0 ? 0.0 : -INFINITY;
                    for (int64_t b = 0; b < n; ++b) {
                        double dot = 0.0;
                        for (int t = 0; t < d; ++t)
                            dot = dot + Q[a * c + h * d + t] * K[b * c + h * d + t];
                        double l = ((s[a] * s[b]) * dot) / rsd;
                        E[b] = l;
                        if (l > m) m = l;
                    }
                    double z = 0.0;
                    for (int64_t b = 0; b < n; ++b) {
                        E[b] = exp(E[b] - m);
                        z = z + E[b];
                    }
                    if (phi > 0) z = z + (double)phi * exp(-m);  /* m >= 0 here */
                    for (int t = 0; t < d; ++t) {
                        double acc = 0.0;
                        for (int64_t b = 0; b < n; ++b) acc = acc + (E[b] / z) * V[b * c + h * d + t];
                        out[(base + a) * c + h * d + t] = acc;
                    }
                }
        }
        free(Q); free(K); free(V); free(E);
    }
    return err;
}
