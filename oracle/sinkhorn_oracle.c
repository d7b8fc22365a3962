/*
 * CPU oracle for banded log-domain Sinkhorn attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the graft smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or helper
 * with the CUDA library.
 *
 * What it computes (one problem = one (batch, head) pair), all in double:
 *
 *   S_ij = <q_i, k_j> / (sqrt(d) * eps)    on the band support
 *   Omega = {(i, j) : |i - j| <= W, token i and token j both valid}.
 *   (Block-Wise Differentiable Sinkhorn Attention, gist.science/de technical
 *   summary, section 2.1: the support is a fixed band of half-width W and the
 *   temperature eps is folded into the scores.)
 *
 *   Stopped base: v = 0; T times { u <- -LSE_j(S + v); v <- -LSE_i(S + u) };
 *   (u0, v0) = (u, v), held constant under differentiation (section 2.1).
 *   Tail: for r = 1..R: u^(r) = -LSE_j(S + v^(r-1)), v^(r) = -LSE_i(S + u^(r)),
 *   started from the stopped base (section 2.1).
 *   Output O = P^(R,R) V with P^(a,b)_ij = exp(S_ij + u^(a)_i + v^(b)_j).
 *
 *   Backward for an arbitrary cotangent dO, by reverse mode through the tail:
 *   the staircase plans P^(R,R), P^(R,R-1), ..., P^(1,0) (for R = 2 the four
 *   factors P^(2,2), P^(2,1), P^(1,1), P^(1,0) of section 2.2), each one formed
 *   by its own exponential ("direct" schedule), and the one-reference schedule
 *   that forms only P^(R,R) and rescales it with the transport-orbit identity
 *   P^(a,b) = P^(R,R) * exp(u^(a) - u^(R)) * exp(v^(b) - v^(R)) (section 2.2).
 *
 *   Dustbin support (section 2.3: the dustbin path is the same surrogate on
 *   an enlarged state space, one learned dustbin token added): one
 *   extra row and one extra column, index L in every dual vector, with the
 *   constant score dustbin_score on every dustbin entry (i, dustbin),
 *   (dustbin, j) and on the corner, and unit target mass like every other row
 *   and column.  Its value vector v_dust enters O; its query row is not an
 *   output (its cotangent is zero).
 *
 * Readings where the pages are silent (each one is listed in the design
 * notes): one iteration is a u-update followed by a v-update; the base starts
 * from v = 0; T = 0 means u0 = v0 = 0; the dustbin score is used as given (it
 * is not divided by eps); masked tokens have zero duals, outputs and
 * gradients.
 *
 * Layouts: q, k, v, o, dO, dq, dk, dv are [L][d] row-major.  The band score
 * matrix is [L][2W+1] with entry (i, t) holding S(i, i - W + t); entries
 * outside Omega hold -INFINITY.  The dual state is [(2R+2)][L + dustbin]:
 * row 2r is u^(r), row 2r+1 is v^(r), r = 0..R.
 *
 * Each pass parallelises over rows (or columns) with OpenMP; every individual
 * sum is sequential in index order, so results do not depend on the thread
 * count.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int L;              /* sequence length (tokens, including padding) */
    int d;              /* head dimension */
    int W;              /* band half-width, >= 0 */
    int T;              /* stopped base iterations, >= 0 */
    int R;              /* tail iterations, >= 1 */
    double eps;         /* entropic temperature, > 0 */
    int dustbin;        /* 0 or 1 */
    double dustbin_score;
} orc_params;

/* ------------------------------------------------------------------------ */
/* small helpers                                                            */
/* ------------------------------------------------------------------------ */

static int band_w(const orc_params* p) { return 2 * p->W + 1; }
static int nd(const orc_params* p) { return p->L + (p->dustbin ? 1 : 0); }

static int valid(const unsigned char* mask, int i) { return mask == NULL || mask[i] != 0; }

/* log(sum(exp(x))) over n values, shifted by the maximum; -inf if empty. */
static double lse(const double* x, int n) {
    double m = -INFINITY;
    for (int t = 0; t < n; ++t)
        if (x[t] > m) m = x[t];
    if (m == -INFINITY) return -INFINITY;
    double s = 0.0;
    for (int t = 0; t < n; ++t) s += exp(x[t] - m);
    return m + log(s);
}

/* S on the band (section 2.1 of the technical summary). */
static void scores(const orc_params* p, const double* q, const double* k,
                   const unsigned char* mask, double* S) {
    const int L = p->L, d = p->d, W = p->W, bw = band_w(p);
    const double c = 1.0 / (sqrt((double)d) * p->eps);
#pragma omp parallel for schedule(static)
    for (int i = 0; i < L; ++i) {
        for (int t = 0; t < bw; ++t) {
            int j = i - W + t;
            double s = -INFINITY;
            if (j >= 0 && j < L && valid(mask, i) && valid(mask, j)) {
                double acc = 0.0;
                for (int e = 0; e < d; ++e) acc += q[(size_t)i * d + e] * k[(size_t)j * d + e];
                s = c * acc;
            }
            S[(size_t)i * bw + t] = s;
        }
    }
}

static long long support_size(const orc_params* p, const unsigned char* mask) {
    long long n = 0, cnt = 0;
    for (int i = 0; i < p->L; ++i) {
        if (!valid(mask, i)) continue;
        ++n;
        for (int j = i - p->W; j <= i + p->W; ++j)
            if (j >= 0 && j < p->L && valid(mask, j)) ++cnt;
    }
    if (p->dustbin) cnt += 2 * n + 1;
    return cnt;
}

/* u_i = -LSE_j (S_ij + v_j) over row i of the (augmented) support. */
static void row_update(const orc_params* p, const double* S, const unsigned char* mask,
                       const double* v, double* u, long long* visits) {
    const int L = p->L, W = p->W, bw = band_w(p);
    const double sd = p->dustbin_score;
    long long cnt = 0;
#pragma omp parallel for schedule(static) reduction(+ : cnt)
    for (int i = 0; i < L; ++i) {
        if (!valid(mask, i)) { u[i] = 0.0; continue; }
        double x[bw + 1];
        int n = 0;
        for (int t = 0; t < bw; ++t) {
            double s = S[(size_t)i * bw + t];
            if (s == -INFINITY) continue;
            x[n++] = s + v[i - W + t];
        }
        if (p->dustbin) x[n++] = sd + v[L];
        cnt += n;
        u[i] = -lse(x, n);
    }
    if (p->dustbin) {
        double* x = (double*)malloc(sizeof(double) * (size_t)(L + 1));
        int n = 0;
        for (int j = 0; j < L; ++j)
            if (valid(mask, j)) x[n++] = sd + v[j];
        x[n++] = sd + v[L];
        cnt += n;
        u[L] = -lse(x, n);
        free(x);
    }
    if (visits) *visits += cnt;
}

/* v_j = -LSE_i (S_ij + u_i) over column j of the (augmented) support. */
static void col_update(const orc_params* p, const double* S, const unsigned char* mask,
                       const double* u, double* v, long long* visits) {
    const int L = p->L, W = p->W, bw = band_w(p);
    const double sd = p->dustbin_score;
    long long cnt = 0;
#pragma omp parallel for schedule(static) reduction(+ : cnt)
    for (int j = 0; j < L; ++j) {
        if (!valid(mask, j)) { v[j] = 0.0; continue; }
        double x[bw + 1];
        int n = 0;
        for (int i = j - W; i <= j + W; ++i) {
            if (i < 0 || i >= L) continue;
            double s = S[(size_t)i * bw + (j - i + W)];
            if (s == -INFINITY) continue;
            x[n++] = s + u[i];
        }
        if (p->dustbin) x[n++] = sd + u[L];
        cnt += n;
        v[j] = -lse(x, n);
    }
    if (p->dustbin) {
        double* x = (double*)malloc(sizeof(double) * (size_t)(L + 1));
        int n = 0;
        for (int i = 0; i < L; ++i)
            if (valid(mask, i)) x[n++] = sd + u[i];
        x[n++] = sd + u[L];
        cnt += n;
        v[L] = -lse(x, n);
        free(x);
    }
    if (visits) *visits += cnt;
}

/* Plan P^(a,b) = exp(S + u^(a) + v^(b)) on the support, 0 elsewhere.
 * band: [L][2W+1]; dcol: [L] entries (i, dustbin); drow: [L+1] entries
 * (dustbin, j) with drow[L] the corner.  dcol/drow only when dustbin. */
static void plan(const orc_params* p, const double* S, const unsigned char* mask,
                 const double* ua, const double* vb, double* band, double* dcol, double* drow) {
    const int L = p->L, W = p->W, bw = band_w(p);
    const double sd = p->dustbin_score;
#pragma omp parallel for schedule(static)
    for (int i = 0; i < L; ++i) {
        for (int t = 0; t < bw; ++t) {
            double s = S[(size_t)i * bw + t];
            band[(size_t)i * bw + t] = (s == -INFINITY) ? 0.0 : exp(s + ua[i] + vb[i - W + t]);
        }
        if (p->dustbin) dcol[i] = valid(mask, i) ? exp(sd + ua[i] + vb[L]) : 0.0;
    }
    if (p->dustbin) {
        for (int j = 0; j < L; ++j) drow[j] = valid(mask, j) ? exp(sd + ua[L] + vb[j]) : 0.0;
        drow[L] = exp(sd + ua[L] + vb[L]);
    }
}

/* ------------------------------------------------------------------------ */
/* forward                                                                  */
/* ------------------------------------------------------------------------ */

static double* U(const orc_params* p, double* st, int r) { return st + (size_t)(2 * r) * nd(p); }
static double* V(const orc_params* p, double* st, int r) { return st + (size_t)(2 * r + 1) * nd(p); }

/*
 * base_in: NULL for the stopped T-step solve from v = 0, or [2][L+db] holding
 * a frozen (u0, v0) that replaces it (used to differentiate the surrogate by
 * finite differences with the base held fixed).
 * visits: optional counter of support entries visited (exp evaluations).
 */
int orc_forward(const orc_params* p, const double* q, const double* k, const double* v,
                const unsigned char* mask, const double* v_dust, const double* base_in,
                double* o, double* state, long long* visits) {
    if (p->L < 0 || p->d <= 0 || p->W < 0 || p->T < 0 || p->R < 1 || !(p->eps > 0)) return -1;
    const int L = p->L, d = p->d, W = p->W, bw = band_w(p), n = nd(p);
    double* S = (double*)malloc(sizeof(double) * (size_t)L * bw + 1);
    scores(p, q, k, mask, S);

    double* u0 = U(p, state, 0);
    double* v0 = V(p, state, 0);
    if (base_in) {
        memcpy(u0, base_in, sizeof(double) * n);
        memcpy(v0, base_in + n, sizeof(double) * n);
    } else {
        for (int j = 0; j < n; ++j) { u0[j] = 0.0; v0[j] = 0.0; }
        for (int it = 0; it < p->T; ++it) {
            row_update(p, S, mask, v0, u0, visits);
            col_update(p, S, mask, u0, v0, visits);
        }
    }
    for (int r = 1; r <= p->R; ++r) {
        row_update(p, S, mask, V(p, state, r - 1), U(p, state, r), visits);
        col_update(p, S, mask, U(p, state, r), V(p, state, r), visits);
    }

    /* O = P^(R,R) V (+ the dustbin column times v_dust) for valid rows. */
    const double* uR = U(p, state, p->R);
    const double* vR = V(p, state, p->R);
    long long cnt = 0;
#pragma omp parallel for schedule(static) reduction(+ : cnt)
    for (int i = 0; i < L; ++i) {
        double* oi = o + (size_t)i * d;
        for (int e = 0; e < d; ++e) oi[e] = 0.0;
        if (!valid(mask, i)) continue;
        for (int t = 0; t < bw; ++t) {
            double s = S[(size_t)i * bw + t];
            if (s == -INFINITY) continue;
            int j = i - W + t;
            double pij = exp(s + uR[i] + vR[j]);
            ++cnt;
            for (int e = 0; e < d; ++e) oi[e] += pij * v[(size_t)j * d + e];
        }
        if (p->dustbin) {
            double pid = exp(p->dustbin_score + uR[i] + vR[L]);
            ++cnt;
            if (v_dust)
                for (int e = 0; e < d; ++e) oi[e] += pid * v_dust[e];
        }
    }
    if (visits) *visits += cnt;
    free(S);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* backward                                                                 */
/* ------------------------------------------------------------------------ */

typedef struct {      /* one plan on the augmented support */
    double* band;     /* [L][2W+1] */
    double* dcol;     /* [L]   (i, dustbin) */
    double* drow;     /* [L+1] (dustbin, j), corner last */
} plan_t;

static plan_t plan_alloc(const orc_params* p) {
    plan_t P;
    P.band = (double*)calloc((size_t)p->L * band_w(p) + 1, sizeof(double));
    P.dcol = (double*)calloc((size_t)p->L + 1, sizeof(double));
    P.drow = (double*)calloc((size_t)p->L + 2, sizeof(double));
    return P;
}
static void plan_free(plan_t* P) { free(P->band); free(P->dcol); free(P->drow); }

/* y_i = sum_j P_ij x_j over the augmented support (rows 0..L, row L = dustbin). */
static void plan_matvec(const orc_params* p, const unsigned char* mask, const plan_t* P,
                        const double* x, double* y) {
    const int L = p->L, W = p->W, bw = band_w(p);
#pragma omp parallel for schedule(static)
    for (int i = 0; i < L; ++i) {
        double s = 0.0;
        for (int t = 0; t < bw; ++t) {
            int j = i - W + t;
            if (j < 0 || j >= L) continue;
            s += P->band[(size_t)i * bw + t] * x[j];
        }
        if (p->dustbin) s += P->dcol[i] * x[L];
        y[i] = valid(mask, i) ? s : 0.0;
    }
    if (p->dustbin) {
        double s = 0.0;
        for (int j = 0; j <= L; ++j) s += P->drow[j] * x[j];
        y[L] = s;
    }
}

/* y_j = sum_i P_ij x_i over the augmented support (columns 0..L). */
static void plan_rmatvec(const orc_params* p, const unsigned char* mask, const plan_t* P,
                         const double* x, double* y) {
    const int L = p->L, W = p->W, bw = band_w(p);
#pragma omp parallel for schedule(static)
    for (int j = 0; j < L; ++j) {
        double s = 0.0;
        for (int i = j - W; i <= j + W; ++i) {
            if (i < 0 || i >= L) continue;
            s += P->band[(size_t)i * bw + (j - i + W)] * x[i];
        }
        if (p->dustbin) s += P->drow[j] * x[L];
        y[j] = valid(mask, j) ? s : 0.0;
    }
    if (p->dustbin) {
        double s = 0.0;
        for (int i = 0; i < L; ++i) s += P->dcol[i] * x[i];
        s += P->drow[L] * x[L];
        y[L] = s;
    }
}

/* dQ = c dS K and dK = c dS^T Q over the band. */
static void score_vjp(const orc_params* p, const double* q, const double* k, const double* dS,
                      double* dq, double* dk) {
    const int L = p->L, d = p->d, W = p->W, bw = band_w(p);
    const double c = 1.0 / (sqrt((double)d) * p->eps);
#pragma omp parallel for schedule(static)
    for (int i = 0; i < L; ++i) {
        double* g = dq + (size_t)i * d;
        for (int e = 0; e < d; ++e) g[e] = 0.0;
        for (int t = 0; t < bw; ++t) {
            int j = i - W + t;
            if (j < 0 || j >= L) continue;
            double w = dS[(size_t)i * bw + t];
            if (w == 0.0) continue;
            for (int e = 0; e < d; ++e) g[e] += c * w * k[(size_t)j * d + e];
        }
    }
#pragma omp parallel for schedule(static)
    for (int j = 0; j < L; ++j) {
        double* g = dk + (size_t)j * d;
        for (int e = 0; e < d; ++e) g[e] = 0.0;
        for (int i = j - W; i <= j + W; ++i) {
            if (i < 0 || i >= L) continue;
            double w = dS[(size_t)i * bw + (j - i + W)];
            if (w == 0.0) continue;
            for (int e = 0; e < d; ++e) g[e] += c * w * q[(size_t)i * d + e];
        }
    }
}

/*
 * Exact reverse mode through the tail (stopped base held constant).
 * schedule 1 = direct: every staircase plan P^(r,r), P^(r,r-1) is formed by
 * its own exponential.  schedule 0 = one-reference: only P^(R,R) is formed;
 * every other plan entry it needs is P^(R,R) times the orbit factors
 * exp(u^(a)_i - u^(R)_i) exp(v^(b)_j - v^(R)_j).
 *
 * G_ij = <dO_i, V_j> (and <dO_i, v_dust> on the dustbin column), A = P^(R,R)*G.
 *   dV_j = sum_i P^(R,R)_ij dO_i,  dv_dust = sum_i P^(R,R)_(i,dustbin) dO_i
 *   vbar^R = colsum(A);  ubar^R = rowsum(A) - P^(R,R) vbar^R
 *   for r = R..2:  vbar^(r-1) = -P^(r,r-1)^T ubar^r;  ubar^(r-1) = -P^(r-1,r-1) vbar^(r-1)
 *   dS = A - P^(R,R)*(1 vbar^R^T) - sum_{r=1..R} P^(r,r-1)*(ubar^r 1^T)
 *          - sum_{r=1..R-1} P^(r,r)*(1 vbar^r^T)
 *   dQ = c dS K;  dK = c dS^T Q.
 * With a dustbin, d_score (if not NULL, two doubles) receives in d_score[0]
 * the cotangent of the dustbin score (section 2.3: one learned dustbin token):
 * the score enters every dustbin entry -- column (i, dustbin), row
 * (dustbin, j) and the corner -- with weight 1, so its cotangent is the sum of
 * dS over those entries, dS as above (A is zero on the dustbin row, which has
 * no output).  d_score[1] = the sum of |dS| over the same entries, the size
 * of what cancels in d_score[0] (an error scale for comparisons).
 */
int orc_backward(const orc_params* p, int schedule, const double* q, const double* k,
                 const double* v, const unsigned char* mask, const double* v_dust,
                 const double* state_in, const double* dO, double* dq, double* dk, double* dv,
                 double* dv_dust, double* d_score, long long* visits) {
    if (p->L < 0 || p->d <= 0 || p->W < 0 || p->R < 1 || !(p->eps > 0)) return -1;
    const int L = p->L, d = p->d, W = p->W, bw = band_w(p), n = nd(p), R = p->R;
    double* state = (double*)state_in; /* read only */
    double* S = (double*)malloc(sizeof(double) * (size_t)L * bw + 1);
    scores(p, q, k, mask, S);
    long long cnt = 0;

    /* the reference plan P^(R,R) */
    plan_t P = plan_alloc(p);
    plan(p, S, mask, U(p, state, R), V(p, state, R), P.band, P.dcol, P.drow);
    cnt += support_size(p, mask);

    /* G and A on the augmented support (the dustbin query row has dO = 0) */
    plan_t A = plan_alloc(p);
    double* G = (double*)calloc((size_t)L * bw + 1, sizeof(double));
#pragma omp parallel for schedule(static)
    for (int i = 0; i < L; ++i) {
        for (int t = 0; t < bw; ++t) {
            int j = i - W + t;
            if (S[(size_t)i * bw + t] == -INFINITY) continue;
            double g = 0.0;
            for (int e = 0; e < d; ++e) g += dO[(size_t)i * d + e] * v[(size_t)j * d + e];
            G[(size_t)i * bw + t] = g;
            A.band[(size_t)i * bw + t] = P.band[(size_t)i * bw + t] * g;
        }
        if (p->dustbin && valid(mask, i)) {
            double g = 0.0;
            if (v_dust)
                for (int e = 0; e < d; ++e) g += dO[(size_t)i * d + e] * v_dust[e];
            A.dcol[i] = P.dcol[i] * g;
        }
    }

    /* dV and dv_dust */
#pragma omp parallel for schedule(static)
    for (int j = 0; j < L; ++j) {
        double* g = dv + (size_t)j * d;
        for (int e = 0; e < d; ++e) g[e] = 0.0;
        for (int i = j - W; i <= j + W; ++i) {
            if (i < 0 || i >= L) continue;
            double pij = P.band[(size_t)i * bw + (j - i + W)];
            if (pij == 0.0) continue;
            for (int e = 0; e < d; ++e) g[e] += pij * dO[(size_t)i * d + e];
        }
    }
    if (dv_dust) {
        for (int e = 0; e < d; ++e) dv_dust[e] = 0.0;
        if (p->dustbin)
            for (int i = 0; i < L; ++i)
                for (int e = 0; e < d; ++e) dv_dust[e] += P.dcol[i] * dO[(size_t)i * d + e];
    }

    /* vector cotangents ubar^r, vbar^r, r = 1..R, each of length L + db */
    double* ub = (double*)calloc((size_t)(R + 1) * n, sizeof(double));
    double* vb = (double*)calloc((size_t)(R + 1) * n, sizeof(double));
    double* tmp = (double*)calloc((size_t)n, sizeof(double));
    double* ones = (double*)malloc(sizeof(double) * (size_t)n);
    for (int j = 0; j < n; ++j) ones[j] = 1.0;
    double* ubR = ub + (size_t)R * n;
    double* vbR = vb + (size_t)R * n;
    plan_rmatvec(p, mask, &A, ones, vbR);            /* vbar^R = colsum(A) */
    plan_matvec(p, mask, &A, ones, ubR);             /* rowsum(A) */
    plan_matvec(p, mask, &P, vbR, tmp);              /* - P^(R,R) vbar^R */
    for (int i = 0; i < n; ++i) ubR[i] -= tmp[i];
    cnt += support_size(p, mask);

    /* the staircase plans, direct schedule only */
    plan_t* Prr1 = NULL; /* P^(r,r-1), r = 1..R */
    plan_t* Prr = NULL;  /* P^(r,r),   r = 1..R-1 */
    if (schedule == 1) {
        Prr1 = (plan_t*)malloc(sizeof(plan_t) * (size_t)(R + 1));
        Prr = (plan_t*)malloc(sizeof(plan_t) * (size_t)(R + 1));
        for (int r = 1; r <= R; ++r) {
            Prr1[r] = plan_alloc(p);
            plan(p, S, mask, U(p, state, r), V(p, state, r - 1), Prr1[r].band, Prr1[r].dcol,
                 Prr1[r].drow);
            cnt += support_size(p, mask);
        }
        for (int r = 1; r < R; ++r) {
            Prr[r] = plan_alloc(p);
            plan(p, S, mask, U(p, state, r), V(p, state, r), Prr[r].band, Prr[r].dcol,
                 Prr[r].drow);
            cnt += support_size(p, mask);
        }
    }

    /* orbit factors for the one-reference schedule: exp(u^(a) - u^(R)), exp(v^(b) - v^(R)) */
    double* eu = (double*)calloc((size_t)(R + 1) * n, sizeof(double));
    double* ev = (double*)calloc((size_t)(R + 1) * n, sizeof(double));
    for (int a = 0; a <= R; ++a)
        for (int i = 0; i < n; ++i) {
            eu[(size_t)a * n + i] = exp(U(p, state, a)[i] - U(p, state, R)[i]);
            ev[(size_t)a * n + i] = exp(V(p, state, a)[i] - V(p, state, R)[i]);
        }

    for (int r = R; r >= 2; --r) {
        double* ubr = ub + (size_t)r * n;
        double* vbm = vb + (size_t)(r - 1) * n;
        double* ubm = ub + (size_t)(r - 1) * n;
        if (schedule == 1) {
            plan_rmatvec(p, mask, &Prr1[r], ubr, tmp);
            for (int j = 0; j < n; ++j) vbm[j] = -tmp[j];
            plan_matvec(p, mask, &Prr[r - 1], vbm, tmp);
            for (int i = 0; i < n; ++i) ubm[i] = -tmp[i];
        } else {
            /* P^(r,r-1)^T x = ev^(r-1) * (P^(R,R)^T (eu^r * x)) */
            double* x = (double*)malloc(sizeof(double) * (size_t)n);
            for (int i = 0; i < n; ++i) x[i] = eu[(size_t)r * n + i] * ubr[i];
            plan_rmatvec(p, mask, &P, x, tmp);
            for (int j = 0; j < n; ++j) vbm[j] = -ev[(size_t)(r - 1) * n + j] * tmp[j];
            /* P^(r-1,r-1) y = eu^(r-1) * (P^(R,R) (ev^(r-1) * y)) */
            for (int j = 0; j < n; ++j) x[j] = ev[(size_t)(r - 1) * n + j] * vbm[j];
            plan_matvec(p, mask, &P, x, tmp);
            for (int i = 0; i < n; ++i) ubm[i] = -eu[(size_t)(r - 1) * n + i] * tmp[i];
            free(x);
        }
        cnt += 2 * support_size(p, mask);
    }

    /* score cotangent on the band */
    double* dS = (double*)calloc((size_t)L * bw + 1, sizeof(double));
#pragma omp parallel for schedule(static)
    for (int i = 0; i < L; ++i) {
        for (int t = 0; t < bw; ++t) {
            if (S[(size_t)i * bw + t] == -INFINITY) continue;
            int j = i - W + t;
            size_t idx = (size_t)i * bw + t;
            double g;
            if (schedule == 1) {
                g = A.band[idx] - P.band[idx] * vbR[j];
                for (int r = 1; r <= R; ++r) g -= Prr1[r].band[idx] * ub[(size_t)r * n + i];
                for (int r = 1; r < R; ++r) g -= Prr[r].band[idx] * vb[(size_t)r * n + j];
            } else {
                /* dS = P^(R,R) * M, M = G - vbar^R_j - sum_r eu^r_i ev^(r-1)_j ubar^r_i
                 *                        - sum_{r<R} eu^r_i ev^r_j vbar^r_j */
                double M = G[idx] - vbR[j];
                for (int r = 1; r <= R; ++r)
                    M -= eu[(size_t)r * n + i] * ev[(size_t)(r - 1) * n + j] * ub[(size_t)r * n + i];
                for (int r = 1; r < R; ++r)
                    M -= eu[(size_t)r * n + i] * ev[(size_t)r * n + j] * vb[(size_t)r * n + j];
                g = P.band[idx] * M;
            }
            dS[idx] = g;
        }
    }
    cnt += support_size(p, mask);
    score_vjp(p, q, k, dS, dq, dk);

    /* the dustbin score's cotangent: dS summed over the dustbin entries.  An
     * entry is (row i, column j) with i or j equal to L; pref its P^(R,R) value
     * and a its A value. */
    if (d_score) {
        double g = 0.0, gabs = 0.0;
        if (p->dustbin) {
            for (int e = 0; e < 2 * L + 1; ++e) {
                int i, j;
                double pref, a;
                if (e < L) {            /* column entry (e, dustbin) */
                    if (!valid(mask, e)) continue;
                    i = e; j = L; pref = P.dcol[e]; a = A.dcol[e];
                } else if (e < 2 * L) { /* row entry (dustbin, e - L) */
                    if (!valid(mask, e - L)) continue;
                    i = L; j = e - L; pref = P.drow[j]; a = 0.0;
                } else {                /* the corner */
                    i = L; j = L; pref = P.drow[L]; a = 0.0;
                }
                double ds;
                if (schedule == 1) {
                    ds = a - pref * vbR[j];
                    for (int r = 1; r <= R; ++r) {
                        const double pr = (i == L) ? Prr1[r].drow[j] : Prr1[r].dcol[i];
                        ds -= pr * ub[(size_t)r * n + i];
                    }
                    for (int r = 1; r < R; ++r) {
                        const double pr = (i == L) ? Prr[r].drow[j] : Prr[r].dcol[i];
                        ds -= pr * vb[(size_t)r * n + j];
                    }
                } else {
                    double M = -vbR[j];
                    for (int r = 1; r <= R; ++r)
                        M -= eu[(size_t)r * n + i] * ev[(size_t)(r - 1) * n + j] * ub[(size_t)r * n + i];
                    for (int r = 1; r < R; ++r)
                        M -= eu[(size_t)r * n + i] * ev[(size_t)r * n + j] * vb[(size_t)r * n + j];
                    ds = a + pref * M;
                }
                g += ds;
                gabs += fabs(ds);
            }
        }
        d_score[0] = g;
        d_score[1] = gabs;
    }

    if (visits) *visits += cnt;
    if (schedule == 1) {
        for (int r = 1; r <= R; ++r) plan_free(&Prr1[r]);
        for (int r = 1; r < R; ++r) plan_free(&Prr[r]);
        free(Prr1);
        free(Prr);
    }
    free(eu); free(ev); free(dS); free(ub); free(vb); free(tmp); free(ones);
    free(G);
    plan_free(&A);
    plan_free(&P);
    free(S);
    return 0;
}

/* P^(a,b) on the augmented support, from a finished forward state. */
int orc_plan(const orc_params* p, int a, int b, const double* q, const double* k,
             const unsigned char* mask, const double* state_in, double* band, double* dcol,
             double* drow) {
    if (a < 0 || b < 0 || a > p->R || b > p->R) return -1;
    double* state = (double*)state_in;
    double* S = (double*)malloc(sizeof(double) * (size_t)p->L * band_w(p) + 1);
    scores(p, q, k, mask, S);
    plan(p, S, mask, U(p, state, a), V(p, state, b), band, dcol, drow);
    free(S);
    return 0;
}

/* |Omega| of the augmented support. */
long long orc_support_size(const orc_params* p, const unsigned char* mask) {
    return support_size(p, mask);
}
