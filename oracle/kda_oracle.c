/*
 * FP64 CPU oracle for the Kimi Delta Attention (KDA) core.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * CPU-baseline leg of bench.py may load this library.  The CUDA library never
 * links, includes or calls it, and it shares no code with the CUDA library.
 *
 * What it computes is the plain token-by-token definition of KDA, in double
 * precision, from the exact input values the GPU receives (bf16/fp32 widened):
 *
 *   preprocessing (each step only if its switch is set; page "KDAAttention 层",
 *   section "chunk_kda 内部做了什么", three in-kernel switches):
 *     q <- q / sqrt(sum q^2 + eps),  k <- k / sqrt(sum k^2 + eps)
 *     beta <- 1 / (1 + exp(-beta_logit))
 *     g <- g_min / (1 + exp(-exp(A_log[hv]) * (z + dt_bias[hv,:])))
 *       (bounded decay, page "KDA 模块交互式演示" section 1.4 Eq. 5 and
 *        page "Implémenter KDA" section "La décroissance bornée")
 *     alpha = exp(g)
 *
 *   recurrence, in the order fixed by page "Implémenter KDA", sections
 *   "La forme récurrente de référence" and "Trois pièges" (decay BEFORE the
 *   delta erase; the output reads the state AFTER the update):
 *     S <- Diag(alpha_t) S
 *     u <- S^T k_t
 *     S <- S + beta_t k_t (v_t - u)^T
 *     o_t <- scale * S^T q_t
 *
 *   cumulative transition (page "Implémenter KDA", "Test 2 - l'identité de
 *   composition"):  M_T = prod_{t=T-1..0} (I - beta_t k_t k_t^T) Diag(alpha_t),
 *   each new factor multiplied on the left.
 *
 *   segment combine (page "KDA 模块交互式演示" section 1.6 KCP, page
 *   "Implémenter KDA" "Test 3 - le balayage préfixe"):
 *     S_in[0] = S_init;  S_in[s+1] = M_s S_in[s] + S_seg[s]
 *
 * Chains (b, hv) are independent; OpenMP runs them in parallel.  Value head hv
 * reads q/k head h = hv / (HV / H) (contiguous groups of value heads share one
 * q/k head).
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int B, T, H, HV, Dk, Dv;
    double g_min, scale, l2_eps;
    int qk_l2norm_in_kernel, beta_sigmoid_in_kernel, gate_in_kernel;
    const double *q;       /* [B,T,H,Dk]  */
    const double *k;       /* [B,T,H,Dk]  */
    const double *v;       /* [B,T,HV,Dv] */
    const double *g;       /* [B,T,HV,Dk]: log-decay g, or raw z when gate_in_kernel */
    const double *beta;    /* [B,T,HV]: beta, or its logit when beta_sigmoid_in_kernel */
    const double *A_log;   /* [HV], read iff gate_in_kernel */
    const double *dt_bias; /* [HV,Dk] or NULL (= 0), read iff gate_in_kernel */
    const double *S0;      /* [B,HV,Dk,Dv] or NULL (= 0) */
    double *o;             /* [B,T,HV,Dv] */
    double *S_T;           /* [B,HV,Dk,Dv] or NULL */
    double *M_T;           /* [B,HV,Dk,Dk] or NULL */
} oracle_kda_args;

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* x / sqrt(sum x^2 + eps) */
static void l2_normalise(const double *x, double *out, int D, double eps) {
    double ss = 0.0;
    for (int c = 0; c < D; ++c) ss += x[c] * x[c];
    double inv = 1.0 / sqrt(ss + eps);
    for (int c = 0; c < D; ++c) out[c] = x[c] * inv;
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* Preprocess one token of one chain into (qn, kn, alpha, beta). */
static void prepare_token(const oracle_kda_args *a, int b, int t, int hv,
                          double *qn, double *kn, double *alpha, double *beta_out) {
    const int H = a->H, HV = a->HV, Dk = a->Dk, T = a->T;
    const int h = hv / (HV / H);
    const double *qs = a->q + (((size_t)b * T + t) * H + h) * Dk;
    const double *ks = a->k + (((size_t)b * T + t) * H + h) * Dk;
    const double *gs = a->g + (((size_t)b * T + t) * HV + hv) * Dk;
    double bt = a->beta[((size_t)b * T + t) * HV + hv];

    if (a->qk_l2norm_in_kernel) {
        l2_normalise(qs, qn, Dk, a->l2_eps);
        l2_normalise(ks, kn, Dk, a->l2_eps);
    } else {
        memcpy(qn, qs, sizeof(double) * Dk);
        memcpy(kn, ks, sizeof(double) * Dk);
    }
    *beta_out = a->beta_sigmoid_in_kernel ? sigmoid(bt) : bt;
    if (a->gate_in_kernel) {
        double ea = exp(a->A_log[hv]);
        for (int c = 0; c < Dk; ++c) {
            double zb = gs[c] + (a->dt_bias ? a->dt_bias[(size_t)hv * Dk + c] : 0.0);
            double g = a->g_min * sigmoid(ea * zb);
            alpha[c] = exp(g);
        }
    } else {
        for (int c = 0; c < Dk; ++c) alpha[c] = exp(gs[c]);
    }
}

/* One recurrence step on a state S [Dk x Dv] (row c = key channel), in the
 * order decay -> erase along k -> write, then read with q. */
static void recurrence_step(double *S, const double *qn, const double *kn,
                            const double *vt, const double *alpha, double beta,
                            double scale, int Dk, int Dv, double *u, double *o_out) {
    for (int c = 0; c < Dk; ++c)
        for (int j = 0; j < Dv; ++j) S[(size_t)c * Dv + j] *= alpha[c];
    for (int j = 0; j < Dv; ++j) u[j] = 0.0;
    for (int c = 0; c < Dk; ++c)
        for (int j = 0; j < Dv; ++j) u[j] += S[(size_t)c * Dv + j] * kn[c];
    for (int c = 0; c < Dk; ++c)
        for (int j = 0; j < Dv; ++j) S[(size_t)c * Dv + j] += beta * kn[c] * (vt[j] - u[j]);
    if (o_out) {
        for (int j = 0; j < Dv; ++j) {
            double acc = 0.0;
            for (int c = 0; c < Dk; ++c) acc += S[(size_t)c * Dv + j] * qn[c];
            o_out[j] = scale * acc;
        }
    }
}

/* M <- (I - beta k k^T) Diag(alpha) M  for M [Dk x Dk].
 * The product with the rank-one-corrected diagonal is expanded exactly:
 * (I - b k k^T) Diag(a) M = Diag(a) M - b k ((a*k)^T M). */
static void transition_left_multiply(double *M, const double *kn, const double *alpha,
                                     double beta, int Dk, double *w) {
    for (int j = 0; j < Dk; ++j) w[j] = 0.0;
    for (int c = 0; c < Dk; ++c)
        for (int j = 0; j < Dk; ++j) w[j] += alpha[c] * kn[c] * M[(size_t)c * Dk + j];
    for (int c = 0; c < Dk; ++c)
        for (int j = 0; j < Dk; ++j)
            M[(size_t)c * Dk + j] = alpha[c] * M[(size_t)c * Dk + j] - beta * kn[c] * w[j];
}

int oracle_kda_fwd(const oracle_kda_args *a) {
    if (!a || a->B < 0 || a->T < 0 || a->H <= 0 || a->HV <= 0 || a->Dk <= 0 || a->Dv <= 0)
        return 1;
    if (a->HV % a->H != 0) return 2;
    if (a->B == 0) return 0;
    const int B = a->B, T = a->T, HV = a->HV, Dk = a->Dk, Dv = a->Dv;
    const int nchains = B * HV;
    int err = 0;

#pragma omp parallel for schedule(dynamic, 1)
    for (int chain = 0; chain < nchains; ++chain) {
        const int b = chain / HV, hv = chain % HV;
        double *S = (double *)calloc((size_t)Dk * Dv, sizeof(double));
        double *M = a->M_T ? (double *)calloc((size_t)Dk * Dk, sizeof(double)) : NULL;
        double *qn = (double *)malloc(sizeof(double) * Dk);
        double *kn = (double *)malloc(sizeof(double) * Dk);
        double *al = (double *)malloc(sizeof(double) * Dk);
        double *u = (double *)malloc(sizeof(double) * (Dv > Dk ? Dv : Dk));
        if (!S || (a->M_T && !M) || !qn || !kn || !al || !u) {
#pragma omp atomic write
            err = 3;
        } else {
            if (a->S0) memcpy(S, a->S0 + (size_t)chain * Dk * Dv, sizeof(double) * Dk * Dv);
            if (M) for (int c = 0; c < Dk; ++c) M[(size_t)c * Dk + c] = 1.0;
            for (int t = 0; t < T; ++t) {
                double bt;
                prepare_token(a, b, t, hv, qn, kn, al, &bt);
                const double *vt = a->v + (((size_t)b * T + t) * HV + hv) * Dv;
                double *ot = a->o ? a->o + (((size_t)b * T + t) * HV + hv) * Dv : NULL;
                recurrence_step(S, qn, kn, vt, al, bt, a->scale, Dk, Dv, u, ot);
                if (M) transition_left_multiply(M, kn, al, bt, Dk, u);
            }
            if (a->S_T) memcpy(a->S_T + (size_t)chain * Dk * Dv, S, sizeof(double) * Dk * Dv);
            if (M) memcpy(a->M_T + (size_t)chain * Dk * Dk, M, sizeof(double) * Dk * Dk);
        }
        free(S); free(M); free(qn); free(kn); free(al); free(u);
    }
    return err;
}

/* One decode step for B*HV independent chains: the state S [B,HV,Dk,Dv] is
 * updated in place and o [B,HV,Dv] is written.  Inputs are one token each:
 * q,k [B,H,Dk], v [B,HV,Dv], g [B,HV,Dk], beta [B,HV]. */
int oracle_kda_step(const oracle_kda_args *a, double *S) {
    if (!a || !S || a->H <= 0 || a->HV <= 0 || a->HV % a->H != 0) return 1;
    oracle_kda_args one = *a;
    one.T = 1;
    one.S0 = S;
    one.S_T = S;     /* in place: each chain copies in, runs, copies out */
    one.M_T = NULL;
    return oracle_kda_fwd(&one);
}

/* Sequential segment combine: S_in[0] = S_init (or 0); S_in[s+1] = M_s S_in[s] + S_seg[s].
 * M [n_seg,BH,Dk,Dk], S_seg [n_seg,BH,Dk,Dv], S_init [BH,Dk,Dv] or NULL,
 * S_in [n_seg+1,BH,Dk,Dv]. */
int oracle_kda_compose(int n_seg, int BH, int Dk, int Dv, const double *M,
                       const double *S_seg, const double *S_init, double *S_in) {
    if (n_seg < 0 || BH < 0 || Dk <= 0 || Dv <= 0 || !S_in) return 1;
    const size_t st = (size_t)Dk * Dv, mt = (size_t)Dk * Dk;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < BH; ++bh) {
        double *cur = S_in + (size_t)bh * st;
        if (S_init) memcpy(cur, S_init + (size_t)bh * st, sizeof(double) * st);
        else memset(cur, 0, sizeof(double) * st);
        for (int s = 0; s < n_seg; ++s) {
            const double *Ms = M + ((size_t)s * BH + bh) * mt;
            const double *Ss = S_seg + ((size_t)s * BH + bh) * st;
            const double *prev = S_in + ((size_t)s * BH + bh) * st;
            double *next = S_in + ((size_t)(s + 1) * BH + bh) * st;
            for (int c = 0; c < Dk; ++c)
                for (int j = 0; j < Dv; ++j) {
                    double acc = Ss[(size_t)c * Dv + j];
                    for (int m = 0; m < Dk; ++m) acc += Ms[(size_t)c * Dk + m] * prev[(size_t)m * Dv + j];
                    next[(size_t)c * Dv + j] = acc;
                }
        }
    }
    return 0;
}
