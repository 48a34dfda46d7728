/*
 * FP64 CPU oracle of Kimi Delta Attention (KDA).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; only the tests, the package's smoke check and the CPU
 * baseline leg of the benchmark do.  It shares no code, header or table
 * with the CUDA implementation.
 *
 * What it computes, per sequence i and head h, over the packed tokens
 * t = cu[i] .. cu[i+1]-1, in double precision:
 *
 *     alpha_t = exp(g_t)                                   (per key channel)
 *     S_t     = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t     = S_t^T q_t
 *
 * with S a D_k x D_v matrix (row = key channel).  Sources:
 *  - "LLM - Semianalysis, Kimi K3 아키텍처" (charstring.tistory.com/2557),
 *    Background:
 *    KDA is Gated DeltaNet with the scalar forget gate widened to a diagonal
 *    matrix (one decay per channel); the delta rule is one gradient step on
 *    the L2 value-retrieval loss 1/2 |S^T k - v|^2, which expands to the
 *    (I - beta k k^T) S + beta k v^T form above with the gate applied first.
 *  - Same page, Methods 1 (FlashKDA): decode runs this recurrence as is; the
 *    state is FP32 on the GPU (here FP64).
 *  - "MoonshotAI/Kimi-K3 딥다이브" (fiv.co.kr/repos/kimi-k3-deep-dive.html),
 *    section 4-1: per-channel decay with a
 *    lower bound; prefill in 16-token tiles with a recurrence between tiles.
 *  - The first page, Methods 3: the state is cached only at coarse positions
 *    (e.g. every 32K tokens) for prefix caching -> checkpoints below.
 *
 * Checkpoints: when (t + 1 - cu[i]) is a positive multiple of ckpt_interval,
 * a copy of S_t is stored.  Checkpoints are packed sequence by sequence, in
 * position order, as [n_ckpt, H, D_k, D_v]; sequence i's first slot is
 * sum_{j<i} floor(T_j / ckpt_interval).
 *
 * Two forms are provided: kda_oracle_recurrent (the definition, token by
 * token) and kda_oracle_chunked (the same result regrouped into C-token
 * chunks: a unit lower-triangular solve inside each chunk and a state carry
 * between chunks, written from the algebra of the recurrence; used to check
 * that regrouping, with plain exp of gate differences and no factoring).
 *
 * All arrays are dense row-major doubles:
 *   q, k, g [T_tot, H, Dk]; v, out [T_tot, H, Dv]; beta [T_tot, H];
 *   init_state, final_state [N, H, Dk, Dv] (init_state may be NULL = zeros).
 * Returns 0 on success, a negative value on a bad argument.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int64_t H, Dk, Dv;
    const double *q, *k, *v, *g, *beta, *init;
    double *out, *fin, *ckpt;
    int64_t ckpt_interval;
    /* optional explicit positions: sequence i stores its state after
       pos[pos_cu[i]], ..., pos[pos_cu[i+1]-1] tokens into pos_states */
    const int64_t *pos_cu, *pos;
    double *pos_states;
} problem;

static int64_t ckpt_base(const int64_t *cu, int64_t seq, int64_t interval) {
    int64_t base = 0;
    if (interval <= 0) return 0;
    for (int64_t j = 0; j < seq; ++j) base += (cu[j + 1] - cu[j]) / interval;
    return base;
}

static void store_ckpt(const problem *p, int64_t slot, int64_t h, const double *S) {
    double *dst = p->ckpt + (slot * p->H + h) * p->Dk * p->Dv;
    memcpy(dst, S, sizeof(double) * (size_t)(p->Dk * p->Dv));
}

static void store_pos(const problem *p, int64_t j, int64_t h, const double *S) {
    double *dst = p->pos_states + (j * p->H + h) * p->Dk * p->Dv;
    memcpy(dst, S, sizeof(double) * (size_t)(p->Dk * p->Dv));
}

/* One (sequence, head) unit of the token-by-token recurrence. */
static void recurrent_unit(const problem *p, const int64_t *cu, int64_t seq, int64_t h,
                           double *S, double *y) {
    const int64_t H = p->H, Dk = p->Dk, Dv = p->Dv;
    const int64_t t0 = cu[seq], t1 = cu[seq + 1];
    int64_t slot = ckpt_base(cu, seq, p->ckpt_interval);
    int64_t pj = p->pos ? p->pos_cu[seq] : 0, pe = p->pos ? p->pos_cu[seq + 1] : 0;
    if (p->init) memcpy(S, p->init + (seq * H + h) * Dk * Dv, sizeof(double) * (size_t)(Dk * Dv));
    else memset(S, 0, sizeof(double) * (size_t)(Dk * Dv));
    /* positions at or before the start store the initial state */
    while (pj < pe && p->pos[pj] <= 0) store_pos(p, pj++, h, S);
    for (int64_t t = t0; t < t1; ++t) {
        const double *qt = p->q + (t * H + h) * Dk;
        const double *kt = p->k + (t * H + h) * Dk;
        const double *gt = p->g + (t * H + h) * Dk;
        const double *vt = p->v + (t * H + h) * Dv;
        const double bt = p->beta[t * H + h];
        /* S <- Diag(alpha_t) S : row c scaled by exp(g_tc). */
        for (int64_t c = 0; c < Dk; ++c) {
            const double a = exp(gt[c]);
            for (int64_t j = 0; j < Dv; ++j) S[c * Dv + j] *= a;
        }
        /* y = S^T k_t (what the gated state currently retrieves for k_t). */
        for (int64_t j = 0; j < Dv; ++j) y[j] = 0.0;
        for (int64_t c = 0; c < Dk; ++c)
            for (int64_t j = 0; j < Dv; ++j) y[j] += S[c * Dv + j] * kt[c];
        /* S <- S + beta k (v - y)^T  ==  (I - beta k k^T) S + beta k v^T. */
        for (int64_t c = 0; c < Dk; ++c)
            for (int64_t j = 0; j < Dv; ++j) S[c * Dv + j] += bt * kt[c] * (vt[j] - y[j]);
        /* o_t = S_t^T q_t. */
        double *ot = p->out + (t * H + h) * Dv;
        for (int64_t j = 0; j < Dv; ++j) ot[j] = 0.0;
        for (int64_t c = 0; c < Dk; ++c)
            for (int64_t j = 0; j < Dv; ++j) ot[j] += S[c * Dv + j] * qt[c];
        if (p->ckpt_interval > 0 && (t + 1 - t0) % p->ckpt_interval == 0)
            store_ckpt(p, slot++, h, S);
        while (pj < pe && p->pos[pj] <= t + 1 - t0) store_pos(p, pj++, h, S);
    }
    /* positions past the end store the final state */
    while (pj < pe) store_pos(p, pj++, h, S);
    if (p->fin) memcpy(p->fin + (seq * H + h) * Dk * Dv, S, sizeof(double) * (size_t)(Dk * Dv));
}

/*
 * One (sequence, head) unit of the chunked form.  Inside a chunk of L tokens
 * starting from state S0, with Gam_r = sum_{s<=r} g_s (inclusive, per channel):
 *
 *   Kt_r = k_r * exp(Gam_r)        Qt_r = q_r * exp(Gam_r)
 *   Kh_r = k_r * exp(Gam_L - Gam_r)
 *   M_ri = beta_r sum_c k_rc k_ic exp(Gam_rc - Gam_ic)   (i < r)
 *   P_ri = sum_c q_rc k_ic exp(Gam_rc - Gam_ic)          (i <= r)
 *   (I + M) U = diag(beta) (V - Kt S0)        -- forward substitution
 *   O = Qt S0 + P U
 *   S_L = Diag(exp(Gam_L)) S0 + Kh^T U
 *
 * Row r of U is the delta-rule correction of token r: S_r = Diag(alpha_r)
 * S_{r-1} + k_r u_r^T.  Chunks restart at each sequence start; the last
 * chunk of a sequence may be shorter than C.
 */
static void chunked_unit(const problem *p, const int64_t *cu, int64_t seq, int64_t h,
                         int64_t C, double *S, double *work) {
    const int64_t H = p->H, Dk = p->Dk, Dv = p->Dv;
    const int64_t t0 = cu[seq], t1 = cu[seq + 1];
    int64_t slot = ckpt_base(cu, seq, p->ckpt_interval);
    double *Gam = work;               /* C x Dk */
    double *M = Gam + C * Dk;         /* C x C  */
    double *P = M + C * C;            /* C x C  */
    double *U = P + C * C;            /* C x Dv */
    double *S1 = U + C * Dv;          /* Dk x Dv */
    if (p->init) memcpy(S, p->init + (seq * H + h) * Dk * Dv, sizeof(double) * (size_t)(Dk * Dv));
    else memset(S, 0, sizeof(double) * (size_t)(Dk * Dv));
    for (int64_t c0 = t0; c0 < t1; c0 += C) {
        const int64_t L = (t1 - c0 < C) ? (t1 - c0) : C;
#define Q_(r, c) p->q[((c0 + (r)) * H + h) * Dk + (c)]
#define K_(r, c) p->k[((c0 + (r)) * H + h) * Dk + (c)]
#define G_(r, c) p->g[((c0 + (r)) * H + h) * Dk + (c)]
#define V_(r, j) p->v[((c0 + (r)) * H + h) * Dv + (j)]
#define B_(r) p->beta[(c0 + (r)) * H + h]
        for (int64_t c = 0; c < Dk; ++c) {
            double acc = 0.0;
            for (int64_t r = 0; r < L; ++r) { acc += G_(r, c); Gam[r * Dk + c] = acc; }
        }
        for (int64_t r = 0; r < L; ++r)
            for (int64_t i = 0; i < L; ++i) {
                double m = 0.0, pr = 0.0;
                if (i <= r)
                    for (int64_t c = 0; c < Dk; ++c) {
                        const double e = exp(Gam[r * Dk + c] - Gam[i * Dk + c]);
                        m += K_(r, c) * K_(i, c) * e;
                        pr += Q_(r, c) * K_(i, c) * e;
                    }
                M[r * C + i] = (i < r) ? B_(r) * m : 0.0;
                P[r * C + i] = (i <= r) ? pr : 0.0;
            }
        /* Right-hand side diag(beta)(V - Kt S0), then forward substitution. */
        for (int64_t r = 0; r < L; ++r) {
            for (int64_t j = 0; j < Dv; ++j) {
                double w = 0.0;
                for (int64_t c = 0; c < Dk; ++c) w += K_(r, c) * exp(Gam[r * Dk + c]) * S[c * Dv + j];
                double u = B_(r) * (V_(r, j) - w);
                for (int64_t i = 0; i < r; ++i) u -= M[r * C + i] * U[i * Dv + j];
                U[r * Dv + j] = u;
            }
        }
        /* Outputs O = Qt S0 + P U. */
        for (int64_t r = 0; r < L; ++r) {
            double *ot = p->out + ((c0 + r) * H + h) * Dv;
            for (int64_t j = 0; j < Dv; ++j) {
                double o = 0.0;
                for (int64_t c = 0; c < Dk; ++c) o += Q_(r, c) * exp(Gam[r * Dk + c]) * S[c * Dv + j];
                for (int64_t i = 0; i <= r; ++i) o += P[r * C + i] * U[i * Dv + j];
                ot[j] = o;
            }
        }
        /* State carry S_L = Diag(exp(Gam_L)) S0 + Kh^T U. */
        for (int64_t c = 0; c < Dk; ++c) {
            const double gl = Gam[(L - 1) * Dk + c];
            for (int64_t j = 0; j < Dv; ++j) {
                double s = exp(gl) * S[c * Dv + j];
                for (int64_t r = 0; r < L; ++r) s += K_(r, c) * exp(gl - Gam[r * Dk + c]) * U[r * Dv + j];
                S1[c * Dv + j] = s;
            }
        }
        memcpy(S, S1, sizeof(double) * (size_t)(Dk * Dv));
        if (p->ckpt_interval > 0 && (c0 + L - t0) % p->ckpt_interval == 0)
            store_ckpt(p, slot++, h, S);
#undef Q_
#undef K_
#undef G_
#undef V_
#undef B_
    }
    if (p->fin) memcpy(p->fin + (seq * H + h) * Dk * Dv, S, sizeof(double) * (size_t)(Dk * Dv));
}

static int check_args(int64_t num_seqs, const int64_t *cu, int64_t H, int64_t Dk, int64_t Dv,
                      const problem *p) {
    if (num_seqs < 0 || H <= 0 || Dk <= 0 || Dv <= 0 || !cu) return -1;
    if (cu[0] != 0) return -1;
    for (int64_t i = 0; i < num_seqs; ++i)
        if (cu[i + 1] < cu[i]) return -1;
    if (cu[num_seqs] > 0 && (!p->q || !p->k || !p->v || !p->g || !p->beta || !p->out)) return -1;
    if (p->ckpt_interval < 0) return -1;
    if (p->ckpt_interval > 0 && !p->ckpt) return -1;
    return 0;
}

static int run(int64_t num_seqs, const int64_t *cu, int64_t H, int64_t Dk, int64_t Dv,
               const double *q, const double *k, const double *v, const double *g,
               const double *beta, const double *init, int64_t ckpt_interval, double *out,
               double *fin, double *ckpt, int nthreads, int64_t chunk, const int64_t *pos_cu,
               const int64_t *pos, double *pos_states) {
    problem p = {H, Dk, Dv, q, k, v, g, beta, init, out, fin, ckpt, ckpt_interval,
                 pos_cu, pos, pos_states};
    if (pos && (!pos_cu || !pos_states || chunk != 0)) return -1;
    if (check_args(num_seqs, cu, H, Dk, Dv, &p)) return -1;
    if (chunk < 0) return -1;
    const int64_t units = num_seqs * H;
    const size_t per_unit = (size_t)(Dk * Dv + Dv) +
        (chunk > 0 ? (size_t)(chunk * Dk + 2 * chunk * chunk + chunk * Dv + Dk * Dv) : 0);
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#else
    nthreads = 1;
#endif
    int failed = 0;
#pragma omp parallel num_threads(nthreads)
    {
        double *buf = (double *)malloc(sizeof(double) * per_unit);
        if (!buf) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t u = 0; u < units; ++u) {
            if (!buf) continue;
            const int64_t seq = u / H, h = u % H;
            if (chunk == 0) recurrent_unit(&p, cu, seq, h, buf, buf + Dk * Dv);
            else chunked_unit(&p, cu, seq, h, chunk, buf, buf + Dk * Dv);
        }
        free(buf);
    }
    return failed ? -2 : 0;
}

int kda_oracle_recurrent(int64_t num_seqs, const int64_t *cu_seqlens, int64_t H, int64_t Dk,
                         int64_t Dv, const double *q, const double *k, const double *v,
                         const double *g, const double *beta, const double *init_state,
                         int64_t ckpt_interval, double *out, double *final_state,
                         double *ckpt_states, int nthreads) {
    return run(num_seqs, cu_seqlens, H, Dk, Dv, q, k, v, g, beta, init_state, ckpt_interval,
               out, final_state, ckpt_states, nthreads, 0, NULL, NULL, NULL);
}

/* The recurrence with states also stored at explicit per-sequence positions:
 * entries pos[pos_cu[i]] .. pos[pos_cu[i+1]-1] are token counts of sequence i;
 * pos_states[j] receives the state after pos[j] tokens (the initial state for
 * pos[j] <= 0, the final state for pos[j] >= T_i).  Prefix caching keeps the
 * state at prompt boundaries as well as at the coarse interval ("LLM -
 * Semianalysis, Kimi K3 아키텍처", Conclusion table, "32K interval (+prompt
 * boundaries)"). */
int kda_oracle_recurrent_pos(int64_t num_seqs, const int64_t *cu_seqlens, int64_t H, int64_t Dk,
                             int64_t Dv, const double *q, const double *k, const double *v,
                             const double *g, const double *beta, const double *init_state,
                             int64_t ckpt_interval, double *out, double *final_state,
                             double *ckpt_states, int nthreads, const int64_t *pos_cu,
                             const int64_t *pos, double *pos_states) {
    return run(num_seqs, cu_seqlens, H, Dk, Dv, q, k, v, g, beta, init_state, ckpt_interval,
               out, final_state, ckpt_states, nthreads, 0, pos_cu, pos, pos_states);
}

int kda_oracle_chunked(int64_t num_seqs, const int64_t *cu_seqlens, int64_t H, int64_t Dk,
                       int64_t Dv, const double *q, const double *k, const double *v,
                       const double *g, const double *beta, const double *init_state,
                       int64_t ckpt_interval, double *out, double *final_state,
                       double *ckpt_states, int nthreads, int64_t chunk) {
    if (chunk <= 0) return -1;
    if (ckpt_interval > 0 && ckpt_interval % chunk != 0) return -1;
    return run(num_seqs, cu_seqlens, H, Dk, Dv, q, k, v, g, beta, init_state, ckpt_interval,
               out, final_state, ckpt_states, nthreads, chunk, NULL, NULL, NULL);
}

/*
 * Backward pass of the recurrence (the training direction; the pages give no
 * detail of it, so it is derived here from the forward definition above and
 * pinned in the tests against central finite differences of the forward).
 *
 * Per token, with P_t = Diag(alpha_t) S_{t-1}, y_t = P_t^T k_t,
 * u_t = beta_t (v_t - y_t), S_t = P_t + k_t u_t^T and o_t = S_t^T q_t, and
 * dS the gradient of the loss with respect to S_t coming from later tokens
 * (d_final_state for the last one):
 *
 *   dS    += q_t do_t^T                 dq_t   = S_t do_t
 *   du     = dS^T k_t                   dk_t   = dS u_t - beta_t P_t du
 *   dbeta_t = du . (v_t - y_t)          dv_t   = beta_t du
 *   dP     = dS - beta_t k_t du^T       dg_t,c = alpha_t,c sum_j dP_cj S_{t-1,cj}
 *   dS    <- Diag(alpha_t) dP           (the gradient with respect to S_{t-1})
 *
 * After the first token of a sequence dS is the gradient with respect to its
 * initial state.  Arrays as for the forward (d_out [T_tot, H, Dv],
 * d_final_state and d_init_state [N, H, Dk, Dv], either may be NULL).
 */
static void backward_unit(int64_t H, int64_t Dk, int64_t Dv, const double *q, const double *k,
                          const double *v, const double *g, const double *beta,
                          const double *init, const double *dout, const double *dfin,
                          double *dq, double *dk, double *dv, double *dg, double *dbeta,
                          double *dinit, const int64_t *cu, int64_t seq, int64_t h,
                          double *states, double *dS, double *vec) {
    const int64_t t0 = cu[seq], T = cu[seq + 1] - cu[seq], DD = Dk * Dv;
    double *y = vec, *u = vec + Dv, *du = vec + 2 * Dv, *alpha = vec + 3 * Dv;
    /* forward, keeping S_{t} for t = -1 .. T-1 (states[t + 1]) */
    if (init) memcpy(states, init + (seq * H + h) * DD, sizeof(double) * (size_t)DD);
    else memset(states, 0, sizeof(double) * (size_t)DD);
    for (int64_t t = 0; t < T; ++t) {
        const int64_t tt = t0 + t;
        const double *kt = k + (tt * H + h) * Dk, *gt = g + (tt * H + h) * Dk;
        const double *vt = v + (tt * H + h) * Dv;
        const double bt = beta[tt * H + h];
        const double *Sp = states + t * DD;
        double *Sn = states + (t + 1) * DD;
        for (int64_t c = 0; c < Dk; ++c) {
            const double a = exp(gt[c]);
            for (int64_t j = 0; j < Dv; ++j) Sn[c * Dv + j] = a * Sp[c * Dv + j];
        }
        for (int64_t j = 0; j < Dv; ++j) y[j] = 0.0;
        for (int64_t c = 0; c < Dk; ++c)
            for (int64_t j = 0; j < Dv; ++j) y[j] += Sn[c * Dv + j] * kt[c];
        for (int64_t c = 0; c < Dk; ++c)
            for (int64_t j = 0; j < Dv; ++j) Sn[c * Dv + j] += bt * kt[c] * (vt[j] - y[j]);
    }
    /* backward */
    if (dfin) memcpy(dS, dfin + (seq * H + h) * DD, sizeof(double) * (size_t)DD);
    else memset(dS, 0, sizeof(double) * (size_t)DD);
    for (int64_t t = T - 1; t >= 0; --t) {
        const int64_t tt = t0 + t;
        const double *qt = q + (tt * H + h) * Dk, *kt = k + (tt * H + h) * Dk;
        const double *gt = g + (tt * H + h) * Dk, *vt = v + (tt * H + h) * Dv;
        const double *dot = dout + (tt * H + h) * Dv;
        const double bt = beta[tt * H + h];
        const double *Sp = states + t * DD, *Sn = states + (t + 1) * DD;
        for (int64_t c = 0; c < Dk; ++c) alpha[c] = exp(gt[c]);
        /* y and u of this token, from P = Diag(alpha) S_{t-1} */
        for (int64_t j = 0; j < Dv; ++j) y[j] = 0.0;
        for (int64_t c = 0; c < Dk; ++c)
            for (int64_t j = 0; j < Dv; ++j) y[j] += alpha[c] * Sp[c * Dv + j] * kt[c];
        for (int64_t j = 0; j < Dv; ++j) u[j] = bt * (vt[j] - y[j]);
        /* o_t = S_t^T q_t */
        double *dqt = dq + (tt * H + h) * Dk;
        for (int64_t c = 0; c < Dk; ++c) {
            double a = 0.0;
            for (int64_t j = 0; j < Dv; ++j) a += Sn[c * Dv + j] * dot[j];
            dqt[c] = a;
        }
        for (int64_t c = 0; c < Dk; ++c)
            for (int64_t j = 0; j < Dv; ++j) dS[c * Dv + j] += qt[c] * dot[j];
        /* S_t = P + k u^T */
        for (int64_t j = 0; j < Dv; ++j) du[j] = 0.0;
        for (int64_t c = 0; c < Dk; ++c)
            for (int64_t j = 0; j < Dv; ++j) du[j] += dS[c * Dv + j] * kt[c];
        double db = 0.0;
        double *dvt = dv + (tt * H + h) * Dv;
        for (int64_t j = 0; j < Dv; ++j) {
            db += du[j] * (vt[j] - y[j]);
            dvt[j] = bt * du[j];
        }
        dbeta[tt * H + h] = db;
        double *dkt = dk + (tt * H + h) * Dk, *dgt = dg + (tt * H + h) * Dk;
        for (int64_t c = 0; c < Dk; ++c) {
            double a = 0.0, b = 0.0, da = 0.0;
            for (int64_t j = 0; j < Dv; ++j) {
                a += dS[c * Dv + j] * u[j];
                b += alpha[c] * Sp[c * Dv + j] * du[j];
                da += (dS[c * Dv + j] - bt * kt[c] * du[j]) * Sp[c * Dv + j];
            }
            dkt[c] = a - bt * b;
            dgt[c] = alpha[c] * da;
        }
        /* the gradient with respect to S_{t-1} */
        for (int64_t c = 0; c < Dk; ++c)
            for (int64_t j = 0; j < Dv; ++j)
                dS[c * Dv + j] = alpha[c] * (dS[c * Dv + j] - bt * kt[c] * du[j]);
    }
    if (dinit) memcpy(dinit + (seq * H + h) * DD, dS, sizeof(double) * (size_t)DD);
}

int kda_oracle_backward(int64_t num_seqs, const int64_t *cu, int64_t H, int64_t Dk, int64_t Dv,
                        const double *q, const double *k, const double *v, const double *g,
                        const double *beta, const double *init_state, const double *d_out,
                        const double *d_final_state, double *dq, double *dk, double *dv,
                        double *dg, double *dbeta, double *d_init_state, int nthreads) {
    if (num_seqs < 0 || H <= 0 || Dk <= 0 || Dv <= 0 || !cu || cu[0] != 0) return -1;
    int64_t maxT = 0;
    for (int64_t i = 0; i < num_seqs; ++i) {
        if (cu[i + 1] < cu[i]) return -1;
        if (cu[i + 1] - cu[i] > maxT) maxT = cu[i + 1] - cu[i];
    }
    if (cu[num_seqs] > 0 && (!q || !k || !v || !g || !beta || !d_out || !dq || !dk || !dv ||
                             !dg || !dbeta))
        return -1;
    const size_t per_unit = (size_t)((maxT + 2) * Dk * Dv + 3 * Dv + Dk);
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#else
    nthreads = 1;
#endif
    int failed = 0;
    const int64_t units = num_seqs * H;
#pragma omp parallel num_threads(nthreads)
    {
        double *buf = (double *)malloc(sizeof(double) * per_unit);
        if (!buf) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t w = 0; w < units; ++w) {
            if (!buf) continue;
            const int64_t DD = Dk * Dv;
            backward_unit(H, Dk, Dv, q, k, v, g, beta, init_state, d_out, d_final_state, dq, dk, dv,
                          dg, dbeta, d_init_state, cu, w / H, w % H, buf, buf + (maxT + 1) * DD,
                          buf + (maxT + 2) * DD);
        }
        free(buf);
    }
    return failed ? -2 : 0;
}

int kda_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
