/*
 * wkv7_oracle.c -- plain, slow, fp64 CPU oracle for the RWKV-7 "generalized
 * delta rule" (WKV7) recurrence.  TEST INFRASTRUCTURE ONLY: it is built and
 * called by the tests, by the smoke check and by the benchmark's CPU-baseline
 * leg, never by the product path.  It shares no code, header or constant with
 * the CUDA library.
 *
 * What it computes (rwkv-ops 0.9.0 README, "rwkv7op 使用方法": the
 * generalized_delta_rule signature and docstring; rwkv-ops 0.7.4 README, same
 * section).  Per (sequence, head) a K x V state S, stored row-major [k][v]
 * exactly like the documented initial_state / final_state layout [N, H, K, V],
 * evolves token by token:
 *
 *     u_t = S_{t-1}^T a_t                            (read the old state with a)
 *     S_t = diag(exp(w_t)) S_{t-1} + b_t u_t^T + k_t v_t^T
 *     o_t = S_t^T r_t
 *
 * w is the decay "in log space" (docstring: gk is the decay term in log
 * space), so the per-step factor is exp(w).  The docstring's mask[B,T]
 * decides whether the state is updated (1 update, 0 no update); at a masked
 * step the state is carried unchanged and the output is read from it,
 * o_t = S_{t-1}^T r_t.  initial_state=None means a zero state.  With
 * cu_seqlens (the packed variable-length form: initial_state has one entry
 * per sequence, N = number of sequences), sequence n occupies packed rows
 * [cu_seqlens[n], cu_seqlens[n+1]) of a batch of one and starts from its own
 * initial state.
 *
 * Layouts (all dense, row-major): r,w,k,a,b [B,T,H,K]; v [B,T,H,V];
 * o [B,T,H,V]; s0 / sT [N,H,K,V]; mask [B,T] (nonzero = update).
 * Without cu_seqlens N == B.  With cu_seqlens B == 1 and T == cu_seqlens[N].
 *
 * gdn_oracle_fwd, at the end of this file, is the Gated DeltaNet operator of
 * the same README, written on its own (it does not call the function above).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* One (sequence, head) unit, rows [bos, eos) of batch row bb. */
static void oracle_unit(const double* r, const double* w, const double* k,
                        const double* v, const double* a, const double* b,
                        const double* s0, const unsigned char* mask,
                        double* o, double* sT, int T, int H, int K, int V,
                        int bb, int bos, int eos, int n, int h, double* S,
                        double* u) {
    const size_t state_off = ((size_t)n * H + h) * (size_t)K * V;
    if (s0)
        memcpy(S, s0 + state_off, sizeof(double) * (size_t)K * V);
    else
        memset(S, 0, sizeof(double) * (size_t)K * V);

    for (int t = bos; t < eos; ++t) {
        const size_t rowK = (((size_t)bb * T + t) * H + h) * (size_t)K;
        const size_t rowV = (((size_t)bb * T + t) * H + h) * (size_t)V;
        const int update = mask ? (mask[(size_t)bb * T + t] != 0) : 1;
        if (update) {
            /* u = S^T a  (uses the state before this token) */
            for (int j = 0; j < V; ++j) u[j] = 0.0;
            for (int i = 0; i < K; ++i) {
                const double ai = a[rowK + i];
                for (int j = 0; j < V; ++j) u[j] += S[(size_t)i * V + j] * ai;
            }
            /* S = diag(exp(w)) S + b u^T + k v^T */
            for (int i = 0; i < K; ++i) {
                const double di = exp(w[rowK + i]);
                const double bi = b[rowK + i];
                const double ki = k[rowK + i];
                for (int j = 0; j < V; ++j) {
                    double* s = &S[(size_t)i * V + j];
                    *s = di * (*s) + bi * u[j] + ki * v[rowV + j];
                }
            }
        }
        /* o = S^T r */
        for (int j = 0; j < V; ++j) {
            double acc = 0.0;
            for (int i = 0; i < K; ++i) acc += S[(size_t)i * V + j] * r[rowK + i];
            o[rowV + j] = acc;
        }
    }
    if (sT) memcpy(sT + state_off, S, sizeof(double) * (size_t)K * V);
}

/*
 * Returns 0 on success, 1 on an invalid argument.  nthreads <= 0 lets OpenMP
 * choose; the number of threads actually used is written to *threads_used
 * when that pointer is non-NULL.
 */
int wkv7_oracle_fwd(const double* r, const double* w, const double* k,
                    const double* v, const double* a, const double* b,
                    const double* s0, const unsigned char* mask, double* o,
                    double* sT, int B, int T, int H, int K, int V,
                    const int32_t* cu_seqlens, int N, int nthreads,
                    int* threads_used) {
    if (!r || !w || !k || !v || !a || !b || !o) return 1;
    if (B < 0 || T < 0 || H <= 0 || K <= 0 || V <= 0) return 1;
    if (cu_seqlens) {
        if (B != 1 || N < 0 || cu_seqlens[0] != 0 || cu_seqlens[N] != T) return 1;
        for (int n = 0; n < N; ++n)
            if (cu_seqlens[n + 1] < cu_seqlens[n]) return 1;
    } else {
        N = B;
    }
    const long units = (long)N * H;
    int used = 1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
    {
#pragma omp single
        used = omp_get_num_threads();
        double* S = (double*)malloc(sizeof(double) * ((size_t)K * V + V));
#pragma omp for schedule(dynamic, 1)
        for (long unit = 0; unit < units; ++unit) {
            const int n = (int)(unit / H), h = (int)(unit % H);
            const int bb = cu_seqlens ? 0 : n;
            const int bos = cu_seqlens ? cu_seqlens[n] : 0;
            const int eos = cu_seqlens ? cu_seqlens[n + 1] : T;
            oracle_unit(r, w, k, v, a, b, s0, mask, o, sT, T, H, K, V, bb, bos,
                        eos, n, h, S, S + (size_t)K * V);
        }
        free(S);
    }
#else
    (void)nthreads;
    {
        double* S = (double*)malloc(sizeof(double) * ((size_t)K * V + V));
        for (long unit = 0; unit < units; ++unit) {
            const int n = (int)(unit / H), h = (int)(unit % H);
            const int bb = cu_seqlens ? 0 : n;
            const int bos = cu_seqlens ? cu_seqlens[n] : 0;
            const int eos = cu_seqlens ? cu_seqlens[n + 1] : T;
            oracle_unit(r, w, k, v, a, b, s0, mask, o, sT, T, H, K, V, bb, bos,
                        eos, n, h, S, S + (size_t)K * V);
        }
        free(S);
    }
#endif
    if (threads_used) *threads_used = used;
    return 0;
}

/*
 * Gated DeltaNet (rwkv-ops 0.9.0 README, "gdn_recurrent 使用方法" and
 * "gdn_chunk 使用方法": gated_delta_net_recurrent / _chunk / _single_step).
 * q, k [B,T,H,K] are L2-normalised over K inside the op; v [B,T,H,V]; g [B,T,H]
 * is the log-space decay gate; beta [B,T,H] the write strength, already in (0,1).
 * initial_state is [N,H,K,V], or [1,H,K,V] shared by every sequence.  The
 * README names the operator but prints no formula; this is the Gated DeltaNet
 * rule in its delta-rule form, per (sequence, head) and token:
 *
 *     qh = q / |q|,  kh = k / |k|          (a zero vector stays zero)
 *     S  <- exp(g) S                        (the gate decays the old state)
 *     e   = v - S^T kh                      (what the gated state predicts for kh)
 *     S  <- S + beta kh e^T                 (delta-rule correction)
 *     o   = S^T qh
 *
 * No further scaling of q (the README states none).
 */
static void unit_normalise(const double* x, double* y, int n) {
    double ss = 0.0;
    for (int i = 0; i < n; ++i) ss += x[i] * x[i];
    const double nrm = sqrt(ss);
    for (int i = 0; i < n; ++i) y[i] = nrm > 0.0 ? x[i] / nrm : 0.0;
}

static void gdn_unit(const double* q, const double* k, const double* v,
                     const double* g, const double* beta, const double* s0,
                     int s0_shared, double* o, double* sT, int T, int H, int K,
                     int V, int bb, int bos, int eos, int n, int h, double* S,
                     double* work) {
    double* qh = work;
    double* kh = work + K;
    double* e = work + 2 * (size_t)K;
    const size_t state_off = ((size_t)n * H + h) * (size_t)K * V;
    const size_t init_off = ((size_t)(s0_shared ? 0 : n) * H + h) * (size_t)K * V;
    if (s0)
        memcpy(S, s0 + init_off, sizeof(double) * (size_t)K * V);
    else
        memset(S, 0, sizeof(double) * (size_t)K * V);

    for (int t = bos; t < eos; ++t) {
        const size_t tok = ((size_t)bb * T + t) * H + h;
        unit_normalise(q + tok * K, qh, K);
        unit_normalise(k + tok * K, kh, K);
        const double alpha = exp(g[tok]);
        const double bt = beta[tok];
        for (size_t i = 0; i < (size_t)K * V; ++i) S[i] *= alpha;
        for (int j = 0; j < V; ++j) {
            double pred = 0.0;
            for (int i = 0; i < K; ++i) pred += S[(size_t)i * V + j] * kh[i];
            e[j] = v[tok * V + j] - pred;
        }
        for (int i = 0; i < K; ++i)
            for (int j = 0; j < V; ++j) S[(size_t)i * V + j] += bt * kh[i] * e[j];
        for (int j = 0; j < V; ++j) {
            double acc = 0.0;
            for (int i = 0; i < K; ++i) acc += S[(size_t)i * V + j] * qh[i];
            o[tok * V + j] = acc;
        }
    }
    if (sT) memcpy(sT + state_off, S, sizeof(double) * (size_t)K * V);
}

/* Same conventions and return codes as wkv7_oracle_fwd; s0_shared != 0 means
 * s0 holds one [H,K,V] state used by every sequence. */
int gdn_oracle_fwd(const double* q, const double* k, const double* v,
                   const double* g, const double* beta, const double* s0,
                   int s0_shared, double* o, double* sT, int B, int T, int H,
                   int K, int V, const int32_t* cu_seqlens, int N, int nthreads,
                   int* threads_used) {
    if (!q || !k || !v || !g || !beta || !o) return 1;
    if (B < 0 || T < 0 || H <= 0 || K <= 0 || V <= 0) return 1;
    if (cu_seqlens) {
        if (B != 1 || N < 0 || cu_seqlens[0] != 0 || cu_seqlens[N] != T) return 1;
        for (int n = 0; n < N; ++n)
            if (cu_seqlens[n + 1] < cu_seqlens[n]) return 1;
    } else {
        N = B;
    }
    const long units = (long)N * H;
    const size_t scratch = (size_t)K * V + 2 * (size_t)K + V;
    int used = 1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
    {
#pragma omp single
        used = omp_get_num_threads();
        double* S = (double*)malloc(sizeof(double) * scratch);
#pragma omp for schedule(dynamic, 1)
        for (long unit = 0; unit < units; ++unit) {
            const int n = (int)(unit / H), h = (int)(unit % H);
            gdn_unit(q, k, v, g, beta, s0, s0_shared, o, sT, T, H, K, V,
                     cu_seqlens ? 0 : n, cu_seqlens ? cu_seqlens[n] : 0,
                     cu_seqlens ? cu_seqlens[n + 1] : T, n, h, S, S + (size_t)K * V);
        }
        free(S);
    }
#else
    (void)nthreads;
    {
        double* S = (double*)malloc(sizeof(double) * scratch);
        for (long unit = 0; unit < units; ++unit) {
            const int n = (int)(unit / H), h = (int)(unit % H);
            gdn_unit(q, k, v, g, beta, s0, s0_shared, o, sT, T, H, K, V,
                     cu_seqlens ? 0 : n, cu_seqlens ? cu_seqlens[n] : 0,
                     cu_seqlens ? cu_seqlens[n + 1] : T, n, h, S, S + (size_t)K * V);
        }
        free(S);
    }
#endif
    if (threads_used) *threads_used = used;
    return 0;
}

/*
 * Backward of the generalized delta rule above (the README: the chunked
 * generalized_delta_rule entry supports backpropagation; rwkv-ops 0.9.0 README,
 * "rwkv7op 使用方法").  Given dL/do (dout, [B,T,H,V]) and dL/dS_T (dsT, [N,H,K,V]
 * or NULL), returns dL/dr, dw, dk, dv, da, db ([B,T,H,*]) and dL/ds0 ([N,H,K,V]).
 * Plain reverse-mode differentiation of the forward recurrence, token by token,
 * with every state of the unit kept (S_0 .. S_L):
 *
 *   o_t = S_t^T r_t            ->  G += r_t do_t^T,   dr_t = S_t do_t
 *   S_t = D_t S_{t-1} + b_t u_t^T + k_t v_t^T,  u_t = S_{t-1}^T a_t,  D_t = diag(e^{w_t}):
 *        dv_t = G^T k_t,   dk_t = G v_t,   du_t = G^T b_t,   db_t = G u_t,
 *        da_t = S_{t-1} du_t,   dw_t = e^{w_t} * rowsum(G * S_{t-1}),
 *        G <- D_t G + a_t du_t^T                 (G becomes dL/dS_{t-1})
 *   a masked token passes G through unchanged and has zero dw, dk, dv, da, db.
 * At the end dL/ds0 = G.
 */
static void oracle_unit_bwd(const double* r, const double* w, const double* k,
                            const double* v, const double* a, const double* b,
                            const double* s0, const unsigned char* mask,
                            const double* dout, const double* dsT, double* dr,
                            double* dw, double* dk, double* dv, double* da,
                            double* db, double* ds0, int T, int H, int K, int V,
                            int bb, int bos, int eos, int n, int h) {
    const size_t KV = (size_t)K * V;
    const size_t state_off = ((size_t)n * H + h) * KV;
    const int L = eos - bos;
    double* S = (double*)malloc(sizeof(double) * KV * (size_t)(L + 1));
    double* G = (double*)malloc(sizeof(double) * KV);
    double* u = (double*)malloc(sizeof(double) * V);
    double* du = (double*)malloc(sizeof(double) * V);
    if (s0)
        memcpy(S, s0 + state_off, sizeof(double) * KV);
    else
        memset(S, 0, sizeof(double) * KV);
    for (int p = 0; p < L; ++p) {  /* forward, keeping S_{p+1} */
        const int t = bos + p;
        const size_t rowK = (((size_t)bb * T + t) * H + h) * (size_t)K;
        const size_t rowV = (((size_t)bb * T + t) * H + h) * (size_t)V;
        const double* Sp = S + KV * (size_t)p;
        double* Sn = S + KV * (size_t)(p + 1);
        if (mask && mask[(size_t)bb * T + t] == 0) {
            memcpy(Sn, Sp, sizeof(double) * KV);
            continue;
        }
        for (int j = 0; j < V; ++j) {
            u[j] = 0.0;
            for (int i = 0; i < K; ++i) u[j] += Sp[(size_t)i * V + j] * a[rowK + i];
        }
        for (int i = 0; i < K; ++i)
            for (int j = 0; j < V; ++j)
                Sn[(size_t)i * V + j] = exp(w[rowK + i]) * Sp[(size_t)i * V + j] +
                                        b[rowK + i] * u[j] + k[rowK + i] * v[rowV + j];
    }
    if (dsT)
        memcpy(G, dsT + state_off, sizeof(double) * KV);
    else
        memset(G, 0, sizeof(double) * KV);
    for (int p = L - 1; p >= 0; --p) {
        const int t = bos + p;
        const size_t rowK = (((size_t)bb * T + t) * H + h) * (size_t)K;
        const size_t rowV = (((size_t)bb * T + t) * H + h) * (size_t)V;
        const double* Sp = S + KV * (size_t)p;        /* S_{t-1} */
        const double* St = S + KV * (size_t)(p + 1);  /* S_t */
        for (int i = 0; i < K; ++i) {
            double acc = 0.0;
            for (int j = 0; j < V; ++j) {
                G[(size_t)i * V + j] += r[rowK + i] * dout[rowV + j];
                acc += St[(size_t)i * V + j] * dout[rowV + j];
            }
            dr[rowK + i] = acc;
        }
        if (mask && mask[(size_t)bb * T + t] == 0) {
            for (int i = 0; i < K; ++i) dw[rowK + i] = dk[rowK + i] = da[rowK + i] = db[rowK + i] = 0.0;
            for (int j = 0; j < V; ++j) dv[rowV + j] = 0.0;
            continue;
        }
        for (int j = 0; j < V; ++j) {
            double su = 0.0, sv = 0.0, sd = 0.0;
            for (int i = 0; i < K; ++i) {
                su += Sp[(size_t)i * V + j] * a[rowK + i];
                sv += G[(size_t)i * V + j] * k[rowK + i];
                sd += G[(size_t)i * V + j] * b[rowK + i];
            }
            u[j] = su;
            dv[rowV + j] = sv;
            du[j] = sd;
        }
        for (int i = 0; i < K; ++i) {
            double sk = 0.0, sb = 0.0, sa = 0.0, sw = 0.0;
            for (int j = 0; j < V; ++j) {
                const double g = G[(size_t)i * V + j];
                sk += g * v[rowV + j];
                sb += g * u[j];
                sa += Sp[(size_t)i * V + j] * du[j];
                sw += g * Sp[(size_t)i * V + j];
            }
            const double di = exp(w[rowK + i]);
            dk[rowK + i] = sk;
            db[rowK + i] = sb;
            da[rowK + i] = sa;
            dw[rowK + i] = di * sw;
            for (int j = 0; j < V; ++j)
                G[(size_t)i * V + j] = di * G[(size_t)i * V + j] + a[rowK + i] * du[j];
        }
    }
    if (ds0) memcpy(ds0 + state_off, G, sizeof(double) * KV);
    free(S);
    free(G);
    free(u);
    free(du);
}

/* Same conventions and return codes as wkv7_oracle_fwd.  dout is required; dsT
 * and ds0 may be NULL. */
int wkv7_oracle_bwd(const double* r, const double* w, const double* k,
                    const double* v, const double* a, const double* b,
                    const double* s0, const unsigned char* mask, const double* dout,
                    const double* dsT, double* dr, double* dw, double* dk,
                    double* dv, double* da, double* db, double* ds0, int B,
                    int T, int H, int K, int V, const int32_t* cu_seqlens, int N,
                    int nthreads, int* threads_used) {
    if (!r || !w || !k || !v || !a || !b || !dout) return 1;
    if (!dr || !dw || !dk || !dv || !da || !db) return 1;
    if (B < 0 || T < 0 || H <= 0 || K <= 0 || V <= 0) return 1;
    if (cu_seqlens) {
        if (B != 1 || N < 0 || cu_seqlens[0] != 0 || cu_seqlens[N] != T) return 1;
        for (int n = 0; n < N; ++n)
            if (cu_seqlens[n + 1] < cu_seqlens[n]) return 1;
    } else {
        N = B;
    }
    const long units = (long)N * H;
    int used = 1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
    {
#pragma omp single
        used = omp_get_num_threads();
#pragma omp for schedule(dynamic, 1)
        for (long unit = 0; unit < units; ++unit) {
            const int n = (int)(unit / H), h = (int)(unit % H);
            oracle_unit_bwd(r, w, k, v, a, b, s0, mask, dout, dsT, dr, dw, dk, dv, da, db,
                            ds0, T, H, K, V, cu_seqlens ? 0 : n,
                            cu_seqlens ? cu_seqlens[n] : 0,
                            cu_seqlens ? cu_seqlens[n + 1] : T, n, h);
        }
    }
#else
    (void)nthreads;
    for (long unit = 0; unit < units; ++unit) {
        const int n = (int)(unit / H), h = (int)(unit % H);
        oracle_unit_bwd(r, w, k, v, a, b, s0, mask, dout, dsT, dr, dw, dk, dv, da, db, ds0,
                        T, H, K, V, cu_seqlens ? 0 : n, cu_seqlens ? cu_seqlens[n] : 0,
                        cu_seqlens ? cu_seqlens[n + 1] : T, n, h);
    }
#endif
    if (threads_used) *threads_used = used;
    return 0;
}

/*
 * The generalized delta rule with State Anomaly Neutralization (SANE; rwkv-ops
 * 0.9.0 README, "rwkv7op_sane 使用方法" and "rwkv7_op_sane_rnn 使用方法"): the
 * recurrence of wkv7_oracle_fwd, and after every 16th token of a sequence (a chunk
 * boundary) the state is soft-clipped with that chunk's tau[b, c, h] > 0 when the
 * chunk's flag sane_mask[b, c] is nonzero (NULL: every chunk).  The outputs are read
 * from the state before the clip (README: "output based on the state before SANE").
 * The README defers the clip function to an external paper; the reading here is the
 * elementwise soft clip S <- tau * tanh(S / tau).  A partial last chunk is not
 * clipped (tau has T / 16 entries per sequence).  No token mask: padding is input
 * values (README: k = 0, a = 0, w = -inf).
 *
 * Layouts: r, w, k, a, b [B,T,H,K]; v, o [B,T,H,V]; tau [B, T/16, H] (fp64 here);
 * sane_mask [B, T/16] or NULL; s0 / sT [B,H,K,V].
 */
int wkv7_oracle_sane_fwd(const double* r, const double* w, const double* k,
                         const double* v, const double* a, const double* b,
                         const double* tau, const unsigned char* sane_mask,
                         const double* s0, double* o, double* sT, int B, int T,
                         int H, int K, int V) {
    if (!r || !w || !k || !v || !a || !b || !tau || !o) return 1;
    if (B < 0 || T < 0 || H <= 0 || K <= 0 || V <= 0) return 1;
    const int C = T / 16;  /* full 16-token chunks */
    const size_t KV = (size_t)K * V;
    double* S = (double*)malloc(sizeof(double) * (KV + V));
    double* u = S + KV;
    for (int bb = 0; bb < B; ++bb) {
        for (int h = 0; h < H; ++h) {
            const size_t state_off = ((size_t)bb * H + h) * KV;
            if (s0)
                memcpy(S, s0 + state_off, sizeof(double) * KV);
            else
                memset(S, 0, sizeof(double) * KV);
            for (int t = 0; t < T; ++t) {
                const size_t rowK = (((size_t)bb * T + t) * H + h) * (size_t)K;
                const size_t rowV = (((size_t)bb * T + t) * H + h) * (size_t)V;
                for (int j = 0; j < V; ++j) {
                    u[j] = 0.0;
                    for (int i = 0; i < K; ++i) u[j] += S[(size_t)i * V + j] * a[rowK + i];
                }
                for (int i = 0; i < K; ++i)
                    for (int j = 0; j < V; ++j)
                        S[(size_t)i * V + j] = exp(w[rowK + i]) * S[(size_t)i * V + j] +
                                               b[rowK + i] * u[j] + k[rowK + i] * v[rowV + j];
                for (int j = 0; j < V; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < K; ++i) acc += S[(size_t)i * V + j] * r[rowK + i];
                    o[rowV + j] = acc;
                }
                const int c = t / 16;
                if (t % 16 == 15 && c < C &&
                    (!sane_mask || sane_mask[(size_t)bb * C + c] != 0)) {
                    const double tc = tau[((size_t)bb * C + c) * H + h];
                    for (size_t e = 0; e < KV; ++e) S[e] = tc * tanh(S[e] / tc);
                }
            }
            if (sT) memcpy(sT + state_off, S, sizeof(double) * KV);
        }
    }
    free(S);
    return 0;
}
