/*
 * Oracle for the gated delta rule -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, fp64, token-by-token CPU recurrence. Only the tests, the smoke
 * check and the benchmark's CPU-baseline leg may load this library; the CUDA
 * product path never does, and this file shares no code with it.
 *
 * What it computes (column convention, state S is d_v x d_k):
 *
 *   S_t = (S_{t-1} D_t)(I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = S_t q_t
 *
 * with D_t = exp(g_t) I for a scalar gate (Gated DeltaNet) and
 * D_t = Diag(exp(g_t)) for a per-key-channel gate (Kimi Delta Attention).
 * Sources:
 *   - "Gated DeltaNet: Householder Transitions and the Arithmetic of Forgetting",
 *     section "The gated delta rule": S_t = S_{t-1} alpha_t (I - beta k k^T) + beta v k^T
 *     in the column convention used here.
 *   - "Linear Attention, Visualized", section "DeltaNet / Recurrent form"
 *     (prediction, scaled correction u_t, additive write, readout) and section
 *     "Gated DeltaNet (GDN) / Decay also changes the correction rows"
 *     (u_t = beta_t (v_t - a_t k_t S_{t-1})).
 *   - "Linear Attention, Visualized", section "Kimi Delta Attention (KDA)":
 *     the state is decayed channel by channel first, then corrected.
 *
 * The update is evaluated in the additive form that the "Recurrent form"
 * section gives, after the decay has been applied:
 *     S' = S D_t;  p = S' k_t;  u = beta_t (v_t - p);  S = S' + u k_t^T;  o_t = S q_t.
 *
 * Layouts (row-major, the same as the library's C-ABI):
 *   q, k  [B, T, H, d_k]     v, out [B, T, H, d_v]
 *   g     [B, T, H] (scalar gate) or [B, T, H, d_k] (per-channel gate), log-decay
 *   beta  [B, T, H]
 *   S0, S_final [n_seq, H, d_v, d_k]  (S0 may be NULL: zero initial state)
 *   cu_seqlens: NULL (B sequences of length T) or [n_seq + 1] token offsets
 *               into a packed batch (then B must be 1).
 * Work is split over (sequence, head) pairs with POSIX threads.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const double *q, *k, *v, *g, *beta, *S0;
    double *out, *S_final;
    int B, T, H, dk, dv, n_seq, per_channel;
    const int *cu;
    int next_unit; /* guarded by lock */
    pthread_mutex_t lock;
} fwd_job;

static void run_unit(fwd_job *J, int unit, double *S, double *Sd, double *p, double *u) {
    const int H = J->H, dk = J->dk, dv = J->dv;
    const int s = unit / H, h = unit % H;
    long t_begin, t_end;
    if (J->cu) {
        t_begin = J->cu[s];
        t_end = J->cu[s + 1];
    } else {
        t_begin = (long)s * J->T;
        t_end = t_begin + J->T;
    }
    const size_t state_off = ((size_t)s * H + h) * (size_t)dv * dk;
    if (J->S0)
        memcpy(S, J->S0 + state_off, sizeof(double) * (size_t)dv * dk);
    else
        memset(S, 0, sizeof(double) * (size_t)dv * dk);

    for (long t = t_begin; t < t_end; ++t) {
        const size_t tok = (size_t)t * H + h;
        const double *qt = J->q + tok * dk;
        const double *kt = J->k + tok * dk;
        const double *vt = J->v + tok * dv;
        const double bt = J->beta[tok];
        /* decay: S' = S D_t */
        if (J->per_channel) {
            const double *gt = J->g + tok * dk;
            for (int j = 0; j < dk; ++j) Sd[j] = exp(gt[j]);
            for (int i = 0; i < dv; ++i)
                for (int j = 0; j < dk; ++j) S[(size_t)i * dk + j] *= Sd[j];
        } else {
            const double a = exp(J->g[tok]);
            for (size_t e = 0; e < (size_t)dv * dk; ++e) S[e] *= a;
        }
        /* prediction p = S' k_t and correction u = beta (v - p) */
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * kt[j];
            p[i] = acc;
            u[i] = bt * (vt[i] - acc);
        }
        /* write S = S' + u k^T, then read o = S q */
        double *ot = J->out + tok * dv;
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            double *row = S + (size_t)i * dk;
            for (int j = 0; j < dk; ++j) {
                row[j] += u[i] * kt[j];
                acc += row[j] * qt[j];
            }
            ot[i] = acc;
        }
    }
    if (J->S_final) memcpy(J->S_final + state_off, S, sizeof(double) * (size_t)dv * dk);
}

static void *fwd_worker(void *arg) {
    fwd_job *J = (fwd_job *)arg;
    const size_t n = (size_t)J->dv * J->dk;
    double *S = (double *)malloc(sizeof(double) * n);
    double *Sd = (double *)malloc(sizeof(double) * (size_t)J->dk);
    double *p = (double *)malloc(sizeof(double) * (size_t)J->dv);
    double *u = (double *)malloc(sizeof(double) * (size_t)J->dv);
    const int n_units = J->n_seq * J->H;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int unit = J->next_unit++;
        pthread_mutex_unlock(&J->lock);
        if (unit >= n_units) break;
        run_unit(J, unit, S, Sd, p, u);
    }
    free(S);
    free(Sd);
    free(p);
    free(u);
    return NULL;
}

/* Returns 0 on success, nonzero on invalid arguments. */
int oracle_gdr_fwd(const double *q, const double *k, const double *v, const double *g,
                   const double *beta, const double *S0, double *out, double *S_final, int B, int T,
                   int H, int dk, int dv, const int *cu_seqlens, int n_seq, int per_channel,
                   int n_threads) {
    if (!q || !k || !v || !g || !beta || !out) return 1;
    if (B <= 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return 1;
    if (cu_seqlens) {
        if (B != 1 || n_seq <= 0 || cu_seqlens[0] != 0 || cu_seqlens[n_seq] != T) return 1;
        for (int i = 0; i < n_seq; ++i)
            if (cu_seqlens[i + 1] < cu_seqlens[i]) return 1;
    } else {
        n_seq = B;
    }
    fwd_job J;
    J.q = q; J.k = k; J.v = v; J.g = g; J.beta = beta; J.S0 = S0;
    J.out = out; J.S_final = S_final;
    J.B = B; J.T = T; J.H = H; J.dk = dk; J.dv = dv; J.n_seq = n_seq;
    J.per_channel = per_channel; J.cu = cu_seqlens; J.next_unit = 0;
    pthread_mutex_init(&J.lock, NULL);
    if (n_threads < 1) n_threads = 1;
    if (n_threads > n_seq * H) n_threads = n_seq * H;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    for (int i = 0; i < n_threads; ++i) pthread_create(&th[i], NULL, fwd_worker, &J);
    for (int i = 0; i < n_threads; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.lock);
    return 0;
}

/*
 * One decode step for n independent sequences: the same token update as above,
 * applied once, in place on S_inout [n, H, d_v, d_k].
 *   q, k [n, H, d_k]; v, out [n, H, d_v]; g [n, H] or [n, H, d_k]; beta [n, H].
 * Single-threaded (a step is small); the caller parallelises if it wants to.
 */
int oracle_gdr_decode_step(const double *q, const double *k, const double *v, const double *g,
                           const double *beta, double *S_inout, double *out, int n, int H, int dk,
                           int dv, int per_channel) {
    if (!q || !k || !v || !g || !beta || !S_inout || !out) return 1;
    if (n <= 0 || H <= 0 || dk <= 0 || dv <= 0) return 1;
    double *p = (double *)malloc(sizeof(double) * (size_t)dv);
    for (int s = 0; s < n; ++s) {
        for (int h = 0; h < H; ++h) {
            const size_t tok = (size_t)s * H + h;
            double *S = S_inout + tok * (size_t)dv * dk;
            const double *qt = q + tok * dk, *kt = k + tok * dk, *vt = v + tok * dv;
            if (per_channel) {
                const double *gt = g + tok * dk;
                for (int i = 0; i < dv; ++i)
                    for (int j = 0; j < dk; ++j) S[(size_t)i * dk + j] *= exp(gt[j]);
            } else {
                const double a = exp(g[tok]);
                for (size_t e = 0; e < (size_t)dv * dk; ++e) S[e] *= a;
            }
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * kt[j];
                p[i] = beta[tok] * (vt[i] - acc);
            }
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                double *row = S + (size_t)i * dk;
                for (int j = 0; j < dk; ++j) {
                    row[j] += p[i] * kt[j];
                    acc += row[j] * qt[j];
                }
                out[tok * dv + i] = acc;
            }
        }
    }
    free(p);
    return 0;
}

/*
 * Gated DeltaProduct ("Linear Attention, Visualized", section "Gated Delta
 * Product (GDP)"): per token t, decay once (S' = S D_t), then n_h substeps
 *     p = S k_tj;  u = beta_tj (v_tj - p);  S = S + u k_tj^T      (j = 1..n_h)
 * and read o_t = S q_t after the last substep.  Written from that definition,
 * not from the virtual-sequence mapping, so the mapping can be checked
 * against it.
 *   q [B,T,H,dk]; k [B,T,nh,H,dk]; v [B,T,nh,H,dv]; g [B,T,H] or [B,T,H,dk];
 *   beta [B,T,nh,H]; S0/S_final [n_seq,H,dv,dk]; out [B,T,H,dv].
 * Single-threaded over (sequence, head).
 */
int oracle_gdp_fwd(const double *q, const double *k, const double *v, const double *g,
                   const double *beta, const double *S0, double *out, double *S_final, int B,
                   int T, int H, int nh, int dk, int dv, const int *cu_seqlens, int n_seq,
                   int per_channel) {
    if (!q || !k || !v || !g || !beta || !out || nh < 1) return 1;
    if (B <= 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return 1;
    if (cu_seqlens) {
        if (B != 1 || n_seq <= 0 || cu_seqlens[0] != 0 || cu_seqlens[n_seq] != T) return 1;
        for (int i = 0; i < n_seq; ++i)
            if (cu_seqlens[i + 1] < cu_seqlens[i]) return 1;
    } else {
        n_seq = B;
    }
    double *S = (double *)malloc(sizeof(double) * (size_t)dv * dk);
    double *u = (double *)malloc(sizeof(double) * (size_t)dv);
    for (int s = 0; s < n_seq; ++s) {
        long t0 = cu_seqlens ? cu_seqlens[s] : (long)s * T;
        long t1 = cu_seqlens ? cu_seqlens[s + 1] : t0 + T;
        for (int h = 0; h < H; ++h) {
            const size_t soff = ((size_t)s * H + h) * (size_t)dv * dk;
            if (S0) memcpy(S, S0 + soff, sizeof(double) * (size_t)dv * dk);
            else memset(S, 0, sizeof(double) * (size_t)dv * dk);
            for (long t = t0; t < t1; ++t) {
                const size_t tok = (size_t)t * H + h;
                for (int j = 0; j < dk; ++j) {
                    const double a = per_channel ? exp(g[tok * dk + j]) : exp(g[tok]);
                    for (int i = 0; i < dv; ++i) S[(size_t)i * dk + j] *= a;
                }
                for (int jj = 0; jj < nh; ++jj) {
                    const size_t sub = ((size_t)t * nh + jj) * H + h;
                    const double *kt = k + sub * dk, *vt = v + sub * dv;
                    const double bt = beta[sub];
                    for (int i = 0; i < dv; ++i) {
                        double acc = 0.0;
                        for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * kt[j];
                        u[i] = bt * (vt[i] - acc);
                    }
                    for (int i = 0; i < dv; ++i)
                        for (int j = 0; j < dk; ++j) S[(size_t)i * dk + j] += u[i] * kt[j];
                }
                const double *qt = q + tok * dk;
                for (int i = 0; i < dv; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * qt[j];
                    out[tok * dv + i] = acc;
                }
            }
            if (S_final) memcpy(S_final + soff, S, sizeof(double) * (size_t)dv * dk);
        }
    }
    free(S);
    free(u);
    return 0;
}

/*
 * Gated DeltaNet-2 ("Gated DeltaNet-2, and the gate that was doing two jobs",
 * section "What decoupling actually means here"): the scalar step size splits
 * into an erase gate b_t (per key channel) and a write gate w_t (per value
 * channel), e_t = b_t . k_t, z_t = w_t . v_t, and in the page's row convention
 *     S_t = (I - k_t e_t^T) D_t S_{t-1} + k_t z_t^T,   o_t = S_t^T q_t.
 * Transposed to the column convention used here (S is d_v x d_k):
 *     S' = S D_t;  p = S' e_t;  u = z_t - p;  S = S' + u k_t^T;  o_t = S q_t.
 *   q, k [B,T,H,dk]; v, out [B,T,H,dv]; g [B,T,H] or [B,T,H,dk];
 *   b [B,T,H,dk]; w [B,T,H,dv]; S0/S_final [n_seq,H,dv,dk].
 * Single-threaded over (sequence, head).
 */
int oracle_gdn2_fwd(const double *q, const double *k, const double *v, const double *g,
                    const double *b, const double *w, const double *S0, double *out,
                    double *S_final, int B, int T, int H, int dk, int dv, const int *cu_seqlens,
                    int n_seq, int per_channel) {
    if (!q || !k || !v || !g || !b || !w || !out) return 1;
    if (B <= 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return 1;
    if (cu_seqlens) {
        if (B != 1 || n_seq <= 0 || cu_seqlens[0] != 0 || cu_seqlens[n_seq] != T) return 1;
        for (int i = 0; i < n_seq; ++i)
            if (cu_seqlens[i + 1] < cu_seqlens[i]) return 1;
    } else {
        n_seq = B;
    }
    double *S = (double *)malloc(sizeof(double) * (size_t)dv * dk);
    double *e = (double *)malloc(sizeof(double) * (size_t)dk);
    double *u = (double *)malloc(sizeof(double) * (size_t)dv);
    for (int s = 0; s < n_seq; ++s) {
        long t0 = cu_seqlens ? cu_seqlens[s] : (long)s * T;
        long t1 = cu_seqlens ? cu_seqlens[s + 1] : t0 + T;
        for (int h = 0; h < H; ++h) {
            const size_t soff = ((size_t)s * H + h) * (size_t)dv * dk;
            if (S0) memcpy(S, S0 + soff, sizeof(double) * (size_t)dv * dk);
            else memset(S, 0, sizeof(double) * (size_t)dv * dk);
            for (long t = t0; t < t1; ++t) {
                const size_t tok = (size_t)t * H + h;
                const double *kt = k + tok * dk, *vt = v + tok * dv, *qt = q + tok * dk;
                for (int j = 0; j < dk; ++j) {
                    const double a = per_channel ? exp(g[tok * dk + j]) : exp(g[tok]);
                    for (int i = 0; i < dv; ++i) S[(size_t)i * dk + j] *= a;
                    e[j] = b[tok * dk + j] * kt[j];
                }
                for (int i = 0; i < dv; ++i) {
                    double p = 0.0;
                    for (int j = 0; j < dk; ++j) p += S[(size_t)i * dk + j] * e[j];
                    u[i] = w[tok * dv + i] * vt[i] - p;
                }
                for (int i = 0; i < dv; ++i) {
                    double acc = 0.0;
                    double *row = S + (size_t)i * dk;
                    for (int j = 0; j < dk; ++j) {
                        row[j] += u[i] * kt[j];
                        acc += row[j] * qt[j];
                    }
                    out[tok * dv + i] = acc;
                }
            }
            if (S_final) memcpy(S_final + soff, S, sizeof(double) * (size_t)dv * dk);
        }
    }
    free(S);
    free(e);
    free(u);
    return 0;
}

/*
 * Implicit frame-level update ("video-delta-rule", sections "A First Attempt
 * at Frame-Level Updates" and "A Different Route"): the tokens of a sequence
 * are grouped into frames of n consecutive tokens (the last frame may be
 * shorter); with the frame's erasure G_t = sum_i gamma_i k_i k_i^T and write
 * C_t = sum_i gamma_i v_i k_i^T, the state takes one backward-Euler step
 *     S_t (I + G_t) = S_{t-1} D_t + C_t
 * (the frame's decay D_t first, as the forget gate at the frame boundary), and
 * every query of frame t reads the same S_t: o_i = S_t q_i.  I + G_t is
 * symmetric positive definite; it is factorised as L L^T (Cholesky) and each
 * row of S_t solves x (L L^T) = b by forward then backward substitution.
 *   q, k [B,T,H,dk]; v, out [B,T,H,dv]; gamma [B,T,H];
 *   g [B,F,H] or [B,F,H,dk] with F = ceil(T / n) (log-decay per frame);
 *   S0/S_final [B,H,dv,dk].
 */
int oracle_frame_fwd(const double *q, const double *k, const double *v, const double *g,
                     const double *gamma, const double *S0, double *out, double *S_final, int B,
                     int T, int H, int dk, int dv, int n, int per_channel) {
    if (!q || !k || !v || !g || !gamma || !out || n < 1) return 1;
    if (B <= 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return 1;
    const int F = (T + n - 1) / n;
    double *S = (double *)malloc(sizeof(double) * (size_t)dv * dk);
    double *Bm = (double *)malloc(sizeof(double) * (size_t)dv * dk);
    double *A = (double *)malloc(sizeof(double) * (size_t)dk * dk);
    double *y = (double *)malloc(sizeof(double) * (size_t)dk);
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            const size_t soff = ((size_t)b * H + h) * (size_t)dv * dk;
            if (S0) memcpy(S, S0 + soff, sizeof(double) * (size_t)dv * dk);
            else memset(S, 0, sizeof(double) * (size_t)dv * dk);
            for (int f = 0; f < F; ++f) {
                const int t0 = f * n, t1 = (t0 + n < T) ? t0 + n : T;
                const size_t fo = ((size_t)b * F + f) * H + h;
                /* B = S D_t, A = I */
                for (int i = 0; i < dv; ++i)
                    for (int j = 0; j < dk; ++j) {
                        const double a = per_channel ? exp(g[fo * dk + j]) : exp(g[fo]);
                        Bm[(size_t)i * dk + j] = S[(size_t)i * dk + j] * a;
                    }
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dk; ++j) A[(size_t)i * dk + j] = (i == j) ? 1.0 : 0.0;
                /* A += gamma k k^T, B += gamma v k^T over the frame's tokens */
                for (int t = t0; t < t1; ++t) {
                    const size_t tok = ((size_t)b * T + t) * H + h;
                    const double *kt = k + tok * dk, *vt = v + tok * dv, gm = gamma[tok];
                    for (int i = 0; i < dk; ++i)
                        for (int j = 0; j < dk; ++j) A[(size_t)i * dk + j] += gm * kt[i] * kt[j];
                    for (int i = 0; i < dv; ++i)
                        for (int j = 0; j < dk; ++j) Bm[(size_t)i * dk + j] += gm * vt[i] * kt[j];
                }
                /* Cholesky A = L L^T, L stored in the lower triangle of A */
                for (int j = 0; j < dk; ++j) {
                    double d = A[(size_t)j * dk + j];
                    for (int m = 0; m < j; ++m) d -= A[(size_t)j * dk + m] * A[(size_t)j * dk + m];
                    if (!(d > 0.0)) {
                        free(S); free(Bm); free(A); free(y);
                        return 2;
                    }
                    const double ljj = sqrt(d);
                    A[(size_t)j * dk + j] = ljj;
                    for (int i = j + 1; i < dk; ++i) {
                        double s = A[(size_t)i * dk + j];
                        for (int m = 0; m < j; ++m) s -= A[(size_t)i * dk + m] * A[(size_t)j * dk + m];
                        A[(size_t)i * dk + j] = s / ljj;
                    }
                }
                /* each row r of S_t: (L L^T) x = b_r^T (A is symmetric) */
                for (int r = 0; r < dv; ++r) {
                    const double *br = Bm + (size_t)r * dk;
                    for (int i = 0; i < dk; ++i) {
                        double s = br[i];
                        for (int m = 0; m < i; ++m) s -= A[(size_t)i * dk + m] * y[m];
                        y[i] = s / A[(size_t)i * dk + i];
                    }
                    double *xr = S + (size_t)r * dk;
                    for (int i = dk - 1; i >= 0; --i) {
                        double s = y[i];
                        for (int m = i + 1; m < dk; ++m) s -= A[(size_t)m * dk + i] * xr[m];
                        xr[i] = s / A[(size_t)i * dk + i];
                    }
                }
                /* every query of the frame reads S_t */
                for (int t = t0; t < t1; ++t) {
                    const size_t tok = ((size_t)b * T + t) * H + h;
                    const double *qt = q + tok * dk;
                    for (int i = 0; i < dv; ++i) {
                        double acc = 0.0;
                        for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * qt[j];
                        out[tok * dv + i] = acc;
                    }
                }
            }
            if (S_final) memcpy(S_final + soff, S, sizeof(double) * (size_t)dv * dk);
        }
    }
    free(S); free(Bm); free(A); free(y);
    return 0;
}
