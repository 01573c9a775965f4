/*
 * gdr_oracle.c -- plain, slow, fp64 CPU oracle for the gated delta-rule
 * recurrent memory (DeltaNet / Gated DeltaNet / Kimi Delta Attention).
 *
 * TEST INFRASTRUCTURE ONLY. This file is called from the test-suite, the
 * package's smoke check and the benchmark's CPU-baseline leg, never from the
 * product path. It shares no code, header, table or helper with the CUDA
 * library, and the CUDA library never links or calls it.
 *
 * What it computes (one head, state S in R^{d_v x d_k}, o = S q):
 *
 *   S_t = S_{t-1} Diag(alpha_t) (I - e_t k_t k_t^T) + w_t v_t k_t^T
 *   o_t = scale * S_t q_t                      (read after the token's write)
 *
 * with alpha_t = exp(g_t) (a scalar for Gated DeltaNet, a d_k-vector acting
 * on the key dimension for Kimi Delta Attention, 1 for DeltaNet) and the
 * delta-rule mixer using e_t = w_t = beta_t. Sources:
 *   - "linear attention and its gated descendants", sections "DeltaNet"
 *     (the error-correcting update S_t = S_{t-1} + beta_t (v_t - S_{t-1}k_t)k_t^T
 *     and its erase/write reading), "Gated DeltaNet" (decay applied before the
 *     prediction: S_t = alpha_t S_{t-1} + beta_t (v_t - alpha_t S_{t-1} k_t) k_t^T)
 *     and "Kimi Delta Attention" (Diag(alpha_t) on the key/address dimension);
 *   - "Linear Attention Architectures: Mechanisms, Trade-offs, and Cross-Layer
 *     Routing", Sec. 3 (Kimi Delta Attention: "the diagonal decay matrix
 *     multiplies on the right ... along the key-feature dimension");
 *   - "Linear Attention & DeltaNet", How it works, items 1, 3 and 4 (the read
 *     out_t from the state after the update, and the erase-then-write form).
 * The generalised erase/write pair (e_t, w_t) exists for self-checks only:
 * (e, w) = (0, 1) with alpha = 1 is plain linear attention, S_t = S_{t-1} + v_t k_t^T.
 *
 * Row form used here (row j of S is s_j in R^{d_k}; rows never interact):
 *   s_bar = s_j (.) alpha_t ;  p = s_bar . k_t ;
 *   s_j   = s_bar - e_t p k_t + w_t v_{t,j} k_t ;  o_{t,j} = scale * (s_j . q_t)
 *
 * Layouts (row-major, contiguous): q, k [B,T,H,d_k]; v [B,T,H,d_v];
 * g [B,T,H] (scalar) or [B,T,H,d_k] (channel) or NULL (none);
 * erase, write [B,T,H]; S0, S_T [B,H,d_v,d_k]; o [B,T,H,d_v].
 * Inputs are float32 (in_f64 = 0) or float64 (in_f64 = 1); S0/S_T/o are fp64.
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_MODE_NONE 0
#define ORACLE_MODE_SCALAR 1
#define ORACLE_MODE_CHANNEL 2

/* rows of S handled by one task: a block of rows shares one pass over the tokens */
#define ORACLE_ROW_BLOCK 16

static inline double ld_in(const void* p, size_t i, int f64) {
    return f64 ? ((const double*)p)[i] : (double)((const float*)p)[i];
}

int gdr_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Returns 0 on success, -1 on an invalid argument, -2 on allocation failure. */
int gdr_oracle_recurrent(int B, int T, int H, int dk, int dv,
                         const void* q, const void* k, const void* v,
                         const void* g, int mode,
                         const void* erase, const void* write, int in_f64,
                         const double* S0, double scale,
                         double* o, double* S_T, int nthreads) {
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    if (mode != ORACLE_MODE_NONE && mode != ORACLE_MODE_SCALAR && mode != ORACLE_MODE_CHANNEL) return -1;
    if (mode != ORACLE_MODE_NONE && g == NULL) return -1;
    if ((T > 0) && (q == NULL || k == NULL || v == NULL || erase == NULL || write == NULL || o == NULL)) return -1;
    const int nblk = (dv + ORACLE_ROW_BLOCK - 1) / ORACLE_ROW_BLOCK;
    const long ntask = (long)B * H * nblk;
    int status = 0;
    if (nthreads <= 0) nthreads = gdr_oracle_max_threads();

#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (long task = 0; task < ntask; ++task) {
        const int blk = (int)(task % nblk);
        const int h = (int)((task / nblk) % H);
        const int b = (int)(task / ((long)nblk * H));
        const int j0 = blk * ORACLE_ROW_BLOCK;
        const int j1 = (j0 + ORACLE_ROW_BLOCK < dv) ? j0 + ORACLE_ROW_BLOCK : dv;
        const int nr = j1 - j0;
        double* s = (double*)malloc(sizeof(double) * (size_t)nr * dk);
        double* kt = (double*)malloc(sizeof(double) * (size_t)dk);
        double* qt = (double*)malloc(sizeof(double) * (size_t)dk);
        double* at = (double*)malloc(sizeof(double) * (size_t)dk);
        if (!s || !kt || !qt || !at) {
            free(s); free(kt); free(qt); free(at);
#pragma omp atomic write
            status = -2;
            continue;
        }
        /* initial state rows */
        for (int r = 0; r < nr; ++r)
            for (int c = 0; c < dk; ++c)
                s[(size_t)r * dk + c] =
                    S0 ? S0[(((size_t)b * H + h) * dv + (j0 + r)) * dk + c] : 0.0;

        for (int t = 0; t < T; ++t) {
            const size_t tok = ((size_t)b * T + t) * H + h; /* (b, t, h) index */
            for (int c = 0; c < dk; ++c) {
                kt[c] = ld_in(k, tok * dk + c, in_f64);
                qt[c] = ld_in(q, tok * dk + c, in_f64);
                if (mode == ORACLE_MODE_NONE) at[c] = 1.0;
                else if (mode == ORACLE_MODE_SCALAR) at[c] = exp(ld_in(g, tok, in_f64));
                else at[c] = exp(ld_in(g, tok * dk + c, in_f64));
            }
            const double e = ld_in(erase, tok, in_f64);
            const double w = ld_in(write, tok, in_f64);
            for (int r = 0; r < nr; ++r) {
                double* sj = s + (size_t)r * dk;
                const double vj = ld_in(v, tok * dv + (j0 + r), in_f64);
                /* decay: s_bar = s_j (.) alpha_t */
                for (int c = 0; c < dk; ++c) sj[c] *= at[c];
                /* prediction from the decayed memory: p = s_bar . k_t */
                double p = 0.0;
                for (int c = 0; c < dk; ++c) p += sj[c] * kt[c];
                /* erase e_t p k_t, write w_t v_{t,j} k_t */
                const double coef = w * vj - e * p;
                for (int c = 0; c < dk; ++c) sj[c] += coef * kt[c];
                /* read after write */
                double a = 0.0;
                for (int c = 0; c < dk; ++c) a += sj[c] * qt[c];
                o[tok * dv + (j0 + r)] = scale * a;
            }
        }
        if (S_T)
            for (int r = 0; r < nr; ++r)
                for (int c = 0; c < dk; ++c)
                    S_T[(((size_t)b * H + h) * dv + (j0 + r)) * dk + c] = s[(size_t)r * dk + c];
        free(s); free(kt); free(qt); free(at);
    }
    return status;
}

/*
 * Gradients of the mixer recurrence (e_t = w_t = beta_t) for a loss whose gradients with respect
 * to the outputs are dO [B,T,H,d_v] and dS_T [B,H,d_v,d_k] (NULL: zero). Reverse-mode
 * differentiation of the row form above, written out step by step: a forward sweep keeps the state
 * before every token, then the tokens are taken from the last to the first. With ds the gradient
 * of row j of the state after token t, the forward steps
 *     s_bar = s (.) a ;  p = s_bar . k ;  delta = beta (v_j - p) ;  s' = s_bar + delta k ;
 *     o_j = scale (s' . q)
 * give, in reverse order,
 *     ds'    = ds + scale do_j q            dq += scale do_j s'
 *     ddelta = ds' . k                      dk += delta ds'
 *     dbeta += ddelta (v_j - p)             dv_j = beta ddelta
 *     dp     = -beta ddelta
 *     ds_bar = ds' + dp k                   dk += dp s_bar
 *     ds     = ds_bar (.) a                 dg += ds_bar (.) s_bar   (a = exp(g): da/dg = a)
 * summed over the rows j for dq, dk, dbeta and dg (over the channels too for the scalar gate).
 * Outputs: dq, dk [B,T,H,d_k]; dv [B,T,H,d_v]; dbeta [B,T,H]; dg [B,T,H] (scalar) or [B,T,H,d_k]
 * (channel), unused for NONE (may be NULL); dS0 [B,H,d_v,d_k] or NULL. All fp64.
 * Returns 0, -1 on an invalid argument, -2 on allocation failure.
 */
int gdr_oracle_backward(int B, int T, int H, int dk, int dv,
                        const void* q, const void* k, const void* v, const void* g, int mode,
                        const void* beta, int in_f64, const double* S0, double scale,
                        const double* dO, const double* dST,
                        double* dq, double* dk_out, double* dv_out, double* dg, double* dbeta,
                        double* dS0, int nthreads) {
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    if (mode != ORACLE_MODE_NONE && mode != ORACLE_MODE_SCALAR && mode != ORACLE_MODE_CHANNEL) return -1;
    if (mode != ORACLE_MODE_NONE && (g == NULL || dg == NULL)) return -1;
    if (T > 0 && (q == NULL || k == NULL || v == NULL || beta == NULL || dO == NULL || dq == NULL ||
                  dk_out == NULL || dv_out == NULL || dbeta == NULL))
        return -1;
    const long nhead = (long)B * H;
    int status = 0;
    if (nthreads <= 0) nthreads = gdr_oracle_max_threads();

#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (long bh = 0; bh < nhead; ++bh) {
        const int h = (int)(bh % H);
        const int b = (int)(bh / H);
        const size_t sz = (size_t)dv * dk;
        double* hist = (double*)malloc(sizeof(double) * sz * (size_t)(T > 0 ? T : 1));
        double* s = (double*)malloc(sizeof(double) * sz);
        double* ds = (double*)malloc(sizeof(double) * sz);
        double* vec = (double*)malloc(sizeof(double) * (size_t)dk * 8);
        if (!hist || !s || !ds || !vec) {
            free(hist); free(s); free(ds); free(vec);
#pragma omp atomic write
            status = -2;
            continue;
        }
        double *kt = vec, *qt = vec + dk, *at = vec + 2 * dk, *sbar = vec + 3 * dk, *dsp = vec + 4 * dk;
        double *gq = vec + 5 * dk, *gk = vec + 6 * dk, *gg = vec + 7 * dk;
        for (size_t i = 0; i < sz; ++i) {
            s[i] = S0 ? S0[(size_t)bh * sz + i] : 0.0;
            ds[i] = dST ? dST[(size_t)bh * sz + i] : 0.0;
        }
        /* forward sweep: the state before each token */
        for (int t = 0; t < T; ++t) {
            const size_t tok = ((size_t)b * T + t) * H + h;
            memcpy(hist + (size_t)t * sz, s, sizeof(double) * sz);
            const double bt = ld_in(beta, tok, in_f64);
            for (int c = 0; c < dk; ++c) {
                kt[c] = ld_in(k, tok * dk + c, in_f64);
                if (mode == ORACLE_MODE_NONE) at[c] = 1.0;
                else if (mode == ORACLE_MODE_SCALAR) at[c] = exp(ld_in(g, tok, in_f64));
                else at[c] = exp(ld_in(g, tok * dk + c, in_f64));
            }
            for (int j = 0; j < dv; ++j) {
                double* sj = s + (size_t)j * dk;
                double p = 0.0;
                for (int c = 0; c < dk; ++c) {
                    sj[c] *= at[c];
                    p += sj[c] * kt[c];
                }
                const double delta = bt * (ld_in(v, tok * dv + j, in_f64) - p);
                for (int c = 0; c < dk; ++c) sj[c] += delta * kt[c];
            }
        }
        /* reverse sweep */
        for (int t = T - 1; t >= 0; --t) {
            const size_t tok = ((size_t)b * T + t) * H + h;
            const double bt = ld_in(beta, tok, in_f64);
            for (int c = 0; c < dk; ++c) {
                kt[c] = ld_in(k, tok * dk + c, in_f64);
                qt[c] = ld_in(q, tok * dk + c, in_f64);
                if (mode == ORACLE_MODE_NONE) at[c] = 1.0;
                else if (mode == ORACLE_MODE_SCALAR) at[c] = exp(ld_in(g, tok, in_f64));
                else at[c] = exp(ld_in(g, tok * dk + c, in_f64));
                gq[c] = gk[c] = gg[c] = 0.0;
            }
            double gb = 0.0;
            for (int j = 0; j < dv; ++j) {
                const double* sj = hist + (size_t)t * sz + (size_t)j * dk;
                double* dsj = ds + (size_t)j * dk;
                const double vj = ld_in(v, tok * dv + j, in_f64);
                const double doj = dO[tok * dv + j];
                double p = 0.0;
                for (int c = 0; c < dk; ++c) {
                    sbar[c] = sj[c] * at[c];
                    p += sbar[c] * kt[c];
                }
                const double delta = bt * (vj - p);
                double ddelta = 0.0;
                for (int c = 0; c < dk; ++c) {
                    const double spc = sbar[c] + delta * kt[c];
                    dsp[c] = dsj[c] + scale * doj * qt[c];
                    gq[c] += scale * doj * spc;
                    gk[c] += delta * dsp[c];
                    ddelta += dsp[c] * kt[c];
                }
                gb += ddelta * (vj - p);
                dv_out[tok * dv + j] = bt * ddelta;
                const double dp = -bt * ddelta;
                for (int c = 0; c < dk; ++c) {
                    const double dsb = dsp[c] + dp * kt[c];
                    gk[c] += dp * sbar[c];
                    gg[c] += dsb * sbar[c];
                    dsj[c] = dsb * at[c];
                }
            }
            for (int c = 0; c < dk; ++c) {
                dq[tok * dk + c] = gq[c];
                dk_out[tok * dk + c] = gk[c];
            }
            dbeta[tok] = gb;
            if (mode == ORACLE_MODE_SCALAR) {
                double sum = 0.0;
                for (int c = 0; c < dk; ++c) sum += gg[c];
                dg[tok] = sum;
            } else if (mode == ORACLE_MODE_CHANNEL) {
                for (int c = 0; c < dk; ++c) dg[tok * dk + c] = gg[c];
            }
        }
        if (dS0)
            for (size_t i = 0; i < sz; ++i) dS0[(size_t)bh * sz + i] = ds[i];
        free(hist); free(s); free(ds); free(vec);
    }
    return status;
}

/*
 * Gated DeltaNet-2: the delta rule with a channel-wise erase gate on the key side and a
 * channel-wise write gate on the value side ("Linear Attention Architectures: Mechanisms,
 * Trade-offs, and Cross-Layer Routing", Sec. 3, the Gated DeltaNet-2 paragraph and its gate
 * definitions). With the decay-adjusted memory S_bar = S_{t-1} Diag(alpha_t), the gated erase
 * direction e_t (.) k_t and the gated write target w_t (.) v_t, the residual written to memory is
 * r_t = w_t (.) v_t - S_bar (e_t (.) k_t), and
 *
 *     S_t = S_bar + r_t k_t^T ,    o_t = scale * S_t q_t .
 *
 * (The page's formulas are stripped; this is the reading under which one residual is written
 * along k_t, e_t = w_t = beta_t 1 gives Kimi Delta Attention and a scalar alpha then gives Gated
 * DeltaNet, as the page states.) Row form: s_bar = s_j (.) alpha ; p = s_bar . (e (.) k) ;
 * s_j = s_bar + (w_j v_{t,j} - p) k ; o_{t,j} = scale (s_j . q).
 * erase: [B,T,H,d_k]; write: [B,T,H,d_v]; other arguments as gdr_oracle_recurrent.
 */
int gdr_oracle_recurrent_gdn2(int B, int T, int H, int dk, int dv,
                              const void* q, const void* k, const void* v,
                              const void* g, int mode,
                              const void* erase, const void* write, int in_f64,
                              const double* S0, double scale,
                              double* o, double* S_T, int nthreads) {
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    if (mode != ORACLE_MODE_NONE && mode != ORACLE_MODE_SCALAR && mode != ORACLE_MODE_CHANNEL) return -1;
    if (mode != ORACLE_MODE_NONE && g == NULL) return -1;
    if ((T > 0) && (q == NULL || k == NULL || v == NULL || erase == NULL || write == NULL || o == NULL)) return -1;
    const long nhead = (long)B * H;
    int status = 0;
    if (nthreads <= 0) nthreads = gdr_oracle_max_threads();

#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (long bh = 0; bh < nhead; ++bh) {
        const int h = (int)(bh % H);
        const int b = (int)(bh / H);
        double* s = (double*)malloc(sizeof(double) * (size_t)dv * dk);
        double* vec = (double*)malloc(sizeof(double) * (size_t)dk * 4);
        if (!s || !vec) {
            free(s); free(vec);
#pragma omp atomic write
            status = -2;
            continue;
        }
        double *kt = vec, *qt = vec + dk, *at = vec + 2 * dk, *ek = vec + 3 * dk;
        for (size_t i = 0; i < (size_t)dv * dk; ++i) s[i] = S0 ? S0[(size_t)bh * dv * dk + i] : 0.0;
        for (int t = 0; t < T; ++t) {
            const size_t tok = ((size_t)b * T + t) * H + h;
            for (int c = 0; c < dk; ++c) {
                kt[c] = ld_in(k, tok * dk + c, in_f64);
                qt[c] = ld_in(q, tok * dk + c, in_f64);
                ek[c] = ld_in(erase, tok * dk + c, in_f64) * kt[c]; /* gated erase direction */
                if (mode == ORACLE_MODE_NONE) at[c] = 1.0;
                else if (mode == ORACLE_MODE_SCALAR) at[c] = exp(ld_in(g, tok, in_f64));
                else at[c] = exp(ld_in(g, tok * dk + c, in_f64));
            }
            for (int j = 0; j < dv; ++j) {
                double* sj = s + (size_t)j * dk;
                /* decay-adjusted memory, then its prediction along the gated erase direction */
                double p = 0.0;
                for (int c = 0; c < dk; ++c) {
                    sj[c] *= at[c];
                    p += sj[c] * ek[c];
                }
                /* residual: gated write target minus that prediction, written along k_t */
                const double r = ld_in(write, tok * dv + j, in_f64) * ld_in(v, tok * dv + j, in_f64) - p;
                double a = 0.0;
                for (int c = 0; c < dk; ++c) {
                    sj[c] += r * kt[c];
                    a += sj[c] * qt[c];
                }
                o[tok * dv + j] = scale * a;
            }
        }
        if (S_T)
            for (size_t i = 0; i < (size_t)dv * dk; ++i) S_T[(size_t)bh * dv * dk + i] = s[i];
        free(s); free(vec);
    }
    return status;
}
