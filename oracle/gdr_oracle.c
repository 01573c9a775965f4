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
