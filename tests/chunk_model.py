"""fp64 NumPy model of the chunkwise-parallel algebra (test helper, not the oracle).

It restates, per head and per chunk of C tokens, the UT/WY chunk form that the
CUDA kernels implement, so that the derivation can be checked against the
token-by-token oracle on the CPU. Sources: "linear attention and its gated
descendants", "Chunkwise Parallel Form" (boundary state plus a masked
intra-chunk part, O = Q S^T + (Q K^T (.) M) V for plain linear attention) and
"Linear Attention & DeltaNet", item 3 (a chunk of delta-rule updates folds into
a WY/Householder compact form).

Derivation (value-by-key state, o = S q, positions r = 1..C in a chunk,
Gamma_r = inclusive cumulative log-decay, gamma_r = exp(Gamma_r)):
  delta_r = beta_r (v_r - S_{r-1} Diag(alpha_r) k_r)
  S_r     = S_0 Diag(gamma_r) + sum_{i<=r} delta_i (k_i (.) gamma_r / gamma_i)^T
  => (I + A) Delta = diag(beta) V - diag(beta) (K (.) gamma) S_0^T,
     A_ri = beta_r (k_r (.) gamma_r).(k_i / gamma_i) for i < r  (strictly lower)
  => Delta = U - W S_0^T,  T = (I + A)^-1,  W = T diag(beta)(K (.) gamma),  U = T diag(beta) V
  O      = scale [ (Q (.) gamma) S_0^T + (M (.) (Q (.) gamma)(K / gamma)^T) Delta ]   (M includes the diagonal)
  S_next = S_0 Diag(gamma_C) + Delta^T (K (.) gamma_C / gamma)
"""
import numpy as np


def chunk_forward_head(q, k, v, g, beta, mode, S0, C, scale):
    """One head: q,k [T,dk], v [T,dv], beta [T], g [T] / [T,dk] / None; S0 [dv,dk]."""
    T, dk = k.shape
    S = np.array(S0, dtype=np.float64, copy=True)
    O = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        sl = slice(c0, min(T, c0 + C))
        Qc, Kc, Vc, bc = q[sl], k[sl], v[sl], beta[sl]
        n = Kc.shape[0]
        if mode == "none":
            Gam = np.zeros((n, dk))
        elif mode == "scalar":
            Gam = np.repeat(np.cumsum(g[sl])[:, None], dk, axis=1)
        else:
            Gam = np.cumsum(g[sl], axis=0)
        gam = np.exp(Gam)
        if mode == "channel":
            KK = (Kc * gam) @ (Kc / gam).T
            QK = (Qc * gam) @ (Kc / gam).T
        else:  # pairwise exp(Gamma_r - Gamma_i), safe for r >= i
            D = np.exp(np.minimum(Gam[:, :1] - Gam[:, :1].T, 0.0))
            KK = (Kc @ Kc.T) * D
            QK = (Qc @ Kc.T) * D
        A = np.tril(bc[:, None] * KK, -1)
        Tm = np.linalg.inv(np.eye(n) + A)
        W = Tm @ (bc[:, None] * (Kc * gam))
        U = Tm @ (bc[:, None] * Vc)
        Delta = U - W @ S.T
        P = np.tril(QK)
        O[sl] = scale * ((Qc * gam) @ S.T + P @ Delta)
        Ktil = Kc * np.exp(Gam[-1][None, :] - Gam)
        S = S * gam[-1][None, :] + Delta.T @ Ktil
    return O, S


def chunk_forward(q, k, v, g, beta, mode, S0, C, scale=None):
    """Batched wrapper: q,k [B,T,H,dk], v [B,T,H,dv]; returns o [B,T,H,dv], S [B,H,dv,dk]."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    scale = 1.0 / np.sqrt(dk) if scale is None else scale
    o = np.zeros((B, T, H, dv))
    S_T = np.zeros((B, H, dv, dk))
    for b in range(B):
        for h in range(H):
            gg = None if mode == "none" else g[b, :, h]
            s0 = np.zeros((dv, dk)) if S0 is None else S0[b, h]
            o[b, :, h], S_T[b, h] = chunk_forward_head(q[b, :, h], k[b, :, h], v[b, :, h], gg,
                                                       beta[b, :, h], mode, s0, C, scale)
    return o, S_T
