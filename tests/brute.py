"""Brute-force restatements of the recurrence for tiny sizes (test helpers).

Independent of the oracle's row loop: the state evolution is written as the
affine transition S_t = S_{t-1} A_t + B_t ("linear attention and its gated
descendants", section "where does this leave us?": from DeltaNet onward the
update is a multiplicative transition plus a write, A_t = (I - beta k k^T) Diag(alpha)
in the key-by-value orientation; here the value-by-key orientation o = S q is
used, so A_t = Diag(alpha_t)(I - e_t k_t k_t^T) acts from the right). Two forms:

* explicit products:   S_t = S0 A_1...A_t + sum_{i<=t} B_i A_{i+1}...A_t
* Kronecker form:      vec(S_t) = (A_t^T kron I) vec(S_{t-1}) + vec(B_t)   (column-major vec)
"""
import numpy as np


def transitions(k, v, g, mode, erase, write):
    """Per-token (A_t [dk,dk], B_t [dv,dk]) for one head; k [T,dk], v [T,dv]."""
    T, dk = k.shape
    As, Bs = [], []
    for t in range(T):
        if mode == "none":
            alpha = np.ones(dk)
        elif mode == "scalar":
            alpha = np.full(dk, np.exp(g[t]))
        else:
            alpha = np.exp(g[t])
        kt = k[t][:, None]
        As.append(np.diag(alpha) @ (np.eye(dk) - erase[t] * (kt @ kt.T)))
        Bs.append(write[t] * (v[t][:, None] @ kt.T))
    return As, Bs


def states_by_product(S0, As, Bs):
    """All S_t (t = 1..T) from explicit products of the transitions."""
    T = len(As)
    out = []
    for t in range(T):
        P = np.eye(As[0].shape[0])
        for s in range(t + 1):
            P = P @ As[s]
        St = S0 @ P
        for i in range(t + 1):
            Q = np.eye(As[0].shape[0])
            for s in range(i + 1, t + 1):
                Q = Q @ As[s]
            St = St + Bs[i] @ Q
        out.append(St)
    return out


def states_by_kron(S0, As, Bs):
    """All S_t from the d_v*d_k-dimensional linear system, column-major vec."""
    dv, dk = S0.shape
    x = S0.reshape(-1, order="F")
    out = []
    for A, Bm in zip(As, Bs):
        x = np.kron(A.T, np.eye(dv)) @ x + Bm.reshape(-1, order="F")
        out.append(x.reshape(dv, dk, order="F"))
    return out


def transitions_gdn2(k, v, g, mode, erase, write):
    """Gated DeltaNet-2 per-token (A_t, B_t) for one head: A_t = Diag(alpha_t)(I - (e_t * k_t) k_t^T)
    and B_t = (w_t * v_t) k_t^T, with erase e_t [dk] and write w_t [dv] channel-wise gates."""
    T, dk = k.shape
    As, Bs = [], []
    for t in range(T):
        if mode == "none":
            alpha = np.ones(dk)
        elif mode == "scalar":
            alpha = np.full(dk, np.exp(g[t]))
        else:
            alpha = np.exp(g[t])
        kt = k[t][:, None]
        As.append(np.diag(alpha) @ (np.eye(dk) - (erase[t][:, None] * kt) @ kt.T))
        Bs.append((write[t] * v[t])[:, None] @ kt.T)
    return As, Bs
