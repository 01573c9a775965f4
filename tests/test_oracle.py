"""Pins for the fp64 oracle (CPU only).

Each test checks the oracle against something other than itself: a closed
form, a brute-force restatement, a hand-worked example or a limiting case the
pages state. Together they fail on a dropped term, a wrong sign, a transposed
operand, a misplaced decay or a read-before-write.
"""
import json
import os

import numpy as np
import pytest

import oracle
from brute import states_by_kron, states_by_product, transitions

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples_d2.json")
MODES = ("none", "scalar", "channel")


def _rand_problem(rng, B, T, H, dk, dv, mode, unit_keys=True, g_scale=0.3):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    if unit_keys:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    beta = rng.uniform(0.0, 1.0, (B, T, H))
    if mode == "scalar":
        g = -g_scale * rng.uniform(0, 1, (B, T, H))
    elif mode == "channel":
        g = -g_scale * rng.uniform(0, 1, (B, T, H, dk))
    else:
        g = None
    return q, k, v, g, beta


def _run(q, k, v, g, beta, mode, S0=None, **kw):
    return oracle.recurrent(q, k, v, g, beta, mode, S0=S0, f64_inputs=True, **kw)


# ---------------------------------------------------------------- golden ---
def test_hand_worked_examples():
    """Hand-worked tiny examples of the update rule (tests/golden)."""
    spec = json.load(open(GOLDEN))
    for case in spec["cases"]:
        k = np.array(case["k"], float)[None, :, None, :]
        v = np.array(case["v"], float)[None, :, None, :]
        q = np.array(case["q"], float)[None, :, None, :]
        beta = np.array(case["beta"], float)[None, :, None]
        g = np.log(np.array(case["alpha"], float))
        g = g[None, :, None] if case["mode"] == "scalar" else g[None, :, None, :]
        S0 = None if case["S0"] is None else np.array(case["S0"], float)[None, None]
        T = k.shape[1]
        for t in range(1, T + 1):  # every prefix: intermediate states too
            o, S = _run(q[:, :t], k[:, :t], v[:, :t], g[:, :t], beta[:, :t], case["mode"], S0,
                        scale=case["scale"])
            np.testing.assert_allclose(o[0, :, 0], np.array(case["o"], float)[:t], atol=1e-12)
            np.testing.assert_allclose(S[0, 0], np.array(case["S"], float)[t - 1], atol=1e-12)


# ----------------------------------------------------------- brute force ---
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("generalised", [False, True])
def test_matches_transition_products(mode, generalised):
    """Per-token states and outputs equal the explicit product of affine
    transitions and the d_v*d_k Kronecker form on tiny T (T<=8, d<=6)."""
    rng = np.random.default_rng(11 + MODES.index(mode) + 7 * generalised)
    B, T, H, dk, dv = 2, 7, 2, 5, 4
    q, k, v, g, beta = _rand_problem(rng, B, T, H, dk, dv, mode, unit_keys=not generalised, g_scale=0.7)
    S0 = rng.standard_normal((B, H, dv, dk))
    erase = rng.uniform(0, 1.2, (B, T, H)) if generalised else beta
    write = rng.uniform(-1, 1, (B, T, H)) if generalised else beta
    scale = 0.37
    o, S_T = _run(q, k, v, g, beta, mode, S0, erase=erase, write=write, scale=scale)
    for b in range(B):
        for h in range(H):
            gg = None if g is None else g[b, :, h]
            As, Bs = transitions(k[b, :, h], v[b, :, h], gg, mode, erase[b, :, h], write[b, :, h])
            Sp = states_by_product(S0[b, h], As, Bs)
            Sk = states_by_kron(S0[b, h], As, Bs)
            for t in range(T):
                np.testing.assert_allclose(Sp[t], Sk[t], atol=1e-12)
                np.testing.assert_allclose(o[b, t, h], scale * Sp[t] @ q[b, t, h], atol=1e-12)
            np.testing.assert_allclose(S_T[b, h], Sp[-1], atol=1e-12)


# ---------------------------------------------------------- closed forms ---
@pytest.mark.parametrize("mode", MODES)
def test_erase_free_is_decayed_linear_attention(mode):
    """Erase-free mode (e=0, w=1) is (decayed) linear attention, whose output has
    the closed form scale * (Q K^T (.) D) V with D_ti = exp(Gamma_t - Gamma_i) for
    i <= t (D = causal mask incl. the diagonal when alpha = 1): "linear attention
    and its gated descendants", Chunkwise Parallel Form, and "Linear Attention &
    DeltaNet", item 1."""
    rng = np.random.default_rng(3 + MODES.index(mode))
    B, T, H, dk, dv = 1, 41, 2, 8, 6
    q, k, v, g, beta = _rand_problem(rng, B, T, H, dk, dv, mode, unit_keys=False)
    zeros, ones = np.zeros((B, T, H)), np.ones((B, T, H))
    o, S_T = _run(q, k, v, g, beta, mode, erase=zeros, write=ones, scale=1.0)
    for h in range(H):
        Q, K, V = q[0, :, h], k[0, :, h], v[0, :, h]
        if mode == "channel":
            Gam = np.cumsum(g[0, :, h], axis=0)  # [T, dk]
            ref = np.zeros((T, dv))
            for t in range(T):
                for i in range(t + 1):
                    ref[t] += V[i] * np.dot(K[i] * np.exp(Gam[t] - Gam[i]), Q[t])
            Sref = sum(np.outer(V[i], K[i] * np.exp(Gam[-1] - Gam[i])) for i in range(T))
        else:
            Gam = np.zeros(T) if mode == "none" else np.cumsum(g[0, :, h])
            D = np.tril(np.exp(Gam[:, None] - Gam[None, :]))
            ref = ((Q @ K.T) * D) @ V
            Sref = (V * np.exp(Gam[-1] - Gam)[:, None]).T @ K
        np.testing.assert_allclose(o[0, :, h], ref, atol=1e-11)
        np.testing.assert_allclose(S_T[0, h], Sref, atol=1e-11)


def test_plain_linear_attention_mask_includes_diagonal():
    """With alpha = 1, e = 0, w = 1: o = (Q K^T (.) M) V, M lower-triangular with the
    diagonal (token t reads its own write). A strictly-lower mask must fail."""
    rng = np.random.default_rng(5)
    T, d = 16, 4
    q, k, v, _, beta = _rand_problem(rng, 1, T, 1, d, d, "none", unit_keys=False)
    o, _ = _run(q, k, v, None, beta, "none", erase=np.zeros_like(beta), write=np.ones_like(beta), scale=1.0)
    Q, K, V = q[0, :, 0], k[0, :, 0], v[0, :, 0]
    np.testing.assert_allclose(o[0, :, 0], np.tril(Q @ K.T) @ V, atol=1e-12)
    assert np.abs(o[0, :, 0] - np.tril(Q @ K.T, -1) @ V).max() > 1e-3


# --------------------------------------------------- delta-rule semantics ---
def test_exact_recall_orthonormal_keys():
    """alpha=1, beta=1 and orthonormal keys: the memory stores and recalls each
    value exactly, S_T k_i = v_i; a query equal to k_i reads v_i / sqrt(d_k)
    ("linear attention and its gated descendants", DeltaNet: orthogonal keys
    isolate v_j; "Linear Attention & DeltaNet", item 3)."""
    rng = np.random.default_rng(7)
    dk, dv, T = 16, 9, 12
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Qm[:, :T].T  # T orthonormal rows
    k = keys[None, :, None, :]
    v = rng.standard_normal((1, T, 1, dv))
    q = keys[rng.permutation(T)][None, :, None, :]  # query some earlier or later key
    beta = np.ones((1, T, 1))
    o, S_T = _run(q, k, v, None, beta, "none")
    for i in range(T):
        np.testing.assert_allclose(S_T[0, 0] @ keys[i], v[0, i, 0], atol=1e-12)
    qidx = [int(np.argmax(np.abs(keys @ q[0, t, 0]))) for t in range(T)]
    for t in range(T):
        want = v[0, qidx[t], 0] / np.sqrt(dk) if qidx[t] <= t else np.zeros(dv)
        np.testing.assert_allclose(o[0, t, 0], want, atol=1e-12)


def test_overwrite_same_key_recalls_latest():
    rng = np.random.default_rng(8)
    dk, dv = 8, 5
    kk = rng.standard_normal(dk); kk /= np.linalg.norm(kk)
    k = np.stack([kk, kk])[None, :, None, :]
    v = rng.standard_normal((1, 2, 1, dv))
    _, S_T = _run(k, k, v, None, np.ones((1, 2, 1)), "none")
    np.testing.assert_allclose(S_T[0, 0] @ kk, v[0, 1, 0], atol=1e-12)


@pytest.mark.parametrize("mode", MODES)
def test_beta_blend_at_current_key(mode):
    """For a unit key: S_t k_t = (1 - beta) Sbar k_t + beta v_t (beta = 1 replaces,
    beta = 0 keeps, 0 < beta < 1 blends -- the DeltaNet section)."""
    rng = np.random.default_rng(9 + MODES.index(mode))
    B, T, H, dk, dv = 1, 6, 1, 7, 3
    q, k, v, g, beta = _rand_problem(rng, B, T, H, dk, dv, mode)
    S0 = rng.standard_normal((B, H, dv, dk))
    S = S0[0, 0].copy()
    for t in range(T):
        _, St = _run(q[:, t:t + 1], k[:, t:t + 1], v[:, t:t + 1], None if g is None else g[:, t:t + 1],
                     beta[:, t:t + 1], mode, S[None, None])
        if mode == "none":
            a = np.ones(dk)
        elif mode == "scalar":
            a = np.full(dk, np.exp(g[0, t, 0]))
        else:
            a = np.exp(g[0, t, 0])
        kt = k[0, t, 0]
        Sbar = S * a[None, :]
        want = (1 - beta[0, t, 0]) * (Sbar @ kt) + beta[0, t, 0] * v[0, t, 0]
        np.testing.assert_allclose(St[0, 0] @ kt, want, atol=1e-12)
        S = St[0, 0]


@pytest.mark.parametrize("mode", ("scalar", "channel"))
def test_beta_zero_only_decays(mode):
    """beta = 0 writes nothing: S_T = S0 Diag(prod alpha), o_t = scale S0 Diag(prod_{s<=t} alpha) q_t."""
    rng = np.random.default_rng(12)
    B, T, H, dk, dv = 1, 9, 2, 6, 5
    q, k, v, g, _ = _rand_problem(rng, B, T, H, dk, dv, mode)
    S0 = rng.standard_normal((B, H, dv, dk))
    o, S_T = _run(q, k, v, g, np.zeros((B, T, H)), mode, S0)
    for h in range(H):
        Gam = np.cumsum(g[0, :, h], axis=0)
        Gam = Gam[:, None] * np.ones(dk) if mode == "scalar" else Gam
        for t in range(T):
            np.testing.assert_allclose(o[0, t, h], (S0[0, h] * np.exp(Gam[t])[None, :]) @ q[0, t, h] / np.sqrt(dk),
                                       atol=1e-12)
        np.testing.assert_allclose(S_T[0, h], S0[0, h] * np.exp(Gam[-1])[None, :], atol=1e-12)


@pytest.mark.parametrize("mode", ("scalar", "channel"))
def test_alpha_zero_resets_every_token(mode):
    """alpha = 0 (g = -1e4, exp underflows to exactly 0): S_t = beta_t v_t k_t^T and
    o_t = scale beta_t (k_t . q_t) v_t, whatever came before."""
    rng = np.random.default_rng(13)
    B, T, H, dk, dv = 2, 8, 2, 6, 4
    q, k, v, g, beta = _rand_problem(rng, B, T, H, dk, dv, mode)
    g = np.full_like(g, -1e4)
    S0 = rng.standard_normal((B, H, dv, dk))
    o, S_T = _run(q, k, v, g, beta, mode, S0)
    want_o = (beta * np.einsum("bthd,bthd->bth", k, q))[..., None] * v / np.sqrt(dk)
    np.testing.assert_allclose(o, want_o, atol=1e-12)
    want_S = beta[:, -1, :, None, None] * np.einsum("bhv,bhk->bhvk", v[:, -1], k[:, -1])
    np.testing.assert_allclose(S_T, want_S, atol=1e-12)


# ------------------------------------------------------------- reductions ---
def test_channel_with_constant_channels_is_scalar():
    """KDA whose per-channel gate is constant across channels is Gated DeltaNet."""
    rng = np.random.default_rng(14)
    B, T, H, dk, dv = 2, 30, 2, 8, 8
    q, k, v, g, beta = _rand_problem(rng, B, T, H, dk, dv, "scalar")
    S0 = rng.standard_normal((B, H, dv, dk))
    o1, s1 = _run(q, k, v, g, beta, "scalar", S0)
    o2, s2 = _run(q, k, v, np.repeat(g[..., None], dk, axis=-1), beta, "channel", S0)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(s1, s2, atol=1e-13)


def test_scalar_with_zero_log_decay_is_deltanet():
    rng = np.random.default_rng(15)
    B, T, H, dk, dv = 1, 25, 3, 8, 4
    q, k, v, _, beta = _rand_problem(rng, B, T, H, dk, dv, "none")
    S0 = rng.standard_normal((B, H, dv, dk))
    o1, s1 = _run(q, k, v, None, beta, "none", S0)
    o2, s2 = _run(q, k, v, np.zeros((B, T, H)), beta, "scalar", S0)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(s1, s2)


def test_first_order_small_beta_limit():
    """beta = eps, alpha = 1, S0 = 0: o / eps -> scale (Q K^T (.) M) V with error O(eps)."""
    rng = np.random.default_rng(16)
    T, dk, dv = 20, 8, 5
    q, k, v, _, _ = _rand_problem(rng, 1, T, 1, dk, dv, "none")
    eps = 1e-6
    o, _ = _run(q, k, v, None, np.full((1, T, 1), eps), "none")
    Q, K, V = q[0, :, 0], k[0, :, 0], v[0, :, 0]
    ref = np.tril(Q @ K.T) @ V / np.sqrt(dk)
    err = np.abs(o[0, :, 0] / eps - ref).max()
    assert err < 50 * eps * T, err


# ---------------------------------------------------------- structure ------
@pytest.mark.parametrize("mode", MODES)
def test_state_carry_split(mode):
    """Running T1 then T2 from the carried state equals running T1+T2 at once
    (state additivity over splits, the Chunk-Boundary State step)."""
    rng = np.random.default_rng(17)
    B, T, H, dk, dv = 2, 37, 2, 8, 6
    q, k, v, g, beta = _rand_problem(rng, B, T, H, dk, dv, mode)
    S0 = rng.standard_normal((B, H, dv, dk))
    o, S_T = _run(q, k, v, g, beta, mode, S0)
    t1 = 15
    sl1, sl2 = slice(0, t1), slice(t1, T)
    gs = (lambda s: None) if g is None else (lambda s: g[:, s])
    o1, s1 = _run(q[:, sl1], k[:, sl1], v[:, sl1], gs(sl1), beta[:, sl1], mode, S0)
    o2, s2 = _run(q[:, sl2], k[:, sl2], v[:, sl2], gs(sl2), beta[:, sl2], mode, s1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), o, atol=1e-12)
    np.testing.assert_allclose(s2, S_T, atol=1e-12)


@pytest.mark.parametrize("mode", MODES)
def test_linear_in_values_and_initial_state(mode):
    rng = np.random.default_rng(18)
    B, T, H, dk, dv = 1, 19, 2, 6, 5
    q, k, v1, g, beta = _rand_problem(rng, B, T, H, dk, dv, mode)
    v2 = rng.standard_normal(v1.shape)
    s01, s02 = rng.standard_normal((2, B, H, dv, dk))
    a, b = 0.7, -1.3
    o1, S1 = _run(q, k, v1, g, beta, mode, s01)
    o2, S2 = _run(q, k, v2, g, beta, mode, s02)
    o3, S3 = _run(q, k, a * v1 + b * v2, g, beta, mode, a * s01 + b * s02)
    np.testing.assert_allclose(o3, a * o1 + b * o2, atol=1e-12)
    np.testing.assert_allclose(S3, a * S1 + b * S2, atol=1e-12)


def test_value_rows_are_independent():
    """Permuting the value channels (rows of S) permutes the outputs the same way."""
    rng = np.random.default_rng(19)
    B, T, H, dk, dv = 1, 21, 1, 6, 7
    q, k, v, g, beta = _rand_problem(rng, B, T, H, dk, dv, "channel")
    S0 = rng.standard_normal((B, H, dv, dk))
    perm = rng.permutation(dv)
    o, S = _run(q, k, v, g, beta, "channel", S0)
    op, Sp = _run(q, k, v[..., perm], g, beta, "channel", S0[:, :, perm])
    np.testing.assert_allclose(op, o[..., perm], atol=1e-13)
    np.testing.assert_allclose(Sp, S[:, :, perm], atol=1e-13)


def test_state_norm_bound():
    """For unit keys, beta in [0,1], alpha <= 1 the erase factor is a contraction:
    ||S_t||_2 <= ||S_{t-1}||_2 + beta_t ||v_t||."""
    rng = np.random.default_rng(20)
    dk, dv, T = 8, 8, 40
    q, k, v, g, beta = _rand_problem(rng, 1, T, 1, dk, dv, "channel")
    S = rng.standard_normal((1, 1, dv, dk))
    for t in range(T):
        _, Sn = _run(q[:, t:t + 1], k[:, t:t + 1], v[:, t:t + 1], g[:, t:t + 1], beta[:, t:t + 1], "channel", S)
        assert np.linalg.norm(Sn[0, 0], 2) <= np.linalg.norm(S[0, 0], 2) + beta[0, t, 0] * np.linalg.norm(v[0, t, 0]) + 1e-12
        S = Sn


@pytest.mark.parametrize("mode", MODES)
def test_decode_steps_equal_forward(mode):
    """The recurrent decode step applied T times equals the forward over T tokens."""
    rng = np.random.default_rng(21)
    B, T, H, dk, dv = 2, 5, 3, 6, 4
    q, k, v, g, beta = _rand_problem(rng, B, T, H, dk, dv, mode)
    S0 = rng.standard_normal((B, H, dv, dk))
    o, S_T = _run(q, k, v, g, beta, mode, S0)
    S = S0
    for t in range(T):
        od, S = oracle.decode_step(q[:, t], k[:, t], v[:, t], None if g is None else g[:, t], beta[:, t], S,
                                   mode, f64_inputs=True)
        np.testing.assert_allclose(od, o[:, t], atol=1e-13)
    np.testing.assert_allclose(S, S_T, atol=1e-13)


def test_float32_inputs_read_exactly():
    """bf16/fp32 inputs are read as their exact values (float32 path == float64 path)."""
    rng = np.random.default_rng(22)
    q, k, v, g, beta = _rand_problem(rng, 1, 13, 2, 8, 8, "scalar")
    f = lambda x: x.astype(np.float32)
    o32, s32 = oracle.recurrent(f(q), f(k), f(v), f(g), f(beta), "scalar")
    o64, s64 = oracle.recurrent(*(f(x).astype(np.float64) for x in (q, k, v, g, beta)), "scalar", f64_inputs=True)
    np.testing.assert_array_equal(o32, o64)
    np.testing.assert_array_equal(s32, s64)


def test_threads_do_not_change_results():
    rng = np.random.default_rng(23)
    q, k, v, g, beta = _rand_problem(rng, 2, 30, 3, 8, 40, "channel")
    o1, s1 = _run(q, k, v, g, beta, "channel", threads=1)
    o2, s2 = _run(q, k, v, g, beta, "channel", threads=4)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(s1, s2)


def test_bad_arguments_raise():
    rng = np.random.default_rng(24)
    q, k, v, g, beta = _rand_problem(rng, 1, 4, 1, 4, 4, "scalar")
    with pytest.raises(ValueError):
        _run(q, k, v, g[..., None].repeat(4, -1), beta, "scalar")
    with pytest.raises(ValueError):
        _run(q, k, v, g, beta, "bogus")


# ---- the mixer prologue (q/k L2 normalisation, beta = sigmoid(logit), softplus decay gate)

def test_prologue_l2norm_worked_and_invariants():
    # worked example: (3, 4) / 5; a zero vector stays zero; every (b, t, h) vector of q and of k
    # comes out with unit norm and the same direction, whatever its input scale
    q = np.zeros((1, 2, 2, 2))
    q[0, 0, 0] = (3.0, 4.0)
    q[0, 0, 1] = (-6.0, 8.0)
    q[0, 1, 0] = (0.0, 0.0)
    q[0, 1, 1] = (1e-3, 0.0)
    k = q[:, ::-1].copy()
    qn, kn, _, _ = oracle.prologue(q, k, np.zeros((1, 2, 2)), None, "none", l2norm_qk=True)
    assert np.array_equal(qn[0, 0, 0], [0.6, 0.8])
    assert np.array_equal(qn[0, 0, 1], [-0.6, 0.8])
    assert np.array_equal(qn[0, 1, 0], [0.0, 0.0])
    assert np.array_equal(qn[0, 1, 1], [1.0, 0.0])
    assert np.array_equal(kn, qn[:, ::-1])
    rng = np.random.default_rng(11)
    x = rng.standard_normal((2, 5, 3, 16)) * 10.0 ** rng.integers(-3, 4, (2, 5, 3, 1))
    xn, _, _, _ = oracle.prologue(x, x, np.zeros((2, 5, 3)), None, "none", l2norm_qk=True)
    np.testing.assert_allclose(np.linalg.norm(xn, axis=-1), 1.0, rtol=0, atol=1e-15)
    x32 = x.astype(np.float32).astype(np.float64)  # the oracle reads inputs as float32
    np.testing.assert_allclose(xn * np.linalg.norm(x32, axis=-1, keepdims=True), x32, rtol=1e-14, atol=0)
    # flags off: values pass through (widened from float32)
    xo, _, bo, _ = oracle.prologue(x, x, np.full((2, 5, 3), 0.25), None, "none")
    assert np.array_equal(xo, x32) and np.all(bo == 0.25)


def test_prologue_beta_sigmoid_closed_forms():
    b = np.array([0.0, np.log(3.0), -np.log(3.0), 800.0, -800.0, 2.5, -2.5]).reshape(1, 7, 1)
    _, _, s, _ = oracle.prologue(np.ones((1, 7, 1, 2)), np.ones((1, 7, 1, 2)), b, None, "none", beta_sigmoid=True)
    s = s.ravel()
    b32 = b.ravel().astype(np.float32).astype(np.float64)
    assert s[0] == 0.5
    np.testing.assert_allclose(s[1], 1.0 / (1.0 + np.exp(-b32[1])), rtol=1e-15)  # ~0.75
    assert abs(s[1] - 0.75) < 1e-7 and abs(s[2] - 0.25) < 1e-7  # ln 3 rounded to float32
    assert s[3] == 1.0 and 0.0 <= s[4] < 1e-300 and np.all(np.isfinite(s))
    np.testing.assert_allclose(s[5] + s[6], 1.0, rtol=0, atol=1e-15)  # sigma(x) + sigma(-x) = 1
    np.testing.assert_allclose(s[5], np.exp(2.5) / (1.0 + np.exp(2.5)), rtol=1e-15)


@pytest.mark.parametrize("mode", ["scalar", "channel"])
def test_prologue_softplus_gate_closed_forms(mode):
    # a = 0 gives g = -A ln 2; a = ln(e^2 - 1) gives g = -2 A; a = 40 gives -40 A (to 1e-17
    # relative); a = -40 gives -A e^-40; per-head A broadcasts over tokens (and channels)
    vals = np.array([0.0, np.log(np.e ** 2 - 1.0), 40.0, -40.0], dtype=np.float32).astype(np.float64)
    A = np.array([0.05, 1.0, 3.0])
    H = 3
    shape = (1, 4, H) if mode == "scalar" else (1, 4, H, 2)
    a = np.broadcast_to(vals.reshape((1, 4, 1) + ((1,) if mode == "channel" else ())), shape).copy()
    _, _, _, g = oracle.prologue(np.ones((1, 4, H, 2)), np.ones((1, 4, H, 2)), np.zeros((1, 4, H)), a, mode,
                                 gate_softplus=True, gate_scale=A)
    sp = np.array([np.log(2.0), np.log1p(np.exp(vals[1])), 40.0 + np.log1p(np.exp(-40.0)), np.exp(-40.0)])
    A32 = A.astype(np.float32).astype(np.float64)  # gate_scale is read as float32 too
    for h in range(H):
        gh = g[0, :, h] if mode == "scalar" else g[0, :, h, 1]
        np.testing.assert_allclose(gh, -A32[h] * sp, rtol=1e-15)
    assert abs(sp[1] - 2.0) < 1e-6  # ln(e^2 - 1) rounded to float32
    # the pages' gate alpha = sigmoid(x) is A = 1, a = -x: exp(g) = sigmoid(x)
    x = np.linspace(-30, 30, 61).reshape(1, 61, 1)
    _, _, _, g1 = oracle.prologue(np.ones((1, 61, 1, 2)), np.ones((1, 61, 1, 2)), np.zeros((1, 61, 1)), -x, "scalar",
                                  gate_softplus=True)
    x32 = x.astype(np.float32).astype(np.float64)
    np.testing.assert_allclose(np.exp(g1), 1.0 / (1.0 + np.exp(-x32)), rtol=1e-14)
    # the small Gated DeltaNet workload's decay exp(-0.05 softplus(z))
    z = np.random.default_rng(3).standard_normal((1, 50, 1))
    _, _, _, g2 = oracle.prologue(np.ones((1, 50, 1, 2)), np.ones((1, 50, 1, 2)), np.zeros((1, 50, 1)), z, "scalar",
                                  gate_softplus=True, gate_scale=np.array([0.05]))
    z32 = z.astype(np.float32).astype(np.float64)
    a05 = float(np.float32(0.05))
    np.testing.assert_allclose(np.exp(g2), np.exp(-a05 * np.log(1.0 + np.exp(z32))), rtol=1e-14)
    with pytest.raises(ValueError):
        oracle.prologue(np.ones((1, 1, 1, 2)), np.ones((1, 1, 1, 2)), np.zeros((1, 1, 1)), None, "none",
                        gate_softplus=True)


def test_prologue_then_recurrence_exact_recall_with_raw_keys():
    # orthogonal keys of arbitrary lengths (rows of an 8 x 8 Hadamard matrix times lengths that
    # float32 holds exactly), beta logits large enough that sigmoid rounds to 1, no decay: after
    # the prologue, S_T k_i / |k_i| = v_i for every i (exact recall)
    rng = np.random.default_rng(5)
    dk, T = 8, 6
    Hd = np.array([[1.0]])
    for _ in range(3):
        Hd = np.block([[Hd, Hd], [Hd, -Hd]])
    lengths = np.array([0.1, 0.3, 2.5, 7.0, 10.0, 0.7], dtype=np.float32).astype(np.float64)
    k = (Hd[:T] * lengths[:, None]).reshape(1, T, 1, dk)
    v = rng.standard_normal((1, T, 1, 3))
    q, kk, b, _ = oracle.prologue(k, k, np.full((1, T, 1), 60.0), None, "none", l2norm_qk=True, beta_sigmoid=True)
    assert np.all(b == 1.0)
    _, S = oracle.recurrent(q, kk, v, None, b, "none", f64_inputs=True)
    k32 = k.astype(np.float32).astype(np.float64)
    for i in range(T):
        ki = k32[0, i, 0] / np.linalg.norm(k32[0, i, 0])
        np.testing.assert_allclose(S[0, 0] @ ki, v[0, i, 0], rtol=0, atol=1e-12)


# ---- the backward pass (reverse-mode gradients of the recurrence)

def _loss_and_grads(x, mode, R1, R2, S0):
    o, st = oracle.recurrent(x["q"], x["k"], x["v"], x["g"], x["beta"], mode, S0=S0, f64_inputs=True)
    return float(np.sum(o * R1) + np.sum(st * R2))


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("with_dst", [True, False])
def test_backward_matches_central_differences(mode, with_dst):
    """Every gradient (q, k, v, g, beta, S0) of L = <o, R1> + <S_T, R2> against central finite
    differences of the forward oracle, h = 1e-6, on a tiny problem (error O(h^2) + rounding)."""
    rng = np.random.default_rng(21 + MODES.index(mode) + (10 if with_dst else 0))
    B, T, H, dk, dv = 1, 5, 2, 3, 2
    q, k, v, g, beta = _rand_problem(rng, B, T, H, dk, dv, mode, unit_keys=False, g_scale=0.7)
    S0 = 0.5 * rng.standard_normal((B, H, dv, dk))
    R1 = rng.standard_normal((B, T, H, dv))
    R2 = rng.standard_normal((B, H, dv, dk)) if with_dst else np.zeros((B, H, dv, dk))
    x = {"q": q, "k": k, "v": v, "g": g, "beta": beta}
    grads = oracle.backward(q, k, v, g, beta, mode, R1, S0=S0, dS_T=R2 if with_dst else None, f64_inputs=True)
    h = 1e-6
    targets = [("q", "dq"), ("k", "dk"), ("v", "dv"), ("beta", "dbeta")] + ([("g", "dg")] if mode != "none" else [])
    for name, gname in targets:
        base = x[name]
        fd = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            xp = dict(x); xm = dict(x)
            xp[name] = base.copy(); xm[name] = base.copy()
            xp[name][idx] += h
            xm[name][idx] -= h
            fd[idx] = (_loss_and_grads(xp, mode, R1, R2, S0) - _loss_and_grads(xm, mode, R1, R2, S0)) / (2 * h)
        np.testing.assert_allclose(grads[gname], fd, rtol=1e-6, atol=1e-7, err_msg=name)
    fd = np.zeros_like(S0)
    for idx in np.ndindex(S0.shape):
        sp = S0.copy(); sm = S0.copy()
        sp[idx] += h
        sm[idx] -= h
        fd[idx] = (_loss_and_grads(x, mode, R1, R2, sp) - _loss_and_grads(x, mode, R1, R2, sm)) / (2 * h)
    np.testing.assert_allclose(grads["dS0"], fd, rtol=1e-6, atol=1e-7, err_msg="S0")


def test_backward_no_write_closed_form():
    """beta = 0 and alpha = 1: the state stays S0, o_t = scale S0 q_t, so dq_t = scale S0^T do_t,
    dk = dv = 0 and dS0 = dS_T + scale sum_t do_t q_t^T (closed forms)."""
    rng = np.random.default_rng(33)
    B, T, H, dk, dv = 2, 7, 2, 4, 3
    q, k, v, _, _ = _rand_problem(rng, B, T, H, dk, dv, "none")
    beta = np.zeros((B, T, H))
    S0 = rng.standard_normal((B, H, dv, dk))
    dO = rng.standard_normal((B, T, H, dv))
    dST = rng.standard_normal((B, H, dv, dk))
    gr = oracle.backward(q, k, v, None, beta, "none", dO, S0=S0, dS_T=dST, f64_inputs=True)
    sc = 1.0 / np.sqrt(dk)
    np.testing.assert_allclose(gr["dq"], sc * np.einsum("bhjc,bthj->bthc", S0, dO), rtol=1e-13, atol=1e-13)
    assert np.all(gr["dk"] == 0) and np.all(gr["dv"] == 0)
    np.testing.assert_allclose(gr["dS0"], dST + sc * np.einsum("bthj,bthc->bhjc", dO, q), rtol=1e-13, atol=1e-13)
    assert gr["dg"] is None


# ---- Gated DeltaNet-2 (channel-wise erase and write gates)

def _gdn2_problem(rng, B, T, H, dk, dv, mode):
    q, k, v, g, _ = _rand_problem(rng, B, T, H, dk, dv, mode, unit_keys=True, g_scale=0.5)
    erase = rng.uniform(0.0, 1.0, (B, T, H, dk))
    write = rng.uniform(0.0, 1.0, (B, T, H, dv))
    return q, k, v, g, erase, write


@pytest.mark.parametrize("mode", MODES)
def test_gdn2_matches_transition_products(mode):
    """S_T from explicit products and from the Kronecker-form linear system of the transitions
    A_t = Diag(alpha_t)(I - (e_t k_t) k_t^T), B_t = (w_t v_t) k_t^T; o_t = scale S_t q_t."""
    from brute import transitions_gdn2
    rng = np.random.default_rng(41 + MODES.index(mode))
    B, T, H, dk, dv = 1, 6, 2, 4, 3
    q, k, v, g, e, w = _gdn2_problem(rng, B, T, H, dk, dv, mode)
    S0 = rng.standard_normal((B, H, dv, dk))
    o, st = oracle.recurrent_gdn2(q, k, v, g, e, w, mode, S0=S0, f64_inputs=True)
    sc = 1.0 / np.sqrt(dk)
    for h in range(H):
        gh = None if g is None else g[0, :, h]
        As, Bs = transitions_gdn2(k[0, :, h], v[0, :, h], gh, mode, e[0, :, h], w[0, :, h])
        by_prod = states_by_product(S0[0, h], As, Bs)
        by_kron = states_by_kron(S0[0, h], As, Bs)
        for t in range(T):
            np.testing.assert_allclose(by_prod[t], by_kron[t], rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(o[0, t, h], sc * by_prod[t] @ q[0, t, h], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(st[0, h], by_prod[-1], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mode", MODES)
def test_gdn2_equal_gates_is_the_delta_rule(mode):
    """e_t = w_t = beta_t 1 gives the delta rule with the same decay (Kimi Delta Attention for the
    channel gate, Gated DeltaNet for the scalar one, DeltaNet without decay)."""
    rng = np.random.default_rng(51 + MODES.index(mode))
    B, T, H, dk, dv = 2, 9, 2, 5, 3
    q, k, v, g, beta = _rand_problem(rng, B, T, H, dk, dv, mode)
    S0 = rng.standard_normal((B, H, dv, dk))
    e = np.repeat(beta[..., None], dk, axis=-1)
    w = np.repeat(beta[..., None], dv, axis=-1)
    o2, s2 = oracle.recurrent_gdn2(q, k, v, g, e, w, mode, S0=S0, f64_inputs=True)
    o1, s1 = _run(q, k, v, g, beta, mode, S0=S0)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(s2, s1, rtol=1e-12, atol=1e-13)


def test_gdn2_erase_free_is_gated_linear_attention():
    """e = 0, alpha = 1: nothing is erased and o_t = scale sum_{i<=t} (k_i . q_t) (w_i v_i) (closed form)."""
    rng = np.random.default_rng(61)
    B, T, H, dk, dv = 1, 7, 2, 4, 3
    q, k, v, g, e, w = _gdn2_problem(rng, B, T, H, dk, dv, "none")
    e = np.zeros_like(e)
    o, st = oracle.recurrent_gdn2(q, k, v, None, e, w, "none", f64_inputs=True)
    sc = 1.0 / np.sqrt(dk)
    for t in range(T):
        ref = sc * sum((k[0, i] * q[0, t]).sum(-1)[:, None] * (w[0, i] * v[0, i]) for i in range(t + 1))
        np.testing.assert_allclose(o[0, t], ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(st[0], np.einsum("thj,thc->hjc", w[0] * v[0], k[0]), rtol=1e-12, atol=1e-13)


def test_gdn2_erase_only_projects_out_written_keys():
    """w = 0, e = 1, alpha = 1, orthonormal keys: each token projects its key direction out of the
    memory, so S_T k_i = 0 for every key written and S_T x = S0 x for x orthogonal to all of them."""
    rng = np.random.default_rng(71)
    dk, dv, T = 6, 3, 4
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm[:T].reshape(1, T, 1, dk)
    q = rng.standard_normal((1, T, 1, dk))
    v = rng.standard_normal((1, T, 1, dv))
    S0 = rng.standard_normal((1, 1, dv, dk))
    _, st = oracle.recurrent_gdn2(q, k, v, None, np.ones((1, T, 1, dk)), np.zeros((1, T, 1, dv)), "none", S0=S0,
                                  f64_inputs=True)
    for i in range(T):
        np.testing.assert_allclose(st[0, 0] @ Qm[i], 0.0, atol=1e-13)
    for i in range(T, dk):
        np.testing.assert_allclose(st[0, 0] @ Qm[i], S0[0, 0] @ Qm[i], atol=1e-13)
