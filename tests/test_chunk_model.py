"""The chunked (UT/WY) algebra that the CUDA kernels implement, in fp64 NumPy,
equals the token-by-token oracle for every chunk size: C = 1 is the recurrent
form and C = T the fully parallel masked form ("linear attention and its gated
descendants", Chunkwise Parallel Form, limiting cases). T is chosen so most
chunk sizes leave a ragged tail."""
import numpy as np
import pytest

import oracle
from chunk_model import chunk_forward

MODES = ("none", "scalar", "channel")


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("C", [1, 4, 16, 64, 75])
def test_chunk_model_equals_oracle(mode, C):
    rng = np.random.default_rng(100 + 10 * MODES.index(mode) + C)
    B, T, H, dk, dv = 2, 75, 2, 16, 12
    q = rng.standard_normal((B, T, H, dk)); q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k = rng.standard_normal((B, T, H, dk)); k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    beta = rng.uniform(0, 1, (B, T, H))
    g = None
    if mode == "scalar":
        g = -0.2 * rng.uniform(0, 1, (B, T, H))
    elif mode == "channel":
        g = -0.2 * rng.uniform(0, 1, (B, T, H, dk))
    S0 = rng.standard_normal((B, H, dv, dk))
    o_ref, s_ref = oracle.recurrent(q, k, v, g, beta, mode, S0=S0, f64_inputs=True)
    o, s = chunk_forward(q, k, v, g, beta, mode, S0, C)
    np.testing.assert_allclose(o, o_ref, atol=1e-10)
    np.testing.assert_allclose(s, s_ref, atol=1e-10)


def test_chunk_model_tail_padding_is_neutral():
    """A padded token with k = 0, beta = 0, g = 0 leaves the state unchanged, so a
    ragged tail may be handled as zero padding."""
    rng = np.random.default_rng(7)
    B, T, H, d = 1, 10, 1, 8
    q = rng.standard_normal((B, T, H, d)); k = rng.standard_normal((B, T, H, d))
    v = rng.standard_normal((B, T, H, d)); beta = rng.uniform(0, 1, (B, T, H))
    g = -0.1 * rng.uniform(0, 1, (B, T, H))
    S0 = rng.standard_normal((B, H, d, d))
    o, s = oracle.recurrent(q, k, v, g, beta, "scalar", S0=S0, f64_inputs=True)
    pad = lambda x: np.concatenate([x, np.zeros((B, 6) + x.shape[2:])], axis=1)
    op, sp = oracle.recurrent(pad(q), pad(k), pad(v), pad(g), pad(beta), "scalar", S0=S0, f64_inputs=True)
    np.testing.assert_allclose(op[:, :T], o, atol=1e-13)
    np.testing.assert_allclose(sp, s, atol=1e-13)
