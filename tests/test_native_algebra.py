"""The chunked ("native mixed") output form, checked in float64 (CPU).

gdn_native_forward evaluates each chunk's outputs from the state entering
it by products of C x C and C x d matrices instead of the token loop:
    o_i = scale (e^{G_i} S q_i + sum_{j <= i} e^{G_i - G_j} (q_i . k_j) u_j),
with u_j the rows of U from the chunk boundary's UT system, and prepares a
sequence's trailing partial chunk zero-padded.  oracle.chunked_outputs and
oracle.native_forward write that form out in float64; here they must equal
the oracle's token loop (oracle.forward, the C recurrence) to ~1e-12, and
padding tokens (k = v = 0, beta = g = 0) must be identity steps.  A dropped
diagonal term (j < i instead of j <= i), the decay taken from G_j instead of
G_i, or U built without the S-dependent part each miss that bound by many
orders of magnitude (checked below on the same inputs).
"""
import numpy as np
import pytest

import oracle


def _batch(lens, H, d, seed, strong=False):
    rng = np.random.default_rng(seed)
    T = sum(lens)
    q = rng.normal(size=(T, H, d))
    k = rng.normal(size=(T, H, d))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.normal(size=(T, H, d))
    beta = 1.0 / (1.0 + np.exp(-rng.normal(size=(T, H))))
    g = -np.log1p(np.exp((2.5 if strong else 1.0) * rng.normal(size=(T, H))))
    if strong:
        g = np.maximum(g, -8.0)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    h0 = rng.normal(size=(len(lens), H, d, d)) * 0.3
    return q, k, v, beta, g, cu, h0


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.sqrt(np.mean(b * b)), 1e-300))


@pytest.mark.parametrize("strong", [False, True])
@pytest.mark.parametrize("C", [1, 4, 16, 64])
def test_native_forward_equals_the_token_loop(C, strong):
    lens = [1, 63, 64, 65, 130, 0, 7]
    q, k, v, beta, g, cu, h0 = _batch(lens, 2, 8, 100 + C, strong)
    o_ref, s_ref = oracle.forward(q, k, v, beta, g, cu, h0=h0, scale=0.7)
    o, s_fin, s_bnd = oracle.native_forward(q, k, v, beta, g, cu, C, h0=h0, scale=0.7)
    assert _rel(o, o_ref) < 1e-11
    assert _rel(s_fin, s_ref) < 1e-11
    _, _, s_bnd_cpr, _ = oracle.cpr_forward(q, k, v, beta, g, cu, C, h0=h0)
    assert _rel(s_bnd, s_bnd_cpr) < 1e-12


def test_zero_padding_is_identity():
    q, k, v, beta, g, cu, h0 = _batch([37], 1, 8, 7)
    S0 = h0[0, 0]
    o, S = oracle.chunked_outputs(S0, q[:, 0], k[:, 0], v[:, 0], beta[:, 0], g[:, 0])
    pad = lambda x: np.concatenate([x, np.zeros((64 - 37,) + x.shape[1:])])  # noqa: E731
    o_p, S_p = oracle.chunked_outputs(S0, pad(q[:, 0]), pad(k[:, 0]), pad(v[:, 0]),
                                      pad(beta[:, 0]), pad(g[:, 0]))
    assert _rel(o_p[:37], o) < 1e-13 and _rel(S_p, S) < 1e-13
    assert np.all(o_p[37:] == 0.0)


def _planted(S0, Q, K, V, beta, g, which):
    cb = oracle.chunk_boundary(S0, K, V, beta, g)
    G, U = cb["G"], cb["U"]
    n = len(G)
    if which == "no_state_in_U":
        U = cb["Ut"]
    Pm = np.zeros((n, n))
    for i in range(n):
        for j in range(i + (0 if which == "strict_lower" else 1)):
            Gi = G[j] if which == "decay_from_j" else G[i]
            Pm[i, j] = np.exp(Gi - G[j]) * (Q[i] @ K[j])
    return np.exp(G)[:, None] * (Q @ S0.T) + Pm @ U


@pytest.mark.parametrize("which", ["strict_lower", "decay_from_j", "no_state_in_U"])
def test_plausible_mistakes_miss_the_bound(which):
    q, k, v, beta, g, cu, h0 = _batch([64], 1, 8, 9)
    S0 = h0[0, 0]
    o_ref, _ = oracle.forward(q, k, v, beta, g, cu, h0=h0)
    o_bad = _planted(S0, q[:, 0], k[:, 0], v[:, 0], beta[:, 0], g[:, 0], which)
    assert _rel(o_bad, o_ref[:, 0]) > 1e-3
