"""Pins of the CPU oracle against facts that do not come from the oracle itself.

The recurrence is the one of "NovaSky's IsoExec Fixes the Hidden Math Bug
Corrupting AI Training Runs", section "Solving the linear-attention headache"
(Gated DeltaNet, evaluated by CPR with the recurrence as the primary
algorithm):  S_t = alpha_t S_{t-1}(I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
o_t = scale * S_t q_t.

Pins (each a property the mathematics fixes, independent of the token loop):
  decay      beta = 0: S_T = (prod alpha) S_0 and o_t = gamma_t S_0 q_t
  store      alpha = 1, beta = 1, orthonormal keys: S_T k_i = v_i and
             o_t = v_t when q_t = k_t (the delta rule overwrites)
  placement  orthonormal keys, S_0 orthogonal to them: S_T is the explicit
             decayed sum of beta_i v_i k_i^T (locates alpha and beta)
  resets     alpha = 0 at reset positions: after the last reset the state is
             the explicit sum of beta_i v_i k_i^T since that reset
  product    the unrolled product of explicit transition matrices (fp64)
  exact      exact-rational fixtures in tests/golden (Fraction arithmetic)
Each pin is applied to the C oracle, to the numpy token loop, and to versions
of the token loop with a planted mistake, every one of which must fail at
least one pin.
"""
import glob
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ----------------------------------------------------------------------------
# Implementations under test: impl(S0, q, k, v, beta, alpha, scale) -> (o, S_T)
# ----------------------------------------------------------------------------

def c_oracle_alpha(S0, q, k, v, beta, alpha, scale=1.0):
    T = len(beta)
    o, s = oracle.forward_alpha(q[:, None, :], k[:, None, :], v[:, None, :], beta[:, None],
                                alpha[:, None], np.array([0, T], np.int32),
                                h0=np.asarray(S0)[None, None], scale=scale, threads=1)
    return o[:, 0, :], s[0, 0]


def c_oracle_g(S0, q, k, v, beta, alpha, scale=1.0):
    """The g entry point: alpha enters as g = log(alpha) (alpha = 0 -> g = -inf)."""
    with np.errstate(divide="ignore"):
        g = np.log(np.asarray(alpha, dtype=np.float64))
    T = len(beta)
    o, s = oracle.forward(q[:, None, :], k[:, None, :], v[:, None, :], beta[:, None],
                          g[:, None], np.array([0, T], np.int32),
                          h0=np.asarray(S0)[None, None], scale=scale, threads=1)
    return o[:, 0, :], s[0, 0]


def make_loop(mutation=None):
    """numpy token loop; `mutation` plants one mistake (for the pins' own test)."""
    def impl(S0, q, k, v, beta, alpha, scale=1.0):
        S = np.array(S0, dtype=np.float64, copy=True)
        T = len(beta)
        o = np.zeros((T, S.shape[0]))
        for t in range(T):
            a, b = alpha[t], beta[t]
            if mutation == "alpha_lag":
                a = alpha[t - 1] if t > 0 else 1.0
            p = S.T @ k[t] if mutation == "transpose" else S @ k[t]
            S_prev = S
            if mutation == "drop_alpha_state":
                S = (S - b * np.outer(p, k[t])) + b * np.outer(v[t], k[t])
            elif mutation == "alpha_on_write":
                S = a * (S - b * np.outer(p, k[t]) + b * np.outer(v[t], k[t]))
            elif mutation == "sign":
                S = a * (S + b * np.outer(p, k[t])) + b * np.outer(v[t], k[t])
            elif mutation == "drop_beta_write":
                S = a * (S - b * np.outer(p, k[t])) + np.outer(v[t], k[t])
            else:
                S = a * (S - b * np.outer(p, k[t])) + b * np.outer(v[t], k[t])
            if mutation == "o_before_update":
                o[t] = scale * (S_prev @ q[t])
            elif mutation == "o_uses_key":
                o[t] = scale * (S @ k[t])
            else:
                o[t] = scale * (S @ q[t])
        return o, S
    return impl


MUTATIONS = ["drop_alpha_state", "alpha_on_write", "sign", "transpose", "o_before_update",
             "o_uses_key", "drop_beta_write", "alpha_lag"]


# ----------------------------------------------------------------------------
# Pins: each returns the max relative error of `impl` on its case
# ----------------------------------------------------------------------------

def _rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(1e-300, float(np.max(np.abs(b)))))


def _orthonormal(rng, n, d):
    Q, _ = np.linalg.qr(rng.standard_normal((d, d)))
    return Q[:n]  # n orthonormal rows


def pin_decay(impl, seed=0, d=6, T=9):
    rng = np.random.default_rng(seed)
    S0 = rng.standard_normal((d, d))
    q, k = rng.standard_normal((T, d)), rng.standard_normal((T, d))
    v = rng.standard_normal((T, d))
    alpha = rng.uniform(0.3, 0.99, T)
    beta = np.zeros(T)
    o, S = impl(S0, q, k, v, beta, alpha, 1.0)
    gam = np.cumprod(alpha)
    o_ref = gam[:, None] * (q @ S0.T)
    return max(_rel(S, gam[-1] * S0), _rel(o, o_ref))


def pin_store(impl, seed=1, d=5):
    rng = np.random.default_rng(seed)
    K = _orthonormal(rng, d, d)
    S0 = rng.standard_normal((d, d))
    v = rng.standard_normal((d, d))
    o, S = impl(S0, K.copy(), K, v, np.ones(d), np.ones(d), 1.0)
    return max(_rel(o, v), _rel(K @ S.T, v))


def pin_placement(impl, seed=2, d=7, n=4):
    rng = np.random.default_rng(seed)
    K = _orthonormal(rng, n, d)
    P = np.eye(d) - K.T @ K  # projector onto the keys' orthogonal complement
    S0 = rng.standard_normal((d, d)) @ P
    q = rng.standard_normal((n, d))
    v = rng.standard_normal((n, d))
    beta = rng.uniform(0.1, 0.9, n)
    alpha = rng.uniform(0.2, 0.95, n)
    o, S = impl(S0, q, K, v, beta, alpha, 1.0)

    def state_at(t):  # explicit decayed sum after tokens 0..t
        acc = np.prod(alpha[:t + 1]) * S0
        for i in range(t + 1):
            acc = acc + np.prod(alpha[i + 1:t + 1]) * beta[i] * np.outer(v[i], K[i])
        return acc
    o_ref = np.stack([state_at(t) @ q[t] for t in range(n)])
    return max(_rel(S, state_at(n - 1)), _rel(o, o_ref))


def pin_resets(impl, seed=3, d=6, seg=(3, 5, 4)):
    rng = np.random.default_rng(seed)
    T = sum(seg)
    K = np.concatenate([_orthonormal(rng, s, d) for s in seg])
    S0 = rng.standard_normal((d, d))
    q = rng.standard_normal((T, d))
    v = rng.standard_normal((T, d))
    beta = rng.uniform(0.1, 1.0, T)
    alpha = np.ones(T)
    starts = np.cumsum((0,) + seg[:-1])
    alpha[starts[1:]] = 0.0  # a reset opens every segment after the first
    o, S = impl(S0, q, K, v, beta, alpha, 1.0)
    last = starts[-1]
    S_ref = sum(beta[i] * np.outer(v[i], K[i]) for i in range(last, T))
    o_ref_last = S_ref @ q[-1]
    return max(_rel(S, S_ref), _rel(o[-1], o_ref_last))


def pin_product(impl, seed=4, d=3, T=10):
    rng = np.random.default_rng(seed)
    S0 = rng.standard_normal((d, d + 1))
    q, k = rng.standard_normal((T, d + 1)), rng.standard_normal((T, d + 1)) * 0.6
    v = rng.standard_normal((T, d))
    beta = rng.uniform(0.05, 1.0, T)
    alpha = rng.uniform(0.5, 1.0, T)
    o, S = impl(S0, q, k, v, beta, alpha, 0.75)
    S_ref = oracle.explicit_product_state(S0, k, v, beta, alpha)
    o_ref = np.stack([0.75 * (oracle.explicit_product_state(S0, k[:t + 1], v[:t + 1],
                                                            beta[:t + 1], alpha[:t + 1]) @ q[t])
                      for t in range(T)])
    return max(_rel(S, S_ref), _rel(o, o_ref))


def _load_golden(path):
    with open(path) as f:
        c = json.load(f)
    F = lambda M: np.array([[float(Fraction(x)) for x in row] for row in M])  # noqa: E731
    exact = lambda M: [[Fraction(x) for x in row] for row in M]  # noqa: E731
    return c, F, exact


def pin_exact(impl):
    worst = 0.0
    for path in sorted(glob.glob(os.path.join(GOLDEN, "exact_*.json"))):
        c, F, exact = _load_golden(path)
        o, S = impl(F(c["S0"]), F(c["q"]), F(c["k"]), F(c["v"]),
                    np.array([float(Fraction(x)) for x in c["beta"]]),
                    np.array([float(Fraction(x)) for x in c["alpha"]]), 1.0)
        worst = max(worst, _rel(S, F(c["S_T"])), _rel(o, F(c["o"])))
    return worst


PINS = {"decay": pin_decay, "store": pin_store, "placement": pin_placement,
        "resets": pin_resets, "product": pin_product, "exact": pin_exact}
TOL = 1e-12


# ----------------------------------------------------------------------------
# Tests
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("pin", sorted(PINS))
@pytest.mark.parametrize("impl_name", ["c_alpha", "c_g", "numpy_loop"])
def test_oracle_meets_pin(pin, impl_name):
    impl = {"c_alpha": c_oracle_alpha, "c_g": c_oracle_g, "numpy_loop": make_loop()}[impl_name]
    err = PINS[pin](impl)
    assert err <= TOL, f"{impl_name} fails pin {pin}: rel err {err:.3e}"


@pytest.mark.parametrize("mutation", MUTATIONS)
def test_planted_mistake_is_caught(mutation):
    impl = make_loop(mutation)
    errs = {}
    for name, pin in PINS.items():
        try:
            errs[name] = pin(impl)
        except ValueError:  # a shape error (non-square state) also exposes the mistake
            errs[name] = float("inf")
    assert max(errs.values()) > 1e-6, f"no pin detects mutation {mutation}: {errs}"


def test_golden_fixtures_present():
    files = glob.glob(os.path.join(GOLDEN, "exact_*.json"))
    assert len(files) >= 4


def test_exact_fixture_matches_exact_loop():
    """The fixtures' product form equals an exact-rational token loop (Fraction)."""
    for path in sorted(glob.glob(os.path.join(GOLDEN, "exact_*.json"))):
        c, F, exact = _load_golden(path)
        S = exact(c["S0"])
        q, k, v = exact(c["q"]), exact(c["k"]), exact(c["v"])
        beta = [Fraction(x) for x in c["beta"]]
        alpha = [Fraction(x) for x in c["alpha"]]
        dv, dk = len(S), len(S[0])
        for t in range(c["T"]):
            p = [sum((S[r][j] * k[t][j] for j in range(dk)), Fraction(0)) for r in range(dv)]
            S = [[alpha[t] * (S[r][j] - beta[t] * p[r] * k[t][j]) + beta[t] * v[t][r] * k[t][j]
                  for j in range(dk)] for r in range(dv)]
            o_t = [sum((S[r][j] * q[t][j] for j in range(dk)), Fraction(0)) for r in range(dv)]
            assert o_t == [Fraction(x) for x in c["o"][t]]
        assert S == exact(c["S_T"])


def test_oracle_packing_and_empty_sequences():
    """Several sequences and heads, including empty ones: each unit equals its own run."""
    rng = np.random.default_rng(5)
    lens = [0, 3, 0, 7, 1]
    H, dk, dv = 2, 4, 3
    T = sum(lens)
    cu = np.cumsum([0] + lens).astype(np.int32)
    q, k = rng.standard_normal((T, H, dk)), rng.standard_normal((T, H, dk)) * 0.5
    v = rng.standard_normal((T, H, dv))
    beta, g = rng.uniform(0, 1, (T, H)), -rng.uniform(0, 2, (T, H))
    h0 = rng.standard_normal((len(lens), H, dv, dk))
    o, s = oracle.forward(q, k, v, beta, g, cu, h0=h0, threads=2)
    for n, L in enumerate(lens):
        for h in range(H):
            sl = slice(cu[n], cu[n + 1])
            oo, ss = make_loop()(h0[n, h], q[sl, h], k[sl, h], v[sl, h], beta[sl, h],
                                 np.exp(g[sl, h]), 1.0)
            assert _rel(ss, s[n, h]) <= TOL
            if L:
                assert _rel(oo, o[sl, h]) <= TOL
            else:
                assert np.array_equal(s[n, h], h0[n, h])


# ----------------------------------------------------------------------------
# The CPR schedule in fp64 (chunk boundary in UT/WY form) against the token loop
# ----------------------------------------------------------------------------

def _rand_batch(rng, lens, H, d):
    T = sum(lens)
    q = rng.standard_normal((T, H, d))
    k = rng.standard_normal((T, H, d))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, d))
    beta = 1 / (1 + np.exp(-rng.standard_normal((T, H))))
    g = -np.log1p(np.exp(rng.standard_normal((T, H))))
    return q, k, v, beta, g, np.cumsum([0] + lens).astype(np.int32)


@pytest.mark.parametrize("C", [1, 2, 3, 8, 64])
def test_cpr_algebra_equals_token_loop(C):
    rng = np.random.default_rng(100 + C)
    lens = [0, 1, C - 1 if C > 1 else 2, C, C + 1, 3 * C + 2, 130]
    H, d = 2, 8
    q, k, v, beta, g, cu = _rand_batch(rng, lens, H, d)
    h0 = rng.standard_normal((len(lens), H, d, d)) * 0.3
    o_ref, s_ref = oracle.forward(q, k, v, beta, g, cu, h0=h0)
    o, s_run, s_bnd, bstates = oracle.cpr_forward(q, k, v, beta, g, cu, C, h0=h0)
    scale = float(np.sqrt(np.mean(o_ref ** 2)))
    assert np.max(np.abs(o - o_ref)) <= 1e-12 * max(scale, 1.0)
    assert np.max(np.abs(s_run - s_ref)) <= 1e-12 * max(1.0, float(np.max(np.abs(s_ref))))
    for n, L in enumerate(lens):
        nf = L // C
        # the boundary state after nf chunks is the token-loop state after nf*C tokens
        sub = slice(cu[n], cu[n] + nf * C)
        _, s_pref = oracle.forward(q[sub], k[sub], v[sub], beta[sub], g[sub],
                                   np.array([0, nf * C], np.int32), h0=h0[n:n + 1])
        assert np.max(np.abs(s_bnd[n] - s_pref[0])) <= 1e-12 * max(1.0, np.max(np.abs(s_pref)))
        assert bstates[n].shape[0] == nf + 1


def test_chunk_boundary_size_one_is_one_step():
    """With C = 1 the UT system is 1x1 (T = I) and the boundary is one recurrence step."""
    rng = np.random.default_rng(7)
    d = 5
    S0 = rng.standard_normal((d, d))
    k, v = rng.standard_normal((1, d)), rng.standard_normal((1, d))
    beta, g = np.array([0.7]), np.array([-0.4])
    out = oracle.chunk_boundary(S0, k, v, beta, g)
    assert np.array_equal(out["T"], np.eye(1))
    a = math.exp(-0.4)
    S1 = a * (S0 - 0.7 * np.outer(S0 @ k[0], k[0])) + 0.7 * np.outer(v[0], k[0])
    assert np.max(np.abs(out["S"] - S1)) <= 1e-14 * np.max(np.abs(S1))


def test_chunk_boundary_after_resets_is_explicit_sum():
    """Chunked schedule with resets inside chunks: the state after the last reset
    is the explicit sum of beta_i v_i k_i^T (orthonormal keys, alpha = 1 elsewhere)."""
    rng = np.random.default_rng(8)
    d, C = 8, 4
    seg = [5, 6, 5]
    T = sum(seg)
    K = np.concatenate([_orthonormal(rng, s, d) for s in seg])
    V = rng.standard_normal((T, d))
    beta = rng.uniform(0.2, 1.0, T)
    g = np.zeros(T)
    starts = np.cumsum([0] + seg[:-1])
    g[starts[1:]] = -1e4  # exp underflows to exactly 0: a hard reset
    q = rng.standard_normal((T, d))
    o, s_run, s_bnd, _ = oracle.cpr_forward(q[:, None], K[:, None], V[:, None], beta[:, None],
                                            g[:, None], np.array([0, T], np.int32), C)
    S_ref = sum(beta[i] * np.outer(V[i], K[i]) for i in range(starts[-1], T))
    assert np.max(np.abs(s_run[0, 0] - S_ref)) <= 1e-12
