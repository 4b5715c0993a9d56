"""Pins of the oracle's reverse mode (CPU): the gradient of a loss through
the token loop, checked against what fixes it independently of the
derivation coded in oracle/gdn_oracle.c:

* central finite differences of the forward oracle (the definition of the
  gradient), for every input element of a small ragged batch;
* reverse mode derived by torch.autograd through an fp64 PyTorch token loop;
* closed forms at beta = 0, where S_t = (prod_{s<=t} exp(g_s)) h0;
* planted mistakes in a copy of the reverse step are caught by the same
  finite-difference test.
"""
import numpy as np
import pytest
import torch

import oracle


def _batch(lens, H, dk, dv, seed):
    rng = np.random.default_rng(seed)
    T = sum(lens)
    q = rng.normal(size=(T, H, dk))
    k = rng.normal(size=(T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.normal(size=(T, H, dv))
    beta = 1.0 / (1.0 + np.exp(-rng.normal(size=(T, H))))
    g = -np.log1p(np.exp(rng.normal(size=(T, H))))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    h0 = rng.normal(size=(len(lens), H, dv, dk))
    return dict(q=q, k=k, v=v, beta=beta, g=g, cu=cu, h0=h0)


def _loss(b, do, dsf, scale):
    o, s = oracle.forward(b["q"], b["k"], b["v"], b["beta"], b["g"], b["cu"], h0=b["h0"],
                          scale=scale, threads=1)
    return float(np.sum(o * do) + np.sum(s * dsf))


def _grads(b, do, dsf, scale):
    return oracle.backward(b["q"], b["k"], b["v"], b["beta"], b["g"], b["cu"], do, h0=b["h0"],
                           ds_final=dsf, scale=scale, threads=1)


NAMES = {"q": "dq", "k": "dk", "v": "dv", "beta": "dbeta", "g": "dg", "h0": "dh0"}


def _fd_check(b, do, dsf, scale, grads, eps=1e-6, tol=1e-6):
    worst = 0.0
    for name, gname in NAMES.items():
        x = b[name]
        for idx in np.ndindex(x.shape):
            keep = x[idx]
            x[idx] = keep + eps
            lp = _loss(b, do, dsf, scale)
            x[idx] = keep - eps
            lm = _loss(b, do, dsf, scale)
            x[idx] = keep
            fd = (lp - lm) / (2 * eps)
            err = abs(fd - grads[gname][idx]) / max(1.0, abs(fd))
            worst = max(worst, err)
            if err > tol:
                return False, (name, idx, fd, grads[gname][idx])
    return True, worst


def test_backward_matches_finite_differences():
    b = _batch([5, 3, 0, 4], H=2, dk=3, dv=2, seed=11)
    rng = np.random.default_rng(12)
    do = rng.normal(size=b["v"].shape)
    dsf = rng.normal(size=b["h0"].shape)
    ok, info = _fd_check(b, do, dsf, 0.7, _grads(b, do, dsf, 0.7))
    assert ok, info


def test_backward_across_checkpoints_matches_autograd():
    """Lengths around the 64-token checkpoint spacing, d = 8: fp64 autograd."""
    lens, H, dk, dv, scale = [1, 63, 64, 65, 130], 2, 8, 6, 0.5
    b = _batch(lens, H, dk, dv, seed=13)
    rng = np.random.default_rng(14)
    do = rng.normal(size=b["v"].shape)
    dsf = rng.normal(size=b["h0"].shape)
    got = _grads(b, do, dsf, scale)
    t = {n: torch.tensor(b[n], dtype=torch.float64, requires_grad=True)
         for n in ("q", "k", "v", "beta", "g", "h0")}
    loss = torch.zeros((), dtype=torch.float64)
    cu = b["cu"].tolist()
    for n in range(len(lens)):
        for h in range(H):
            S = t["h0"][n, h]
            for i in range(cu[n], cu[n + 1]):
                kt, vt, qt = t["k"][i, h], t["v"][i, h], t["q"][i, h]
                a, bt = torch.exp(t["g"][i, h]), t["beta"][i, h]
                p = S @ kt
                S = a * (S - bt * torch.outer(p, kt)) + bt * torch.outer(vt, kt)
                loss = loss + scale * torch.dot(torch.tensor(do[i, h]), S @ qt)
            loss = loss + torch.sum(torch.tensor(dsf[n, h]) * S)
    loss.backward()
    for name, gname in NAMES.items():
        ref = t[name].grad.numpy()
        assert np.max(np.abs(got[gname] - ref)) <= 1e-10 * max(1.0, np.max(np.abs(ref))), name


def test_backward_closed_forms_at_beta_zero():
    """beta = 0: S_t = A_t h0 with A_t = prod_{s<=t} exp(g_s); o_t = scale A_t h0 q_t.
    Then dv = dk = 0, dq_t = scale A_t h0^T do_t, dh0 = sum_t scale A_t do_t q_t^T + A_L dS_end,
    dg_s = sum_{t>=s} scale A_t <do_t, h0 q_t> + A_L <dS_end, h0>."""
    b = _batch([9], H=1, dk=4, dv=3, seed=15)
    b["beta"][:] = 0.0
    rng = np.random.default_rng(16)
    do = rng.normal(size=b["v"].shape)
    dsf = rng.normal(size=b["h0"].shape)
    scale = 1.3
    got = _grads(b, do, dsf, scale)
    h0 = b["h0"][0, 0]
    A = np.exp(np.cumsum(b["g"][:, 0]))
    assert np.max(np.abs(got["dv"])) == 0.0 and np.max(np.abs(got["dk"])) == 0.0
    for t in range(9):
        np.testing.assert_allclose(got["dq"][t, 0], scale * A[t] * h0.T @ do[t, 0], rtol=1e-12)
    dh0 = sum(scale * A[t] * np.outer(do[t, 0], b["q"][t, 0]) for t in range(9)) + A[-1] * dsf[0, 0]
    np.testing.assert_allclose(got["dh0"][0, 0], dh0, rtol=1e-12)
    term = np.array([scale * A[t] * do[t, 0] @ (h0 @ b["q"][t, 0]) for t in range(9)])
    dg = np.array([term[s:].sum() + A[-1] * np.sum(dsf[0, 0] * h0) for s in range(9)])
    np.testing.assert_allclose(got["dg"][:, 0], dg, rtol=1e-11, atol=1e-13)


def _mutated_backward(b, do, dsf, scale, mutation):
    """A numpy copy of the reverse step with one planted mistake."""
    q, k, v, beta, g, cu = b["q"], b["k"], b["v"], b["beta"], b["g"], b["cu"]
    T, H, dk = q.shape
    out = {"dq": np.zeros_like(q), "dk": np.zeros_like(k), "dv": np.zeros_like(v),
           "dbeta": np.zeros_like(beta), "dg": np.zeros_like(g), "dh0": np.zeros_like(b["h0"])}
    for n in range(len(cu) - 1):
        for h in range(H):
            S = [b["h0"][n, h].copy()]
            for i in range(cu[n], cu[n + 1]):
                a, bt = np.exp(g[i, h]), beta[i, h]
                p = S[-1] @ k[i, h]
                S.append(a * (S[-1] - bt * np.outer(p, k[i, h])) + bt * np.outer(v[i, h], k[i, h]))
            dS = dsf[n, h].copy()
            for i in range(cu[n + 1] - 1, cu[n] - 1, -1):
                j = i - cu[n]
                Sp, Sc = S[j], S[j + 1]
                a, bt = np.exp(g[i, h]), beta[i, h]
                dS = dS + scale * np.outer(do[i, h], q[i, h])
                out["dq"][i, h] = scale * Sc.T @ do[i, h]
                w, p = dS @ k[i, h], Sp @ k[i, h]
                da = np.sum(dS * Sp) - bt * w @ p
                if mutation == "sign_da":
                    da = np.sum(dS * Sp) + bt * w @ p
                out["dbeta"][i, h] = w @ (v[i, h] - a * p)
                out["dv"][i, h] = bt * w
                dp = -a * bt * w
                out["dk"][i, h] = dS.T @ (bt * (v[i, h] - a * p)) + Sp.T @ dp
                if mutation == "drop_p_path":
                    out["dk"][i, h] = dS.T @ (bt * (v[i, h] - a * p))
                out["dg"][i, h] = a * da
                dS = a * dS + np.outer(dp, k[i, h])
                if mutation == "no_p_in_ds":
                    dS = dS - np.outer(dp, k[i, h])  # the p path left out of dS_{t-1}
            out["dh0"][n, h] = dS
    return out


def test_unmutated_numpy_copy_equals_oracle():
    b = _batch([5, 3], H=2, dk=3, dv=2, seed=17)
    rng = np.random.default_rng(18)
    do, dsf = rng.normal(size=b["v"].shape), rng.normal(size=b["h0"].shape)
    got, ref = _mutated_backward(b, do, dsf, 0.9, None), _grads(b, do, dsf, 0.9)
    for name in got:
        np.testing.assert_allclose(got[name], ref[name], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mutation", ["sign_da", "drop_p_path", "no_p_in_ds"])
def test_planted_mistakes_are_caught_by_finite_differences(mutation):
    b = _batch([5, 3], H=2, dk=3, dv=2, seed=17)
    rng = np.random.default_rng(18)
    do, dsf = rng.normal(size=b["v"].shape), rng.normal(size=b["h0"].shape)
    ok, _ = _fd_check(b, do, dsf, 0.9, _mutated_backward(b, do, dsf, 0.9, mutation))
    assert not ok, mutation
