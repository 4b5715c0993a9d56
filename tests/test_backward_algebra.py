"""The algebra of the CUDA backward, checked in float64 against the oracle (CPU).

gdn_cpr_backward does not run the reverse token loop that oracle.backward
runs.  It splits the gradient into (i) an adjoint recurrence per state row,
mu_{t-1} = alpha_t (Lambda_t - beta_t w_t k_t^T), (ii) per-chunk recomputed
states, (iii) dg as a telescoped sum Z_{t-1} = Z_t + do_t.o_t - beta_t v_t.w_t
and (iv) dq, dk of a chunk as products of C x C and C x d matrices
(Y = DO U^T, X = W U^T, A, B).  This test writes that schedule out in float64
numpy and requires it to equal the oracle's reverse mode to 1e-12 on ragged
batches with chunk sizes that leave partial chunks, so the identities the
kernels rely on are exact, independently of the GPU.
"""
import numpy as np
import pytest

import oracle


def _batch(lens, H, d, seed):
    rng = np.random.default_rng(seed)
    T = sum(lens)
    q = rng.normal(size=(T, H, d))
    k = rng.normal(size=(T, H, d))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.normal(size=(T, H, d))
    beta = 1.0 / (1.0 + np.exp(-rng.normal(size=(T, H))))
    g = -np.log1p(np.exp(rng.normal(size=(T, H))))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    h0 = rng.normal(size=(len(lens), H, d, d))
    do = rng.normal(size=(T, H, d))
    dsf = rng.normal(size=h0.shape)
    return q, k, v, beta, g, cu, h0, do, dsf


def chunked_backward(q, k, v, beta, g, cu, do, h0, dsf, scale, C):
    T, H, d = q.shape
    out = {n: np.zeros_like(x) for n, x in
           [("dq", q), ("dk", k), ("dv", v), ("dbeta", beta), ("dg", g), ("dh0", h0)]}
    for n in range(len(cu) - 1):
        a0, e0 = int(cu[n]), int(cu[n + 1])
        for h in range(H):
            # boundary states S_a at every chunk start (the forward's first pass)
            S, Sb = h0[n, h].copy(), {}
            for j in range(a0, e0):
                if (j - a0) % C == 0:
                    Sb[j] = S.copy()
                al = np.exp(g[j, h])
                S = al * S + np.outer(beta[j, h] * (v[j, h] - al * (S @ k[j, h])), k[j, h])
            # (i) adjoint recurrence, last token first: w per token, mu at chunk ends
            mu, W, mu_end = dsf[n, h].copy(), np.zeros((e0 - a0, d)), {}
            for j in range(e0 - 1, a0 - 1, -1):
                if (j - a0) % C == C - 1 or j == e0 - 1:
                    mu_end[j + 1] = mu.copy()
                lam = mu + scale * np.outer(do[j, h], q[j, h])
                W[j - a0] = lam @ k[j, h]
                mu = np.exp(g[j, h]) * (lam - beta[j, h] * np.outer(W[j - a0], k[j, h]))
            out["dh0"][n, h] = mu
            out["dv"][a0:e0, h] = beta[a0:e0, h, None] * W
            for a in range(a0, e0, C):
                e = min(a + C, e0)
                L = e - a
                # (ii) the chunk's states recomputed from S_a: p, u, o per token
                S = Sb[a].copy()
                P, U, O = np.zeros((L, d)), np.zeros((L, d)), np.zeros((L, d))
                for j in range(a, e):
                    al = np.exp(g[j, h])
                    P[j - a] = S @ k[j, h]
                    U[j - a] = beta[j, h] * (v[j, h] - al * P[j - a])
                    S = al * S + np.outer(U[j - a], k[j, h])
                    O[j - a] = scale * S @ q[j, h]
                Wc, al, bt = W[a - a0:e - a0], np.exp(g[a:e, h]), beta[a:e, h]
                out["dbeta"][a:e, h] = np.sum(Wc * (v[a:e, h] - al[:, None] * P), 1)
                # (iii) dg_t = Z_{t-1}, telescoped from Z at the chunk's end
                Z = np.sum(mu_end[e] * S)
                for j in range(e - 1, a - 1, -1):
                    Z = Z + do[j, h] @ O[j - a] - bt[j - a] * (v[j, h] @ Wc[j - a])
                    out["dg"][j, h] = Z
                # (iv) dq, dk from the chunk products
                G = np.cumsum(g[a:e, h])
                DO, Q, K = do[a:e, h], q[a:e, h], k[a:e, h]
                ii = np.arange(L)
                dec = np.exp(G[:, None] - G[None, :])
                A = np.where(ii[:, None] >= ii[None, :], dec, 0.0) * (DO @ U.T)
                B = np.where(ii[:, None] > ii[None, :], dec, 0.0) * (Wc @ U.T) * bt[:, None]
                out["dq"][a:e, h] = scale * (np.exp(G)[:, None] * (DO @ Sb[a]) + A @ K)
                out["dk"][a:e, h] = (scale * A.T @ Q - (B + B.T) @ K
                                     - (bt * np.exp(G))[:, None] * (Wc @ Sb[a])
                                     + np.exp(G[-1] - G)[:, None] * (U @ mu_end[e]))
    return out


@pytest.mark.parametrize("C", [1, 3, 16, 64])
def test_chunked_schedule_equals_the_oracles_reverse_mode(C):
    q, k, v, beta, g, cu, h0, do, dsf = _batch([1, 63, 64, 65, 130, 0, 7], 2, 6, seed=C)
    scale = 0.6
    ref = oracle.backward(q, k, v, beta, g, cu, do, h0=h0, ds_final=dsf, scale=scale, threads=1)
    got = chunked_backward(q, k, v, beta, g, cu, do, h0, dsf, scale, C)
    for name in ref:
        err = np.max(np.abs(got[name] - ref[name])) / max(1.0, np.max(np.abs(ref[name])))
        assert err < 1e-12, (name, C, err)


def test_adjoint_chunk_map_is_the_transposed_boundary_map():
    """The adjoint crosses a chunk as mu_a = mu_e P^T + W_loc, where P is the
    chunk's state transition (S_end = S_a P with v = 0), W_loc the adjoint the
    chunk's own outputs produce from mu_e = 0, and P^T has the closed form
    e^{G_n} I - K^T diag(e^{G_n - G}) T diag(beta e^G) K in the quantities of
    the forward's boundary computation (T = (I + A)^{-1}).  So a reverse walk
    over chunk boundaries can run on the forward's boundary data."""
    rng = np.random.default_rng(5)
    n, d, scale = 13, 5, 0.7
    K = rng.normal(size=(n, d))
    K /= np.linalg.norm(K, axis=1, keepdims=True)
    Q = rng.normal(size=(n, d))
    beta = 1.0 / (1.0 + np.exp(-rng.normal(size=n)))
    g = -np.log1p(np.exp(rng.normal(size=n)))
    DO = rng.normal(size=(n, d))
    cb = oracle.chunk_boundary(np.zeros((d, d)), K, np.zeros((n, d)), beta, g)
    T, G = cb["T"], cb["G"]
    # P from the token loop: S -> S F_1 ... F_n with F_t = a_t (I - b_t k_t k_t^T)
    P = np.eye(d)
    for t in range(n):
        P = P @ (np.exp(g[t]) * (np.eye(d) - beta[t] * np.outer(K[t], K[t])))
    S0 = rng.normal(size=(d, d))
    assert np.allclose(S0 @ P, oracle.chunk_boundary(S0, K, np.zeros((n, d)), beta, g)["S"],
                       rtol=0, atol=1e-12)
    Pt = (np.exp(G[-1]) * np.eye(d)
          - K.T @ (np.exp(G[-1] - G)[:, None] * T * (beta * np.exp(G))[None, :]) @ K)
    assert np.allclose(Pt, P.T, rtol=0, atol=1e-12)

    def adjoint(mu_e):
        mu = mu_e.copy()
        for t in range(n - 1, -1, -1):
            lam = mu + scale * np.outer(DO[t], Q[t])
            w = lam @ K[t]
            mu = np.exp(g[t]) * (lam - beta[t] * np.outer(w, K[t]))
        return mu

    mu_e = rng.normal(size=(d, d))
    W_loc = adjoint(np.zeros((d, d)))
    assert np.allclose(adjoint(mu_e), mu_e @ Pt + W_loc, rtol=0, atol=1e-12)


def chunked_adjoint(q, k, beta, g, cu, do, dsf, scale, C, n, h):
    """The chunk form of the adjoint (the CUDA backward runs the token
    recurrence; this form is what a chunk-parallel adjoint evaluates): per
    chunk (in parallel)
    Z = (I + A)^{-T} R, Y = (I + A)^{-T} diag(e^{G_{L-1} - G}) K and
    W_loc = scale DO^T diag(e^G) Q - Z^T diag(beta e^G) K; then a reverse walk
    over the chunks, mu_a = e^{G_{L-1}} mu_e - (mu_e Y^T) diag(beta e^G) K + W_loc;
    then W = Z + Y mu_e^T per chunk.  Returns (W, mu at every chunk end, dh0)."""
    a0, e0 = int(cu[n]), int(cu[n + 1])
    d = q.shape[2]
    W, mu_end, pre = np.zeros((e0 - a0, d)), {}, {}
    for a in range(a0, e0, C):
        e = min(a + C, e0)
        L = e - a
        G = np.cumsum(g[a:e, h])
        K, Q, DO, bt = k[a:e, h], q[a:e, h], do[a:e, h], beta[a:e, h]
        ii = np.arange(L)
        A = (np.where(ii[:, None] > ii[None, :], np.exp(G[:, None] - G[None, :]), 0.0)
             * (K @ K.T) * bt[:, None])                        # A[r, t], r > t
        M = np.where(ii[None, :] >= ii[:, None], np.exp(G[None, :] - G[:, None]), 0.0) * (K @ Q.T)
        I_A = np.eye(L) + A
        Z = np.linalg.solve(I_A.T, scale * M @ DO)
        Y = np.linalg.solve(I_A.T, np.exp(G[-1] - G)[:, None] * K)
        bg = bt * np.exp(G)
        Wl = scale * DO.T @ (np.exp(G)[:, None] * Q) - Z.T @ (bg[:, None] * K)
        pre[a] = (Z, Y, bg, K, np.exp(G[-1]), Wl)
    mu = dsf[n, h].copy()
    for a in reversed(range(a0, e0, C)):
        e = min(a + C, e0)
        Z, Y, bg, K, gam, Wl = pre[a]
        mu_end[e] = mu.copy()
        W[a - a0:e - a0] = Z + Y @ mu.T
        mu = gam * mu - ((mu @ Y.T) * bg[None, :]) @ K + Wl
    return W, mu_end, mu


@pytest.mark.parametrize("C", [1, 3, 16, 64])
def test_chunked_adjoint_equals_the_token_recurrence(C):
    q, k, v, beta, g, cu, h0, do, dsf = _batch([1, 63, 64, 65, 130, 0, 7], 2, 6, seed=10 + C)
    scale = 0.6
    for n in range(len(cu) - 1):
        a0, e0 = int(cu[n]), int(cu[n + 1])
        for h in range(2):
            mu, W, ends = dsf[n, h].copy(), np.zeros((e0 - a0, 6)), {}
            for j in range(e0 - 1, a0 - 1, -1):
                if (j - a0) % C == C - 1 or j == e0 - 1:
                    ends[j + 1] = mu.copy()
                lam = mu + scale * np.outer(do[j, h], q[j, h])
                W[j - a0] = lam @ k[j, h]
                mu = np.exp(g[j, h]) * (lam - beta[j, h] * np.outer(W[j - a0], k[j, h]))
            W2, ends2, mu2 = chunked_adjoint(q, k, beta, g, cu, do, dsf, scale, C, n, h)
            assert np.max(np.abs(W2 - W), initial=0.0) < 1e-12
            assert np.max(np.abs(mu2 - mu)) < 1e-12
            assert ends.keys() == ends2.keys()
            for e in ends:
                assert np.max(np.abs(ends2[e] - ends[e])) < 1e-12


def kernel_adjoint(q, k, beta, g, cu, do, dsf, scale, C, n, h):
    """The chunk form of the adjoint as the bf16-input CUDA backward evaluates
    it (k_adj_prep, k_adj_walk, k_adj_w), with T = (I + A)^{-1} from the
    forward prep, Tb = T diag(beta e^G), dvec = e^{G_{L-1} - G} and
    Pm[r][t] = [t <= r] e^{G_r - G_t} q_r . k_t:
      X   = scale (diag(e^G) Q - Pm Tb K)                      (per chunk)
      mu <- e^{G_{L-1}} mu - ((mu K^T) diag(dvec)) Tb K + DO^T X  (serial walk)
      W   = T^T (diag(dvec) (mu_e K^T)^T + scale Pm^T DO)        (per chunk)
    Returns (W, mu at every chunk end, dh0)."""
    a0, e0 = int(cu[n]), int(cu[n + 1])
    d = q.shape[2]
    W, mu_end, pre = np.zeros((e0 - a0, d)), {}, {}
    for a in range(a0, e0, C):
        e = min(a + C, e0)
        L = e - a
        G = np.cumsum(g[a:e, h])
        K, Q, DO, bt = k[a:e, h], q[a:e, h], do[a:e, h], beta[a:e, h]
        ii = np.arange(L)
        A = (np.where(ii[:, None] > ii[None, :], np.exp(G[:, None] - G[None, :]), 0.0)
             * (K @ K.T) * bt[:, None])
        T = np.linalg.inv(np.eye(L) + A)
        Tb = T * (bt * np.exp(G))[None, :]
        dvec = np.exp(G[-1] - G)
        Pm = np.where(ii[None, :] <= ii[:, None], np.exp(G[:, None] - G[None, :]), 0.0) * (Q @ K.T)
        X = scale * (np.exp(G)[:, None] * Q - Pm @ Tb @ K)
        pre[a] = (K, DO, T, Tb, dvec, Pm, X, np.exp(G[-1]))
    mu = dsf[n, h].copy()
    for a in reversed(range(a0, e0, C)):
        e = min(a + C, e0)
        K, DO, T, Tb, dvec, Pm, X, gam = pre[a]
        mu_end[e] = mu.copy()
        Ydv = (mu @ K.T) * dvec[None, :]                       # [row][t]
        W[a - a0:e - a0] = T.T @ (Ydv.T + scale * Pm.T @ DO)
        mu = gam * mu - (Ydv @ Tb) @ K + DO.T @ X
    return W, mu_end, mu


@pytest.mark.parametrize("C", [1, 3, 16, 64])
def test_kernel_adjoint_form_equals_the_token_recurrence(C):
    q, k, v, beta, g, cu, h0, do, dsf = _batch([1, 63, 64, 65, 130, 0, 7], 2, 6, seed=30 + C)
    scale = 0.6
    for n in range(len(cu) - 1):
        a0, e0 = int(cu[n]), int(cu[n + 1])
        for h in range(2):
            mu, W, ends = dsf[n, h].copy(), np.zeros((e0 - a0, 6)), {}
            for j in range(e0 - 1, a0 - 1, -1):
                if (j - a0) % C == C - 1 or j == e0 - 1:
                    ends[j + 1] = mu.copy()
                lam = mu + scale * np.outer(do[j, h], q[j, h])
                W[j - a0] = lam @ k[j, h]
                mu = np.exp(g[j, h]) * (lam - beta[j, h] * np.outer(W[j - a0], k[j, h]))
            W2, ends2, mu2 = kernel_adjoint(q, k, beta, g, cu, do, dsf, scale, C, n, h)
            assert np.max(np.abs(W2 - W), initial=0.0) < 1e-12
            assert np.max(np.abs(mu2 - mu)) < 1e-12
            assert ends.keys() == ends2.keys()
            for e in ends:
                assert np.max(np.abs(ends2[e] - ends[e])) < 1e-12



def kernel_rows(q, k, v, beta, g, S_a, W, mu_e, do, scale):
    """The per-chunk u, dbeta and dg of the bf16-input CUDA backward (k_bwd_u,
    then the epilogue of k_bwd_gemm_tc), for one chunk of length L from its
    entry state S_a, its w rows W, the adjoint mu_e at its end and its do rows:
      U       = T diag(beta) (V - diag(e^G) K S_a^T),  T = (I + A)^{-1},
                A_ts = [s < t] beta_t e^{G_t - G_s} k_t . k_s
      DQ      = scale (diag(e^G) DO S_a + Ad K),  Ad_ts = [s <= t] e^{G_t - G_s} do_t . u_s
      dbeta_t = w_t . v_t - e^{G_t} k_t . (W S_a)_t - sum_{s<t} A'_ts X_ts,
                A'_ts = e^{G_t - G_s} k_t . k_s,  X = W U^T
      Z_end   = e^{G_{L-1}} <mu_e, S_a> + sum_t e^{G_{L-1} - G_t} k_t . (U mu_e)_t
      dg_t    = Z_end + sum_{s >= t} (q_s . dq_s - beta_s v_s . w_s).
    Returns (U, DQ, dbeta, Z_end, dg)."""
    L, d = k.shape
    G = np.cumsum(g)
    ii = np.arange(L)
    low = ii[:, None] > ii[None, :]
    dec = np.exp(G[:, None] - G[None, :])
    KK = k @ k.T
    A = np.where(low, dec, 0.0) * KK * beta[:, None]
    T = np.linalg.inv(np.eye(L) + A)
    U = T @ (beta[:, None] * (v - np.exp(G)[:, None] * (k @ S_a.T)))
    Ad = np.where(ii[:, None] >= ii[None, :], dec, 0.0) * (do @ U.T)
    DQ = scale * (np.exp(G)[:, None] * (do @ S_a) + Ad @ k)
    X = W @ U.T
    dbeta = (np.sum(W * v, axis=1) - np.exp(G) * np.sum(k * (W @ S_a), axis=1)
             - np.sum(np.where(low, dec, 0.0) * KK * X, axis=1))
    dvec = np.exp(G[-1] - G)
    Z_end = np.exp(G[-1]) * np.sum(mu_e * S_a) + np.sum(dvec * np.sum(k * (U @ mu_e), axis=1))
    term = np.sum(q * DQ, axis=1) - beta * np.sum(v * W, axis=1)
    dg = Z_end + np.cumsum(term[::-1])[::-1]
    return U, DQ, dbeta, Z_end, dg


def test_kernel_rows_form_equals_the_token_recurrence():
    """u, dq, dbeta = w . (v - alpha S_{t-1} k) and dg = <mu_{t-1}, S_{t-1}> of the
    kernels' product form against the token recurrence and its adjoint."""
    rng = np.random.default_rng(41)
    for L in (1, 7, 64):
        d, scale = 6, 0.7
        k = rng.normal(size=(L, d)); k /= np.linalg.norm(k, axis=1, keepdims=True)
        q, v, do = rng.normal(size=(L, d)), rng.normal(size=(L, d)), rng.normal(size=(L, d))
        beta = 1.0 / (1.0 + np.exp(-rng.normal(size=L)))
        g = -np.log1p(np.exp(2.0 * rng.normal(size=L)))
        S_a, mu_e = rng.normal(size=(d, d)), rng.normal(size=(d, d))
        # The adjoint inside the chunk, last token first (mu_t, Lambda_t, w_t).
        states = [S_a]
        for t in range(L):
            a = np.exp(g[t])
            u = beta[t] * (v[t] - a * (states[-1] @ k[t]))
            states.append(a * states[-1] + np.outer(u, k[t]))
        mu = mu_e.copy()
        W = np.zeros((L, d))
        dg_ref = np.zeros(L)
        for t in range(L - 1, -1, -1):
            Lam = mu + scale * np.outer(do[t], q[t])
            W[t] = Lam @ k[t]
            mu = np.exp(g[t]) * (Lam - beta[t] * np.outer(W[t], k[t]))
            dg_ref[t] = np.sum(mu * states[t])  # <mu_{t-1}, S_{t-1}>
        U, DQ, dbeta, Z_end, dg = kernel_rows(q, k, v, beta, g, S_a, W, mu_e, do, scale)
        for t in range(L):
            S_prev, S_t = states[t], states[t + 1]
            r = v[t] - np.exp(g[t]) * (S_prev @ k[t])
            assert np.max(np.abs(U[t] - beta[t] * r)) < 1e-12
            assert np.max(np.abs(DQ[t] - scale * (S_t.T @ do[t]))) < 1e-12
            assert abs(dbeta[t] - W[t] @ r) < 1e-12
        assert abs(Z_end - np.sum(mu_e * states[-1])) < 1e-12 * max(1.0, abs(Z_end))
        assert np.max(np.abs(dg - dg_ref)) < 1e-11 * max(1.0, np.max(np.abs(dg_ref)))
