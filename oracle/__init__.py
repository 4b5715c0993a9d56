"""CPU oracle for the CPR Gated DeltaNet layer.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this package.  The CUDA
library and its Python binding never import, link or call it, and it imports
nothing from them: the two implementations share no code, tables or constants.

What the layer computes
-----------------------
"NovaSky's IsoExec Fixes the Hidden Math Bug Corrupting AI Training Runs",
section "Solving the linear-attention headache": Gated DeltaNet is evaluated
by CPR (chunkwise-parallel recurrent): the token recurrence defines the
result, a serial sweep gives the state entering each chunk, the chunks then
replay the recurrence from those states, and decode swaps its running state
for the chunk-start computation after each chunk's worth of tokens.  The
section also says that the chunked and the token-by-token forms agree in
exact arithmetic, so the oracle for every output is the plain recurrence

    S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
    o_t = scale * S_t q_t,          alpha_t = exp(g_t),

evaluated token by token in float64 with no chunking (``forward``).

The module ``oracle.pik`` is the oracle of the parallelism-invariant K-leaf
GEMM (section "Making kernels parallelism-invariant" of the same page).

Functions
---------
forward / forward_alpha   the token loop, in C (``gdn_oracle.c``), OpenMP
                          over (sequence, head) units.
backward                  its reverse mode (the gradient of a loss through the
                          token loop), in C, fp64, with the states recomputed
                          from checkpoints every 64 tokens.
explicit_product_state    the closed product form of the recurrence with the
                          per-token transition matrices written out, in
                          float64 (numpy matmul) or exact rationals
                          (``fractions.Fraction``); a structurally different
                          evaluation of the same definition, used to pin the
                          token loop.
chunk_boundary / cpr_forward
                          the CPR schedule in float64: the boundary state of a
                          C-token chunk from the UT (WY) form of the same
                          recurrence, then the per-token fill inside each
                          chunk from the boundary states.  Pinned against the
                          token loop; it documents the boundary formula the
                          CUDA kernels evaluate in fp32 on tensor cores.

Every input is a float64 copy of exactly the values the GPU sees (bf16 and
fp32 widen exactly).  Outputs are float64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from fractions import Fraction
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "libgdn_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (-O2 -fopenmp).  Returns the .so path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", _SRC, "-o", _LIB, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int32)
        for name in ("gdn_oracle_forward", "gdn_oracle_forward_alpha"):
            fn = getattr(lib, name)
            fn.restype = ctypes.c_int
            fn.argtypes = [dp, dp, dp, dp, dp, ip, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                           ctypes.c_int, ctypes.c_double, dp, dp, dp, ctypes.c_int]
        fb = lib.gdn_oracle_backward
        fb.restype = ctypes.c_int
        fb.argtypes = [dp, dp, dp, dp, dp, ip, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                       ctypes.c_int, ctypes.c_double, dp, dp, dp, dp, dp, dp, dp, dp, dp,
                       ctypes.c_int]
        lib.gdn_oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def max_threads() -> int:
    """Threads the C oracle uses when ``threads`` is not given."""
    return int(_load().gdn_oracle_max_threads())


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor: widen exactly through float64
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _run(entry: str, q, k, v, beta, gate, cu_seqlens, h0, scale, threads, want_state=True):
    q, k, v, beta, gate = (_f64(a) for a in (q, k, v, beta, gate))
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    T, H, dk = q.shape
    dv = v.shape[2]
    n = cu.shape[0] - 1
    assert k.shape == (T, H, dk) and v.shape[:2] == (T, H)
    assert beta.shape == (T, H) and gate.shape == (T, H)
    assert n >= 0 and int(cu[0]) == 0 and int(cu[-1]) == T
    o = np.zeros((T, H, dv), dtype=np.float64)
    s_final = np.zeros((n, H, dv, dk), dtype=np.float64) if want_state else None
    h0a = None if h0 is None else _f64(h0)
    if h0a is not None:
        assert h0a.shape == (n, H, dv, dk)
    dp = ctypes.POINTER(ctypes.c_double)

    def ptr(a):
        return None if a is None else a.ctypes.data_as(dp)

    rc = getattr(_load(), entry)(
        ptr(q), ptr(k), ptr(v), ptr(beta), ptr(gate),
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), n, H, dk, dv, float(scale),
        ptr(h0a), ptr(o), ptr(s_final), int(threads or 0))
    if rc != 0:
        raise ValueError(f"{entry} failed with status {rc}")
    return o, s_final


def forward(q, k, v, beta, g, cu_seqlens, h0=None, scale: float = 1.0,
            threads: Optional[int] = None):
    """Token-by-token fp64 recurrence over packed sequences.

    Shapes: q,k [T,H,dk]; v [T,H,dv]; beta,g [T,H]; cu_seqlens [N+1];
    h0 [N,H,dv,dk] or None (zeros).  Returns (o [T,H,dv], S_final [N,H,dv,dk]).
    alpha_t = exp(g_t) in double.
    """
    return _run("gdn_oracle_forward", q, k, v, beta, g, cu_seqlens, h0, scale, threads)


def forward_alpha(q, k, v, beta, alpha, cu_seqlens, h0=None, scale: float = 1.0,
                  threads: Optional[int] = None):
    """Same recurrence with the decay alpha_t given directly (alpha = 0 allowed)."""
    return _run("gdn_oracle_forward_alpha", q, k, v, beta, alpha, cu_seqlens, h0, scale, threads)


def backward(q, k, v, beta, g, cu_seqlens, do, h0=None, ds_final=None, scale: float = 1.0,
             threads: Optional[int] = None):
    """Reverse mode of the token loop (fp64): the gradient of a loss L given
    do = dL/do [T,H,dv] and ds_final = dL/dS_final [N,H,dv,dk] (None = 0).
    Returns dict(dq, dk [T,H,dk], dv [T,H,dv], dbeta, dg [T,H], dh0 [N,H,dv,dk])."""
    q, k, v, beta, g, do = (_f64(a) for a in (q, k, v, beta, g, do))
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    T, H, dk = q.shape
    dv = v.shape[2]
    n = cu.shape[0] - 1
    assert k.shape == (T, H, dk) and v.shape == (T, H, dv) and do.shape == (T, H, dv)
    assert beta.shape == (T, H) and g.shape == (T, H)
    assert n >= 0 and int(cu[0]) == 0 and int(cu[-1]) == T
    h0a = None if h0 is None else _f64(h0)
    dsf = None if ds_final is None else _f64(ds_final)
    out = {"dq": np.zeros((T, H, dk)), "dk": np.zeros((T, H, dk)), "dv": np.zeros((T, H, dv)),
           "dbeta": np.zeros((T, H)), "dg": np.zeros((T, H)), "dh0": np.zeros((n, H, dv, dk))}
    dp = ctypes.POINTER(ctypes.c_double)

    def ptr(a):
        return None if a is None else a.ctypes.data_as(dp)

    rc = _load().gdn_oracle_backward(
        ptr(q), ptr(k), ptr(v), ptr(beta), ptr(g),
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), n, H, dk, dv, float(scale),
        ptr(h0a), ptr(do), ptr(dsf), ptr(out["dq"]), ptr(out["dk"]), ptr(out["dv"]),
        ptr(out["dbeta"]), ptr(out["dg"]), ptr(out["dh0"]), int(threads or 0))
    if rc != 0:
        raise ValueError(f"gdn_oracle_backward failed with status {rc}")
    return out


# ---------------------------------------------------------------------------
# Explicit product form (pins the token loop)
# ---------------------------------------------------------------------------

def explicit_product_state(S0, K, V, beta, alpha, exact: bool = False):
    """Final state of one (sequence, head) from the unrolled product form.

    Writing M_t = alpha_t (I - beta_t k_t k_t^T), the recurrence
    S_t = S_{t-1} M_t + beta_t v_t k_t^T unrolls to

        S_T = S_0 M_1 M_2 ... M_T + sum_t beta_t v_t k_t^T M_{t+1} ... M_T.

    Every M_t is formed as an explicit d_k x d_k matrix and the products are
    taken as matrix products.  With ``exact=True`` all arithmetic is done in
    ``fractions.Fraction`` (inputs must then be exact rationals or floats,
    which convert exactly).  Returns an object array of Fractions when exact,
    else float64.
    """
    T = len(beta)
    if exact:
        S0 = [[Fraction(x) for x in row] for row in S0]
        K = [[Fraction(x) for x in row] for row in K]
        V = [[Fraction(x) for x in row] for row in V]
        beta = [Fraction(b) for b in beta]
        alpha = [Fraction(a) for a in alpha]
        dv, dk = len(S0), len(S0[0])

        def matmul(A, B):
            n, m, p = len(A), len(B), len(B[0])
            return [[sum((A[i][l] * B[l][j] for l in range(m)), Fraction(0)) for j in range(p)]
                    for i in range(n)]

        def madd(A, B):
            return [[a + b for a, b in zip(ra, rb)] for ra, rb in zip(A, B)]

        M = []
        for t in range(T):
            Mt = [[alpha[t] * ((1 if i == j else 0) - beta[t] * K[t][i] * K[t][j])
                   for j in range(dk)] for i in range(dk)]
            M.append(Mt)
        acc = S0
        for t in range(T):
            acc = matmul(acc, M[t])
        for t in range(T):
            term = [[beta[t] * V[t][r] * K[t][j] for j in range(dk)] for r in range(dv)]
            for s in range(t + 1, T):
                term = matmul(term, M[s])
            acc = madd(acc, term)
        return np.array(acc, dtype=object)

    S0 = np.asarray(S0, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    dk = S0.shape[1]
    M = [alpha[t] * (np.eye(dk) - beta[t] * np.outer(K[t], K[t])) for t in range(T)]
    acc = S0.copy()
    for t in range(T):
        acc = acc @ M[t]
    for t in range(T):
        term = beta[t] * np.outer(V[t], K[t])
        for s in range(t + 1, T):
            term = term @ M[s]
        acc = acc + term
    return acc


# ---------------------------------------------------------------------------
# CPR schedule in fp64 (UT / WY form of the chunk boundary)
# ---------------------------------------------------------------------------

def chunk_boundary(S0, K, V, beta, g):
    """State after one chunk of n tokens, from the state S0 at its start.

    Derivation (from the recurrence; the pages give only the idea of a
    first pass that computes the state at chunk boundaries):
    with u_i = beta_i (v_i - alpha_i S_{i-1} k_i) the recurrence reads
    S_i = alpha_i S_{i-1} + u_i k_i^T.  With G_i = g_1 + ... + g_i and
    gamma_i = exp(G_i), unrolling gives
        S_i = gamma_i S0 + sum_{j<=i} exp(G_i - G_j) u_j k_j^T,
    and substituting S_{i-1} into u_i gives the unit lower-triangular system
        (I + A) U = diag(beta) V - diag(beta * gamma) K S0^T,
        A_ij = beta_i exp(G_i - G_j) (k_i . k_j)   for j < i.
    With T = (I + A)^{-1}, W = T diag(beta gamma) K and U~ = T diag(beta) V:
        U   = U~ - W S0^T
        S_n = exp(G_n) S0 + U^T diag(exp(G_n - G)) K.
    Gate ratios are always exp of a difference of cumulative sums, never a
    ratio of two exponentials (those underflow on long decays).

    Returns a dict with the boundary state and the intermediates.
    """
    S0 = np.asarray(S0, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    beta = np.asarray(beta, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    n = len(g)
    G = np.cumsum(g)
    P = K @ K.T
    A = np.zeros((n, n))
    for i in range(n):
        for j in range(i):
            A[i, j] = beta[i] * np.exp(G[i] - G[j]) * P[i, j]
    # Forward substitution of (I + A) T = I, row by row.
    Tm = np.eye(n)
    for i in range(n):
        for j in range(i):
            Tm[i, j] = -sum(A[i, m] * Tm[m, j] for m in range(j, i))
    W = Tm @ ((beta * np.exp(G))[:, None] * K)
    Ut = Tm @ (beta[:, None] * V)
    U = Ut - W @ S0.T
    S_end = np.exp(G[-1]) * S0 + U.T @ (np.exp(G[-1] - G)[:, None] * K)
    return {"S": S_end, "G": G, "A": A, "T": Tm, "W": W, "Ut": Ut, "U": U}


def _unit_recurrence(S, q, k, v, beta, g, scale):
    """Token loop for one unit (float64, numpy); returns (o, S_end)."""
    S = np.array(S, dtype=np.float64, copy=True)
    o = np.zeros((len(g), S.shape[0]))
    for t in range(len(g)):
        a = np.exp(g[t])
        p = S @ k[t]
        S = a * (S - beta[t] * np.outer(p, k[t])) + beta[t] * np.outer(v[t], k[t])
        o[t] = scale * (S @ q[t])
    return o, S


def cpr_forward(q, k, v, beta, g, cu_seqlens, C: int, h0=None, scale: float = 1.0):
    """CPR forward in float64.

    Pass 1: walk the full chunks of every sequence with ``chunk_boundary``
    (chunks start at each sequence's token 0 and never cross cu_seqlens).
    Pass 2: from each chunk's boundary state, run the token recurrence over
    the chunk's tokens to produce its outputs.
    Returns (o, S_run_final, S_bnd_final, boundary_states) where
    S_bnd_final is the boundary state after the last full chunk, S_run_final
    is that same state when the length is a multiple of C and otherwise the
    recurrent state after the trailing partial chunk, and boundary_states is
    a list (per sequence) of [n_full+1, H, dv, dk] arrays.
    """
    q, k, v, beta, g = (_f64(a) for a in (q, k, v, beta, g))
    cu = [int(x) for x in np.asarray(cu_seqlens)]
    T, H, dk = q.shape
    dv = v.shape[2]
    N = len(cu) - 1
    o = np.zeros((T, H, dv))
    s_run = np.zeros((N, H, dv, dk))
    s_bnd = np.zeros((N, H, dv, dk))
    bstates = []
    for n in range(N):
        t0, t1 = cu[n], cu[n + 1]
        L = t1 - t0
        nf = L // C
        seq_b = np.zeros((nf + 1, H, dv, dk))
        for h in range(H):
            S = np.zeros((dv, dk)) if h0 is None else _f64(h0)[n, h]
            seq_b[0, h] = S
            for c in range(nf):
                a, b = t0 + c * C, t0 + (c + 1) * C
                S = chunk_boundary(S, k[a:b, h], v[a:b, h], beta[a:b, h], g[a:b, h])["S"]
                seq_b[c + 1, h] = S
            s_bnd[n, h] = S
            s_run[n, h] = S
            for c in range((L + C - 1) // C):
                a, b = t0 + c * C, min(t0 + (c + 1) * C, t1)
                oc, Se = _unit_recurrence(seq_b[c, h], q[a:b, h], k[a:b, h], v[a:b, h],
                                          beta[a:b, h], g[a:b, h], scale)
                o[a:b, h] = oc
                if c == nf:  # trailing partial chunk
                    s_run[n, h] = Se
        bstates.append(seq_b)
    return o, s_run, s_bnd, bstates


def chunked_outputs(S0, Q, K, V, beta, g, scale: float = 1.0):
    """Outputs of one chunk of n tokens from the state S0 at its start, by
    the chunkwise-parallel (UT / WY) products (float64).

    This is how the usual ("native mixed") layout of the per-layer table in
    "NovaSky's IsoExec Fixes the Hidden Math Bug Corrupting AI Training
    Runs" (section "Solving the linear-attention headache") evaluates a
    chunk in training and prefill.  From the unrolled recurrence of
    ``chunk_boundary``, S_i = gamma_i S0 + sum_{j<=i} exp(G_i - G_j) u_j k_j^T,
    so o_i = scale S_i q_i is
        o_i = scale (exp(G_i) S0 q_i + sum_{j<=i} exp(G_i - G_j) (q_i . k_j) u_j)
    with U the rows u_j of ``chunk_boundary``.  Returns (o [n, dv], S_n).
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    S0 = np.asarray(S0, dtype=np.float64)
    cb = chunk_boundary(S0, K, V, beta, g)
    G, U = cb["G"], cb["U"]
    n = len(G)
    Pm = np.zeros((n, n))
    for i in range(n):
        for j in range(i + 1):
            Pm[i, j] = np.exp(G[i] - G[j]) * (Q[i] @ K[j])
    o = scale * (np.exp(G)[:, None] * (Q @ S0.T) + Pm @ U)
    return o, cb["S"]


def native_forward(q, k, v, beta, g, cu_seqlens, C: int, h0=None, scale: float = 1.0):
    """The chunked ("native mixed") forward in float64: the boundary states of
    ``cpr_forward``'s first pass, then every chunk's outputs (trailing partial
    chunks included) by ``chunked_outputs``.  Returns (o, S_final, S_bnd_final)."""
    q, k, v, beta, g = (_f64(a) for a in (q, k, v, beta, g))
    cu = [int(x) for x in np.asarray(cu_seqlens)]
    T, H, dk = q.shape
    dv = v.shape[2]
    N = len(cu) - 1
    o = np.zeros((T, H, dv))
    s_fin = np.zeros((N, H, dv, dk))
    s_bnd = np.zeros((N, H, dv, dk))
    for n in range(N):
        t0, t1 = cu[n], cu[n + 1]
        for h in range(H):
            S = np.zeros((dv, dk)) if h0 is None else _f64(h0)[n, h]
            s_bnd[n, h] = S
            for a in range(t0, t1, C):
                b = min(a + C, t1)
                oc, Se = chunked_outputs(S, q[a:b, h], k[a:b, h], v[a:b, h], beta[a:b, h],
                                         g[a:b, h], scale)
                o[a:b, h] = oc
                if b - a == C:
                    s_bnd[n, h] = Se
                S = Se
            s_fin[n, h] = S
    return o, s_fin, s_bnd


__all__ = ["build", "forward", "forward_alpha", "max_threads", "explicit_product_state",
           "chunk_boundary", "cpr_forward", "chunked_outputs", "native_forward"]
