"""CPU oracle of the parallelism-invariant K-leaf GEMM.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline and reference legs may import this module.
The CUDA library and its binding never import, link or call it, and it
imports nothing from them.

What the GEMM computes
----------------------
"NovaSky's IsoExec Fixes the Hidden Math Bug Corrupting AI Training Runs",
section "Making kernels parallelism-invariant" (and its reduction-tree
figure): the K dimension of a GEMM is cut into contiguous leaves; each leaf
is a tensor-core product accumulated in fp32; the leaves are combined by one
fixed binary tree, and every rank always owns the same leaves, so the result
has the same bits however many ranks share the work.  Here

    C[m, n] = sum_k A[m, k] B[n, k]          (A is M x K, B is N x K)

with K cut into L leaves of K / L consecutive indices, L a power of two, and
the tree the balanced one: level by level, neighbours (2i, 2i + 1) are added.
R ranks (R a power of two dividing L) own contiguous blocks of L / R leaves,
each block a complete subtree, so a rank's partial is a node of the same tree.

Functions
---------
gemm_fp64          the definition, A B^T in float64 (numpy matmul).
leaf_bounds        the K ranges of the L leaves.
tree_f32           the fixed balanced tree over a list of float32 arrays, each
                   addition rounded to float32 (numpy float32 arithmetic).
ranked_tree_f32    the same tree evaluated as R ranks would: each rank's
                   subtree first, then the levels above the ranks.
leaf_partials_fp64 each leaf's exact product A[:, leaf] B[:, leaf]^T (float64).
"""
from __future__ import annotations

import numpy as np


def gemm_fp64(A, B) -> np.ndarray:
    """C = A B^T in float64: the plain definition."""
    return np.asarray(A, dtype=np.float64) @ np.asarray(B, dtype=np.float64).T


def leaf_bounds(K: int, L: int):
    """[(k0, k1)] of the L contiguous leaves of K (L must divide K)."""
    if L < 1 or K % L:
        raise ValueError("L must be >= 1 and divide K")
    w = K // L
    return [(l * w, (l + 1) * w) for l in range(L)]


def _is_pow2(x: int) -> bool:
    return x >= 1 and (x & (x - 1)) == 0


def tree_f32(parts):
    """Balanced binary tree over a power-of-two count of float32 arrays:
    each level adds neighbours (2i, 2i + 1), every sum rounded to float32."""
    level = [np.asarray(p, dtype=np.float32) for p in parts]
    if not _is_pow2(len(level)):
        raise ValueError("the tree needs a power-of-two number of leaves")
    while len(level) > 1:
        level = [np.add(level[2 * i], level[2 * i + 1], dtype=np.float32)
                 for i in range(len(level) // 2)]
    return level[0]


def ranked_tree_f32(parts, R: int):
    """The tree of ``tree_f32`` evaluated as R ranks do: rank r first sums
    its contiguous block of L / R leaves (a subtree), then the R rank partials
    go through the levels above them."""
    L = len(parts)
    if not (_is_pow2(R) and L % R == 0):
        raise ValueError("R must be a power of two dividing L")
    per = L // R
    ranks = [tree_f32(parts[r * per:(r + 1) * per]) for r in range(R)]
    return tree_f32(ranks)


def leaf_partials_fp64(A, B, L: int):
    """Exact (float64) product of every leaf."""
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    return [A[:, k0:k1] @ B[:, k0:k1].T for k0, k1 in leaf_bounds(A.shape[1], L)]
