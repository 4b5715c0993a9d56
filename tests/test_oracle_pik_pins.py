"""Pins of the K-leaf GEMM oracle (oracle/pik.py), CPU only.

The definition C = A B^T is checked against a brute-force triple loop on
exact small integers and against identity and permutation matrices; the tree
against hand-worked float32 cases whose bits depend on the pairing (a
left-to-right sum, an exact sum or another pairing gives other values); the
ranked evaluation against the plain tree, bit for bit.
"""
import numpy as np
import pytest

from oracle import pik


def test_gemm_is_a_times_b_transposed_brute_force():
    rng = np.random.default_rng(0)
    A = rng.integers(-5, 6, size=(3, 7))
    B = rng.integers(-5, 6, size=(4, 7))
    C = pik.gemm_fp64(A, B)
    assert C.shape == (3, 4)
    for m in range(3):
        for n in range(4):
            assert C[m, n] == sum(int(A[m, k]) * int(B[n, k]) for k in range(7))


def test_gemm_identity_and_permutation():
    rng = np.random.default_rng(1)
    A = rng.normal(size=(5, 6))
    assert np.array_equal(pik.gemm_fp64(A, np.eye(6)), A)
    perm = rng.permutation(6)
    P = np.eye(6)[perm]  # row n of P selects column perm[n] of A
    assert np.array_equal(pik.gemm_fp64(A, P), A[:, perm])


def test_leaf_bounds_partition_k():
    assert pik.leaf_bounds(512, 4) == [(0, 128), (128, 256), (256, 384), (384, 512)]
    assert pik.leaf_bounds(64, 1) == [(0, 64)]
    with pytest.raises(ValueError):
        pik.leaf_bounds(100, 8)


def test_tree_pairs_neighbours_level_by_level():
    f = np.float32
    # balanced: (1 + 1e8) + (-1e8 + 1) = 1e8 + (-1e8) = 0 in float32
    # (left to right gives 1, the exact sum is 2)
    assert pik.tree_f32([f(1), f(1e8), f(-1e8), f(1)]) == f(0)
    # pairing (0,1),(2,3) and not (0,2),(1,3): the latter would give 2
    assert pik.tree_f32([f(1e8), f(1), f(-1e8), f(1)]) == f(0)
    # one level: a single rounded addition
    assert pik.tree_f32([f(1.5), f(2 ** -24)]) == f(1.5) + f(2 ** -24)
    assert pik.tree_f32([f(3.25)]) == f(3.25)
    with pytest.raises(ValueError):
        pik.tree_f32([f(1), f(2), f(3)])


def test_eight_leaf_tree_hand_worked():
    f = np.float32
    x = [f(2.0 ** 24), f(1), f(1), f(1), f(-2.0 ** 24), f(1), f(1), f(1)]
    # Level 1: 2^24 + 1 is a tie between 2^24 and 2^24 + 2 and rounds to the even
    # 2^24; 1 + 1 = 2; -2^24 + 1 = -16777215 exactly; 1 + 1 = 2.
    # Level 2: 2^24 + 2 = 16777218 (exact); -16777215 + 2 = -16777213 (exact).
    # Level 3: 16777218 - 16777213 = 5.  (Exact sum 6; left to right 3.)
    assert pik.tree_f32(x) == f(5)


@pytest.mark.parametrize("L", [1, 2, 8, 16])
def test_ranked_tree_equals_tree_bitwise(L):
    rng = np.random.default_rng(L)
    parts = [rng.normal(size=(5, 7)).astype(np.float32) * np.float32(10.0 ** rng.integers(-3, 4))
             for _ in range(L)]
    ref = pik.tree_f32(parts)
    R = 1
    while R <= L:
        assert np.array_equal(pik.ranked_tree_f32(parts, R), ref), R
        R *= 2
    with pytest.raises(ValueError):
        pik.ranked_tree_f32(parts + parts[:1], 2) if L > 1 else pik.ranked_tree_f32(parts, 3)


def test_tree_of_leaves_is_the_product_within_float32():
    rng = np.random.default_rng(7)
    A = rng.normal(size=(6, 256))
    B = rng.normal(size=(5, 256))
    leaves = [p.astype(np.float32) for p in pik.leaf_partials_fp64(A, B, 8)]
    got = pik.tree_f32(leaves).astype(np.float64)
    ref = pik.gemm_fp64(A, B)
    bound = 8 * 2.0 ** -24 * (np.abs(A) @ np.abs(B).T)
    assert np.all(np.abs(got - ref) <= bound)
    assert np.allclose(sum(pik.leaf_partials_fp64(A, B, 8)), ref, rtol=0, atol=1e-12)
