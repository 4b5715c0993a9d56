"""Host-side checks of the K-leaf GEMM's grouping (no GPU).

gdn_pik_gemm runs blocks of G = min(L / R, 2) consecutive leaves and, when
L / G > 1, adds the group sums with a combine kernel that evaluates the tree's
upper levels as a binary counter.  The grouping is read back through
gdn_pik_workspace_bytes (one fp32 M x N slice per group); the counter's order
of additions, transcribed from the combine kernel, must be the balanced tree's
(oracle.pik.tree_f32) bit for bit for every power-of-two group count, and a
group of two leaves followed by the counter must be the tree over the leaves.
"""
import numpy as np
import pytest

from oracle import pik as opik
from rl_train_numerics_b200 import build_lib

build_lib.build()
from rl_train_numerics_b200 import _abi as gdn  # noqa: E402


@pytest.mark.parametrize("L", [1, 2, 4, 8, 16, 32, 64])
def test_group_count_for_every_rank_count(L):
    M, N, K = 256, 512, 64 * L
    R = 1
    while R <= L:
        G = min(L // R, 2)
        want = (L // G) * M * N * 4 if L // G > 1 else 0
        assert gdn.pik_workspace_bytes(M, N, K, L, R) == want, (L, R)
        R *= 2


def binary_counter(parts):
    """The combine kernel's loop: push each group sum; while the two newest
    entries cover equal numbers of groups, replace them by (older + newer)."""
    stack, size = [], []
    for p in parts:
        v, sz = np.asarray(p, dtype=np.float32), 1
        while stack and size[-1] == sz:
            v = np.add(stack.pop(), v, dtype=np.float32)
            size.pop()
            sz *= 2
        stack.append(v)
        size.append(sz)
    assert len(stack) == 1
    return stack[0]


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 32, 64])
def test_combine_counter_is_the_balanced_tree(n):
    rng = np.random.default_rng(n)
    parts = [(rng.normal(size=(3, 5)) * 10.0 ** rng.integers(-4, 5)).astype(np.float32)
             for _ in range(n)]
    assert np.array_equal(binary_counter(parts), opik.tree_f32(parts))


@pytest.mark.parametrize("L", [2, 4, 8, 16])
def test_pairs_then_counter_is_the_tree_over_leaves(L):
    rng = np.random.default_rng(100 + L)
    leaves = [(rng.normal(size=(4, 4)) * 10.0 ** rng.integers(-4, 5)).astype(np.float32)
              for _ in range(L)]
    pairs = [np.add(leaves[2 * i], leaves[2 * i + 1], dtype=np.float32) for i in range(L // 2)]
    assert np.array_equal(binary_counter(pairs), opik.tree_f32(leaves))
