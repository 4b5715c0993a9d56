"""Host-side checks of the K-leaf GEMM's work split (no GPU).

gdn_pik_gemm runs one work unit per 128 x 256 tile and emulated rank: the
rank's L / R leaves, added in the kernel by the balanced tree: leaf pairs
first, then a binary counter over the pair sums (pending subtree sums in a
per-block workspace slice, one 128 x 256 fp32 slot per level above the pairs,
at most 148 persistent blocks).  With
R > 1 the rank sums go to the workspace (one fp32 M x N slice per rank) and a
combine kernel applies the levels above the ranks with the same counter.  The
split is read back through gdn_pik_workspace_bytes; the counter's order of
additions, transcribed from the kernels, must be the balanced tree's
(oracle.pik.tree_f32) bit for bit for every power-of-two count, and rank
subtrees followed by the counter must be the tree over the leaves.
"""
import numpy as np
import pytest

from oracle import pik as opik
from rl_train_numerics_b200 import build_lib

build_lib.build()
from rl_train_numerics_b200 import _abi as gdn  # noqa: E402


@pytest.mark.parametrize("L", [1, 2, 4, 8, 16, 32, 64])
def test_workspace_for_every_rank_count(L):
    M, N, K = 256, 512, 64 * L
    tiles = (M // 128) * (N // 256)
    R = 1
    while R <= L:
        depth = int(np.log2(max(L // R // 2, 1)))  # pending sums over leaf pairs
        blocks = min(tiles * R, 148)
        want = (R * M * N * 4 if R > 1 else 0) + blocks * depth * 128 * 256 * 4
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


@pytest.mark.parametrize("L,R", [(2, 2), (4, 2), (8, 4), (16, 2), (16, 8)])
def test_rank_subtrees_then_counter_is_the_tree_over_leaves(L, R):
    rng = np.random.default_rng(100 + L + R)
    leaves = [(rng.normal(size=(4, 4)) * 10.0 ** rng.integers(-4, 5)).astype(np.float32)
              for _ in range(L)]
    per = L // R
    ranks = [binary_counter(leaves[r * per:(r + 1) * per]) for r in range(R)]
    assert np.array_equal(binary_counter(ranks), opik.tree_f32(leaves))
