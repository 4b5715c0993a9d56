"""GPU K-leaf GEMM (gdn_pik_gemm) against the oracle (oracle/pik.py).

Parity: C against the float64 product A B^T within the float32 error bound of
a sum of K/16 tensor-core steps and the log2(L) tree levels.  Bitwise: the
same C for every number of emulated ranks; C equal to the oracle's float32
tree over the leaves computed one at a time; repeated runs identical.
"""
import numpy as np
import pytest
import torch

from oracle import pik as opik

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gdn():
    from rl_train_numerics_b200 import _abi
    return _abi


def operands(M, N, K, seed):
    gen = torch.Generator().manual_seed(seed)
    A = torch.randn((M, K), generator=gen).to(torch.bfloat16)
    B = torch.randn((N, K), generator=gen).to(torch.bfloat16)
    return A, B


def bound(A, B, L):
    """Float32 bound: each of the K/16 accumulation steps of a leaf and each of
    the log2(L) tree levels rounds once (relative 2^-24 of at most the running
    magnitude, itself at most sum |a||b|); factor 2 for the tensor core's own
    rounding inside a step."""
    a = np.abs(A.double().numpy())
    b = np.abs(B.double().numpy())
    K = A.shape[1]
    steps = K // 16 + int(np.log2(L)) + 2
    return 2 * steps * 2.0 ** -24 * (a @ b.T)


@pytest.mark.parametrize("L", [1, 2, 4, 8, 16])
def test_matches_the_product_within_the_float32_bound(gdn, L):
    M, N, K = 300, 272, 1024  # ragged M; N not a multiple of the tile width
    A, B = operands(M, N, K, 40 + L)
    C, err = gdn.pik_gemm(A.cuda(), B.cuda(), L)
    assert gdn.check_error(err) == 0
    ref = opik.gemm_fp64(A.double().numpy(), B.double().numpy())
    got = C.double().cpu().numpy()
    assert np.all(np.abs(got - ref) <= bound(A, B, L))


def test_same_bits_for_every_rank_count(gdn):
    """L = 16 leaves: 1, 2, 4, 8 and 16 emulated ranks (blocks of 2 leaves with 8 group
    sums combined, down to blocks of 1 leaf with 16)."""
    M, N, K = 256, 320, 16 * 128
    A, B = operands(M, N, K, 50)
    A, B = A.cuda(), B.cuda()
    ref, err = gdn.pik_gemm(A, B, 16, 1)
    for R in (2, 4, 8, 16):
        C, err2 = gdn.pik_gemm(A, B, 16, R)
        assert torch.equal(C, ref), R
        assert gdn.check_error(err2) == 0
    assert gdn.check_error(err) == 0


@pytest.mark.parametrize("L", [2, 8])
def test_leaves_one_at_a_time_then_the_oracle_tree(gdn, L):
    """Each leaf computed alone (its K slice as a one-leaf GEMM), combined by the
    oracle's float32 tree, gives the L-leaf result bit for bit."""
    M, N, K = 200, 256, L * 256
    A, B = operands(M, N, K, 60 + L)
    Ad, Bd = A.cuda(), B.cuda()
    C, err = gdn.pik_gemm(Ad, Bd, L)
    parts = []
    for k0, k1 in opik.leaf_bounds(K, L):
        P, e = gdn.pik_gemm(Ad[:, k0:k1].contiguous(), Bd[:, k0:k1].contiguous(), 1)
        assert gdn.check_error(e) == 0
        parts.append(P.cpu().numpy())
    want = opik.tree_f32(parts)
    assert np.array_equal(C.cpu().numpy(), want)
    assert gdn.check_error(err) == 0


def test_one_leaf_is_a_plain_gemm(gdn):
    M, N, K = 512, 512, 4096
    A, B = operands(M, N, K, 70)
    A, B = A.cuda(), B.cuda()
    C, err = gdn.pik_gemm(A, B, 1)
    assert gdn.check_error(err) == 0
    ref = A.double() @ B.double().T
    rel = ((C.double() - ref).abs().max() / ref.abs().max()).item()
    assert rel < 1e-5


def test_repeat_runs_are_identical_and_empty_k_is_zero(gdn):
    M, N, K = 384, 256, 2048
    A, B = operands(M, N, K, 80)
    A, B = A.cuda(), B.cuda()
    first, _ = gdn.pik_gemm(A, B, 4)
    for _ in range(2):
        again, _ = gdn.pik_gemm(A, B, 4)
        assert torch.equal(first, again)
    C = torch.full((M, N), 7.0, device="cuda")
    gdn.pik_gemm(A[:, :0].contiguous(), B[:, :0].contiguous(), 4, C=C)
    assert torch.count_nonzero(C) == 0
