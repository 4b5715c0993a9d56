"""GPU forward (gdn_cpr_forward, gdn_chunk_boundary) against the fp64 oracle.

Parity bar: tests/gdn_testlib.py (1e-5 x RMS for fp32 inputs, 2e-3 x RMS for
bf16 inputs, on the fp32-output mode).  Bitwise checks: bf16 output equals the
round-to-nearest-even of the fp32 output; repeated runs are identical;
gdn_chunk_boundary equals the forward's first-pass boundary states.
"""
import numpy as np
import pytest
import torch

from rl_train_numerics_b200 import workloads as W
from tests.gdn_testlib import (canaries_intact, guarded, oracle_prefix_state, oracle_unit,
                               rel_err, tol_for)

pytestmark = pytest.mark.gpu
C = 64


@pytest.fixture(scope="module")
def gdn():
    from rl_train_numerics_b200 import _abi
    return _abi


def run(gdn, b, **kw):
    o, srun, sbnd, ws = gdn.forward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens, **kw)
    assert gdn.check_error(ws) == 0
    return o, srun, sbnd


def check_units(gdn, bcpu, o, srun, sbnd, units, h0=None):
    tol = tol_for(bcpu.q.dtype)
    cu = bcpu.cu_seqlens.tolist()
    for n, h in units:
        L = cu[n + 1] - cu[n]
        o_ref, s_ref = oracle_unit(bcpu, n, h, h0=h0)
        if L:
            assert rel_err(o[cu[n]:cu[n + 1], h], o_ref) <= tol, (n, h, L)
        assert rel_err(srun[n, h], s_ref) <= tol, ("s_run_final", n, h, L)
        nf = (L // C) * C
        s_b = s_ref if nf == L else oracle_prefix_state(bcpu, n, h, nf, h0=h0)
        if np.any(s_b):
            assert rel_err(sbnd[n, h], s_b) <= tol, ("s_bnd_final", n, h, L)
        else:
            assert torch.count_nonzero(sbnd[n, h]) == 0


def test_tiny_fp32(gdn):
    """1 sequence, T=256, H=2, d=64, fp32 inputs: 1e-5 x RMS."""
    b = W.tiny()
    o, srun, sbnd = run(gdn, b.to("cuda"), out_dtype=torch.float32)
    check_units(gdn, b, o, srun, sbnd, [(0, 0), (0, 1)])
    assert torch.equal(srun, sbnd)  # length is a multiple of C


@pytest.mark.parametrize("d,dtype", [(128, torch.bfloat16), (64, torch.bfloat16),
                                     (64, torch.float32)])
def test_ragged_lengths(gdn, d, dtype):
    """Lengths around the chunk size, empty sequences, several tiles and a ragged tail."""
    lens = [1, 63, 64, 65, 200, 0, 130, 7, 128]
    b = W.make_batch(lens, 3, d, d, dtype=dtype, seed=11)
    o, srun, sbnd = run(gdn, b.to("cuda"), out_dtype=torch.float32)
    check_units(gdn, b, o, srun, sbnd, [(n, h) for n in range(len(lens)) for h in range(3)])


def test_initial_state_and_scale(gdn):
    lens = [100, 64, 3]
    b = W.make_batch(lens, 2, 128, 128, dtype=torch.bfloat16, seed=12)
    h0 = torch.randn((3, 2, 128, 128), generator=torch.Generator().manual_seed(5)) * 0.2
    o, srun, sbnd = run(gdn, b.to("cuda"), out_dtype=torch.float32, h0=h0.cuda(), scale=0.5)
    cu = b.cu_seqlens.tolist()
    for n in range(3):
        for h in range(2):
            o_ref, s_ref = oracle_unit(b, n, h, h0=h0, scale=0.5)
            assert rel_err(o[cu[n]:cu[n + 1], h], o_ref) <= 2e-3
            assert rel_err(srun[n, h], s_ref) <= 2e-3


def test_bf16_output_is_rounded_fp32(gdn):
    b = W.make_batch([300, 64, 17], 4, 128, 128, seed=13).to("cuda")
    o32, _, _ = run(gdn, b, out_dtype=torch.float32)
    o16, _, _ = run(gdn, b, out_dtype=torch.bfloat16)
    assert torch.equal(o16, o32.to(torch.bfloat16))


def test_repeat_runs_are_identical(gdn):
    b = W.make_batch([500, 129, 64], 4, 128, 128, seed=14).to("cuda")
    first = run(gdn, b)
    for _ in range(2):
        again = run(gdn, b)
        for x, y in zip(first, again):
            assert torch.equal(x, y)


def test_prefill_shape_sampled(gdn):
    """5 x 2048 packed, H=16, d=128, bf16: sampled (sequence, head) units."""
    b = W.prefill()
    o, srun, sbnd = run(gdn, b.to("cuda"), out_dtype=torch.float32)
    check_units(gdn, b, o, srun, sbnd, [(0, 0), (2, 7), (4, 15)])


def test_trainer_shape_sampled(gdn):
    """10240 tokens as 5 documents (Dirichlet lengths), H=16, d=128, bf16."""
    b = W.trainer()
    assert b.total_tokens == 10240 and min(b.lengths) >= 256
    o, srun, sbnd = run(gdn, b.to("cuda"), out_dtype=torch.float32)
    check_units(gdn, b, o, srun, sbnd, [(0, 3), (1, 0), (3, 9), (4, 15)])


def test_canaries_untouched(gdn):
    lens = [70, 0, 64, 5]
    b = W.make_batch(lens, 2, 128, 128, seed=15)
    bd = b.to("cuda")
    ob, o = guarded((b.total_tokens, 2, 128), torch.float32)
    rb, sr = guarded((4, 2, 128, 128), torch.float32)
    bb, sb = guarded((4, 2, 128, 128), torch.float32)
    run(gdn, bd, o=o, s_run_final=sr, s_bnd_final=sb)
    assert canaries_intact(ob) and canaries_intact(rb) and canaries_intact(bb)
    check_units(gdn, b, o, sr, sb, [(n, h) for n in range(4) for h in range(2)])


def test_all_empty_sequences_return_h0(gdn):
    h0 = torch.randn((3, 2, 64, 64), device="cuda")
    z = torch.zeros((0, 2, 64), dtype=torch.bfloat16, device="cuda")
    zb = torch.zeros((0, 2), device="cuda")
    cu = torch.zeros(4, dtype=torch.int32, device="cuda")
    o, srun, sbnd, ws = gdn.forward(z, z, z, zb, zb, cu, h0=h0)
    assert gdn.check_error(ws) == 0
    assert torch.equal(srun, h0) and torch.equal(sbnd, h0)


def test_bad_cu_seqlens_sets_device_error(gdn):
    b = W.make_batch([64, 64], 2, 64, 64, seed=16).to("cuda")
    bad = torch.tensor([0, 100, 64], dtype=torch.int32, device="cuda")  # decreasing
    o = torch.full((128, 2, 64), 7.0, dtype=torch.float32, device="cuda")
    _, _, _, ws = gdn.forward(b.q, b.k, b.v, b.beta, b.g, bad, o=o)
    assert gdn.check_error(ws) == gdn.GDN_DEVERR_CU_SEQLENS
    assert bool((o == 7.0).all())  # nothing was written
    # the error word was cleared; a good call on the same workspace succeeds
    gdn.forward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens, workspace=ws)
    assert gdn.check_error(ws) == 0


@pytest.mark.parametrize("d,dtype", [(128, torch.bfloat16), (64, torch.float32)])
def test_chunk_boundary_matches_forward_bits(gdn, d, dtype):
    """gdn_chunk_boundary(S, chunk) == the forward's boundary state after that chunk."""
    B, H = 3, 2
    b = W.make_batch([C] * B, H, d, d, dtype=dtype, seed=17)
    S = torch.randn((B, H, d, d), generator=torch.Generator().manual_seed(9)) * 0.1
    bd = b.to("cuda")
    _, _, sbnd = run(gdn, bd, h0=S.cuda())
    kc = bd.k.view(B, C, H, d).transpose(1, 2).contiguous()
    vc = bd.v.view(B, C, H, d).transpose(1, 2).contiguous()
    bc = bd.beta.view(B, C, H).transpose(1, 2).contiguous()
    gc = bd.g.view(B, C, H).transpose(1, 2).contiguous()
    out = gdn.chunk_boundary(S.cuda(), kc, vc, bc, gc)
    assert torch.equal(out, sbnd)
    for n in range(B):
        for h in range(H):
            _, s_ref = oracle_unit(b, n, h, h0=S)
            assert rel_err(out[n, h], s_ref) <= tol_for(dtype)
    # in place
    S2 = S.cuda().clone()
    gdn.chunk_boundary(S2, kc, vc, bc, gc, s_end=S2)
    assert torch.equal(S2, out)


def test_running_state_pair(gdn):
    """With s_run_scale the forward returns (mantissa, scale); scale x mantissa,
    rounded once, is bit for bit the state returned without it."""
    lens = [100, 64, 1, 190]
    b = W.make_batch(lens, 4, 128, 128, seed=18).to("cuda")
    _, s_state, _ = run(gdn, b)
    scale = torch.full((4, 4), float("nan"), device="cuda")
    _, s_mant, _ = run(gdn, b, s_run_scale=scale)
    assert torch.isfinite(scale).all()
    assert torch.equal(scale[1], torch.ones(4, device="cuda"))  # chunk-aligned end
    assert torch.equal(scale[:, :, None, None] * s_mant, s_state)


def test_hard_reset_tokens(gdn):
    """g = -1e4 makes exp(g) exactly 0 (a reset) at scattered tokens; long decays
    (g = -8 runs) force the scaled state to renormalise many times."""
    lens = [200, 64, 77]
    b = W.make_batch(lens, 2, 128, 128, seed=19)
    gen = torch.Generator().manual_seed(20)
    pick = torch.rand(b.g.shape, generator=gen)
    g = torch.where(pick < 0.03, torch.full_like(b.g, -1e4), b.g)
    g = torch.where((pick >= 0.03) & (pick < 0.3), torch.full_like(b.g, -8.0), g)
    b = W.Batch(b.q, b.k, b.v, b.beta, g.contiguous(), b.cu_seqlens, b.lengths)
    o, srun, sbnd = run(gdn, b.to("cuda"), out_dtype=torch.float32)
    check_units(gdn, b, o, srun, sbnd, [(n, h) for n in range(3) for h in range(2)])


def test_more_sequences_than_table_threads(gdn):
    """1500 sequences (more than the chunk table's 1024 threads, so each of its
    threads takes several sequences when it orders them and lays out the fill
    order), lengths 0..299 with every seventh empty, unequal chunk counts (the
    fill starts each unit once its walk has ended): each sequence's bits are
    those of a shuffled batch, and sampled units match the oracle."""
    rng = np.random.default_rng(41)
    lens = [int(x) for x in rng.integers(0, 300, size=1500)]
    for i in range(0, len(lens), 7):
        lens[i] = 0
    H, d = 2, 128
    bcpu = W.make_batch(lens, H, d, d, dtype=torch.bfloat16, seed=42)
    b = bcpu.to("cuda")
    o, srun, sbnd = run(gdn, b, out_dtype=torch.float32)
    perm = rng.permutation(len(lens)).tolist()
    bs = b.select(perm)
    o2, srun2, sbnd2 = run(gdn, bs, out_dtype=torch.float32)
    cu, cu2 = b.cu_seqlens.tolist(), bs.cu_seqlens.tolist()
    for i, n in enumerate(perm):
        assert torch.equal(o2[cu2[i]:cu2[i + 1]], o[cu[n]:cu[n + 1]]), ("shuffled", n)
        assert torch.equal(srun2[i], srun[n]) and torch.equal(sbnd2[i], sbnd[n]), n
    picks = [int(x) for x in rng.choice(len(lens), size=6, replace=False)]
    check_units(gdn, bcpu, o.cpu(), srun.cpu(), sbnd.cpu(), [(n, n % H) for n in picks])
