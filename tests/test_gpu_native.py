"""GPU checks of the chunked ("native mixed") forward, gdn_native_forward.

The per-layer table of "NovaSky's IsoExec Fixes the Hidden Math Bug
Corrupting AI Training Runs" (section "Solving the linear-attention
headache") compares CPR with the usual layout, whose prefill evaluates
chunks with the UT / WY products (fast, but rounded differently from
decode).  Here it shares CPR's first pass and replaces the per-token fill by
tensor-core products, so:
  * outputs and final states match the fp64 oracle within the bf16-input
    bound of tests/gdn_testlib.py;
  * the last boundary state is bitwise gdn_cpr_forward's;
  * the outputs are NOT bitwise CPR's (nor the recurrent decode's), which is
    the rounding mismatch the pages describe, but agree within the bound;
  * results do not depend on batch composition or order.
"""
import pytest
import torch

from rl_train_numerics_b200 import workloads as W
from tests.gdn_testlib import oracle_unit, rel_err, tol_for

pytestmark = pytest.mark.gpu
C = 64


@pytest.fixture(scope="module")
def gdn():
    from rl_train_numerics_b200 import _abi
    return _abi


def native(gdn, b, **kw):
    o, s, sb, ws = gdn.native_forward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens, **kw)
    assert gdn.check_error(ws) == 0
    return o, s, sb


def check_vs_oracle(b, o, s, units, h0=None, scale=1.0):
    tol = tol_for(b.q.dtype)
    cu = b.cu_seqlens.tolist()
    for n, h in units:
        o_ref, s_ref = oracle_unit(b, n, h, h0=h0, scale=scale)
        if cu[n + 1] > cu[n]:
            assert rel_err(o[cu[n]:cu[n + 1], h], o_ref) <= tol, (n, h)
        assert rel_err(s[n, h], s_ref) <= tol, ("s_final", n, h)


@pytest.mark.parametrize("g_mode", ["softplus", "stress"])
def test_ragged_lengths(gdn, g_mode):
    """Empty, short, chunk-sized and multi-chunk sequences with ragged tails."""
    lens = [1, 63, 64, 65, 200, 0, 130, 7, 128, 300]
    b = W.make_batch(lens, 3, 128, 128, dtype=torch.bfloat16, seed=31, g_mode=g_mode)
    o, s, sb = native(gdn, b.to("cuda"), out_dtype=torch.float32)
    check_vs_oracle(b, o, s, [(n, h) for n in range(len(lens)) for h in range(3)])


def test_initial_state_scale_and_bf16_output(gdn):
    lens = [100, 64, 3, 257]
    b = W.make_batch(lens, 2, 128, 128, dtype=torch.bfloat16, seed=32)
    h0 = torch.randn((4, 2, 128, 128), generator=torch.Generator().manual_seed(8)) * 0.2
    bg = b.to("cuda")
    o, s, _ = native(gdn, bg, out_dtype=torch.float32, h0=h0.cuda(), scale=0.5)
    check_vs_oracle(b, o, s, [(n, h) for n in range(4) for h in range(2)], h0=h0, scale=0.5)
    o16, _, _ = native(gdn, bg, out_dtype=torch.bfloat16, h0=h0.cuda(), scale=0.5)
    assert torch.equal(o16, o.to(torch.bfloat16))


def test_prefill_shape_sampled(gdn):
    """5 x 2048 tokens, H=16, d=128, bf16: sampled (sequence, head) units."""
    b = W.prefill()
    o, s, _ = native(gdn, b.to("cuda"), out_dtype=torch.float32)
    check_vs_oracle(b, o, s, [(0, 0), (2, 7), (4, 15)])


def test_trainer_shape_sampled(gdn):
    """10240 tokens in 5 ragged documents, H=16: sampled units."""
    b = W.trainer()
    o, s, _ = native(gdn, b.to("cuda"), out_dtype=torch.float32)
    check_vs_oracle(b, o, s, [(0, 3), (3, 9), (4, 0)])


def test_shares_the_first_pass_but_not_the_output_bits(gdn):
    b = W.make_batch([300, 64, 130, 2048], 4, 128, 128, dtype=torch.bfloat16,
                     seed=33).to("cuda")
    o_n, s_n, sb_n = native(gdn, b, out_dtype=torch.float32)
    o_c, s_c, sb_c, ws = gdn.forward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens,
                                     out_dtype=torch.float32)
    assert gdn.check_error(ws) == 0
    assert torch.equal(sb_n, sb_c)  # the same boundary walk
    assert torch.equal(s_n[1], s_c[1])  # length 64: the final state is that boundary
    assert not torch.equal(o_n, o_c)
    tol = tol_for(torch.bfloat16)
    ref = o_c.double()
    err = (o_n.double() - ref).abs().max() / ref.pow(2).mean().sqrt()
    assert float(err) <= tol


def test_batch_invariance(gdn):
    b = W.make_batch([5, 700, 64, 1, 129, 0, 2000, 33], 3, 128, 128, dtype=torch.bfloat16,
                     seed=34).to("cuda")
    o, s, sb = native(gdn, b, out_dtype=torch.float32)
    cu = b.cu_seqlens.tolist()
    order = [6, 0, 3, 7, 1, 5, 2, 4]
    bs = b.select(order)
    o2, s2, sb2 = native(gdn, bs, out_dtype=torch.float32)
    cu2 = bs.cu_seqlens.tolist()
    for i, n in enumerate(order):
        assert torch.equal(o2[cu2[i]:cu2[i + 1]], o[cu[n]:cu[n + 1]]), n
        assert torch.equal(s2[i], s[n]) and torch.equal(sb2[i], sb[n]), n
    b1 = b.select([6])
    o1, s1, _ = native(gdn, b1, out_dtype=torch.float32)
    assert torch.equal(o1, o[cu[6]:cu[7]]) and torch.equal(s1[0], s[6])


def test_bad_cu_seqlens_sets_the_error_word(gdn):
    b = W.make_batch([10, 20], 2, 128, 128, dtype=torch.bfloat16, seed=35).to("cuda")
    bad = torch.tensor([0, 25, 20], dtype=torch.int32, device="cuda")
    _, _, _, ws = gdn.native_forward(b.q, b.k, b.v, b.beta, b.g, bad)
    assert gdn.check_error(ws) & gdn.GDN_DEVERR_CU_SEQLENS
