"""GPU checks of the recurrent-everywhere layer (gdn_recurrent_forward,
gdn_recurrent_decode_step).

The per-layer table of "NovaSky's IsoExec Fixes the Hidden Math Bug
Corrupting AI Training Runs" (section "Solving the linear-attention
headache") compares CPR with a layout that runs the per-token recurrence for
training, prefill and decode alike.  Here it is the CPR fill's step run from
h0 over whole sequences, so:
  * outputs and final states match the fp64 oracle within the forward's
    bounds (tests/gdn_testlib.py);
  * the first 64 tokens of every sequence equal gdn_cpr_forward's bit for bit;
  * prefix forward + recurrent decode steps equal the forward over all tokens
    bit for bit (outputs, final mantissa and scale);
  * results do not depend on batch composition or order.
"""
import numpy as np
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


def recur(gdn, b, **kw):
    o, s, sc, err = gdn.recurrent_forward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens, **kw)
    assert gdn.check_error(err) == 0
    return o, s, sc


def check_vs_oracle(b, o, s, units, h0=None, scale=1.0):
    tol = tol_for(b.q.dtype)
    cu = b.cu_seqlens.tolist()
    for n, h in units:
        o_ref, s_ref = oracle_unit(b, n, h, h0=h0, scale=scale)
        if cu[n + 1] > cu[n]:
            assert rel_err(o[cu[n]:cu[n + 1], h], o_ref) <= tol, (n, h)
        assert rel_err(s[n, h], s_ref) <= tol, ("s_final", n, h)


def test_tiny_fp32(gdn):
    b = W.tiny()
    o, s, _ = recur(gdn, b.to("cuda"), out_dtype=torch.float32)
    check_vs_oracle(b, o, s, [(0, 0), (0, 1)])


@pytest.mark.parametrize("d,dtype", [(128, torch.bfloat16), (64, torch.bfloat16),
                                     (64, torch.float32)])
def test_ragged_lengths(gdn, d, dtype):
    """Empty, short, tile-sized and multi-tile sequences with ragged tails."""
    lens = [1, 31, 32, 33, 200, 0, 130, 7, 64, 97]
    b = W.make_batch(lens, 3, d, d, dtype=dtype, seed=21)
    o, s, _ = recur(gdn, b.to("cuda"), out_dtype=torch.float32)
    check_vs_oracle(b, o, s, [(n, h) for n in range(len(lens)) for h in range(3)])


def test_initial_state_scale_and_bf16_output(gdn):
    lens = [100, 64, 3]
    b = W.make_batch(lens, 2, 128, 128, dtype=torch.bfloat16, seed=22)
    h0 = torch.randn((3, 2, 128, 128), generator=torch.Generator().manual_seed(6)) * 0.2
    bg = b.to("cuda")
    o, s, _ = recur(gdn, bg, out_dtype=torch.float32, h0=h0.cuda(), scale=0.5)
    check_vs_oracle(b, o, s, [(n, h) for n in range(3) for h in range(2)], h0=h0, scale=0.5)
    o16, _, _ = recur(gdn, bg, out_dtype=torch.bfloat16, h0=h0.cuda(), scale=0.5)
    assert torch.equal(o16, o.to(torch.bfloat16))


def test_prefill_shape_sampled(gdn):
    """5 x 2048 tokens, H=16, d=128, bf16: sampled (sequence, head) units."""
    b = W.prefill()
    o, s, _ = recur(gdn, b.to("cuda"), out_dtype=torch.float32)
    check_vs_oracle(b, o, s, [(0, 0), (2, 7), (4, 15)])


@pytest.mark.parametrize("use_h0", [False, True])
def test_first_chunk_is_bitwise_the_cpr_forward(gdn, use_h0):
    lens = [300, 64, 130, 5, 0, 2048]
    b = W.make_batch(lens, 4, 128, 128, dtype=torch.bfloat16, seed=23).to("cuda")
    h0 = None
    if use_h0:
        h0 = (torch.randn((len(lens), 4, 128, 128), generator=torch.Generator().manual_seed(7))
              * 0.3).cuda()
    o_r, _, _ = recur(gdn, b, out_dtype=torch.float32, h0=h0)
    o_c, _, _, ws = gdn.forward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens,
                                out_dtype=torch.float32, h0=h0)
    assert gdn.check_error(ws) == 0
    cu = b.cu_seqlens.tolist()
    for n, L in enumerate(lens):
        m = min(L, C)
        assert torch.equal(o_r[cu[n]:cu[n] + m], o_c[cu[n]:cu[n] + m]), n
    # beyond the first chunk CPR restarts from the boundary state: equal
    # within the bound, not bit for bit
    n = lens.index(2048)
    assert not torch.equal(o_r[cu[n]:cu[n + 1]], o_c[cu[n]:cu[n + 1]])


@pytest.mark.parametrize("d,dtype", [(128, torch.bfloat16), (64, torch.float32)])
def test_prefix_then_decode_is_bitwise_the_forward(gdn, d, dtype):
    """Forward over prefixes (mantissa + scale out), then the same number of
    recurrent decode steps for every sequence == forward over all tokens."""
    H, steps = 4, 150
    prefix = [1, 63, 64, 65, 700, 2000]
    full = [p + steps for p in prefix]
    b = W.make_batch(full, H, d, d, dtype=dtype, seed=24, g_mode="stress").to("cuda")
    o_all, s_all, sc_all = recur(gdn, b, out_dtype=torch.float32,
                                 s_final_scale=torch.empty((len(full), H), device="cuda"))
    cu = b.cu_seqlens.tolist()
    pre_idx = torch.cat([torch.arange(cu[n], cu[n] + prefix[n]) for n in range(len(full))]).cuda()
    pb = W.Batch(b.q[pre_idx], b.k[pre_idx], b.v[pre_idx], b.beta[pre_idx], b.g[pre_idx],
                 W.cu_seqlens_of(prefix, "cuda"), prefix)
    o_pre, s, sc = recur(gdn, pb, out_dtype=torch.float32,
                         s_final_scale=torch.empty((len(full), H), device="cuda"))
    cup = pb.cu_seqlens.tolist()
    for n in range(len(full)):
        assert torch.equal(o_pre[cup[n]:cup[n + 1]], o_all[cu[n]:cu[n] + prefix[n]]), n
    base = torch.tensor([cu[n] + prefix[n] for n in range(len(full))], device="cuda")
    for j in range(steps):
        t = base + j
        o = gdn.recurrent_decode_step(b.q[t], b.k[t], b.v[t], b.beta[t], b.g[t], s, sc,
                                      out_dtype=torch.float32)
        assert torch.equal(o, o_all[t]), j
    assert torch.equal(s, s_all) and torch.equal(sc, sc_all)


def test_batch_invariance(gdn):
    b = W.make_batch([5, 700, 64, 1, 129, 0, 2000, 33], 3, 128, 128, dtype=torch.bfloat16,
                     seed=25).to("cuda")
    o, s, _ = recur(gdn, b, out_dtype=torch.float32)
    cu = b.cu_seqlens.tolist()
    order = [6, 0, 3, 7, 1, 5, 2, 4]
    bs = b.select(order)
    o2, s2, _ = recur(gdn, bs, out_dtype=torch.float32)
    cu2 = bs.cu_seqlens.tolist()
    for i, n in enumerate(order):
        assert torch.equal(o2[cu2[i]:cu2[i + 1]], o[cu[n]:cu[n + 1]]), n
        assert torch.equal(s2[i], s[n]), n
    for n in (1, 6):
        b1 = b.select([n])
        o1, s1, _ = recur(gdn, b1, out_dtype=torch.float32)
        assert torch.equal(o1, o[cu[n]:cu[n + 1]]) and torch.equal(s1[0], s[n])


def test_bad_cu_seqlens_sets_the_error_word(gdn):
    b = W.make_batch([10, 20], 2, 64, 64, dtype=torch.bfloat16, seed=26).to("cuda")
    bad = torch.tensor([0, 25, 20], dtype=torch.int32, device="cuda")  # decreasing
    _, _, _, err = gdn.recurrent_forward(b.q, b.k, b.v, b.beta, b.g, bad)
    torch.cuda.synchronize()
    assert int(err.item()) & gdn.GDN_DEVERR_CU_SEQLENS
    # the next good call clears it
    _, _, _, err = gdn.recurrent_forward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens, error=err)
    assert gdn.check_error(err) == 0


def test_empty_batch(gdn):
    z = torch.zeros((0, 2, 64), dtype=torch.bfloat16, device="cuda")
    zf = torch.zeros((0, 2), device="cuda")
    cu = torch.zeros(1, dtype=torch.int32, device="cuda")
    err = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    gdn.recurrent_forward(z, z, z, zf, zf, cu, n_seqs=0, want_state=False, error=err)
    assert gdn.check_error(err) == 0
