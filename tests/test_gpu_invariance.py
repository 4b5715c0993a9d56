"""Batch invariance on the stress workload.

64 ragged sequences (log-uniform lengths in [1, 8192]), H=32, d=128, bf16,
log-decays with near-0 and near-(-8) tails.  Every sequence's output bits
must be the same whether it runs in the whole batch, in a shuffled batch,
alone, or padded between empty sequences; the same holds for 128 decode
steps continued from each mode's handoff, run as a whole batch and as a
reversed subset.  Sampled units are also checked against the fp64 oracle.
"""
import pytest
import torch

from rl_train_numerics_b200 import workloads as W
from tests.gdn_testlib import oracle_unit, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gdn():
    from rl_train_numerics_b200 import _abi
    return _abi


@pytest.fixture(scope="module")
def stress():
    return W.stress()


def forward(gdn, b, **kw):
    o, srun, sbnd, ws = gdn.forward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens,
                                    out_dtype=torch.float32, **kw)
    assert gdn.check_error(ws) == 0
    return o, srun, sbnd


def per_seq(o, b):
    cu = b.cu_seqlens.tolist()
    return [o[cu[n]:cu[n + 1]] for n in range(len(b.lengths))]


def test_forward_batch_invariance(gdn, stress):
    b = stress.to("cuda")
    n = len(b.lengths)
    o, srun, sbnd = forward(gdn, b)
    whole = per_seq(o, b)

    perm = torch.randperm(n, generator=torch.Generator().manual_seed(31)).tolist()
    bs = b.select(perm)
    o2, srun2, sbnd2 = forward(gdn, bs)
    for i, s in enumerate(per_seq(o2, bs)):
        assert torch.equal(s, whole[perm[i]]), ("shuffled", perm[i])
        assert torch.equal(srun2[i], srun[perm[i]]) and torch.equal(sbnd2[i], sbnd[perm[i]])

    for i in range(n):
        bi = b.select([i])
        oi, ri, bi_ = forward(gdn, bi)
        assert torch.equal(oi, whole[i]), ("alone", i)
        assert torch.equal(ri[0], srun[i]) and torch.equal(bi_[0], sbnd[i])

    # padded: an empty sequence between every pair
    lens = []
    for L in b.lengths:
        lens += [0, L]
    lens.append(0)
    pad = W.Batch(b.q, b.k, b.v, b.beta, b.g, W.cu_seqlens_of(lens, "cuda"), lens)
    op, rp, bp = forward(gdn, pad)
    cu = pad.cu_seqlens.tolist()
    for i in range(n):
        j = 2 * i + 1
        assert torch.equal(op[cu[j]:cu[j + 1]], whole[i]), ("padded", i)
        assert torch.equal(rp[j], srun[i])


def test_stress_parity_sampled(gdn, stress):
    b = stress
    o, srun, _ = forward(gdn, b.to("cuda"))
    lens = b.lengths
    longest = max(range(len(lens)), key=lambda i: lens[i])
    shortest = min(range(len(lens)), key=lambda i: lens[i])
    cu = b.cu_seqlens.tolist()
    for n, h in [(longest, 0), (longest, 31), (shortest, 5), (7, 12)]:
        o_ref, s_ref = oracle_unit(b, n, h)
        if lens[n]:
            assert rel_err(o[cu[n]:cu[n + 1], h], o_ref) <= 2e-3, (n, h)
        assert rel_err(srun[n, h], s_ref) <= 2e-3


def test_decode_batch_invariance(gdn, stress):
    """128 decode steps continued from each forward mode's own handoff (whole
    batch, shuffled batch, one sequence at a time, padded between empty
    sequences), each with that mode's running-state pair and boundary state:
    every slot's decode outputs and states are bit-identical across the modes,
    and also when the whole-batch state is decoded as a reversed subset."""
    b = stress.to("cuda")
    n = len(b.lengths)
    H = b.q.shape[1]
    steps = 128
    toks = W.decode_tokens(steps, n, H, 128, 128, seed=33, g_mode="stress", device="cuda")

    def handoff(batch, slots, n_slots):
        """Forward over `batch`, then its handoff into `n_slots` slots (sequence i
        of the batch goes to slot slots[i])."""
        N = len(batch.lengths)
        sscale = torch.empty((N, H), device="cuda")
        _, srun, sbnd = forward(gdn, batch, s_run_scale=sscale)
        st = gdn.DecodeState(n_slots, H, 128, 128)
        gdn.decode_state_from_prefill(st, batch.k, batch.v, batch.beta, batch.g,
                                      batch.cu_seqlens, srun, sbnd, s_run_scale=sscale,
                                      slot_idx=torch.tensor(slots, dtype=torch.int32,
                                                            device="cuda"))
        return st

    def decode(st, order):
        slots = torch.tensor(order, dtype=torch.int32, device="cuda")
        r = torch.tensor(order, device="cuda")
        outs = []
        for s in range(steps):
            q, k, v, beta, g = (t[s][r].contiguous() for t in toks)
            outs.append(gdn.decode_step(st, q, k, v, beta, g, slot_idx=slots,
                                        out_dtype=torch.float32))
        assert gdn.check_error(st.error) == 0
        return torch.stack(outs)

    every = list(range(n))
    # whole batch
    st_whole = handoff(b, every, n)
    st_sub = st_whole.clone()
    o_whole = decode(st_whole, every)
    states = {"whole": st_whole}
    outs = {}
    # shuffled batch: sequence i of the shuffled batch is original perm[i]
    perm = torch.randperm(n, generator=torch.Generator().manual_seed(31)).tolist()
    st = handoff(b.select(perm), perm, n)
    outs["shuffled"], states["shuffled"] = decode(st, every), st
    # one sequence at a time, each handed off into its own slot of one state
    st = gdn.DecodeState(n, H, 128, 128)
    for i in range(n):
        bi = b.select([i])
        sscale = torch.empty((1, H), device="cuda")
        _, srun, sbnd = forward(gdn, bi, s_run_scale=sscale)
        gdn.decode_state_from_prefill(st, bi.k, bi.v, bi.beta, bi.g, bi.cu_seqlens, srun, sbnd,
                                      s_run_scale=sscale,
                                      slot_idx=torch.tensor([i], dtype=torch.int32,
                                                            device="cuda"))
    outs["alone"], states["alone"] = decode(st, every), st
    # padded: an empty sequence before, between and after the real ones; the
    # empty ones are handed off into extra slots n .. 2n
    lens, slots = [], []
    for i, L in enumerate(b.lengths):
        lens += [0, L]
        slots += [n + i, i]
    lens.append(0)
    slots.append(2 * n)
    pad = W.Batch(b.q, b.k, b.v, b.beta, b.g, W.cu_seqlens_of(lens, "cuda"), lens)
    st = handoff(pad, slots, 2 * n + 1)
    outs["padded"], states["padded"] = decode(st, every), st

    for mode, o in outs.items():
        assert torch.equal(o, o_whole), mode
        for name in ("s_run", "s_scale", "s_bnd", "pos"):
            a = getattr(states[mode], name)[:n]
            assert torch.equal(a, getattr(st_whole, name)), (mode, name)

    sub = list(reversed(range(0, n, 3)))
    o_sub = decode(st_sub, sub)
    for j, i in enumerate(sub):
        assert torch.equal(o_sub[:, j], o_whole[:, i]), i
        assert torch.equal(st_sub.s_bnd[i], st_whole.s_bnd[i])
