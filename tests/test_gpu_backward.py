"""GPU backward (gdn_cpr_backward) against the fp64 oracle's reverse mode.

Every gradient (dq, dk, dv, dbeta, dg, dh0) is compared element by element
with oracle.backward on the same inputs (bf16 inputs widened exactly), as
max|got - ref| <= tol x RMS(ref) per tensor and per (sequence, head), with
the tolerances BWD_TOL below (their reasoning beside them).  Repeated runs must
be bitwise identical (every reduction has a fixed order).
"""
import numpy as np
import pytest
import torch

import oracle
from rl_train_numerics_b200 import workloads as W
from tests.gdn_testlib import rel_err, rms

pytestmark = pytest.mark.gpu

# The backward runs in fp32 (unit roundoff u = 2^-24 = 6e-8) on inputs that
# are exact in fp32 (bf16 inputs widen exactly).  Its longest accumulations
# are the d-term dot products and the <= 64-term chunk sums, so the rounding
# error of one gradient element is a few hundred u of its terms' size; the
# boundary states it starts from carry the forward's first-pass error (three
# bf16 terms per fp32 operand for fp32 inputs, two at d = 128 with bf16
# inputs, ~2^-17 relative per product).  Hence 2e-5 (fp32 inputs) and 1e-4
# (bf16 inputs) of the reference's RMS.
BWD_TOL = {torch.float32: 2e-5, torch.bfloat16: 1e-4}
NAMES = ("dq", "dk", "dv", "dbeta", "dg", "dh0")


def scale_of(name, ref, sl, h):
    """RMS the error of one (sequence, head) is measured against.  dg_t is
    <mu_{t-1}, S_{t-1}>: exactly 0 for a sequence's first token when h0 = 0,
    yet the kernel forms it as a telescoped sum whose terms cancel, so its
    error scales with the head's typical dg, not with that value: dg uses the
    larger of the unit's and the head's RMS over the whole batch."""
    unit = rms(ref[name][sl, h])
    return max(unit, rms(ref[name][:, h])) if name == "dg" else unit


@pytest.fixture(scope="module")
def gdn():
    from rl_train_numerics_b200 import _abi
    return _abi


def _np(t):
    return t.detach().cpu().double().numpy()


def cotangents(b, H, d, seed, dtype):
    gen = torch.Generator().manual_seed(seed)
    T, N = b.total_tokens, b.n_seqs
    d_o = torch.randn((T, H, d), generator=gen).to(dtype)
    dsf = torch.randn((N, H, d, d), generator=gen) * 0.1
    return d_o, dsf


def run_both(gdn, b, d_o, dsf, h0=None, scale=1.0):
    dev = b.to("cuda")
    grads, ws = gdn.backward(dev.q, dev.k, dev.v, dev.beta, dev.g, dev.cu_seqlens, d_o.cuda(),
                             h0=None if h0 is None else h0.cuda(),
                             ds_final=None if dsf is None else dsf.cuda(), scale=scale)
    assert gdn.check_error(ws) == 0
    H, d = b.q.shape[1], b.q.shape[2]
    ref = oracle.backward(_np(b.q), _np(b.k), _np(b.v), _np(b.beta), _np(b.g),
                          b.cu_seqlens.numpy().astype(np.int32), _np(d_o),
                          h0=None if h0 is None else _np(h0),
                          ds_final=None if dsf is None else _np(dsf), scale=scale)
    return grads, ref


def check(grads, ref, b, tol, names=NAMES):
    cu = b.cu_seqlens.tolist()
    H = b.q.shape[1]
    for n in range(b.n_seqs):
        sl = slice(cu[n], cu[n + 1])
        for h in range(H):
            for name in names:
                if name == "dh0":
                    got, want = grads["dh0"][n, h], ref["dh0"][n, h]
                    den = rms(want)
                else:
                    if cu[n + 1] == cu[n]:
                        continue
                    got, want = grads[name][sl, h], ref[name][sl, h]
                    den = scale_of(name, ref, sl, h)
                err = float(np.max(np.abs(_np(got) - want))) / max(den, 1e-30)
                assert err <= tol, (name, n, h, cu[n + 1] - cu[n], err)


@pytest.mark.parametrize("d,dtype", [(128, torch.bfloat16), (64, torch.bfloat16),
                                     (64, torch.float32)])
def test_ragged_lengths(gdn, d, dtype):
    """Lengths around the chunk size, an empty sequence, several chunks and a ragged tail."""
    lens = [1, 63, 64, 65, 200, 0, 130, 7, 128]
    H = 3
    b = W.make_batch(lens, H, d, d, dtype=dtype, seed=21)
    d_o, dsf = cotangents(b, H, d, 22, dtype)
    grads, ref = run_both(gdn, b, d_o, dsf)
    check(grads, ref, b, BWD_TOL[dtype])


def test_initial_state_scale_and_no_final_cotangent(gdn):
    lens = [150, 64, 3]
    H, d = 2, 128
    b = W.make_batch(lens, H, d, d, dtype=torch.bfloat16, seed=23)
    d_o, _ = cotangents(b, H, d, 24, torch.bfloat16)
    h0 = torch.randn((3, H, d, d), generator=torch.Generator().manual_seed(25)) * 0.2
    grads, ref = run_both(gdn, b, d_o, None, h0=h0, scale=0.5)
    check(grads, ref, b, BWD_TOL[torch.bfloat16])


def test_strong_decay(gdn):
    """Decays near zero inside chunks (alpha down to ~e^-8): the chunk products'
    decay factors span many orders of magnitude."""
    lens = [300, 77]
    H, d = 2, 64
    b = W.make_batch(lens, H, d, d, dtype=torch.float32, seed=26)
    b.g.mul_(8.0)
    d_o, dsf = cotangents(b, H, d, 27, torch.float32)
    grads, ref = run_both(gdn, b, d_o, dsf)
    check(grads, ref, b, BWD_TOL[torch.float32])


def test_repeat_runs_are_identical(gdn):
    b = W.make_batch([500, 129, 64], 4, 128, 128, seed=28).to("cuda")
    d_o, dsf = cotangents(b, 4, 128, 29, torch.bfloat16)
    d_o, dsf = d_o.cuda(), dsf.cuda()
    first, ws = gdn.backward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens, d_o, ds_final=dsf)
    first = {k: v.clone() for k, v in first.items()}
    for _ in range(2):
        again, _ = gdn.backward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens, d_o, ds_final=dsf,
                                workspace=ws)
        for k in NAMES:
            assert torch.equal(first[k], again[k]), k


def test_reusing_the_forwards_first_pass_changes_no_bit(gdn):
    """forward() on the backward's workspace, then backward(reuse_forward=True):
    the same bits as a backward that runs the first pass itself, and the
    forward's outputs (written while the backward's adjoint prep may already
    run) the same bits as a forward alone."""
    b = W.make_batch([300, 64, 5, 190], 3, 128, 128, seed=32).to("cuda")
    d_o, dsf = cotangents(b, 3, 128, 33, torch.bfloat16)
    d_o, dsf = d_o.cuda(), dsf.cuda()
    h0 = (torch.randn((4, 3, 128, 128), generator=torch.Generator().manual_seed(34)) * 0.2).cuda()
    ref, _ = gdn.backward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens, d_o, ds_final=dsf, h0=h0)
    ws = torch.zeros(gdn.backward_workspace_bytes(4, b.total_tokens, 3, 128, 128),
                     dtype=torch.uint8, device="cuda")
    o, srun, _, _ = gdn.forward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens, h0=h0, workspace=ws)
    got, _ = gdn.backward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens, d_o, ds_final=dsf, h0=h0,
                          workspace=ws, reuse_forward=True)
    assert gdn.check_error(ws) == 0
    for k in NAMES:
        assert torch.equal(ref[k], got[k]), k
    o_alone, srun_alone, _, ws2 = gdn.forward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens, h0=h0)
    assert gdn.check_error(ws2) == 0
    assert torch.equal(o, o_alone) and torch.equal(srun, srun_alone)


def test_bad_cu_seqlens_sets_the_error_word(gdn):
    b = W.make_batch([64, 64], 2, 64, 64, dtype=torch.float32, seed=30).to("cuda")
    bad = torch.tensor([0, 100, 64], dtype=torch.int32, device="cuda")  # decreasing
    _, ws = gdn.backward(b.q, b.k, b.v, b.beta, b.g, bad, torch.zeros_like(b.v))
    assert gdn.check_error(ws) == gdn.GDN_DEVERR_CU_SEQLENS
    # the same workspace serves a valid call afterwards
    grads, ws = gdn.backward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens, torch.zeros_like(b.v),
                             workspace=ws)
    assert gdn.check_error(ws) == 0
    assert torch.count_nonzero(grads["dq"]) == 0 and torch.count_nonzero(grads["dh0"]) == 0


def test_full_size_sampled_units(gdn):
    """The 5 x 2048 packed batch, H = 16, d = 128, bf16, in one call; three
    (sequence, head) units checked against the oracle run on that unit alone."""
    b = W.prefill()
    H, d = 16, 128
    d_o, dsf = cotangents(b, H, d, 31, torch.bfloat16)
    dev = b.to("cuda")
    grads, ws = gdn.backward(dev.q, dev.k, dev.v, dev.beta, dev.g, dev.cu_seqlens, d_o.cuda(),
                             ds_final=dsf.cuda())
    assert gdn.check_error(ws) == 0
    cu = b.cu_seqlens.tolist()
    for n, h in [(0, 0), (2, 7), (4, 15)]:
        sl = slice(cu[n], cu[n + 1])
        pick = lambda t: _np(t[sl, h:h + 1])  # noqa: E731
        ref = oracle.backward(pick(b.q), pick(b.k), pick(b.v), pick(b.beta), pick(b.g),
                              np.array([0, cu[n + 1] - cu[n]], np.int32), pick(d_o),
                              ds_final=_np(dsf[n:n + 1, h:h + 1]))
        for name in NAMES:
            got = grads[name][n, h] if name == "dh0" else grads[name][sl, h]
            want = ref[name][0, 0] if name == "dh0" else ref[name][:, 0]
            assert rel_err(got, want) <= BWD_TOL[torch.bfloat16], (name, n, h)
