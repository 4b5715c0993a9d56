"""GPU decode (gdn_cpr_decode_step with chunk resync, prefill handoff).

The bitwise contract: decode re-synchronises its state every C tokens with
the same boundary computation as the forward's first pass, so a prefill of P
tokens followed by n decode steps gives exactly the bits of one forward over
the P + n tokens.  Decode outputs are also checked against the fp64 oracle.
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


def forward(gdn, b, **kw):
    o, srun, sbnd, ws = gdn.forward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens, **kw)
    assert gdn.check_error(ws) == 0
    return o, srun, sbnd


def split_batch(full: W.Batch, prefix_lens):
    """Prefix batch (first P_n tokens of each sequence) and per-step decode tokens."""
    cu = full.cu_seqlens.cpu().tolist()
    idx = torch.cat([torch.arange(cu[n], cu[n] + P) for n, P in enumerate(prefix_lens)])
    pre = W.Batch(full.q[idx], full.k[idx], full.v[idx], full.beta[idx], full.g[idx],
                  W.cu_seqlens_of(prefix_lens, full.cu_seqlens.device), list(prefix_lens))
    return pre


def decode_tokens_of(full: W.Batch, prefix_lens, step):
    """Token `step` after the prefix of every sequence, stacked as a decode batch."""
    cu = full.cu_seqlens.cpu().tolist()
    rows = [cu[n] + P + step for n, P in enumerate(prefix_lens)]
    idx = torch.tensor(rows, device=full.q.device)
    return (full.q[idx].contiguous(), full.k[idx].contiguous(), full.v[idx].contiguous(),
            full.beta[idx].contiguous(), full.g[idx].contiguous())


def prefill_pair(gdn, pre, out_dtype=torch.float32):
    """Forward returning the exact running-state pair (mantissa, scale)."""
    scale = torch.empty((len(pre.lengths), pre.q.shape[1]), device=pre.q.device)
    o, srun, sbnd = forward(gdn, pre, out_dtype=out_dtype, s_run_scale=scale)
    return o, srun, scale, sbnd


def run_prefill_then_decode(gdn, full, prefix_lens, n_steps, out_dtype=torch.float32):
    H, d = full.q.shape[1], full.q.shape[2]
    pre = split_batch(full, prefix_lens)
    o_pre, srun, sscale, sbnd = prefill_pair(gdn, pre, out_dtype=out_dtype)
    st = gdn.DecodeState(len(prefix_lens), H, d, d, in_dtype=full.q.dtype)
    gdn.decode_state_from_prefill(st, pre.k, pre.v, pre.beta, pre.g, pre.cu_seqlens, srun, sbnd,
                                  s_run_scale=sscale)
    outs = []
    for s in range(n_steps):
        q, k, v, beta, g = decode_tokens_of(full, prefix_lens, s)
        outs.append(gdn.decode_step(st, q, k, v, beta, g, out_dtype=out_dtype))
    assert gdn.check_error(st.error) == 0
    return o_pre, torch.stack(outs), st


@pytest.mark.parametrize("d,dtype", [(64, torch.float32), (128, torch.bfloat16)])
def test_decode_from_empty_equals_forward(gdn, d, dtype):
    """256 decode steps from the zero state: bitwise the forward over the same tokens."""
    b = W.make_batch([256], 2, d, d, dtype=dtype, seed=0).to("cuda")
    o_fwd, srun, sbnd = forward(gdn, b, out_dtype=torch.float32)
    st = gdn.DecodeState(1, 2, d, d, in_dtype=dtype)
    outs = []
    for t in range(256):
        sl = slice(t, t + 1)
        outs.append(gdn.decode_step(st, b.q[sl], b.k[sl], b.v[sl], b.beta[sl], b.g[sl],
                                    out_dtype=torch.float32))
    o_dec = torch.cat(outs)
    assert torch.equal(o_dec, o_fwd)
    assert torch.equal(st.s_bnd[0], sbnd[0])  # four resyncs: boundary states agree
    assert int(st.pos.max()) == 0
    assert gdn.check_error(st.error) == 0


def test_tiny_config_decode(gdn):
    """The 1 x 256, H=2, d=64 fp32 case: decode with resync vs forward and oracle."""
    b = W.tiny()
    bd = b.to("cuda")
    o_fwd, _, _ = forward(gdn, bd, out_dtype=torch.float32)
    st = gdn.DecodeState(1, 2, 64, 64, in_dtype=torch.float32)
    o_dec = torch.cat([gdn.decode_step(st, bd.q[t:t + 1], bd.k[t:t + 1], bd.v[t:t + 1],
                                       bd.beta[t:t + 1], bd.g[t:t + 1], out_dtype=torch.float32)
                       for t in range(256)])
    assert torch.equal(o_dec, o_fwd)
    for h in range(2):
        o_ref, _ = oracle_unit(b, 0, h)
        assert rel_err(o_dec[:, h], o_ref) <= 1e-5


def test_prefill_plus_decode_equals_trainer_forward(gdn):
    """Trainer-shaped batch: split each document at a seeded point, prefill + decode."""
    full = W.make_batch(W.trainer_lengths(2560, 5, 256, seed=3), 4, 128, 128, seed=21)
    fd = full.to("cuda")
    n_steps = 150
    gen = torch.Generator().manual_seed(22)
    prefix = [int(torch.randint(1, L - n_steps, (1,), generator=gen)) for L in full.lengths]
    o_pre, o_dec, st = run_prefill_then_decode(gdn, fd, prefix, n_steps)
    o_all, _, _ = forward(gdn, fd, out_dtype=torch.float32)
    cu = full.cu_seqlens.tolist()
    for n, P in enumerate(prefix):
        ref = o_all[cu[n] + P: cu[n] + P + n_steps]
        assert torch.equal(o_dec[:, n], ref), n
    # decode parity against the oracle (whole prefix + decoded tokens)
    for n in (0, 3):
        for h in (0, 3):
            o_ref, _ = oracle_unit(full, n, h)
            P = prefix[n]
            assert rel_err(o_dec[:, n, h], o_ref[P:P + n_steps]) <= 2e-3


def effective_running_state(st):
    """The decode state's running state as a (mantissa, scale) pair: after a
    resync (pos == 0) it is the boundary state with scale 1."""
    at_bnd = (st.pos == 0)
    mant = torch.where(at_bnd[..., None, None], st.s_bnd, st.s_run)
    scale = torch.where(at_bnd, torch.ones_like(st.s_scale), st.s_scale)
    return mant, scale


def test_trainer_config_prefill_plus_decode_equals_forward(gdn):
    """The trainer-forward workload at its stated shape: 10240 tokens as 5
    documents (Dirichlet lengths, seed 3), H=16, d=128, bf16.  Each document is
    split at a seeded point; its prefix is prefilled and the rest decoded token
    by token to the document's end (rows leave the decode batch as their
    documents end).  Prefill outputs followed by decode outputs equal one
    forward over all 10240 tokens bit for bit, and so do both final states."""
    full = W.trainer(device="cuda")
    lens = full.lengths
    assert sum(lens) == 10240 and len(lens) == 5 and full.q.shape[1:] == (16, 128)
    gen = torch.Generator().manual_seed(26)
    prefix = [int(torch.randint(1, L - 2 * C + 1, (1,), generator=gen)) for L in lens]
    rest = [L - P for L, P in zip(lens, prefix)]
    assert min(rest) >= 2 * C  # every document crosses at least two resyncs in decode

    fscale = torch.empty((5, 16), device="cuda")
    o_all, srun_all, sbnd_all = forward(gdn, full, out_dtype=torch.float32, s_run_scale=fscale)

    pre = split_batch(full, prefix)
    o_pre, srun, sscale, sbnd = prefill_pair(gdn, pre)
    st = gdn.DecodeState(5, 16, 128, 128)
    gdn.decode_state_from_prefill(st, pre.k, pre.v, pre.beta, pre.g, pre.cu_seqlens, srun, sbnd,
                                  s_run_scale=sscale)
    cu = full.cu_seqlens.tolist()
    o_cat = torch.full_like(o_all, float("nan"))
    cp = pre.cu_seqlens.tolist()
    for n, P in enumerate(prefix):
        o_cat[cu[n]:cu[n] + P] = o_pre[cp[n]:cp[n + 1]]
    for s in range(max(rest)):
        live = [n for n in range(5) if s < rest[n]]
        rows = torch.tensor([cu[n] + prefix[n] + s for n in live], device="cuda")
        slots = torch.tensor(live, dtype=torch.int32, device="cuda")
        o = gdn.decode_step(st, full.q[rows].contiguous(), full.k[rows].contiguous(),
                            full.v[rows].contiguous(), full.beta[rows].contiguous(),
                            full.g[rows].contiguous(), slot_idx=slots, out_dtype=torch.float32)
        o_cat[rows] = o
    assert gdn.check_error(st.error) == 0
    assert torch.equal(o_cat, o_all)
    mant, scale = effective_running_state(st)
    assert torch.equal(mant, srun_all) and torch.equal(scale, fscale)
    assert torch.equal(st.s_bnd, sbnd_all)


def test_rollout_decode_shape_sampled(gdn):
    """256 slots, prefix lengths uniform in [1, 2047], H=16, d=128, bf16, 512 steps."""
    prefix = W.decode_prefix_lengths(256)
    n_steps = 512
    lens = [P + n_steps for P in prefix]
    full = W.make_batch(lens, 16, 128, 128, seed=23).to("cuda")
    o_pre, o_dec, st = run_prefill_then_decode(gdn, full, prefix, n_steps)
    cu = full.cu_seqlens.tolist()
    sample = [0, 17, 100, 255]
    sub = full.select(sample)
    o_sub, _, _ = forward(gdn, sub, out_dtype=torch.float32)
    cs = sub.cu_seqlens.tolist()
    for i, n in enumerate(sample):
        P = prefix[n]
        assert torch.equal(o_dec[:, n], o_sub[cs[i] + P: cs[i] + P + n_steps]), n
    subc = sub.to("cpu")
    for i, n in enumerate(sample[:2]):
        for h in (0, 15):
            o_ref, _ = oracle_unit(subc, i, h)
            P = prefix[n]
            assert rel_err(o_dec[:, n, h], o_ref[P:P + n_steps]) <= 2e-3


def test_decode_slot_order_invariance(gdn):
    """Rows addressed through a permuted slot_idx give each slot the same bits."""
    lens = [90, 64, 1, 200, 33]
    full = W.make_batch([L + 70 for L in lens], 2, 128, 128, seed=24).to("cuda")
    _, o_ref, _ = run_prefill_then_decode(gdn, full, lens, 70)
    pre = split_batch(full, lens)
    _, srun, sscale, sbnd = prefill_pair(gdn, pre)
    perm = [3, 0, 4, 2, 1]
    st = gdn.DecodeState(5, 2, 128, 128)
    slot_of_seq = torch.tensor(perm, dtype=torch.int32, device="cuda")
    gdn.decode_state_from_prefill(st, pre.k, pre.v, pre.beta, pre.g, pre.cu_seqlens, srun, sbnd,
                                  s_run_scale=sscale, slot_idx=slot_of_seq)
    rev = list(reversed(range(5)))  # present the rows in reverse sequence order
    rows = torch.tensor([perm[n] for n in rev], dtype=torch.int32, device="cuda")
    for s in range(70):
        q, k, v, beta, g = decode_tokens_of(full, lens, s)
        r = torch.tensor(rev, device="cuda")
        o = gdn.decode_step(st, q[r].contiguous(), k[r].contiguous(), v[r].contiguous(),
                            beta[r].contiguous(), g[r].contiguous(), slot_idx=rows,
                            out_dtype=torch.float32)
        assert torch.equal(o, o_ref[s][r])


def test_decode_state_save_restore(gdn):
    lens = [40, 100]
    full = W.make_batch([L + 80 for L in lens], 2, 64, 64, seed=25).to("cuda")
    pre = split_batch(full, lens)
    _, srun, sscale, sbnd = prefill_pair(gdn, pre)
    st = gdn.DecodeState(2, 2, 64, 64)
    gdn.decode_state_from_prefill(st, pre.k, pre.v, pre.beta, pre.g, pre.cu_seqlens, srun, sbnd,
                                  s_run_scale=sscale)
    for s in range(30):
        gdn.decode_step(st, *decode_tokens_of(full, lens, s))
    saved = [t.cpu() for t in st.tensors()]
    a = [gdn.decode_step(st, *decode_tokens_of(full, lens, s), out_dtype=torch.float32)
         for s in range(30, 80)]
    st2 = gdn.DecodeState(2, 2, 64, 64)
    for dst, src in zip(st2.tensors(), saved):
        dst.copy_(src)
    b = [gdn.decode_step(st2, *decode_tokens_of(full, lens, s), out_dtype=torch.float32)
         for s in range(30, 80)]
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_bad_position_sets_error(gdn):
    st = gdn.DecodeState(2, 2, 64, 64)
    st.pos[1, 0] = 99
    q = torch.randn(2, 2, 64, dtype=torch.bfloat16, device="cuda")
    o = gdn.decode_step(st, q, q, q, torch.rand(2, 2, device="cuda"),
                        -torch.rand(2, 2, device="cuda"))
    assert gdn.check_error(st.error) == gdn.GDN_DEVERR_POS
    assert int(st.pos[1, 0]) == 99 and int(st.pos[0, 0]) == 1
    assert torch.isfinite(o[0]).all()
