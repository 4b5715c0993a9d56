"""gdn_cpr_forward_noalloc: the forward for callers that cannot allocate.

Some callers of this library cannot call cudaMalloc (a host runtime that
owns the device memory pool, a plugin host without a device allocator, code
that must not allocate on its hot path).  gdn_cpr_forward_noalloc serves them
from a fixed scratch array compiled into the library.  This test calls it
through the C ABI twice in a row, on two different problems (the larger one
first, so the second call runs on scratch that still holds the first call's
data), and checks each result against the regular gdn_cpr_forward (with a
caller workspace).  Both run the same kernels on the same inputs, so the
results must agree bit for bit, which is stricter than the oracle tolerance
of the other GPU tests.  It also checks that a problem larger than the fixed
scratch is refused.  This file is collected last so that a run stopping at
the first failure has already run every other test.
"""
import ctypes

import pytest
import torch

from rl_train_numerics_b200 import workloads as W

pytestmark = pytest.mark.gpu

NOALLOC_LIMIT = 32 << 20  # GDN_NOALLOC_SCRATCH_BYTES in include/gdn_cpr.h


@pytest.fixture(scope="module")
def gdn():
    from rl_train_numerics_b200 import _abi
    return _abi


def p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def call_noalloc(gdn, b, o, srun, sbnd, err):
    T, H, d = b.q.shape
    in_code = gdn.GDN_BF16 if b.q.dtype == torch.bfloat16 else gdn.GDN_F32
    out_code = gdn.GDN_BF16 if o.dtype == torch.bfloat16 else gdn.GDN_F32
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return gdn.lib.gdn_cpr_forward_noalloc(
        p(b.q), p(b.k), p(b.v), in_code, p(b.beta), p(b.g), p(b.cu_seqlens), len(b.lengths), T,
        H, d, d, 64, 1.0, None, p(o), out_code, p(srun), None, p(sbnd), p(err), stream)


def regular(gdn, b):
    o, srun, sbnd, ws = gdn.forward(b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens,
                                    out_dtype=torch.float32)
    assert gdn.check_error(ws) == 0
    return o, srun, sbnd


def test_noalloc_matches_regular_forward_two_calls_in_a_row(gdn):
    cases = [W.make_batch([300, 64, 17, 0, 129], 4, 128, 128, seed=41),
             W.make_batch([256, 70, 1], 2, 64, 64, dtype=torch.float32, seed=42)]
    need = [gdn.forward_workspace_bytes(len(b.lengths), b.total_tokens, b.q.shape[1],
                                        b.q.shape[2], b.q.shape[2], in_dtype=b.q.dtype)
            for b in cases]
    assert 0 < need[1] < need[0] <= NOALLOC_LIMIT  # a smaller problem follows a larger one
    results = []
    for b in [cases[0].to("cuda"), cases[1].to("cuda")]:  # two calls in a row
        T, H, d = b.q.shape
        N = len(b.lengths)
        o = torch.full((T, H, d), float("nan"), device="cuda")
        srun = torch.full((N, H, d, d), float("nan"), device="cuda")
        sbnd = torch.full((N, H, d, d), float("nan"), device="cuda")
        err = torch.full((1,), 7, dtype=torch.int32, device="cuda")
        assert call_noalloc(gdn, b, o, srun, sbnd, err) == gdn.GDN_OK
        assert gdn.check_error(err) == 0
        results.append((b, o, srun, sbnd))
    for b, o, srun, sbnd in results:
        o_ref, srun_ref, sbnd_ref = regular(gdn, b)
        assert torch.equal(o, o_ref)
        assert torch.equal(srun, srun_ref)
        assert torch.equal(sbnd, sbnd_ref)


def test_noalloc_refuses_problems_beyond_its_scratch(gdn):
    T, H, d = 10240, 16, 128
    assert gdn.forward_workspace_bytes(5, T, H, d, d) > NOALLOC_LIMIT
    x = torch.zeros((T, H, d), dtype=torch.bfloat16, device="cuda")
    bg = torch.zeros((T, H), device="cuda")
    cu = W.cu_seqlens_of([2048] * 5, "cuda")
    o = torch.zeros((T, H, d), dtype=torch.bfloat16, device="cuda")
    b = W.Batch(x, x, x, bg, bg, cu, [2048] * 5)
    assert call_noalloc(gdn, b, o, None, None, None) == gdn.GDN_ERR_WORKSPACE


def test_noalloc_empty_batch_clears_the_error_word(gdn):
    """An empty batch launches no kernel but still reports this call's status
    in the caller's error word (zero) instead of an earlier call's bits."""
    err = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    cu = torch.zeros((1,), dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = gdn.lib.gdn_cpr_forward_noalloc(None, None, None, gdn.GDN_BF16, None, None, p(cu), 0, 0,
                                         4, 128, 128, 64, 1.0, None, None, gdn.GDN_BF16, None,
                                         None, None, p(err), stream)
    assert rc == gdn.GDN_OK
    torch.cuda.synchronize()
    assert int(err.item()) == 0
