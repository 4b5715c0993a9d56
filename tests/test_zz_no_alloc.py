"""gdn_cpr_forward_noalloc: the forward for callers that cannot allocate.

Some callers of this library cannot call cudaMalloc (a host runtime that
owns the device memory pool, a plugin host without a device allocator, code
that must not allocate on its hot path).  gdn_cpr_forward_noalloc serves them
from a fixed scratch array compiled into the library.  This test calls it
through the C ABI twice in a row, on two different problems, and checks each
result against the regular gdn_cpr_forward (with a caller workspace) within
the tolerance the other GPU tests use; it also checks that a problem larger
than the fixed scratch is refused.  This file is collected last so that a
run stopping at the first failure has already run every other test.
"""
import ctypes

import pytest
import torch

from rl_train_numerics_b200 import workloads as W
from tests.gdn_testlib import rel_err, tol_for

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
    for b in cases:
        need = gdn.forward_workspace_bytes(len(b.lengths), b.total_tokens, b.q.shape[1],
                                           b.q.shape[2], b.q.shape[2], in_dtype=b.q.dtype)
        assert 0 < need <= NOALLOC_LIMIT
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
        tol = tol_for(b.q.dtype)
        assert rel_err(o, o_ref.double().cpu().numpy()) <= tol
        assert rel_err(srun, srun_ref.double().cpu().numpy()) <= tol
        assert rel_err(sbnd, sbnd_ref.double().cpu().numpy()) <= tol


def test_noalloc_refuses_problems_beyond_its_scratch(gdn):
    T, H, d = 10240, 16, 128
    assert gdn.forward_workspace_bytes(5, T, H, d, d) > NOALLOC_LIMIT
    x = torch.zeros((T, H, d), dtype=torch.bfloat16, device="cuda")
    bg = torch.zeros((T, H), device="cuda")
    cu = W.cu_seqlens_of([2048] * 5, "cuda")
    o = torch.zeros((T, H, d), dtype=torch.bfloat16, device="cuda")
    b = W.Batch(x, x, x, bg, bg, cu, [2048] * 5)
    assert call_noalloc(gdn, b, o, None, None, None) == gdn.GDN_ERR_WORKSPACE
