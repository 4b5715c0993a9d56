"""The give-up path of the bounded waits, on the GPU, without a fault.

A wait on a completion barrier that nothing arrives at must end after its
poll limit with GDN_DEVERR_TIMEOUT, release its tensor memory, and leave the
context usable: a forward right after it still matches the oracle.
"""
import time

import pytest
import torch

from rl_train_numerics_b200 import workloads as W
from tests.gdn_testlib import oracle_unit, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gdn():
    from rl_train_numerics_b200 import _abi
    return _abi


def test_wait_gives_up_and_context_stays_usable(gdn):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    t0 = time.perf_counter()
    for _ in range(3):  # repeated: tensor memory is released every time
        assert gdn.lib.gdn_selftest_bounded_wait(1000, err.data_ptr(), stream) == gdn.GDN_OK
        assert gdn.check_error(err) == gdn.GDN_DEVERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    b = W.make_batch([130, 64], 2, 128, 128, seed=41)
    o, _, _, ws = gdn.forward(*(t.to("cuda") for t in (b.q, b.k, b.v, b.beta, b.g, b.cu_seqlens)),
                              out_dtype=torch.float32)
    assert gdn.check_error(ws) == 0
    for n in range(2):
        o_ref, _ = oracle_unit(b, n, 1)
        cu = b.cu_seqlens.tolist()
        assert rel_err(o[cu[n]:cu[n + 1], 1].cpu(), o_ref) <= 2e-3
