"""Host-side checks of libgdn_cpr.so that need no GPU.

The library must load, export every function include/gdn_cpr.h declares, and
reject bad arguments on the host (before any CUDA call) with the documented
status codes.  Every call below is one the library must refuse; none of them
reaches a kernel launch, so the fake pointers are never dereferenced.
"""
import ctypes
import os
import re

import pytest

from rl_train_numerics_b200 import build_lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn_cpr.h")

build_lib.build()
from rl_train_numerics_b200 import _abi as gdn  # noqa: E402

FAKE = 0x10000  # 16-byte aligned, never dereferenced: every call here is rejected first
MIS = 0x10004   # misaligned


def declared_functions():
    inc = os.path.join(ROOT, "include")
    text = "".join(open(os.path.join(inc, f)).read() for f in sorted(os.listdir(inc))
                   if f.endswith(".h"))
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|size_t|const char\s*\*)\s*(gdn_\w+)\s*\(",
                                 text, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ["gdn_cpr_forward", "gdn_cpr_decode_step", "gdn_chunk_boundary",
              "gdn_cpr_decode_state_from_prefill", "gdn_check_error",
              "gdn_cpr_forward_workspace_bytes", "gdn_status_string", "gdn_cpr_abi_version",
              "gdn_cpr_backward", "gdn_cpr_backward_workspace_bytes", "gdn_pik_gemm",
              "gdn_pik_workspace_bytes"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(build_lib.LIB)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, f"symbols declared in gdn_cpr.h but not exported: {missing}"


def test_abi_version_and_status_strings():
    assert gdn.lib.gdn_cpr_abi_version() == 7
    for code in range(-6, 1):
        assert gdn.status_string(code).startswith("GDN_")
    assert "unknown" in gdn.status_string(42)


def test_workspace_query():
    import torch
    ws = gdn.forward_workspace_bytes
    assert ws(5, 10240, 16, 128, 128) > 0
    assert ws(5, 20480, 16, 128, 128) > ws(5, 10240, 16, 128, 128)
    # chunk states dominate: at least (T/C + N) * H * d * d * 4 bytes
    assert ws(5, 10240, 16, 128, 128) >= (10240 // 64 + 5) * 16 * 128 * 128 * 4
    assert ws(1, 100, 2, 64, 64, 64, torch.float32) > ws(1, 100, 2, 64, 64)  # 3-term splits
    assert ws(1, 100, 2, 128, 128, 64, torch.float32) == 0  # fp32 inputs: d = 64 only
    assert ws(1, 100, 2, 96, 96) == 0          # unsupported head dim
    assert ws(1, 100, 2, 64, 64, 32) == 0      # unsupported chunk size
    assert ws(-1, 100, 2, 64, 64) == 0


def fwd(**over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, in_dtype=gdn.GDN_BF16, beta=FAKE, g=FAKE, cu=FAKE, N=2,
             T=128, H=2, dk=64, dv=64, C=64, scale=1.0, h0=None, o=FAKE,
             out_dtype=gdn.GDN_BF16, srun=None, sscale=None, sbnd=None, ws=FAKE, wsb=1 << 40,
             stream=None)
    a.update(over)
    return gdn.lib.gdn_cpr_forward(a["q"], a["k"], a["v"], a["in_dtype"], a["beta"], a["g"],
                                   a["cu"], a["N"], a["T"], a["H"], a["dk"], a["dv"], a["C"],
                                   a["scale"], a["h0"], a["o"], a["out_dtype"], a["srun"],
                                   a["sscale"], a["sbnd"], a["ws"], a["wsb"], a["stream"])


@pytest.mark.parametrize("over,expect", [
    (dict(H=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(N=-1), gdn.GDN_ERR_INVALID_ARG),
    (dict(T=-5), gdn.GDN_ERR_INVALID_ARG),
    (dict(in_dtype=7), gdn.GDN_ERR_INVALID_ARG),
    (dict(out_dtype=3), gdn.GDN_ERR_INVALID_ARG),
    (dict(scale=float("nan")), gdn.GDN_ERR_INVALID_ARG),
    (dict(dk=96, dv=96), gdn.GDN_ERR_UNSUPPORTED),
    (dict(dk=64, dv=128), gdn.GDN_ERR_UNSUPPORTED),
    (dict(C=32), gdn.GDN_ERR_UNSUPPORTED),
    (dict(in_dtype=gdn.GDN_F32, dk=128, dv=128), gdn.GDN_ERR_UNSUPPORTED),
    (dict(T=1 << 31), gdn.GDN_ERR_UNSUPPORTED),
    (dict(q=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(cu=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(o=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(q=MIS), gdn.GDN_ERR_INVALID_ARG),
    (dict(o=MIS), gdn.GDN_ERR_INVALID_ARG),
    (dict(h0=MIS), gdn.GDN_ERR_INVALID_ARG),
    (dict(srun=MIS), gdn.GDN_ERR_INVALID_ARG),
    (dict(sscale=FAKE), gdn.GDN_ERR_INVALID_ARG),            # scale without a state buffer
    (dict(srun=FAKE, sscale=MIS + 2), gdn.GDN_ERR_INVALID_ARG),
    (dict(ws=None), gdn.GDN_ERR_WORKSPACE),
    (dict(wsb=1024), gdn.GDN_ERR_WORKSPACE),
    (dict(N=0, T=5), gdn.GDN_ERR_INVALID_ARG),
])
def test_forward_rejects_on_host(over, expect):
    assert fwd(**over) == expect


def test_forward_empty_batch_is_a_no_op():
    assert fwd(N=0, T=0, q=None, k=None, v=None, beta=None, g=None, o=None, cu=None,
               ws=None, wsb=0) == gdn.GDN_OK


def test_backward_workspace_query():
    import torch
    fw, bw = gdn.forward_workspace_bytes, gdn.backward_workspace_bytes
    # the forward's workspace plus adjoints at chunk ends and two [T, H, d] fp32 rows
    assert bw(5, 10240, 16, 128, 128) >= fw(5, 10240, 16, 128, 128) + \
        (10240 // 64 + 5) * 16 * 128 * 128 * 4 + 2 * 10240 * 16 * 128 * 4
    assert bw(1, 100, 2, 128, 128, 64, torch.float32) == 0
    assert bw(1, 100, 2, 96, 96) == 0
    assert bw(-1, 100, 2, 64, 64) == 0


def bwd(**over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, in_dtype=gdn.GDN_BF16, beta=FAKE, g=FAKE, cu=FAKE, N=2,
             T=128, H=2, dk=64, dv=64, C=64, scale=1.0, h0=None, do=FAKE, dsf=None, dq=FAKE,
             dk_=FAKE, dv_=FAKE, db=FAKE, dg=FAKE, dh0=None, ws=FAKE, wsb=1 << 40, flags=0,
             stream=None)
    a.update(over)
    return gdn.lib.gdn_cpr_backward(a["q"], a["k"], a["v"], a["in_dtype"], a["beta"], a["g"],
                                    a["cu"], a["N"], a["T"], a["H"], a["dk"], a["dv"], a["C"],
                                    a["scale"], a["h0"], a["do"], a["dsf"], a["dq"], a["dk_"],
                                    a["dv_"], a["db"], a["dg"], a["dh0"], a["ws"], a["wsb"],
                                    a["flags"], a["stream"])


@pytest.mark.parametrize("over,expect", [
    (dict(H=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(N=-1), gdn.GDN_ERR_INVALID_ARG),
    (dict(in_dtype=7), gdn.GDN_ERR_INVALID_ARG),
    (dict(scale=float("inf")), gdn.GDN_ERR_INVALID_ARG),
    (dict(dk=96, dv=96), gdn.GDN_ERR_UNSUPPORTED),
    (dict(in_dtype=gdn.GDN_F32, dk=128, dv=128), gdn.GDN_ERR_UNSUPPORTED),
    (dict(C=128), gdn.GDN_ERR_UNSUPPORTED),
    (dict(T=1 << 31), gdn.GDN_ERR_UNSUPPORTED),
    (dict(do=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(dq=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(dk_=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(dv_=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(db=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(dg=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(do=MIS), gdn.GDN_ERR_INVALID_ARG),
    (dict(dq=MIS), gdn.GDN_ERR_INVALID_ARG),
    (dict(db=MIS + 2), gdn.GDN_ERR_INVALID_ARG),
    (dict(dsf=MIS), gdn.GDN_ERR_INVALID_ARG),
    (dict(dh0=MIS), gdn.GDN_ERR_INVALID_ARG),
    (dict(ws=None), gdn.GDN_ERR_WORKSPACE),
    (dict(wsb=4096), gdn.GDN_ERR_WORKSPACE),
    (dict(ws=MIS), gdn.GDN_ERR_INVALID_ARG),
    (dict(N=0, T=3), gdn.GDN_ERR_INVALID_ARG),
    (dict(flags=2), gdn.GDN_ERR_INVALID_ARG),
    (dict(flags=-1), gdn.GDN_ERR_INVALID_ARG),
])
def test_backward_rejects_on_host(over, expect):
    assert bwd(**over) == expect


def test_backward_empty_batch_is_a_no_op():
    assert bwd(N=0, T=0, q=None, k=None, v=None, beta=None, g=None, do=None, dq=None, dk_=None,
               dv_=None, db=None, dg=None, cu=None, ws=None, wsb=0) == gdn.GDN_OK


def pik(**over):
    a = dict(A=FAKE, B=FAKE, C=FAKE, M=256, N=256, K=1024, L=8, R=1, ws=FAKE, wsb=1 << 40,
             err=FAKE, stream=None)
    a.update(over)
    return gdn.lib.gdn_pik_gemm(a["A"], a["B"], a["C"], a["M"], a["N"], a["K"], a["L"], a["R"],
                                a["ws"], a["wsb"], a["err"], a["stream"])


@pytest.mark.parametrize("over,expect", [
    (dict(M=-1), gdn.GDN_ERR_INVALID_ARG),
    (dict(L=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(L=3), gdn.GDN_ERR_UNSUPPORTED),
    (dict(L=128, K=128 * 64), gdn.GDN_ERR_UNSUPPORTED),
    (dict(R=3), gdn.GDN_ERR_UNSUPPORTED),
    (dict(R=16), gdn.GDN_ERR_UNSUPPORTED),   # more ranks than leaves
    (dict(N=200), gdn.GDN_ERR_UNSUPPORTED),  # not a multiple of 16
    (dict(K=1000), gdn.GDN_ERR_UNSUPPORTED),  # not a multiple of 64 L
    (dict(A=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(err=None), gdn.GDN_ERR_INVALID_ARG),
    (dict(C=MIS), gdn.GDN_ERR_INVALID_ARG),
    (dict(err=MIS + 2), gdn.GDN_ERR_INVALID_ARG),
    (dict(ws=None), gdn.GDN_ERR_WORKSPACE),         # 8 leaves: pending sums above 4 pairs
    (dict(L=16, wsb=16), gdn.GDN_ERR_WORKSPACE),
])
def test_pik_rejects_on_host(over, expect):
    assert pik(**over) == expect


def test_pik_workspace_and_empty_shapes():
    w = gdn.pik_workspace_bytes
    slot = 128 * 256 * 4  # one pending sum of a 128 x 256 tile
    assert w(256, 256, 1024, 2, 1) == 0           # one pair of leaves: no pending sums
    assert w(256, 256, 1024, 1, 1) == 0
    assert w(256, 256, 1024, 8, 1) == 2 * 2 * slot     # 2 blocks x 2 levels above 4 pairs
    assert w(256, 256, 1024, 16, 1) == 2 * 3 * slot
    assert w(256, 256, 1024, 8, 8) == 8 * 256 * 256 * 4   # 8 rank sums, one leaf each
    assert w(256, 200, 1024, 8, 1) == 0 and w(256, 256, 1024, 3, 1) == 0
    assert pik(M=0, A=None, B=None, C=None, err=None) == gdn.GDN_OK
    assert pik(N=0, A=None, B=None, C=None, err=None) == gdn.GDN_OK


def _state(**over):
    f = dict(s_run=FAKE, s_scale=FAKE, s_bnd=FAKE, buf_k=FAKE, buf_v=FAKE, buf_beta=FAKE,
             buf_g=FAKE, pos=FAKE, error=FAKE, resync=FAKE, n_slots=4)
    f.update(over)
    return gdn.DecodeStateStruct(f["s_run"], f["s_scale"], f["s_bnd"], f["buf_k"], f["buf_v"],
                                 f["buf_beta"], f["buf_g"], f["pos"], f["error"], f["resync"],
                                 f["n_slots"])


def dec(st=None, **over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, in_dtype=gdn.GDN_BF16, beta=FAKE, g=FAKE, slot=None, B=4,
             H=2, dk=128, dv=128, C=64, scale=1.0, o=FAKE, out_dtype=gdn.GDN_BF16)
    a.update(over)
    return gdn.lib.gdn_cpr_decode_step(a["q"], a["k"], a["v"], a["in_dtype"], a["beta"],
                                       a["g"], a["slot"], a["B"], a["H"], a["dk"], a["dv"],
                                       a["C"], a["scale"], st or _state(), a["o"],
                                       a["out_dtype"], None)


@pytest.mark.parametrize("over,state_over,expect", [
    (dict(B=-1), {}, gdn.GDN_ERR_INVALID_ARG),
    (dict(dk=32, dv=32), {}, gdn.GDN_ERR_UNSUPPORTED),
    (dict(C=128), {}, gdn.GDN_ERR_UNSUPPORTED),
    (dict(q=None), {}, gdn.GDN_ERR_INVALID_ARG),
    (dict(o=MIS), {}, gdn.GDN_ERR_INVALID_ARG),
    ({}, dict(s_run=None), gdn.GDN_ERR_INVALID_ARG),
    ({}, dict(pos=None), gdn.GDN_ERR_INVALID_ARG),
    ({}, dict(s_scale=None), gdn.GDN_ERR_INVALID_ARG),
    ({}, dict(error=None), gdn.GDN_ERR_INVALID_ARG),
    ({}, dict(resync=None), gdn.GDN_ERR_INVALID_ARG),
    ({}, dict(s_bnd=MIS), gdn.GDN_ERR_INVALID_ARG),
    ({}, dict(n_slots=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(B=5), {}, gdn.GDN_ERR_INVALID_ARG),   # more rows than slots without slot_idx
])
def test_decode_rejects_on_host(over, state_over, expect):
    assert dec(_state(**state_over), **over) == expect


def test_decode_zero_rows_is_a_no_op():
    assert dec(B=0) == gdn.GDN_OK


def test_boundary_and_handoff_reject_on_host():
    L = gdn.lib
    assert L.gdn_chunk_boundary(FAKE, FAKE, FAKE, 0, FAKE, FAKE, -1, 2, 64, 64, 64, FAKE,
                                None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_chunk_boundary(FAKE, FAKE, FAKE, 0, FAKE, FAKE, 1, 2, 64, 64, 16, FAKE,
                                None) == gdn.GDN_ERR_UNSUPPORTED
    assert L.gdn_chunk_boundary(None, FAKE, FAKE, 0, FAKE, FAKE, 1, 2, 64, 64, 64, FAKE,
                                None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_chunk_boundary(FAKE, FAKE, FAKE, 0, FAKE, FAKE, 0, 2, 64, 64, 64, FAKE,
                                None) == gdn.GDN_OK
    assert L.gdn_cpr_decode_state_from_prefill(
        FAKE, FAKE, 0, FAKE, FAKE, FAKE, 8, 100, 2, 64, 64, 64, FAKE, None, FAKE, None,
        _state(n_slots=4), None) == gdn.GDN_ERR_INVALID_ARG  # 8 sequences, 4 slots
    assert L.gdn_cpr_decode_state_from_prefill(
        FAKE, FAKE, 0, FAKE, FAKE, FAKE, 2, 100, 2, 64, 64, 64, None, None, FAKE, None,
        _state(), None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_check_error(None, None, None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_check_error(MIS + 1, None, None) == gdn.GDN_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(4, 2, 64)
    with pytest.raises(ValueError, match="CUDA"):
        gdn.forward(x, x, x, torch.zeros(4, 2), torch.zeros(4, 2),
                    torch.tensor([0, 4], dtype=torch.int32))


def test_selftest_rejects_on_host():
    L = gdn.lib
    assert L.gdn_selftest_bounded_wait(0, FAKE, None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_selftest_bounded_wait((1 << 22) + 1, FAKE, None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_selftest_bounded_wait(10, None, None) == gdn.GDN_ERR_INVALID_ARG


def test_native_forward_host_checks():
    """gdn_native_forward: d = 128 with bf16 inputs only; the forward's argument
    checks and workspace size otherwise (all rejected before any launch)."""
    L = gdn.lib

    def call(**over):
        a = dict(q=FAKE, in_dtype=gdn.GDN_BF16, N=2, T=128, H=2, dk=128, dv=128, C=64,
                 ws=FAKE, wsb=1 << 40)
        a.update(over)
        return L.gdn_native_forward(a["q"], FAKE, FAKE, a["in_dtype"], FAKE, FAKE, FAKE, a["N"],
                                    a["T"], a["H"], a["dk"], a["dv"], a["C"], 1.0, None, FAKE,
                                    gdn.GDN_BF16, None, None, a["ws"], a["wsb"], None, None)
    assert call(dk=64, dv=64) == gdn.GDN_ERR_UNSUPPORTED
    assert call(dk=64, dv=64, in_dtype=gdn.GDN_F32) == gdn.GDN_ERR_UNSUPPORTED
    assert call(q=MIS) == gdn.GDN_ERR_INVALID_ARG
    assert call(C=32) == gdn.GDN_ERR_UNSUPPORTED
    assert call(wsb=16) == gdn.GDN_ERR_WORKSPACE
    assert call(ws=None) == gdn.GDN_ERR_WORKSPACE


def test_recurrent_host_checks():
    L = gdn.lib

    def fwd_call(**over):
        a = dict(q=FAKE, in_dtype=gdn.GDN_BF16, N=2, T=128, dk=128, dv=128, sf=None, sfs=None,
                 err=None)
        a.update(over)
        return L.gdn_recurrent_forward(a["q"], FAKE, FAKE, a["in_dtype"], FAKE, FAKE, FAKE,
                                       a["N"], a["T"], 2, a["dk"], a["dv"], 1.0, None, FAKE,
                                       gdn.GDN_BF16, a["sf"], a["sfs"], a["err"], None)
    assert fwd_call(dk=96, dv=96) == gdn.GDN_ERR_UNSUPPORTED
    assert fwd_call(in_dtype=gdn.GDN_F32) == gdn.GDN_ERR_UNSUPPORTED  # fp32 inputs: d = 64
    assert fwd_call(q=MIS) == gdn.GDN_ERR_INVALID_ARG
    assert fwd_call(sfs=FAKE) == gdn.GDN_ERR_INVALID_ARG  # a scale without the state
    assert fwd_call(err=MIS + 2) == gdn.GDN_ERR_INVALID_ARG  # misaligned error word
    assert fwd_call(N=0, T=5) == gdn.GDN_ERR_INVALID_ARG

    def step_call(**over):
        a = dict(B=4, dk=128, dv=128, in_dtype=gdn.GDN_BF16, s=FAKE, o=FAKE)
        a.update(over)
        return L.gdn_recurrent_decode_step(FAKE, FAKE, FAKE, a["in_dtype"], FAKE, FAKE, a["B"],
                                           2, a["dk"], a["dv"], 1.0, a["s"], FAKE, a["o"],
                                           gdn.GDN_BF16, None)
    assert step_call(dk=96, dv=96) == gdn.GDN_ERR_UNSUPPORTED
    assert step_call(dk=128, dv=64) == gdn.GDN_ERR_UNSUPPORTED
    assert step_call(in_dtype=gdn.GDN_F32) == gdn.GDN_ERR_UNSUPPORTED
    assert step_call(s=MIS) == gdn.GDN_ERR_INVALID_ARG
    assert step_call(s=None) == gdn.GDN_ERR_INVALID_ARG
    assert step_call(B=-1) == gdn.GDN_ERR_INVALID_ARG
    assert step_call(B=0) == gdn.GDN_OK  # nothing to do
