"""Thin Python binding of libgdn_cpr.so (the C ABI in include/gdn_cpr.h).

Argument marshalling only: torch provides device memory and the current CUDA
stream; every step of the layer runs in the library's CUDA kernels.  There is
no CPU or PyTorch fallback: if the shared library is missing, importing this
module raises, and every call checks that its tensors live on a CUDA device.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdn_cpr.so")

GDN_OK = 0
GDN_ERR_INVALID_ARG = -1
GDN_ERR_UNSUPPORTED = -2
GDN_ERR_WORKSPACE = -3
GDN_ERR_CUDA = -4
GDN_ERR_DEVICE_DATA = -5
GDN_ERR_TIMEOUT = -6
GDN_ERR_CONTRACT = -7
GDN_DIGEST_SEMANTIC = 0
GDN_DIGEST_POLICY = 1
GDN_DIGEST_DEPLOYMENT = 2
GDN_BF16 = 0
GDN_F32 = 1
GDN_DEVERR_CU_SEQLENS = 1
GDN_DEVERR_POS = 2
GDN_DEVERR_TIMEOUT = 4
GDN_BWD_REUSE_FORWARD = 1
CHUNK = 64


class GdnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


class DecodeStateStruct(ctypes.Structure):
    _fields_ = [("s_run", ctypes.c_void_p), ("s_scale", ctypes.c_void_p),
                ("s_bnd", ctypes.c_void_p),
                ("buf_k", ctypes.c_void_p), ("buf_v", ctypes.c_void_p),
                ("buf_beta", ctypes.c_void_p), ("buf_g", ctypes.c_void_p),
                ("pos", ctypes.c_void_p), ("error", ctypes.c_void_p),
                ("resync", ctypes.c_void_p), ("n_slots", ctypes.c_int)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run __graft_entry__.build() or "
                          "python -m rl_train_numerics_b200.build_lib")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, f32, sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                             ctypes.c_size_t)
    sigs = {
        "gdn_cpr_abi_version": (i32, []),
        "gdn_status_string": (ctypes.c_char_p, [i32]),
        "gdn_cpr_forward_workspace_bytes": (sz, [i32, i64, i32, i32, i32, i32, i32]),
        "gdn_cpr_forward": (i32, [vp, vp, vp, i32, vp, vp, vp, i32, i64, i32, i32, i32, i32, f32,
                                  vp, vp, i32, vp, vp, vp, vp, sz, vp]),
        "gdn_cpr_forward_ex": (i32, [vp, vp, vp, i32, vp, vp, vp, i32, i64, i32, i32, i32, i32,
                                     f32, vp, vp, i32, vp, vp, vp, vp, sz, vp, vp]),
        "gdn_cpr_forward_noalloc": (i32, [vp, vp, vp, i32, vp, vp, vp, i32, i64, i32, i32, i32,
                                          i32, f32, vp, vp, i32, vp, vp, vp, vp, vp]),
        "gdn_cpr_decode_state_from_prefill": (i32, [vp, vp, i32, vp, vp, vp, i32, i64, i32, i32,
                                                    i32, i32, vp, vp, vp, vp,
                                                    DecodeStateStruct, vp]),
        "gdn_cpr_decode_step": (i32, [vp, vp, vp, i32, vp, vp, vp, i32, i32, i32, i32, i32, f32,
                                      DecodeStateStruct, vp, i32, vp]),
        "gdn_chunk_boundary": (i32, [vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, i32, vp, vp]),
        "gdn_recurrent_forward": (i32, [vp, vp, vp, i32, vp, vp, vp, i32, i64, i32, i32, i32, f32,
                                        vp, vp, i32, vp, vp, vp, vp]),
        "gdn_recurrent_decode_step": (i32, [vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, f32, vp,
                                            vp, vp, i32, vp]),
        "gdn_native_forward": (i32, [vp, vp, vp, i32, vp, vp, vp, i32, i64, i32, i32, i32, i32,
                                     f32, vp, vp, i32, vp, vp, vp, sz, vp, vp]),
        "gdn_cpr_backward_workspace_bytes": (sz, [i32, i64, i32, i32, i32, i32, i32]),
        "gdn_cpr_backward": (i32, [vp, vp, vp, i32, vp, vp, vp, i32, i64, i32, i32, i32, i32,
                                   f32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i32, vp]),
        "gdn_cpr_backward_ex": (i32, [vp, vp, vp, i32, vp, vp, vp, i32, i64, i32, i32, i32,
                                      i32, f32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i32,
                                      vp, vp]),
        "gdn_pik_workspace_bytes": (sz, [i64, i64, i64, i32, i32]),
        "gdn_pik_gemm": (i32, [vp, vp, vp, i64, i64, i64, i32, i32, vp, sz, vp, vp]),
        "gdn_check_error": (i32, [vp, vp, vp]),
        "gdn_cpr_contract_descriptor": (i32, [i32, i32, i32, i32, i32, i32, ctypes.c_char_p, sz,
                                              ctypes.POINTER(ctypes.c_size_t)]),
        "gdn_cpr_contract_digest": (i32, [i32, i32, i32, i32, i32, i32, ctypes.c_char_p]),
        "gdn_cpr_contract_check": (i32, [ctypes.c_char_p, i32, i32, i32, i32, i32]),
        "gdn_sha256": (i32, [ctypes.c_char_p, sz, ctypes.c_char_p]),
        "gdn_selftest_bounded_wait": (i32, [i32, vp, vp]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def status_string(status: int) -> str:
    return lib.gdn_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != GDN_OK:
        raise GdnError(status, what)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("gdn_cpr: tensors must be on a CUDA device (there is no CPU path)")
    if not t.is_contiguous():
        raise ValueError("gdn_cpr: tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    if t.dtype == torch.float32:
        return GDN_F32
    raise ValueError(f"gdn_cpr: unsupported dtype {t.dtype}")


def _out_code(in_code: int, out_dtype, o) -> int:
    """Output dtype code: from `o` when given (must agree with out_dtype), else
    out_dtype, else the input dtype."""
    if o is not None:
        code = _dtype_code(o)
        if out_dtype is not None and _dtype_code(torch.empty(0, dtype=out_dtype)) != code:
            raise ValueError("gdn_cpr: out_dtype disagrees with the dtype of o")
        return code
    if out_dtype is None:
        return in_code
    return _dtype_code(torch.empty(0, dtype=out_dtype))


def _torch_dtype(code: int):
    return torch.bfloat16 if code == GDN_BF16 else torch.float32


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def forward_workspace_bytes(n_seqs: int, total_tokens: int, H: int, dk: int, dv: int,
                            C: int = CHUNK, in_dtype=torch.bfloat16) -> int:
    code = GDN_BF16 if in_dtype == torch.bfloat16 else GDN_F32
    return int(lib.gdn_cpr_forward_workspace_bytes(n_seqs, total_tokens, H, dk, dv, C, code))


def forward(q, k, v, beta, g, cu_seqlens, *, n_seqs: Optional[int] = None, h0=None,
            C: int = CHUNK, scale: float = 1.0, out_dtype=None, o=None, s_run_final=None,
            s_bnd_final=None, s_run_scale=None, want_states: bool = True, workspace=None,
            stream=None, kernel_events=None):
    """gdn_cpr_forward (gdn_cpr_forward_ex when ``kernel_events``, a list of 5
    recorded torch.cuda.Event objects, is given).
    Returns (o, s_run_final, s_bnd_final, workspace).  s_run_final is the
    running state itself, unless an ``s_run_scale`` tensor [N, H] fp32 is
    passed: then s_run_final holds the mantissa and s_run_scale the scale (the
    pair decode needs to continue bit for bit)."""
    T, H, dk = q.shape
    dv = v.shape[2]
    N = (cu_seqlens.numel() - 1) if n_seqs is None else int(n_seqs)
    in_code = _dtype_code(q)
    out_code = _out_code(in_code, out_dtype, o)
    dev = q.device
    if o is None:
        o = torch.empty((T, H, dv), dtype=_torch_dtype(out_code), device=dev)
    if want_states:
        if s_run_final is None:
            s_run_final = torch.empty((N, H, dv, dk), dtype=torch.float32, device=dev)
        if s_bnd_final is None:
            s_bnd_final = torch.empty((N, H, dv, dk), dtype=torch.float32, device=dev)
    need = forward_workspace_bytes(N, T, H, dk, dv, C, q.dtype)
    if workspace is None:
        workspace = torch.zeros(max(need, 256), dtype=torch.uint8, device=dev)
    ev = None
    if kernel_events is not None:
        if len(kernel_events) != 5 or any(e.cuda_event == 0 for e in kernel_events):
            raise ValueError("kernel_events: 5 torch.cuda.Event objects, each recorded once")
        ev = (ctypes.c_void_p * 5)(*[e.cuda_event for e in kernel_events])
    st = lib.gdn_cpr_forward_ex(_ptr(q), _ptr(k), _ptr(v), in_code, _ptr(beta), _ptr(g),
                                _ptr(cu_seqlens), N, T, H, dk, dv, C, float(scale), _ptr(h0),
                                _ptr(o), out_code, _ptr(s_run_final), _ptr(s_run_scale),
                                _ptr(s_bnd_final), _ptr(workspace), workspace.numel(), ev,
                                _stream(stream))
    _check(st, "gdn_cpr_forward")
    return o, s_run_final, s_bnd_final, workspace


def native_forward(q, k, v, beta, g, cu_seqlens, *, n_seqs: Optional[int] = None, h0=None,
                   C: int = CHUNK, scale: float = 1.0, out_dtype=None, o=None, s_final=None,
                   s_bnd_final=None, want_states: bool = True, workspace=None, stream=None,
                   kernel_events=None):
    """gdn_native_forward (the chunked, "native mixed" forward; d = 128, bf16).
    Returns (o, s_final, s_bnd_final, workspace); the workspace is the CPR
    forward's (same size).  kernel_events: 5 recorded torch.cuda.Event objects."""
    T, H, dk = q.shape
    dv = v.shape[2]
    N = (cu_seqlens.numel() - 1) if n_seqs is None else int(n_seqs)
    in_code = _dtype_code(q)
    out_code = _out_code(in_code, out_dtype, o)
    dev = q.device
    if o is None:
        o = torch.empty((T, H, dv), dtype=_torch_dtype(out_code), device=dev)
    if want_states:
        if s_final is None:
            s_final = torch.empty((N, H, dv, dk), dtype=torch.float32, device=dev)
        if s_bnd_final is None:
            s_bnd_final = torch.empty((N, H, dv, dk), dtype=torch.float32, device=dev)
    need = forward_workspace_bytes(N, T, H, dk, dv, C, q.dtype)
    if workspace is None:
        workspace = torch.zeros(max(need, 256), dtype=torch.uint8, device=dev)
    ev = None
    if kernel_events is not None:
        if len(kernel_events) != 5 or any(e.cuda_event == 0 for e in kernel_events):
            raise ValueError("kernel_events: 5 torch.cuda.Event objects, each recorded once")
        ev = (ctypes.c_void_p * 5)(*[e.cuda_event for e in kernel_events])
    st = lib.gdn_native_forward(_ptr(q), _ptr(k), _ptr(v), in_code, _ptr(beta), _ptr(g),
                                _ptr(cu_seqlens), N, T, H, dk, dv, C, float(scale), _ptr(h0),
                                _ptr(o), out_code, _ptr(s_final), _ptr(s_bnd_final),
                                _ptr(workspace), workspace.numel(), ev, _stream(stream))
    _check(st, "gdn_native_forward")
    return o, s_final, s_bnd_final, workspace


def recurrent_forward(q, k, v, beta, g, cu_seqlens, *, n_seqs: Optional[int] = None, h0=None,
                      scale: float = 1.0, out_dtype=None, o=None, s_final=None,
                      s_final_scale=None, want_state: bool = True, error=None, stream=None):
    """gdn_recurrent_forward (the recurrent-everywhere forward).  Returns
    (o, s_final, s_final_scale, error word).  s_final is the state itself
    unless an ``s_final_scale`` tensor [N, H] fp32 is passed: then s_final
    holds the mantissa and s_final_scale the scale."""
    T, H, dk = q.shape
    dv = v.shape[2]
    N = (cu_seqlens.numel() - 1) if n_seqs is None else int(n_seqs)
    in_code = _dtype_code(q)
    out_code = _out_code(in_code, out_dtype, o)
    dev = q.device
    if o is None:
        o = torch.empty((T, H, dv), dtype=_torch_dtype(out_code), device=dev)
    if want_state and s_final is None:
        s_final = torch.empty((N, H, dv, dk), dtype=torch.float32, device=dev)
    if error is None:
        error = torch.zeros(1, dtype=torch.int32, device=dev)
    st = lib.gdn_recurrent_forward(_ptr(q), _ptr(k), _ptr(v), in_code, _ptr(beta), _ptr(g),
                                   _ptr(cu_seqlens), N, T, H, dk, dv, float(scale), _ptr(h0),
                                   _ptr(o), out_code, _ptr(s_final), _ptr(s_final_scale),
                                   _ptr(error), _stream(stream))
    _check(st, "gdn_recurrent_forward")
    return o, s_final, s_final_scale, error


def recurrent_decode_step(q, k, v, beta, g, s, s_scale, *, scale: float = 1.0, out_dtype=None,
                          o=None, stream=None):
    """gdn_recurrent_decode_step: one token per row b; (s, s_scale) updated in
    place.  q, k, v [B, H, d]; beta, g [B, H].  Returns o [B, H, dv]."""
    B, H, dk = q.shape
    dv = v.shape[2]
    in_code = _dtype_code(q)
    out_code = _out_code(in_code, out_dtype, o)
    if o is None:
        o = torch.empty((B, H, dv), dtype=_torch_dtype(out_code), device=q.device)
    st = lib.gdn_recurrent_decode_step(_ptr(q), _ptr(k), _ptr(v), in_code, _ptr(beta), _ptr(g),
                                       B, H, dk, dv, float(scale), _ptr(s), _ptr(s_scale),
                                       _ptr(o), out_code, _stream(stream))
    _check(st, "gdn_recurrent_decode_step")
    return o


def backward_workspace_bytes(n_seqs: int, total_tokens: int, H: int, dk: int, dv: int,
                             C: int = CHUNK, dtype=torch.bfloat16) -> int:
    code = _dtype_code(torch.empty(0, dtype=dtype))
    return int(lib.gdn_cpr_backward_workspace_bytes(n_seqs, total_tokens, H, dk, dv, C, code))


def backward(q, k, v, beta, g, cu_seqlens, d_o, *, n_seqs: Optional[int] = None, h0=None,
             ds_final=None, C: int = CHUNK, scale: float = 1.0, want_dh0: bool = True,
             grads=None, workspace=None, reuse_forward: bool = False, stream=None,
             kernel_events=None):
    """gdn_cpr_backward.  Returns (grads, workspace); grads is a dict of fp32
    tensors dq, dk, dv [T, H, d], dbeta, dg [T, H] and dh0 [N, H, dv, dk]
    (None unless want_dh0).  Pass ``grads`` (the same dict) to reuse buffers.
    reuse_forward=True (GDN_BWD_REUSE_FORWARD): ``workspace`` was last used by
    forward() on this same batch, whose first pass is then reused.
    kernel_events: 5 recorded torch.cuda.Event objects (gdn_cpr_backward_ex)."""
    T, H, dk = q.shape
    dv = v.shape[2]
    N = (cu_seqlens.numel() - 1) if n_seqs is None else int(n_seqs)
    in_code = _dtype_code(q)
    if d_o.dtype != q.dtype:
        raise ValueError("gdn_cpr: d_o must have the dtype of q, k and v")
    dev = q.device
    if grads is None:
        f32 = dict(dtype=torch.float32, device=dev)
        grads = {"dq": torch.empty((T, H, dk), **f32), "dk": torch.empty((T, H, dk), **f32),
                 "dv": torch.empty((T, H, dv), **f32), "dbeta": torch.empty((T, H), **f32),
                 "dg": torch.empty((T, H), **f32),
                 "dh0": torch.empty((N, H, dv, dk), **f32) if want_dh0 else None}
    need = backward_workspace_bytes(N, T, H, dk, dv, C, q.dtype)
    if workspace is None:
        workspace = torch.zeros(max(need, 256), dtype=torch.uint8, device=dev)
    ev = None
    if kernel_events is not None:
        if len(kernel_events) != 5 or any(e.cuda_event == 0 for e in kernel_events):
            raise ValueError("kernel_events: 5 torch.cuda.Event objects, each recorded once")
        ev = (ctypes.c_void_p * 5)(*[e.cuda_event for e in kernel_events])
    st = lib.gdn_cpr_backward_ex(_ptr(q), _ptr(k), _ptr(v), in_code, _ptr(beta), _ptr(g),
                                 _ptr(cu_seqlens), N, T, H, dk, dv, C, float(scale), _ptr(h0),
                                 _ptr(d_o), _ptr(ds_final), _ptr(grads["dq"]),
                                 _ptr(grads["dk"]), _ptr(grads["dv"]), _ptr(grads["dbeta"]),
                                 _ptr(grads["dg"]), _ptr(grads.get("dh0")), _ptr(workspace),
                                 workspace.numel(), GDN_BWD_REUSE_FORWARD if reuse_forward else 0,
                                 ev, _stream(stream))
    _check(st, "gdn_cpr_backward")
    return grads, workspace


def pik_workspace_bytes(M: int, N: int, K: int, n_leaves: int, n_ranks: int = 1) -> int:
    return int(lib.gdn_pik_workspace_bytes(M, N, K, n_leaves, n_ranks))


def pik_gemm(A, B, n_leaves: int, n_ranks: int = 1, *, C=None, workspace=None, error=None,
             stream=None):
    """gdn_pik_gemm: C = A B^T (A [M, K], B [N, K] bf16; C [M, N] fp32) with K in
    n_leaves contiguous leaves combined by the fixed binary tree, computed in the
    layout of n_ranks emulated ranks.  Returns (C, error word tensor)."""
    if A.dtype != torch.bfloat16 or B.dtype != torch.bfloat16:
        raise ValueError("gdn_pik_gemm: A and B must be bf16")
    M, K = A.shape
    N = B.shape[0]
    if B.shape[1] != K:
        raise ValueError("gdn_pik_gemm: A and B must have the same K")
    dev = A.device
    if C is None:
        C = torch.empty((M, N), dtype=torch.float32, device=dev)
    need = pik_workspace_bytes(M, N, K, n_leaves, n_ranks)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if error is None:
        error = torch.zeros(1, dtype=torch.int32, device=dev)
    st = lib.gdn_pik_gemm(_ptr(A) if K else None, _ptr(B) if K else None, _ptr(C), M, N, K,
                          int(n_leaves), int(n_ranks),
                          _ptr(workspace), 0 if workspace is None else workspace.numel(),
                          _ptr(error), _stream(stream))
    _check(st, "gdn_pik_gemm")
    return C, error


def check_error(error_word: torch.Tensor, stream=None) -> int:
    """gdn_check_error: synchronises, returns the device error bits (and clears them)."""
    bits = ctypes.c_int32(0)
    st = lib.gdn_check_error(_ptr(error_word), ctypes.byref(bits), _stream(stream))
    if st not in (GDN_OK, GDN_ERR_DEVICE_DATA):
        _check(st, "gdn_check_error")
    return int(bits.value)


class DecodeState:
    """Caller-owned decode state (device tensors) for n_slots sequences."""

    def __init__(self, n_slots: int, H: int, dk: int, dv: int, in_dtype=torch.bfloat16,
                 C: int = CHUNK, device="cuda"):
        self.n_slots, self.H, self.dk, self.dv, self.C = n_slots, H, dk, dv, C
        self.in_dtype = in_dtype
        f32 = torch.float32
        self.s_run = torch.zeros((n_slots, H, dv, dk), dtype=f32, device=device)
        self.s_scale = torch.ones((n_slots, H), dtype=f32, device=device)
        self.s_bnd = torch.zeros((n_slots, H, dv, dk), dtype=f32, device=device)
        self.buf_k = torch.zeros((n_slots, H, C, dk), dtype=in_dtype, device=device)
        self.buf_v = torch.zeros((n_slots, H, C, dv), dtype=in_dtype, device=device)
        self.buf_beta = torch.zeros((n_slots, H, C), dtype=f32, device=device)
        self.buf_g = torch.zeros((n_slots, H, C), dtype=f32, device=device)
        self.pos = torch.zeros((n_slots, H), dtype=torch.int32, device=device)
        self.error = torch.zeros((1,), dtype=torch.int32, device=device)
        # work list of the resync inside decode_step (scratch, zero between steps)
        self.resync = torch.zeros((4 + n_slots * H,), dtype=torch.int32, device=device)

    def struct(self) -> DecodeStateStruct:
        return DecodeStateStruct(self.s_run.data_ptr(), self.s_scale.data_ptr(),
                                 self.s_bnd.data_ptr(),
                                 self.buf_k.data_ptr(), self.buf_v.data_ptr(),
                                 self.buf_beta.data_ptr(), self.buf_g.data_ptr(),
                                 self.pos.data_ptr(), self.error.data_ptr(),
                                 self.resync.data_ptr(), self.n_slots)

    def tensors(self):
        return (self.s_run, self.s_scale, self.s_bnd, self.buf_k, self.buf_v, self.buf_beta,
                self.buf_g, self.pos)

    def clone(self) -> "DecodeState":
        c = DecodeState.__new__(DecodeState)
        c.__dict__.update({k: (v.clone() if isinstance(v, torch.Tensor) else v)
                           for k, v in self.__dict__.items()})
        return c


def decode_state_from_prefill(state: DecodeState, k, v, beta, g, cu_seqlens, s_run_final,
                              s_bnd_final, *, s_run_scale=None, slot_idx=None, stream=None):
    N = cu_seqlens.numel() - 1
    T, H, dk = k.shape
    st = lib.gdn_cpr_decode_state_from_prefill(
        _ptr(k), _ptr(v), _dtype_code(k), _ptr(beta), _ptr(g), _ptr(cu_seqlens), N, T, H, dk,
        v.shape[2], state.C, _ptr(s_run_final), _ptr(s_run_scale), _ptr(s_bnd_final),
        _ptr(slot_idx), state.struct(), _stream(stream))
    _check(st, "gdn_cpr_decode_state_from_prefill")


def decode_step(state: DecodeState, q, k, v, beta, g, *, slot_idx=None, scale: float = 1.0,
                out_dtype=None, o=None, stream=None):
    """gdn_cpr_decode_step for B rows: q,k [B,H,dk], v [B,H,dv], beta,g [B,H]."""
    B, H, dk = q.shape
    dv = v.shape[2]
    in_code = _dtype_code(q)
    out_code = _out_code(in_code, out_dtype, o)
    if o is None:
        o = torch.empty((B, H, dv), dtype=_torch_dtype(out_code), device=q.device)
    st = lib.gdn_cpr_decode_step(_ptr(q), _ptr(k), _ptr(v), in_code, _ptr(beta), _ptr(g),
                                 _ptr(slot_idx), B, H, dk, dv, state.C, float(scale),
                                 state.struct(), _ptr(o), out_code, _stream(stream))
    _check(st, "gdn_cpr_decode_step")
    return o


def chunk_boundary(s_start, k, v, beta, g, *, s_end=None, stream=None):
    """gdn_chunk_boundary: k [B,H,C,dk], v [B,H,C,dv], beta,g [B,H,C]; s [B,H,dv,dk]."""
    B, H, C, dk = k.shape
    dv = v.shape[3]
    if s_end is None:
        s_end = torch.empty_like(s_start)
    st = lib.gdn_chunk_boundary(_ptr(s_start), _ptr(k), _ptr(v), _dtype_code(k), _ptr(beta),
                                _ptr(g), B, H, dk, dv, C, _ptr(s_end), _stream(stream))
    _check(st, "gdn_chunk_boundary")
    return s_end


def _dt(dtype) -> int:
    return GDN_BF16 if dtype == torch.bfloat16 else GDN_F32 if dtype == torch.float32 else -1


def contract_descriptor(kind: int, in_dtype=torch.bfloat16, out_dtype=torch.bfloat16, dk: int = 128,
                        dv: int = 128, C: int = CHUNK) -> str:
    """gdn_cpr_contract_descriptor: the canonical text a digest hashes."""
    n = ctypes.c_size_t(0)
    args = (kind, _dt(in_dtype), _dt(out_dtype), dk, dv, C)
    _check(lib.gdn_cpr_contract_descriptor(*args, None, 0, ctypes.byref(n)),
           "gdn_cpr_contract_descriptor")
    buf = ctypes.create_string_buffer(n.value + 1)
    _check(lib.gdn_cpr_contract_descriptor(*args, buf, n.value + 1, ctypes.byref(n)),
           "gdn_cpr_contract_descriptor")
    return buf.value.decode()


def contract_digest(kind: int, in_dtype=torch.bfloat16, out_dtype=torch.bfloat16, dk: int = 128,
                    dv: int = 128, C: int = CHUNK) -> bytes:
    """gdn_cpr_contract_digest: 32-byte SHA-256 identity digest."""
    out = ctypes.create_string_buffer(32)
    _check(lib.gdn_cpr_contract_digest(kind, _dt(in_dtype), _dt(out_dtype), dk, dv, C, out),
           "gdn_cpr_contract_digest")
    return out.raw


def contract_check(peer_policy: bytes, in_dtype=torch.bfloat16, out_dtype=torch.bfloat16,
                   dk: int = 128, dv: int = 128, C: int = CHUNK) -> int:
    """gdn_cpr_contract_check: GDN_OK, or GDN_ERR_CONTRACT when the policies differ."""
    if len(peer_policy) != 32:
        raise ValueError("a digest is 32 bytes")
    return lib.gdn_cpr_contract_check(peer_policy, _dt(in_dtype), _dt(out_dtype), dk, dv, C)


def sha256(data: bytes) -> bytes:
    """gdn_sha256 of a byte string."""
    out = ctypes.create_string_buffer(32)
    _check(lib.gdn_sha256(data, len(data), out), "gdn_sha256")
    return out.raw
