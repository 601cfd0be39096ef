"""ctypes binding of libmoe_lowbit.so (argument marshalling only).

Every function forwards torch tensors' device pointers and the current CUDA
stream to the C ABI in include/moe_lowbit.h; all computation happens in the
library's CUDA kernels.  There is no fallback: if the shared library is
missing or the tensors are not CUDA tensors, the calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_lowbit.so")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
                4: "MOE_ERR_CUDA", 5: "MOE_ERR_TIMEOUT", 6: "MOE_ERR_DEVICE_INPUT"}
FMT_AFFINE, FMT_MXFP4 = 0, 1


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({detail})")


class Dims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d_model", ctypes.c_int32), ("d_ff", ctypes.c_int32),
                ("n_experts", ctypes.c_int32), ("top_k", ctypes.c_int32), ("hash_mode", ctypes.c_int32),
                ("vocab", ctypes.c_int32), ("d_ff_shared", ctypes.c_int32), ("router_dtype", ctypes.c_int32)]


class QMatC(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("bits", ctypes.c_int32), ("group", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("q", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("biases", ctypes.c_void_p)]


_lib = None

_VP = ctypes.c_void_p
_SIGS = {
    "moe_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(Dims)]),
    "moe_route": (ctypes.c_int, [ctypes.POINTER(Dims), _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_size_t, _VP]),
    "moe_permute": (ctypes.c_int, [ctypes.POINTER(Dims), _VP, _VP, _VP, _VP, _VP, ctypes.c_size_t, _VP]),
    "moe_expert_ffn": (ctypes.c_int, [ctypes.POINTER(Dims), _VP, _VP, _VP, ctypes.POINTER(QMatC),
                                      ctypes.POINTER(QMatC), ctypes.POINTER(QMatC), _VP, _VP, ctypes.c_size_t, _VP]),
    "moe_expert_ffn_noalloc": (ctypes.c_int, [ctypes.POINTER(Dims), _VP, _VP, _VP, ctypes.POINTER(QMatC),
                                              ctypes.POINTER(QMatC), ctypes.POINTER(QMatC), _VP, _VP]),
    "moe_combine": (ctypes.c_int, [ctypes.POINTER(Dims), _VP, _VP, _VP, _VP, _VP, _VP]),
    "moe_forward": (ctypes.c_int, [ctypes.POINTER(Dims), _VP, _VP, _VP, _VP, _VP, ctypes.POINTER(QMatC),
                                   ctypes.POINTER(QMatC), ctypes.POINTER(QMatC), ctypes.POINTER(QMatC), _VP, _VP,
                                   _VP, _VP, ctypes.c_size_t, _VP]),
    "moe_forward_partial": (ctypes.c_int, [ctypes.POINTER(Dims), ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _VP,
                                           _VP, _VP, _VP, _VP, ctypes.POINTER(QMatC), ctypes.POINTER(QMatC),
                                           ctypes.POINTER(QMatC), ctypes.POINTER(QMatC), _VP, _VP, _VP, _VP,
                                           ctypes.c_size_t, _VP]),
    "moe_dequant_mxfp8": (ctypes.c_int, [_VP, _VP, ctypes.c_int64, ctypes.c_int32, _VP, _VP]),
    "moe_forward_host": (ctypes.c_int, [ctypes.POINTER(Dims), _VP, _VP, _VP, _VP, _VP, ctypes.POINTER(QMatC),
                                        ctypes.POINTER(QMatC), ctypes.POINTER(QMatC), ctypes.POINTER(QMatC), _VP,
                                        _VP, ctypes.c_size_t, _VP]),
    "moe_read_device_error": (ctypes.c_int, [_VP, ctypes.POINTER(ctypes.c_int32), _VP]),
    "moe_read_noalloc_error": (ctypes.c_int, [ctypes.POINTER(ctypes.c_int32), _VP]),
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_last_error_detail": (ctypes.c_char_p, []),
    "moe_set_timing_events": (ctypes.c_int, [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32]),
    "moe_timing_count": (ctypes.c_int32, []),
    "moe_timing_label": (ctypes.c_char_p, [ctypes.c_int32]),
    "moe_set_ffn_path": (ctypes.c_int32, [ctypes.c_int32]),
    "moe_test_stall_fused_wait": (ctypes.c_int32, [ctypes.c_int32]),
    "moe_hc_sinkhorn_mix": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                           ctypes.c_float, _VP, _VP, _VP, _VP, _VP]),
}


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Load (once) and type the shared library; raise if it is missing."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(f"{p} not built: run `python -m bit_quantized_moe_route_b200.build`")
    lib = ctypes.CDLL(p)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


def _check(status: int, where: str):
    if status != MOE_OK:
        detail = load_library().moe_last_error_detail().decode()
        raise MoEError(status, where, detail)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def make_dims(T: int, d_model: int, d_ff: int, n_experts: int, top_k: int, hash_mode: bool = False,
              vocab: int = 0, d_ff_shared: int = 0, router_dtype=None) -> Dims:
    """router_dtype: None/torch.float32 (fp32 router weights) or torch.bfloat16."""
    rd = 1 if router_dtype in (torch.bfloat16, "bf16", 1) else 0
    return Dims(T, d_model, d_ff, n_experts, top_k, int(bool(hash_mode)), vocab, d_ff_shared, rd)


def qmat(m) -> QMatC:
    """Describe a packed matrix: any object with fmt ('affine'|'mxfp4'), bits,
    group and CUDA tensors q, scales, biases (None for mxfp4)."""
    if m.fmt not in ("affine", "mxfp4"):
        raise ValueError(f"packed format {m.fmt!r} is not supported by the library (affine, mxfp4)")
    fmt = FMT_AFFINE if m.fmt == "affine" else FMT_MXFP4
    return QMatC(fmt, m.bits, m.group, 0, _ptr(m.q), _ptr(m.scales),
                 None if m.biases is None else _ptr(m.biases))


def workspace_size(dims: Dims) -> int:
    n = load_library().moe_workspace_size(ctypes.byref(dims))
    if n == 0:
        raise MoEError(1, "moe_workspace_size", "invalid dims")
    return n


def alloc_workspace(dims: Dims, device="cuda") -> torch.Tensor:
    """Zeroed workspace buffer (uint8) of moe_workspace_size bytes."""
    return torch.zeros(workspace_size(dims), dtype=torch.uint8, device=device)


def route(dims, x, router_w, router_b, token_ids, tid2eid, topk_ids, topk_w, ws, stream=None):
    _check(load_library().moe_route(ctypes.byref(dims), _ptr(x), _ptr(router_w), _ptr(router_b),
                                    _ptr(token_ids), _ptr(tid2eid), _ptr(topk_ids), _ptr(topk_w), _ptr(ws),
                                    ws.numel(), _stream(stream)), "moe_route")


def permute(dims, topk_ids, expert_offsets, sorted_rows, inv, ws, stream=None):
    _check(load_library().moe_permute(ctypes.byref(dims), _ptr(topk_ids), _ptr(expert_offsets), _ptr(sorted_rows),
                                      _ptr(inv), _ptr(ws), ws.numel(), _stream(stream)), "moe_permute")


def expert_ffn(dims, x, expert_offsets, sorted_rows, w1, w3, w2, y, ws, stream=None):
    q1, q3, q2 = qmat(w1), qmat(w3), qmat(w2)
    _check(load_library().moe_expert_ffn(ctypes.byref(dims), _ptr(x), _ptr(expert_offsets), _ptr(sorted_rows),
                                         ctypes.byref(q1), ctypes.byref(q3), ctypes.byref(q2), _ptr(y), _ptr(ws),
                                         ws.numel(), _stream(stream)), "moe_expert_ffn")


def expert_ffn_noalloc(dims, x, expert_offsets, sorted_rows, w1, w3, w2, y, stream=None):
    """moe_expert_ffn_noalloc: the expert FFN for callers that cannot allocate
    device memory; its scratch is a fixed 4 MiB static device array shared by
    every call on the device (calls must not overlap on the GPU)."""
    q1, q3, q2 = qmat(w1), qmat(w3), qmat(w2)
    _check(load_library().moe_expert_ffn_noalloc(ctypes.byref(dims), _ptr(x), _ptr(expert_offsets),
                                                 _ptr(sorted_rows), ctypes.byref(q1), ctypes.byref(q3),
                                                 ctypes.byref(q2), _ptr(y), _stream(stream)),
           "moe_expert_ffn_noalloc")


def combine(dims, y, inv, topk_w, y_shared, out, stream=None):
    _check(load_library().moe_combine(ctypes.byref(dims), _ptr(y), _ptr(inv), _ptr(topk_w), _ptr(y_shared),
                                      _ptr(out), _stream(stream)), "moe_combine")


def _shared_arr(shared: Optional[Sequence]):
    if shared is None:
        return None
    arr = (QMatC * 3)(*[qmat(m) for m in shared])
    return arr


def forward(dims, x, token_ids, router_w, router_b, tid2eid, w1, w3, w2, shared, out, ws,
            topk_ids_out=None, topk_w_out=None, stream=None):
    q1, q3, q2 = qmat(w1), qmat(w3), qmat(w2)
    sh = _shared_arr(shared)
    _check(load_library().moe_forward(
        ctypes.byref(dims), _ptr(x), _ptr(token_ids), _ptr(router_w), _ptr(router_b), _ptr(tid2eid),
        ctypes.byref(q1), ctypes.byref(q3), ctypes.byref(q2), sh, _ptr(out), _ptr(topk_ids_out),
        _ptr(topk_w_out), _ptr(ws), ws.numel(), _stream(stream)), "moe_forward")


def forward_partial(dims, expert_begin, expert_end, include_shared, x, token_ids, router_w, router_b, tid2eid,
                    w1, w3, w2, shared, out_partial, ws, topk_ids_out=None, topk_w_out=None, stream=None):
    """moe_forward_partial: the fp32 partial output [T, d_model] of experts
    expert_begin <= e < expert_end (plus the shared expert when include_shared)."""
    if out_partial.dtype != torch.float32:
        raise ValueError("out_partial must be float32")
    q1, q3, q2 = qmat(w1), qmat(w3), qmat(w2)
    sh = _shared_arr(shared)
    _check(load_library().moe_forward_partial(
        ctypes.byref(dims), int(expert_begin), int(expert_end), 1 if include_shared else 0, _ptr(x), _ptr(token_ids),
        _ptr(router_w), _ptr(router_b), _ptr(tid2eid), ctypes.byref(q1), ctypes.byref(q3), ctypes.byref(q2), sh,
        _ptr(out_partial), _ptr(topk_ids_out), _ptr(topk_w_out), _ptr(ws), ws.numel(), _stream(stream)),
        "moe_forward_partial")


def dequant_mxfp8(codes: torch.Tensor, scales: torch.Tensor, out: torch.Tensor, stream=None):
    """moe_dequant_mxfp8: codes uint8 [rows, n_in], scales uint8 [rows, n_in/32], out bf16 [rows, n_in]."""
    if codes.dtype != torch.uint8 or scales.dtype != torch.uint8 or out.dtype != torch.bfloat16:
        raise ValueError("codes and scales must be uint8, out bfloat16")
    rows, n_in = codes.shape
    if tuple(scales.shape) != (rows, n_in // 32) or tuple(out.shape) != (rows, n_in):
        raise ValueError("shape mismatch")
    _check(load_library().moe_dequant_mxfp8(_ptr(codes), _ptr(scales), rows, n_in, _ptr(out), _stream(stream)),
           "moe_dequant_mxfp8")


def forward_host(dims, x_host: torch.Tensor, token_ids_host, router_w, router_b, tid2eid, w1, w3, w2, shared,
                 out_host: torch.Tensor, ws, stream=None):
    """moe_forward_host: x_host/token_ids_host/out_host are CPU tensors (pin them)."""
    for t in (x_host, out_host) + ((token_ids_host,) if token_ids_host is not None else ()):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("host buffers must be contiguous CPU tensors")
    q1, q3, q2 = qmat(w1), qmat(w3), qmat(w2)
    sh = _shared_arr(shared)
    _check(load_library().moe_forward_host(
        ctypes.byref(dims), x_host.data_ptr(), None if token_ids_host is None else token_ids_host.data_ptr(),
        _ptr(router_w), _ptr(router_b), _ptr(tid2eid), ctypes.byref(q1), ctypes.byref(q3), ctypes.byref(q2), sh,
        out_host.data_ptr(), _ptr(ws), ws.numel(), _stream(stream)), "moe_forward_host")


def read_device_error(ws, stream=None) -> int:
    code = ctypes.c_int32(0)
    _check(load_library().moe_read_device_error(_ptr(ws), ctypes.byref(code), _stream(stream)),
           "moe_read_device_error")
    return code.value


def hc_sinkhorn_mix(logits, h, out, iters: int, eps: float = 0.0, P_out=None, stream=None):
    """moe_hc_sinkhorn_mix: logits fp32 [T, n, n], h/out bf16 [T, n, d]."""
    T, n, d = h.shape
    if tuple(logits.shape) != (T, n, n) or tuple(out.shape) != (T, n, d):
        raise ValueError("shapes: logits [T, n, n], h and out [T, n, d]")
    _check(load_library().moe_hc_sinkhorn_mix(T, n, d, int(iters), float(eps), _ptr(logits), _ptr(h), _ptr(P_out),
                                              _ptr(out), _stream(stream)), "moe_hc_sinkhorn_mix")


def read_noalloc_error(stream=None) -> int:
    """Device error word of expert_ffn_noalloc's static scratch (read and cleared)."""
    code = ctypes.c_int32(0)
    _check(load_library().moe_read_noalloc_error(ctypes.byref(code), _stream(stream)), "moe_read_noalloc_error")
    return code.value


FFN_AUTO, FFN_GEMV, FFN_TENSOR_CORE, FFN_DECODE_FUSED = 0, 1, 2, 3


def set_ffn_path(path: int) -> int:
    """Select the expert-FFN implementation (FFN_AUTO / FFN_GEMV /
    FFN_TENSOR_CORE / FFN_DECODE_FUSED) for the calling thread's calls;
    returns its previous setting."""
    prev = load_library().moe_set_ffn_path(int(path))
    if prev < 0:
        raise ValueError(f"unknown FFN path {path}")
    return prev


def status_string(status: int) -> str:
    return load_library().moe_status_string(status).decode()


def set_timing_events(events: Optional[Sequence["torch.cuda.Event"]]):
    """Arm the per-kernel timing hook for the next forward on this thread.

    ``events`` must be CUDA events created with timing enabled; they are
    recorded on the forward's stream around each of its kernels.  Returns the
    ctypes array (keep it alive until the forward has been issued).
    """
    lib = load_library()
    if events is None:
        lib.moe_set_timing_events(None, 0)
        return None
    for ev in events:                 # torch creates the CUDA event on first record
        if not ev.cuda_event:
            ev.record()
    arr = (ctypes.c_void_p * len(events))(*[ev.cuda_event for ev in events])
    lib.moe_set_timing_events(arr, len(events))
    return arr


def timing_labels():
    """Labels of the kernels timed by the last hooked forward."""
    lib = load_library()
    n = lib.moe_timing_count()
    return [lib.moe_timing_label(i).decode() for i in range(max(0, n - 1))]
