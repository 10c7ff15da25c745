"""Python binding of libstrata_moe.so, the B200 MoE expert-layer library.

Argument marshalling only: every function here forwards to the C entry point
of the same name in ``include/strata_moe.h`` and returns its status code.
Tensor arguments may be torch tensors (their ``data_ptr()`` is passed), raw
integer device pointers, or ``None`` for nullable arguments.  PyTorch supplies
device memory and streams; all computation happens in the library's CUDA
kernels.  There is no fallback: if the shared library is missing this module
raises on first use.
"""

from __future__ import annotations

import ctypes
import os
from typing import Any, Optional

__all__ = [
    "STRATA_OK", "STRATA_ERR_INVALID_ARG", "STRATA_ERR_UNSUPPORTED", "STRATA_ERR_WORKSPACE",
    "STRATA_ERR_CUDA", "STRATA_ERR_DEVICE_CHECK", "STRATA_OP_GATE_UP_SWIGLU", "STRATA_OP_DOWN",
    "Dims", "Q4", "StrataError", "lib", "lib_path", "check",
    "strata_moe_workspace_bytes", "strata_status_string", "strata_moe_route",
    "strata_moe_permute", "strata_moe_permute_static", "STRATA_PERMUTE_STATIC_SCRATCH_INTS",
    "strata_moe_expert_gemm_q4", "strata_moe_combine",
    "strata_moe_forward", "strata_moe_device_status", "strata_moe_selftest_wait",
    "strata_moe_gather_rows", "workspace", "AttnDims", "strata_sparse_attention",
    "strata_sparse_attention_workspace_bytes", "attention_workspace",
]

STRATA_OK = 0
STRATA_ERR_INVALID_ARG = 1
STRATA_ERR_UNSUPPORTED = 2
STRATA_ERR_WORKSPACE = 3
STRATA_ERR_CUDA = 4
STRATA_ERR_DEVICE_CHECK = 5
STRATA_OP_GATE_UP_SWIGLU = 0
STRATA_OP_DOWN = 1
STRATA_PERMUTE_STATIC_SCRATCH_INTS = 131072

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libstrata_moe.so"
_lib = None


class StrataError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {strata_status_string(status)} (status {status})")


class Dims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("n", ctypes.c_int32), ("group", ctypes.c_int32)]

    @classmethod
    def of(cls, dims: Any) -> "Dims":
        if isinstance(dims, cls):
            return dims
        if isinstance(dims, dict):
            return cls(int(dims["T"]), int(dims["d"]), int(dims["E"]), int(dims["k"]),
                       int(dims["n"]), int(dims["group"]))
        return cls(*[int(v) for v in dims])


class AttnDims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("L", ctypes.c_int32), ("Hq", ctypes.c_int32),
                ("Hkv", ctypes.c_int32), ("D", ctypes.c_int32), ("P", ctypes.c_int32)]

    @classmethod
    def of(cls, dims: Any) -> "AttnDims":
        if isinstance(dims, cls):
            return dims
        if isinstance(dims, dict):
            return cls(*[int(dims[k]) for k in ("T", "L", "Hq", "Hkv", "D", "P")])
        return cls(*[int(v) for v in dims])


class Q4(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("s", ctypes.c_void_p)]

    @classmethod
    def of(cls, w: Any) -> "Q4":
        if isinstance(w, cls):
            return w
        if w is None:
            return cls(None, None)
        q, s = w
        return cls(_ptr(q), _ptr(s))


def lib_path() -> str:
    return os.path.join(_HERE, _LIB_NAME)


def lib() -> ctypes.CDLL:
    """Load the shared library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    path = lib_path()
    if not os.path.exists(path):
        raise ImportError(f"{path} not found: build it with `python -m local_moe_route_b200.build`"
                          " (there is no non-CUDA fallback)")
    L = ctypes.CDLL(path)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    st = ctypes.c_int
    L.strata_moe_workspace_bytes.argtypes = [Dims]
    L.strata_moe_workspace_bytes.restype = sz
    L.strata_status_string.argtypes = [st]
    L.strata_status_string.restype = ctypes.c_char_p
    L.strata_moe_route.argtypes = [vp, vp, vp, Dims, vp, vp, vp, vp, sz, vp]
    L.strata_moe_route.restype = st
    L.strata_moe_permute.argtypes = [vp, Dims, vp, vp, vp, vp, vp, sz, vp]
    L.strata_moe_permute.restype = st
    L.strata_moe_permute_static.argtypes = [vp, Dims, vp, vp, vp, vp, vp]
    L.strata_moe_permute_static.restype = st
    L.strata_moe_expert_gemm_q4.argtypes = [st, vp, vp, vp, Q4, Q4, vp, Dims, vp, vp, sz, vp]
    L.strata_moe_expert_gemm_q4.restype = st
    L.strata_moe_combine.argtypes = [vp, vp, vp, Dims, vp, vp]
    L.strata_moe_combine.restype = st
    L.strata_moe_forward.argtypes = [vp, vp, vp, Q4, Q4, Q4, Dims, vp, vp, vp, vp, sz, vp]
    L.strata_moe_forward.restype = st
    L.strata_moe_device_status.argtypes = [vp]
    L.strata_moe_device_status.restype = st
    L.strata_moe_selftest_wait.argtypes = [vp, vp, vp]
    L.strata_moe_selftest_wait.restype = st
    i32 = ctypes.c_int32
    L.strata_moe_gather_rows.argtypes = [vp, vp, i32, i32, i32, vp, vp]
    L.strata_moe_gather_rows.restype = st
    L.strata_sparse_attention_workspace_bytes.argtypes = [AttnDims]
    L.strata_sparse_attention_workspace_bytes.restype = sz
    L.strata_sparse_attention.argtypes = [vp, vp, vp, vp, AttnDims, ctypes.c_float, vp, vp, sz,
                                          vp]
    L.strata_sparse_attention.restype = st
    _lib = L
    return L


def _ptr(t: Any) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return int(t.data_ptr())


def _nbytes(t: Any) -> int:
    if t is None:
        return 0
    if isinstance(t, int):
        raise TypeError("pass ws_bytes explicitly with a raw workspace pointer")
    return int(t.numel() * t.element_size())


def _stream(s: Any) -> Optional[int]:
    if s is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream) if torch.cuda.is_available() else None
    if isinstance(s, int):
        return s
    return int(s.cuda_stream)


def check(status: int, what: str = "strata") -> None:
    """Raise StrataError unless status is STRATA_OK."""
    if status != STRATA_OK:
        raise StrataError(status, what)


def strata_moe_workspace_bytes(dims) -> int:
    return int(lib().strata_moe_workspace_bytes(Dims.of(dims)))


def strata_status_string(status: int) -> str:
    return lib().strata_status_string(int(status)).decode()


def strata_moe_route(x, w_router, bias, dims, topk_ids, topk_w, logits_out=None, ws=None,
                     ws_bytes=None, stream=None) -> int:
    return lib().strata_moe_route(
        _ptr(x), _ptr(w_router), _ptr(bias), Dims.of(dims), _ptr(topk_ids), _ptr(topk_w),
        _ptr(logits_out), _ptr(ws), _nbytes(ws) if ws_bytes is None else int(ws_bytes),
        _stream(stream))


def strata_moe_permute(topk_ids, dims, counts, offsets, sorted_token, slot_row, ws=None,
                       ws_bytes=None, stream=None) -> int:
    return lib().strata_moe_permute(
        _ptr(topk_ids), Dims.of(dims), _ptr(counts), _ptr(offsets), _ptr(sorted_token),
        _ptr(slot_row), _ptr(ws), _nbytes(ws) if ws_bytes is None else int(ws_bytes),
        _stream(stream))


def strata_moe_permute_static(topk_ids, dims, counts, offsets, sorted_token, slot_row,
                              stream=None) -> int:
    return lib().strata_moe_permute_static(
        _ptr(topk_ids), Dims.of(dims), _ptr(counts), _ptr(offsets), _ptr(sorted_token),
        _ptr(slot_row), _stream(stream))


def strata_moe_expert_gemm_q4(op, a, sorted_token, offsets, w0, w1, row_scale, dims, out,
                              ws=None, ws_bytes=None, stream=None) -> int:
    return lib().strata_moe_expert_gemm_q4(
        int(op), _ptr(a), _ptr(sorted_token), _ptr(offsets), Q4.of(w0), Q4.of(w1),
        _ptr(row_scale), Dims.of(dims), _ptr(out), _ptr(ws),
        _nbytes(ws) if ws_bytes is None else int(ws_bytes), _stream(stream))


def strata_moe_combine(rows, topk_w, slot_row, dims, y, stream=None) -> int:
    return lib().strata_moe_combine(_ptr(rows), _ptr(topk_w), _ptr(slot_row), Dims.of(dims),
                                    _ptr(y), _stream(stream))


def strata_moe_forward(x, w_router, bias, gate, up, down, dims, y, topk_ids_out=None,
                       topk_w_out=None, ws=None, ws_bytes=None, stream=None) -> int:
    return lib().strata_moe_forward(
        _ptr(x), _ptr(w_router), _ptr(bias), Q4.of(gate), Q4.of(up), Q4.of(down),
        Dims.of(dims), _ptr(y), _ptr(topk_ids_out), _ptr(topk_w_out), _ptr(ws),
        _nbytes(ws) if ws_bytes is None else int(ws_bytes), _stream(stream))


def strata_moe_device_status(stream=None) -> int:
    return lib().strata_moe_device_status(_stream(stream))


def strata_moe_selftest_wait(out, sync_ws, stream=None) -> int:
    return lib().strata_moe_selftest_wait(_ptr(out), _ptr(sync_ws), _stream(stream))


def strata_moe_gather_rows(src, index, src_rows, rows, width, dst, stream=None) -> int:
    return lib().strata_moe_gather_rows(_ptr(src), _ptr(index), int(src_rows), int(rows),
                                        int(width), _ptr(dst), _stream(stream))


def strata_sparse_attention_workspace_bytes(dims) -> int:
    return int(lib().strata_sparse_attention_workspace_bytes(AttnDims.of(dims)))


def strata_sparse_attention(q, k_cache, v_cache, idx, dims, scale, out, ws=None, ws_bytes=None,
                            stream=None) -> int:
    return lib().strata_sparse_attention(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(idx), AttnDims.of(dims), float(scale),
        _ptr(out), _ptr(ws), _nbytes(ws) if ws_bytes is None else int(ws_bytes), _stream(stream))


def attention_workspace(dims, device="cuda"):
    """A torch uint8 buffer of strata_sparse_attention_workspace_bytes(dims) bytes."""
    import torch
    n = strata_sparse_attention_workspace_bytes(dims)
    if n == 0:
        raise StrataError(STRATA_ERR_INVALID_ARG, "attention workspace")
    return torch.empty(n, dtype=torch.uint8, device=device)


def workspace(dims, device="cuda"):
    """A torch uint8 buffer of strata_moe_workspace_bytes(dims) bytes."""
    import torch
    n = strata_moe_workspace_bytes(dims)
    if n == 0:
        raise StrataError(STRATA_ERR_INVALID_ARG, "workspace")
    return torch.empty(n, dtype=torch.uint8, device=device)
