"""fp64 CPU oracle for the MoE expert layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it, and it
never calls the CUDA library: the two share no code.  See ``oracle_moe.cpp``
for the definitions and the passages they follow.

All functions take numpy arrays in the layer's storage formats (bf16 / fp16 as
uint16 bit patterns, packed int4 as uint8) and return fp64 results.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle_moe.cpp")
_LIB_PATH = os.path.join(_HERE, "liboracle_moe.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle (g++ -O2 -fopenmp) next to its source."""
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC",
                               "-shared", _SRC, "-o", tmp])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        L = _lib
        vp, i64 = ctypes.c_void_p, ctypes.c_int64
        L.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_f64.restype = ctypes.c_double
        L.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.oracle_f16_to_f64.restype = ctypes.c_double
        L.oracle_dequant_rows.argtypes = [vp, vp, i64, i64, i64, i64, i64, vp]
        L.oracle_router_logits.argtypes = [vp, vp, vp, i64, i64, i64, vp]
        L.oracle_topk_softmax.argtypes = [vp, i64, i64, i64, vp, vp]
        L.oracle_permute.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp]
        L.oracle_expert_ffn.argtypes = [vp] * 7 + [i64] * 4 + [vp, vp]
        L.oracle_moe_forward.argtypes = [vp] * 9 + [i64] * 6 + [vp, i64, vp, vp, vp, vp, vp, vp, vp]
        ci = ctypes.c_int
        L.oracle_combine.argtypes = [vp, ci, vp, vp, i64, i64, i64, vp]
        L.oracle_gate_up_rows.argtypes = [vp, vp, i64, vp, vp, vp, vp, i64, i64, i64, vp]
        L.oracle_down_rows.argtypes = [vp, ci, vp, i64, vp, vp, vp, i64, i64, i64, vp]
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def bf16_to_f64(b: int) -> float:
    return lib().oracle_bf16_to_f64(int(b))


def f16_to_f64(h: int) -> float:
    return lib().oracle_f16_to_f64(int(h))


def dequant_rows(q, s, K: int, G: int, row0: int = 0, nrows: Optional[int] = None):
    """Rows of one packed matrix q [N][K/2], s [N][K/G] -> fp64 [nrows][K]."""
    q = _c(q, np.uint8).reshape(-1, K // 2)
    s = _c(s, np.uint16).reshape(-1, K // G)
    N = q.shape[0]
    nrows = N - row0 if nrows is None else nrows
    out = np.empty((nrows, K), np.float64)
    lib().oracle_dequant_rows(_p(q), _p(s), N, K, G, row0, nrows, _p(out))
    return out


def router_logits(x, w_router, bias=None):
    x = _c(x, np.uint16)
    w_router = _c(w_router, np.uint16)
    T, d = x.shape
    E = w_router.shape[1]
    b = None if bias is None else _c(bias, np.float32)
    out = np.empty((T, E), np.float64)
    lib().oracle_router_logits(_p(x), _p(w_router), _p(b), T, d, E, _p(out))
    return out


def topk_softmax(logits, k: int):
    logits = _c(logits, np.float64)
    T, E = logits.shape
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    lib().oracle_topk_softmax(_p(logits), T, E, k, _p(ids), _p(w))
    return ids, w


def permute(ids, E: int):
    ids = _c(ids, np.int32)
    T, k = ids.shape
    S = T * k
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    sorted_token = np.empty(S, np.int32)
    slot_row = np.empty(S, np.int32)
    lib().oracle_permute(_p(ids), T, k, E, _p(counts), _p(offsets),
                         _p(sorted_token), _p(slot_row))
    return counts, offsets, sorted_token, slot_row


def _weights(inp):
    return [_c(inp[n], np.uint8 if n.endswith("_q") else np.uint16)
            for n in ("gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s")]


def moe_forward(inp, k: int, group: int, tokens=None, ids=None, w=None,
                want_intermediates: bool = False):
    """The whole layer for `tokens` (default: all) of the input dict produced
    by ``moe_inputs``.  Optional ``ids``/``w`` ([n_sub][k]) replace the
    oracle's own routing.  Returns dict(y, ids, w[, h, o])."""
    x = _c(inp["x"], np.uint16)
    wr = _c(inp["w_router"], np.uint16)
    T, d = x.shape
    E = wr.shape[1]
    gq, gs, uq, us, dq, ds = _weights(inp)
    n = gq.shape[1]
    bias = inp.get("bias")
    b = None if bias is None else _c(bias, np.float32)
    tok = np.arange(T, dtype=np.int32) if tokens is None else _c(tokens, np.int32)
    m = tok.shape[0]
    ids_in = None if ids is None else _c(ids, np.int32).reshape(m, k)
    w_in = None if w is None else _c(w, np.float64).reshape(m, k)
    y = np.empty((m, d), np.float64)
    ids_out = np.empty((m, k), np.int32)
    w_out = np.empty((m, k), np.float64)
    h = np.empty((m, k, n), np.float64) if want_intermediates else None
    o = np.empty((m, k, d), np.float64) if want_intermediates else None
    lib().oracle_moe_forward(_p(x), _p(wr), _p(b), _p(gq), _p(gs), _p(uq), _p(us),
                             _p(dq), _p(ds), T, d, E, k, n, group, _p(tok), m,
                             _p(ids_in), _p(w_in), _p(y), _p(ids_out), _p(w_out),
                             _p(h), _p(o))
    res = dict(y=y, ids=ids_out, w=w_out)
    if want_intermediates:
        res.update(h=h, o=o)
    return res


def combine(rows, w, slot_row, T: int, k: int, rows_fp16: bool = False):
    """rows: [S][d] bf16 bits (or fp16 bits with rows_fp16)."""
    rows = _c(rows, np.uint16)
    d = rows.shape[1]
    wv = None if w is None else _c(w, np.float64)
    sr = _c(slot_row, np.int32)
    y = np.empty((T, d), np.float64)
    lib().oracle_combine(_p(rows), int(rows_fp16), _p(wv), _p(sr), T, k, d, _p(y))
    return y


def gate_up_rows(a, experts, inp, group: int):
    a = _c(a, np.uint16)
    R, d = a.shape
    ex = _c(experts, np.int32)
    gq, gs, uq, us, _, _ = _weights(inp)
    n = gq.shape[1]
    out = np.empty((R, n), np.float64)
    lib().oracle_gate_up_rows(_p(a), _p(ex), R, _p(gq), _p(gs), _p(uq), _p(us),
                              d, n, group, _p(out))
    return out


def down_rows(a, experts, inp, group: int, scale=None, a_fp16: bool = False):
    """a: [R][n] bf16 bits (or fp16 bits with a_fp16)."""
    a = _c(a, np.uint16)
    R, n = a.shape
    ex = _c(experts, np.int32)
    _, _, _, _, dq, ds = _weights(inp)
    d = dq.shape[1]
    sc = None if scale is None else _c(scale, np.float32)
    out = np.empty((R, d), np.float64)
    lib().oracle_down_rows(_p(a), int(a_fp16), _p(ex), R, _p(dq), _p(ds), _p(sc), d, n,
                           group, _p(out))
    return out
