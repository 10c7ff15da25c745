"""Shared helpers for the GPU parity tests: upload seeded inputs, call the
library through its C ABI, and compare with the fp64 oracle."""

from __future__ import annotations

import numpy as np
import torch

import local_moe_route_b200 as sm
from moe_inputs import chunk_sizes, make_custom, make_inputs
from parity_metrics import gate_error, half_ulp, raw_error, rms, round_to, vs_rounded  # noqa: F401

_WEIGHTS = ("gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s")


def dev_tensor(a: np.ndarray, device) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.to(device)


def bf16_dev(bits: np.ndarray, device) -> torch.Tensor:
    return dev_tensor(bits, device).view(torch.bfloat16)


def bf16_host(t: torch.Tensor) -> np.ndarray:
    """bf16 device tensor -> uint16 bit patterns on the host."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f16_host(t: torch.Tensor) -> np.ndarray:
    """fp16 device tensor -> uint16 bit patterns on the host."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f16_to_f64(bits: np.ndarray) -> np.ndarray:
    return bits.view(np.float16).astype(np.float64)


class Layer:
    """A MoE layer's inputs resident on the device."""

    def __init__(self, inp: dict, dims: dict, device):
        self.inp = inp
        self.dims = dict(dims)
        self.device = device
        self.x = bf16_dev(inp["x"], device)
        self.w_router = bf16_dev(inp["w_router"], device)
        self.bias = None if inp.get("bias") is None else dev_tensor(inp["bias"], device)
        self.w = {n: dev_tensor(inp[n], device) for n in _WEIGHTS}

    @classmethod
    def workload(cls, wl, device, T=None):
        return cls(make_inputs(wl, T), wl.dims(T), device)

    @classmethod
    def custom(cls, device, **kw):
        dims = {k: kw[k] for k in ("T", "d", "E", "k", "n", "group")}
        return cls(make_custom(**kw), dims, device)

    def q4(self, name):
        return (self.w[name + "_q"], self.w[name + "_s"])

    def dims_T(self, T):
        d = dict(self.dims)
        d["T"] = T
        return d

    # ------------------------------------------------------------------ calls
    def route(self, x=None, T=None):
        x = self.x if x is None else x
        T = x.shape[0] if T is None else T
        dims = self.dims_T(T)
        k, E = dims["k"], dims["E"]
        ids = torch.empty((T, k), dtype=torch.int32, device=self.device)
        w = torch.empty((T, k), dtype=torch.float32, device=self.device)
        logits = torch.empty((T, E), dtype=torch.float32, device=self.device)
        ws = sm.workspace(dims, self.device)
        sm.check(sm.strata_moe_route(x, self.w_router, self.bias, dims, ids, w, logits, ws),
                 "route")
        return ids, w, logits

    def permute(self, ids, T=None):
        T = ids.shape[0] if T is None else T
        dims = self.dims_T(T)
        E, S = dims["E"], T * dims["k"]
        counts = torch.empty(E, dtype=torch.int32, device=self.device)
        offsets = torch.empty(E + 1, dtype=torch.int32, device=self.device)
        st = torch.empty(max(S, 1), dtype=torch.int32, device=self.device)
        sr = torch.empty(max(S, 1), dtype=torch.int32, device=self.device)
        ws = sm.workspace(dims, self.device)
        sm.check(sm.strata_moe_permute(ids, dims, counts, offsets, st, sr, ws), "permute")
        return counts, offsets, st[:S], sr[:S]

    def gate_up(self, x, sorted_token, offsets, T):
        dims = self.dims_T(T)
        S = T * dims["k"]
        h = torch.empty((S, dims["n"]), dtype=torch.float16, device=self.device)
        ws = sm.workspace(dims, self.device)
        sm.check(sm.strata_moe_expert_gemm_q4(sm.STRATA_OP_GATE_UP_SWIGLU, x, sorted_token,
                                              offsets, self.q4("gate"), self.q4("up"), None,
                                              dims, h, ws), "gate_up")
        return h

    def down(self, h, offsets, T, row_scale=None):
        dims = self.dims_T(T)
        S = T * dims["k"]
        out = torch.empty((S, dims["d"]), dtype=torch.float16, device=self.device)
        ws = sm.workspace(dims, self.device)
        sm.check(sm.strata_moe_expert_gemm_q4(sm.STRATA_OP_DOWN, h, None, offsets,
                                              self.q4("down"), None, row_scale, dims, out, ws),
                 "down")
        return out

    def combine(self, rows, w, slot_row, T):
        dims = self.dims_T(T)
        y = torch.empty((T, dims["d"]), dtype=torch.bfloat16, device=self.device)
        sm.check(sm.strata_moe_combine(rows, w, slot_row, dims, y), "combine")
        return y

    def forward(self, x=None, ws=None, want_routes=True):
        x = self.x if x is None else x
        T = x.shape[0]
        dims = self.dims_T(T)
        y = torch.empty((T, dims["d"]), dtype=torch.bfloat16, device=self.device)
        ids = torch.empty((T, dims["k"]), dtype=torch.int32, device=self.device) if want_routes else None
        w = torch.empty((T, dims["k"]), dtype=torch.float32, device=self.device) if want_routes else None
        ws = sm.workspace(dims, self.device) if ws is None else ws
        sm.check(sm.strata_moe_forward(x, self.w_router, self.bias, self.q4("gate"),
                                       self.q4("up"), self.q4("down"), dims, y, ids, w, ws),
                 "forward")
        return y, ids, w

    def forward_chunked(self, chunk):
        ys, idss = [], []
        for T0, n in zip(np.cumsum([0] + chunk_sizes(self.dims["T"], chunk)[:-1]),
                         chunk_sizes(self.dims["T"], chunk)):
            y, ids, _ = self.forward(self.x[int(T0):int(T0) + n])
            ys.append(y)
            idss.append(ids)
        return torch.cat(ys), torch.cat(idss)


def assert_device_ok():
    torch.cuda.synchronize()
    assert sm.strata_moe_device_status() == sm.STRATA_OK


def near_tie_tokens(logits: np.ndarray, k: int, rel: float = 1e-4) -> np.ndarray:
    """Tokens whose k-th and (k+1)-th largest logits lie closer than rel*RMS."""
    if logits.shape[1] <= k:
        return np.zeros(logits.shape[0], bool)
    srt = -np.sort(-logits, axis=1)
    gap = srt[:, k - 1] - srt[:, k]
    return gap < rel * rms(logits)
