"""fp64 oracle for attention over the KV-cache rows an indexer selected --
TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module; the CUDA library never calls it and it
never calls the library.

The pages: the model's attention is sparse; an indexer picks about 2000
positions for every query, and where llama.cpp still builds a full mask and
runs dense flash attention, Strata's own kernel reads only the selected
KV-cache rows (kongchang.com "两天移植，预填充提速8倍：Strata引擎实测",
section "Strata快在哪", attention paragraph; KV cache background in the note
that follows the "为什么预填充比解码更重要" section).  Both compute the same
thing; this is its plain definition, per query token t and query head h:

    hk      = h // (Hq // Hkv)                   (grouped-query heads share a KV head)
    P_t     = { idx[t][j] : idx[t][j] >= 0 }     (the selected positions; -1 = unused slot)
    s_p     = scale * sum_d q[t][h][d] * K[p][hk][d]        for p in P_t
    o[t][h] = sum_{p in P_t} exp(s_p - max s) V[p][hk] / sum_{p in P_t} exp(s_p - max s)

with scale = 1 / sqrt(D) unless given.  The pages fix no head counts, head
size, precision or index format; those are this library's readings.
Inputs are bf16 bit patterns (uint16) for q, K, V and int32 for idx; the
result is fp64.
"""

from __future__ import annotations

from typing import Optional

import numpy as np


def _bf16(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32) \
        .astype(np.float64)


def sparse_attention(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
                     idx: np.ndarray, scale: Optional[float] = None) -> np.ndarray:
    """q [T][Hq][D], k_cache / v_cache [L][Hkv][D] (bf16 bits), idx [T][P]
    int32 (-1 = unused) -> o [T][Hq][D] fp64.  A query with no selected
    position gets o = 0."""
    qf = _bf16(q)
    kf = _bf16(k_cache)
    vf = _bf16(v_cache)
    T, Hq, D = qf.shape
    L, Hkv, _ = kf.shape
    if Hq % Hkv:
        raise ValueError("query heads must be a multiple of KV heads")
    grp = Hq // Hkv
    sc = 1.0 / np.sqrt(D) if scale is None else float(scale)
    out = np.zeros((T, Hq, D), np.float64)
    for t in range(T):
        sel = idx[t][idx[t] >= 0].astype(np.int64)
        if sel.size == 0:
            continue
        if np.any(sel >= L):
            raise IndexError("selected position beyond the cache")
        for h in range(Hq):
            hk = h // grp
            keys = kf[sel, hk, :]                     # [P][D]
            vals = vf[sel, hk, :]
            s = sc * (keys @ qf[t, h, :])             # [P]
            m = np.max(s)
            e = np.exp(s - m)
            out[t, h, :] = (e @ vals) / np.sum(e)
    return out
