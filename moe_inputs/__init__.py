"""Seeded synthetic inputs for the MoE expert layer.

This module only draws random numbers and stores them in the layer's input
formats (bf16 / fp16 bit patterns, packed int4 bytes).  It holds none of the
layer's arithmetic: both the fp64 oracle and the CUDA library consume what it
produces, and neither is imported here.

Workload shapes follow the write-ups of the Strata local MoE engine: a
125B-class MoE with 512 experts and top-10 routing ("Strata快在哪" section of
the kongchang.com benchmark summary, MoE note), prefill processed in
6144-token chunks (same section), a 34,000-token agent prompt ("为什么预填充比
解码更重要" section) and 1 + 3 MTP draft tokens for verification (same page,
decode paragraph).  Group-wise int4 with per-group scales and group sizes
32/64/128 follow the lqnn.cn review, section 3.1.

Draw order for one workload (numpy PCG64, ``default_rng(seed)``):
  x, W_r, gate q, gate s, up q, up s, down q, down s, then the router bias
  (skewed workload only).
* normals are drawn in fp32 and rounded to bf16 (round-to-nearest-even);
* scales are drawn U(lo, hi) in fp32 and rounded to fp16 (numpy astype);
* int4 codes are uniform in [-8, 7]: every packed byte is a uniform draw in
  [0, 255], whose two nibbles are then two independent uniform two's-complement
  int4 values (low nibble = even k, high nibble = odd k).
* the skewed workload's bias is  b_e = -1.1 * ln(r_e)  for a seeded
  permutation r of 1..E, so exp(b_e) is a Zipf(1.1) popularity.
"""

from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np

__all__ = ["Workload", "WORKLOADS", "make_inputs", "make_custom", "bf16_bits",
           "chunk_sizes", "AttnWorkload", "ATTN_WORKLOADS", "make_attention"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int          # tokens
    d: int          # hidden size
    E: int          # experts
    k: int          # experts per token
    n: int          # expert intermediate size
    group: int      # int4 group size along K (both projections)
    s_lo: float     # scale ~ U(s_lo, s_hi)
    s_hi: float
    seed: int
    zipf: float = 0.0    # > 0: per-expert router bias with Zipf(zipf) popularity
    chunk: int = 0       # > 0: processed in chunks of at most this many tokens
    x_std: float = 1.0
    wr_std: float = 0.02

    @property
    def S(self) -> int:
        return self.T * self.k

    def dims(self, T: Optional[int] = None):
        return dict(T=self.T if T is None else T, d=self.d, E=self.E, k=self.k,
                    n=self.n, group=self.group)


_BIG = dict(d=4096, E=512, k=10, n=1024, group=64, s_lo=0.003, s_hi=0.012)

WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", T=64, d=256, E=16, k=2, n=128, group=64,
                     s_lo=0.005, s_hi=0.02, seed=1),
    "default": Workload("default", T=512, d=2048, E=128, k=8, n=768,
                        group=128, s_lo=0.004, s_hi=0.016, seed=2),
    "large": Workload("large", T=6144, seed=3, **_BIG),
    "verify4": Workload("verify4", T=4, seed=4, **_BIG),
    "decode1": Workload("decode1", T=1, seed=5, **_BIG),
    "skewed": Workload("skewed", T=34000, seed=6, zipf=1.1, chunk=6144, **_BIG),
}


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round-to-nearest-even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounding = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + rounding) >> 16).astype(np.uint16)


def _packed_int4(rng: np.random.Generator, rows: int, K: int) -> np.ndarray:
    return rng.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)


def _scales(rng: np.random.Generator, rows: int, K: int, group: int,
            lo: float, hi: float) -> np.ndarray:
    s = rng.uniform(lo, hi, size=(rows, K // group)).astype(np.float32)
    return s.astype(np.float16).view(np.uint16)


def chunk_sizes(T: int, chunk: int):
    """Chunk lengths for a prompt of T tokens processed <= chunk at a time."""
    if chunk <= 0 or T <= chunk:
        return [T]
    sizes = [chunk] * (T // chunk)
    if T % chunk:
        sizes.append(T % chunk)
    return sizes


def make_custom(T: int, d: int, E: int, k: int, n: int, group: int, seed: int,
                s_lo: float = 0.005, s_hi: float = 0.02, zipf: float = 0.0,
                x_std: float = 1.0, wr_std: float = 0.02) -> Dict[str, np.ndarray]:
    """Inputs for arbitrary dims (edge cases); same recipe as the workloads."""
    if d % group or n % group or group % 2:
        raise ValueError("d and n must be multiples of an even group size")
    rng = np.random.default_rng(seed)
    out: Dict[str, np.ndarray] = {}
    out["x"] = bf16_bits(rng.standard_normal((T, d), dtype=np.float32) * np.float32(x_std))
    out["w_router"] = bf16_bits(rng.standard_normal((d, E), dtype=np.float32) * np.float32(wr_std))
    out["gate_q"] = _packed_int4(rng, E * n, d).reshape(E, n, d // 2)
    out["gate_s"] = _scales(rng, E * n, d, group, s_lo, s_hi).reshape(E, n, d // group)
    out["up_q"] = _packed_int4(rng, E * n, d).reshape(E, n, d // 2)
    out["up_s"] = _scales(rng, E * n, d, group, s_lo, s_hi).reshape(E, n, d // group)
    out["down_q"] = _packed_int4(rng, E * d, n).reshape(E, d, n // 2)
    out["down_s"] = _scales(rng, E * d, n, group, s_lo, s_hi).reshape(E, d, n // group)
    if zipf > 0:
        ranks = rng.permutation(E).astype(np.float64) + 1.0
        out["bias"] = (-zipf * np.log(ranks)).astype(np.float32)
    else:
        out["bias"] = None
    return out


def make_inputs(w: Workload, T: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Inputs for a named workload.  ``T`` overrides the token count (the
    weights and router are drawn after x, so they change with T; callers that
    need one model for several token counts slice ``x`` instead)."""
    return make_custom(w.T if T is None else T, w.d, w.E, w.k, w.n, w.group,
                       w.seed, w.s_lo, w.s_hi, w.zipf, w.x_std, w.wr_std)


# --------------------------------------------------------------------------
# Sparse attention over indexer-selected KV-cache rows (kongchang.com
# benchmark summary, section "Strata快在哪", attention paragraph: the indexer
# picks about 2000 positions per query).  The pages give no head counts or
# head size; the workloads use 32 query heads sharing 4 KV heads (groups of
# 8), head size 128, a 34,000-token context (the agent prompt of the
# "为什么预填充比解码更重要" section) and 2048 selected positions per query.
@dataclasses.dataclass(frozen=True)
class AttnWorkload:
    name: str
    T: int          # query tokens
    L: int          # context length (KV-cache rows)
    Hq: int         # query heads
    Hkv: int        # KV heads
    D: int          # head size
    P: int          # selected positions per query (index slots)
    seed: int


ATTN_WORKLOADS: Dict[str, AttnWorkload] = {
    "attn_tiny": AttnWorkload("attn_tiny", T=3, L=300, Hq=8, Hkv=2, D=64, P=64, seed=11),
    "attn_decode1": AttnWorkload("attn_decode1", T=1, L=34000, Hq=32, Hkv=4, D=128, P=2048,
                                 seed=12),
    "attn_verify4": AttnWorkload("attn_verify4", T=4, L=34000, Hq=32, Hkv=4, D=128, P=2048,
                                 seed=13),
}


def make_attention(T: int, L: int, Hq: int, Hkv: int, D: int, P: int, seed: int,
                   n_valid: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """q [T][Hq][D], k / v [L][Hkv][D] as bf16 bits (values ~N(0,1)), idx
    [T][P] int32: per query a seeded draw of distinct positions in [0, L),
    ascending; with n_valid[t] < P the remaining slots hold -1.
    Draw order: q, k, v, then the positions of each query."""
    rng = np.random.default_rng(seed)
    out: Dict[str, np.ndarray] = {}
    out["q"] = bf16_bits(rng.standard_normal((T, Hq, D), dtype=np.float32))
    out["k"] = bf16_bits(rng.standard_normal((L, Hkv, D), dtype=np.float32))
    out["v"] = bf16_bits(rng.standard_normal((L, Hkv, D), dtype=np.float32))
    idx = np.full((T, P), -1, np.int32)
    for t in range(T):
        m = P if n_valid is None else int(n_valid[t])
        idx[t, :m] = np.sort(rng.choice(L, size=m, replace=False)).astype(np.int32)
    out["idx"] = idx
    return out
