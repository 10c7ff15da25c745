"""Pins for the sparse-attention oracle (CPU only): attention over the
indexer-selected KV rows must equal dense attention with a mask that admits
only those rows (the way the pages say llama.cpp computes it), computed here
by torch's scaled_dot_product_attention in float64, plus closed forms."""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from moe_inputs import bf16_bits, make_attention
from oracle.sparse_attention import sparse_attention


def _f64(bits):
    return torch.from_numpy((bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64))


def dense_masked(q, k, v, idx):
    """Dense attention over the whole cache with a boolean mask (torch SDPA)."""
    T, Hq, D = q.shape
    L, Hkv, _ = k.shape
    grp = Hq // Hkv
    qt = _f64(q).permute(1, 0, 2)                                  # [Hq][T][D]
    kt = _f64(k).permute(1, 0, 2).repeat_interleave(grp, dim=0)    # [Hq][L][D]
    vt = _f64(v).permute(1, 0, 2).repeat_interleave(grp, dim=0)
    mask = torch.zeros((T, L), dtype=torch.bool)
    for t in range(T):
        sel = idx[t][idx[t] >= 0]
        mask[t, torch.from_numpy(sel.astype(np.int64))] = True
    o = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask.unsqueeze(0))
    return o.permute(1, 0, 2).numpy()


@pytest.mark.parametrize("T,L,Hq,Hkv,D,P", [(3, 300, 8, 2, 64, 64), (2, 1000, 4, 4, 32, 200),
                                            (1, 40, 6, 1, 16, 40)])
def test_matches_dense_masked_attention(T, L, Hq, Hkv, D, P):
    a = make_attention(T, L, Hq, Hkv, D, P, seed=T + L)
    got = sparse_attention(a["q"], a["k"], a["v"], a["idx"])
    ref = dense_masked(a["q"], a["k"], a["v"], a["idx"])
    assert np.max(np.abs(got - ref)) <= 1e-12


def test_all_positions_is_dense_attention():
    a = make_attention(2, 50, 4, 2, 16, 50, seed=3)
    assert np.all(np.sort(a["idx"], axis=1) == np.arange(50))
    got = sparse_attention(a["q"], a["k"], a["v"], a["idx"])
    T, Hq, D = a["q"].shape
    qt = _f64(a["q"]).permute(1, 0, 2)
    kt = _f64(a["k"]).permute(1, 0, 2).repeat_interleave(2, dim=0)
    vt = _f64(a["v"]).permute(1, 0, 2).repeat_interleave(2, dim=0)
    ref = F.scaled_dot_product_attention(qt, kt, vt).permute(1, 0, 2).numpy()
    assert np.max(np.abs(got - ref)) <= 1e-12


def test_order_and_padding_do_not_matter():
    a = make_attention(2, 500, 4, 2, 32, 100, seed=5, n_valid=np.array([100, 37]))
    assert np.all(a["idx"][1, 37:] == -1)
    base = sparse_attention(a["q"], a["k"], a["v"], a["idx"])
    rng = np.random.default_rng(0)
    shuffled = np.stack([rng.permutation(r) for r in a["idx"]])    # -1 slots anywhere
    assert np.max(np.abs(sparse_attention(a["q"], a["k"], a["v"], shuffled) - base)) <= 1e-12


def test_closed_forms():
    a = make_attention(2, 64, 4, 2, 16, 8, seed=7)
    # one selected position: the output is that row of V
    one = np.full_like(a["idx"], -1)
    one[:, 0] = [5, 9]
    o = sparse_attention(a["q"], a["k"], a["v"], one)
    v = _f64(a["v"]).numpy()
    assert np.array_equal(o[0], v[5].repeat(2, axis=0))
    assert np.array_equal(o[1], v[9].repeat(2, axis=0))
    # zero queries: equal weights, the mean of the selected rows (per KV head)
    zq = np.zeros_like(a["q"])
    o = sparse_attention(zq, a["k"], a["v"], a["idx"])
    mean = v[a["idx"][0]].mean(axis=0)                              # [Hkv][D]
    assert np.max(np.abs(o[0] - mean.repeat(2, axis=0))) <= 1e-12
    # no selected position: zero output
    none = np.full_like(a["idx"], -1)
    assert not np.any(sparse_attention(a["q"], a["k"], a["v"], none))


def test_query_heads_use_their_own_kv_head():
    """V rows constant per KV head: query head h must return the constant of
    KV head h // (Hq / Hkv)."""
    T, L, Hq, Hkv, D = 1, 20, 8, 4, 16
    a = make_attention(T, L, Hq, Hkv, D, 10, seed=9)
    v = np.zeros((L, Hkv, D), np.float32)
    for hk in range(Hkv):
        v[:, hk, :] = hk + 1
    o = sparse_attention(a["q"], a["k"], bf16_bits(v), a["idx"])
    for h in range(Hq):
        assert np.max(np.abs(o[0, h] - (h // 2 + 1))) <= 1e-12
