"""Pins for the fp64 oracle (CPU only).

Each test checks the oracle against something other than itself: library
conversions over every bit pattern, brute-force sorting in Python, closed
forms on constructed inputs, invariants of a permutation, and a dense SwiGLU
FFN computed with torch float64 matmuls on weights unpacked here, in numpy,
from the documented layout.  A dropped term, a flipped sign, a swapped nibble
or a transposed operand in the oracle fails at least one of them.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from moe_inputs import WORKLOADS, bf16_bits, make_custom, make_inputs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---------------------------------------------------------------- helpers
def unpack_int4(q: np.ndarray) -> np.ndarray:
    """Independent unpack: [..., K/2] bytes -> [..., K] int (low nibble first)."""
    lo = (q & 0xF).astype(np.int64)
    hi = (q >> 4).astype(np.int64)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(q.shape[:-1] + (q.shape[-1] * 2,), np.int64)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def dense_weights(q: np.ndarray, s: np.ndarray, G: int) -> torch.Tensor:
    """q [N][K/2], s [N][K/G] fp16 bits -> fp64 [N][K] via numpy/torch only."""
    vals = unpack_int4(q).astype(np.float64)
    sc = s.view(np.float16).astype(np.float64)
    return torch.from_numpy(vals * np.repeat(sc, G, axis=-1))


def bf16_to_t64(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.copy()).view(torch.bfloat16).to(torch.float64)


# ---------------------------------------------------------------- scalar decoders
def test_bf16_decoder_all_patterns():
    bits = np.arange(65536, dtype=np.uint16)
    ref = bf16_to_t64(bits).numpy()
    got = np.array([oracle.bf16_to_f64(b) for b in bits])
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.all(np.isnan(got[np.isnan(ref)]))


def test_f16_decoder_all_patterns():
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_to_f64(b) for b in bits])
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isinf(got), np.isinf(ref))
    assert np.all(np.isnan(got[np.isnan(ref)]))


# ---------------------------------------------------------------- int4 layout
def _nibble_table():
    rows = []
    with open(os.path.join(GOLDEN, "int4_nibbles.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                b, lo, hi = line.split()
                rows.append((int(b, 16), int(lo), int(hi)))
    return rows


def test_int4_nibble_golden_table():
    rows = _nibble_table()
    q = np.array([[b for b, _, _ in rows]], np.uint8)           # one row, K = 2*len
    K = q.shape[1] * 2
    one = np.float16(1.0).view(np.uint16)
    s = np.full((1, 1), one, np.uint16)                          # group = K
    w = oracle.dequant_rows(q, s, K, K)[0]
    expect = np.array([v for _, lo, hi in rows for v in (lo, hi)], np.float64)
    assert np.array_equal(w, expect)


def test_dequant_matches_independent_unpack():
    inp = make_custom(T=1, d=256, E=2, k=1, n=128, group=32, seed=11)
    for name, K in (("gate", 256), ("down", 128)):
        q = inp[name + "_q"].reshape(-1, K // 2)
        s = inp[name + "_s"].reshape(-1, K // 32)
        got = oracle.dequant_rows(q, s, K, 32)
        ref = dense_weights(q, s, 32).numpy()
        assert np.array_equal(got, ref)


def test_dequant_values_are_q_times_s_range():
    inp = make_custom(T=1, d=128, E=1, k=1, n=128, group=64, seed=12,
                      s_lo=0.5, s_hi=0.5)
    w = oracle.dequant_rows(inp["gate_q"][0], inp["gate_s"][0], 128, 64)
    # scale 0.5 exactly: every weight is an integer in [-8, 7] times 0.5
    assert np.array_equal(w * 2, np.round(w * 2))
    assert w.min() == -4.0 and w.max() == 3.5


# ---------------------------------------------------------------- router
def test_router_logits_vs_float64_matmul():
    inp = make_custom(T=37, d=256, E=24, k=3, n=128, group=64, seed=13, zipf=1.1)
    got = oracle.router_logits(inp["x"], inp["w_router"], inp["bias"])
    ref = (bf16_to_t64(inp["x"]) @ bf16_to_t64(inp["w_router"])).numpy() + \
        inp["bias"].astype(np.float64)[None, :]
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-13)


def test_router_bias_is_added_to_logits():
    inp = make_custom(T=5, d=64, E=8, k=2, n=64, group=64, seed=14)
    base = oracle.router_logits(inp["x"], inp["w_router"], None)
    bias = np.arange(8, dtype=np.float32) * np.float32(0.25)
    got = oracle.router_logits(inp["x"], inp["w_router"], bias)
    assert np.array_equal(got - base, np.broadcast_to(bias.astype(np.float64), got.shape))


# ---------------------------------------------------------------- top-k + softmax
def brute_topk(l, k):
    order = sorted(range(len(l)), key=lambda e: (-l[e], e))
    return order[:k]


@pytest.mark.parametrize("T,E,k", [(64, 16, 2), (33, 8, 8), (50, 32, 5), (7, 5, 1)])
def test_topk_vs_brute_force(T, E, k):
    rng = np.random.default_rng(T * 100 + E)
    logits = rng.standard_normal((T, E))
    ids, w = oracle.topk_softmax(logits, k)
    for t in range(T):
        assert list(ids[t]) == brute_topk(list(logits[t]), k)


def test_topk_ties_lowest_index_wins():
    # duplicated router columns produce exactly equal logits
    rng = np.random.default_rng(5)
    x = bf16_bits(rng.standard_normal((20, 64), dtype=np.float32))
    col = bf16_bits(rng.standard_normal((64, 1), dtype=np.float32))
    other = bf16_bits(rng.standard_normal((64, 3), dtype=np.float32) * np.float32(0.001))
    # experts 1, 3, 6 are copies of the same column; the rest tiny
    wr = np.empty((64, 8), np.uint16)
    wr[:, [0, 2, 4]] = other
    wr[:, [5, 7]] = other[:, :2]
    wr[:, [1, 3, 6]] = col
    logits = oracle.router_logits(x, wr)
    ids, w = oracle.topk_softmax(logits, 2)
    for t in range(20):
        assert logits[t, 1] == logits[t, 3] == logits[t, 6]
        assert list(ids[t]) == brute_topk(list(logits[t]), 2)
        if logits[t, 1] > logits[t, [0, 2, 4, 5, 7]].max():
            assert list(ids[t]) == [1, 3]
            assert w[t, 0] == w[t, 1] == 0.5
    # an all-equal row picks 0..k-1 in order
    ids, w = oracle.topk_softmax(np.zeros((1, 9)), 4)
    assert list(ids[0]) == [0, 1, 2, 3]
    assert np.all(w == 0.25)


def test_softmax_closed_forms():
    rng = np.random.default_rng(6)
    logits = rng.standard_normal((40, 12)) * 3
    ids, w = oracle.topk_softmax(logits, 1)
    assert np.all(w == 1.0)
    ids, w = oracle.topk_softmax(logits, 2)
    for t in range(40):
        l0, l1 = logits[t, ids[t, 0]], logits[t, ids[t, 1]]
        assert math.isclose(w[t, 0], 1.0 / (1.0 + math.exp(l1 - l0)), rel_tol=1e-14)
        assert math.isclose(w[t, 1], 1.0 / (1.0 + math.exp(l0 - l1)), rel_tol=1e-14)
    ids, w = oracle.topk_softmax(logits, 7)
    np.testing.assert_allclose(w.sum(1), 1.0, rtol=0, atol=1e-14)
    assert np.all(np.diff(w, axis=1) <= 0)
    # equals softmax over all E renormalised to the chosen k
    full = np.exp(logits - logits.max(1, keepdims=True))
    full /= full.sum(1, keepdims=True)
    sel = np.take_along_axis(full, ids.astype(np.int64), 1)
    np.testing.assert_allclose(w, sel / sel.sum(1, keepdims=True), rtol=1e-13)


# ---------------------------------------------------------------- permutation
@pytest.mark.parametrize("T,E,k", [(64, 16, 2), (1, 4, 4), (100, 3, 1), (31, 64, 8)])
def test_permute_invariants_and_stable_sort(T, E, k):
    rng = np.random.default_rng(T + E + k)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    counts, offsets, sorted_token, slot_row = oracle.permute(ids, E)
    S = T * k
    assert counts.sum() == S
    assert offsets[0] == 0 and offsets[-1] == S
    assert np.all(np.diff(offsets) == counts)
    assert np.array_equal(np.sort(slot_row), np.arange(S))          # bijection
    # independent definition: stable argsort of the flattened expert ids
    order = np.argsort(ids.reshape(-1), kind="stable")
    assert np.array_equal(sorted_token, (order // k).astype(np.int32))
    inv = np.empty(S, np.int64)
    inv[order] = np.arange(S)
    assert np.array_equal(slot_row, inv.astype(np.int32))
    for e in range(E):
        seg = sorted_token[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(seg) > 0)     # ascending; a token uses e at most once
    flat = ids.reshape(-1)
    assert np.all(flat[np.arange(S)] == np.searchsorted(offsets, slot_row, side="right") - 1)


# ---------------------------------------------------------------- FFN and full layer
def test_zero_scales_give_zero_output():
    inp = make_custom(T=9, d=128, E=4, k=2, n=64, group=32, seed=21)
    for n_ in ("gate_s", "up_s", "down_s"):
        inp[n_] = np.zeros_like(inp[n_])
    res = oracle.moe_forward(inp, k=2, group=32)
    assert np.all(res["y"] == 0.0)
    inp2 = make_custom(T=9, d=128, E=4, k=2, n=64, group=32, seed=21)
    inp2["down_s"] = np.zeros_like(inp2["down_s"])
    assert np.all(oracle.moe_forward(inp2, k=2, group=32)["y"] == 0.0)


def _dense_swiglu_ffn(inp, e, G):
    x = bf16_to_t64(inp["x"])
    Wg = dense_weights(inp["gate_q"][e], inp["gate_s"][e], G)     # [n][d]
    Wu = dense_weights(inp["up_q"][e], inp["up_s"][e], G)
    Wd = dense_weights(inp["down_q"][e], inp["down_s"][e], G)     # [d][n]
    g = x @ Wg.T
    u = x @ Wu.T
    h = torch.nn.functional.silu(g) * u
    return (h @ Wd.T).numpy(), h.numpy()


def test_one_expert_top1_equals_dense_swiglu():
    inp = make_custom(T=16, d=256, E=1, k=1, n=128, group=64, seed=22)
    res = oracle.moe_forward(inp, k=1, group=64, want_intermediates=True)
    y_ref, h_ref = _dense_swiglu_ffn(inp, 0, 64)
    assert np.all(res["ids"] == 0) and np.all(res["w"] == 1.0)
    np.testing.assert_allclose(res["y"], y_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(res["h"][:, 0, :], h_ref, rtol=1e-10, atol=1e-12)


def test_full_layer_vs_dense_mixture():
    # the layer equals sum_j w_j * FFN_{e_j}(x) with dense fp64 FFNs
    inp = make_custom(T=12, d=128, E=6, k=3, n=64, group=32, seed=23, zipf=1.1)
    res = oracle.moe_forward(inp, k=3, group=32)
    logits = (bf16_to_t64(inp["x"]) @ bf16_to_t64(inp["w_router"])).numpy() + \
        inp["bias"].astype(np.float64)
    ffn = [_dense_swiglu_ffn(inp, e, 32)[0] for e in range(6)]
    for t in range(12):
        sel = brute_topk(list(logits[t]), 3)
        assert list(res["ids"][t]) == sel
        z = np.exp(logits[t, sel] - logits[t, sel[0]])
        w = z / z.sum()
        np.testing.assert_allclose(res["w"][t], w, rtol=1e-12)
        y = sum(w[j] * ffn[sel[j]][t] for j in range(3))
        np.testing.assert_allclose(res["y"][t], y, rtol=1e-9, atol=1e-10)


def test_gate_up_and_down_rows_vs_dense():
    inp = make_custom(T=10, d=128, E=3, k=1, n=64, group=64, seed=24)
    ex = np.array([0, 2, 1, 2, 0, 1, 1, 2, 0, 0], np.int32)
    h = oracle.gate_up_rows(inp["x"], ex, inp, 64)
    hb = bf16_bits(h.astype(np.float32))
    scale = np.linspace(0.5, 2.0, 10).astype(np.float32)
    o = oracle.down_rows(hb, ex, inp, 64, scale)
    x = bf16_to_t64(inp["x"])
    for r in range(10):
        e = int(ex[r])
        Wg = dense_weights(inp["gate_q"][e], inp["gate_s"][e], 64)
        Wu = dense_weights(inp["up_q"][e], inp["up_s"][e], 64)
        Wd = dense_weights(inp["down_q"][e], inp["down_s"][e], 64)
        hr = torch.nn.functional.silu(x[r] @ Wg.T) * (x[r] @ Wu.T)
        np.testing.assert_allclose(h[r], hr.numpy(), rtol=1e-10, atol=1e-12)
        orr = (bf16_to_t64(hb[r:r + 1])[0] @ Wd.T) * float(scale[r])
        np.testing.assert_allclose(o[r], orr.numpy(), rtol=1e-10, atol=1e-12)


def test_down_rows_and_combine_accept_fp16():
    rng = np.random.default_rng(28)
    inp = make_custom(T=4, d=128, E=2, k=1, n=64, group=32, seed=29)
    h16 = (rng.standard_normal((5, 64)) * 3).astype(np.float16)
    ex = np.array([1, 0, 1, 1, 0], np.int32)
    o = oracle.down_rows(h16.view(np.uint16), ex, inp, 32, a_fp16=True)
    for r in range(5):
        Wd = dense_weights(inp["down_q"][ex[r]], inp["down_s"][ex[r]], 32)
        ref = Wd @ torch.from_numpy(h16[r].astype(np.float64))
        np.testing.assert_allclose(o[r], ref.numpy(), rtol=1e-12, atol=1e-12)
    rows = (rng.standard_normal((6, 64)) * 10).astype(np.float16)
    sr = np.array([5, 0, 3, 1, 2, 4], np.int32)
    w = rng.uniform(0, 1, (3, 2))
    y = oracle.combine(rows.view(np.uint16), w, sr, 3, 2, rows_fp16=True)
    R = rows.astype(np.float64)[sr.reshape(3, 2)]
    np.testing.assert_allclose(y, np.einsum("tk,tkd->td", w, R), rtol=1e-13, atol=1e-14)


def test_combine_vs_einsum():
    rng = np.random.default_rng(25)
    T, k, d = 11, 3, 64
    rows = bf16_bits(rng.standard_normal((T * k, d), dtype=np.float32))
    slot_row = rng.permutation(T * k).astype(np.int32)
    w = rng.uniform(0, 1, (T, k))
    y = oracle.combine(rows, w, slot_row, T, k)
    R = bf16_to_t64(rows).numpy()[slot_row.reshape(T, k)]          # [T][k][d]
    np.testing.assert_allclose(y, np.einsum("tk,tkd->td", w, R), rtol=1e-13, atol=1e-14)
    y1 = oracle.combine(rows, None, slot_row, T, k)
    np.testing.assert_allclose(y1, R.sum(1), rtol=1e-13, atol=1e-14)


def test_worked_example_golden():
    spec = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    dims = spec["dims"]
    d, n, E = dims["d"], dims["n"], dims["E"]
    bf = lambda v: np.float32(v).view(np.uint32) >> 16
    x = np.empty((2, d), np.uint16)
    x[0] = bf(1.0)
    x[1] = bf(-1.0)
    wr = np.empty((d, E), np.uint16)
    wr[:, 0] = bf(0.5)
    wr[:, 1] = bf(-0.5)
    h16 = lambda v: np.float16(v).view(np.uint16)
    gq = np.zeros((E, n, d // 2), np.uint8)
    uq = np.zeros_like(gq)
    gs = np.zeros((E, n, 1), np.uint16)
    us = np.zeros_like(gs)
    dq = np.zeros((E, d, n // 2), np.uint8)
    ds = np.zeros((E, d, 1), np.uint16)
    gq[0, 0], gs[0, 0] = 0x11, h16(0.5)
    uq[0, 0], us[0, 0] = 0x22, h16(0.25)
    dq[0], ds[0] = 0x11, h16(2.0 ** -10)
    gq[1, 0], gs[1, 0] = 0xFF, h16(0.5)
    uq[1, 0], us[1, 0] = 0x88, h16(0.125)
    dq[1], ds[1] = 0x77, h16(2.0 ** -11)
    inp = dict(x=x, w_router=wr, bias=None, gate_q=gq, gate_s=gs, up_q=uq,
               up_s=us, down_q=dq, down_s=ds)
    res = oracle.moe_forward(inp, k=1, group=64)
    exp = spec["expected"]
    assert res["ids"].tolist() == exp["ids"]
    assert res["w"].tolist() == exp["weights"]
    counts, offsets, st, sr = oracle.permute(res["ids"], E)
    assert counts.tolist() == exp["counts"] and offsets.tolist() == exp["offsets"]
    assert st.tolist() == exp["sorted_token"] and sr.tolist() == exp["slot_row"]
    sig32 = 1.0 / (1.0 + math.exp(-32.0))
    np.testing.assert_allclose(res["y"][0], sig32, rtol=1e-15)
    np.testing.assert_allclose(res["y"][1], 7 * sig32, rtol=1e-15)


def test_token_order_equivariance_and_chunking():
    inp = make_custom(T=24, d=128, E=8, k=2, n=64, group=64, seed=26)
    full = oracle.moe_forward(inp, k=2, group=64)
    perm = np.random.default_rng(1).permutation(24)
    inp_p = dict(inp)
    inp_p["x"] = inp["x"][perm]
    res_p = oracle.moe_forward(inp_p, k=2, group=64)
    assert np.array_equal(res_p["y"], full["y"][perm])
    assert np.array_equal(res_p["ids"], full["ids"][perm])
    a = oracle.moe_forward(inp, k=2, group=64, tokens=np.arange(0, 10))
    b = oracle.moe_forward(inp, k=2, group=64, tokens=np.arange(10, 24))
    assert np.array_equal(np.concatenate([a["y"], b["y"]]), full["y"])


def test_supplied_routes_are_used():
    inp = make_custom(T=6, d=128, E=4, k=2, n=64, group=64, seed=27)
    ids = np.array([[3, 0]] * 6, np.int32)
    w = np.array([[0.75, 0.25]] * 6)
    res = oracle.moe_forward(inp, k=2, group=64, ids=ids, w=w, want_intermediates=True)
    y3, _ = _dense_swiglu_ffn(inp, 3, 64)
    y0, _ = _dense_swiglu_ffn(inp, 0, 64)
    np.testing.assert_allclose(res["y"], 0.75 * y3 + 0.25 * y0, rtol=1e-9, atol=1e-10)


def test_workload_table_shapes():
    w = WORKLOADS["tiny"]
    inp = make_inputs(w)
    assert inp["x"].shape == (64, 256) and inp["w_router"].shape == (256, 16)
    assert inp["gate_q"].shape == (16, 128, 128) and inp["down_q"].shape == (16, 256, 64)
    assert inp["gate_s"].shape == (16, 128, 4) and inp["down_s"].shape == (16, 256, 2)
    s = inp["gate_s"].view(np.float16).astype(np.float64)
    assert s.min() >= 0.005 - 1e-5 and s.max() <= 0.02 + 1e-5
    vals = unpack_int4(inp["gate_q"])
    assert vals.min() == -8 and vals.max() == 7
    assert WORKLOADS["large"].S == 61440
    assert make_inputs(w)["x"].tobytes() == inp["x"].tobytes()      # seeded
