"""GPU parity: every step of the layer, through the C ABI, against the fp64
oracle.  Both sides always receive the same seeded inputs: intermediates that
a step consumes (routes, grouped rows, h, per-row outputs) are drawn by the
test or derived by the oracle, never taken from the GPU.

Bars:
  * expert ids, counts, offsets, sorted_token, slot_row: bit-exact.  With
    integer-valued router inputs the fp32 and fp64 logits coincide, so the
    top-k (including its lowest-index tie-break) must match exactly.  With
    real-valued inputs a route may differ only where the oracle's logits lie
    within the fp32 accumulation error of a tie (several answers are correct
    there; none occur for most seeds and the count is reported);
  * router logits within 1e-4 * RMS of the oracle; routing weights within
    1e-5 where the routes agree;
  * floating-point outputs: max(|gpu - oracle| - half_ulp(oracle)) <= 1.5e-2
    * RMS(oracle), i.e. the layer's 1.5e-2 * RMS gate on top of the output
    format's own correct rounding (bf16 y: half an ulp is 2^-8 relative, and
    these outputs peak near 6 RMS, so even an exactly computed y rounded to
    bf16 can miss a gate that does not allow for it).
Large workloads are checked on seeded samples of rows/tokens (the oracle is
per token, so a sample is exact), in the launch configuration of the bench.
"""

import gc

import numpy as np
import pytest
import torch

import local_moe_route_b200 as sm
import oracle
from gpu_helpers import (Layer, assert_device_ok, bf16_host, bf16_to_f64, f16_host, f16_to_f64,
                         gate_error, raw_error, rms, round_to, vs_rounded)
from moe_inputs import WORKLOADS, bf16_bits, chunk_sizes, make_custom

pytestmark = pytest.mark.gpu

GATE = 1.5e-2
_cache = {}


@pytest.fixture(scope="module")
def dev(cuda_dev):
    from local_moe_route_b200 import build
    build.build()
    return cuda_dev


def layer_for(name, dev):
    """One resident workload at a time for the big shapes (3.4 GB each)."""
    if name not in _cache:
        for key in list(_cache):
            if WORKLOADS[key].d >= 4096:
                del _cache[key]
        gc.collect()
        torch.cuda.empty_cache()
        _cache[name] = Layer.workload(WORKLOADS[name], dev)
    return _cache[name]


def sample(n, m, seed):
    if n <= m:
        return np.arange(n)
    return np.sort(np.random.default_rng(seed).choice(n, m, replace=False))


def oracle_routes(L, tokens=None):
    x = L.inp["x"] if tokens is None else L.inp["x"][tokens]
    lg = oracle.router_logits(x, L.inp["w_router"], L.inp.get("bias"))
    ids, w = oracle.topk_softmax(lg, L.dims["k"])
    return lg, ids, w


def routes_agree(ids_gpu, lg_ref, k, tol):
    """GPU routes equal the oracle's except where a tie lies within `tol`
    (the bound on the GPU's logit error) among the first k+1 sorted logits.
    Returns (near-tie tokens, mismatching tokens)."""
    ids_ref, _ = oracle.topk_softmax(lg_ref, k)
    mism = np.any(ids_gpu != ids_ref, axis=1)
    srt = -np.sort(-lg_ref, axis=1)[:, :k + 1]
    ties = np.any(-np.diff(srt, axis=1) <= 2 * tol, axis=1)
    assert not np.any(mism & ~ties), np.nonzero(mism & ~ties)[0][:10]
    return int(ties.sum()), int(mism.sum())


# --------------------------------------------------------------------------- route
@pytest.mark.parametrize("name", ["tiny", "default", "large", "verify4", "decode1"])
def test_route(name, dev):
    L = layer_for(name, dev)
    wl = WORKLOADS[name]
    ids, w, logits = L.route()
    assert_device_ok()
    rows = sample(wl.T, 1024, 7)
    lg_ref, ids_ref, w_ref = oracle_routes(L, rows)
    lg = logits.cpu().numpy().astype(np.float64)[rows]
    err = np.max(np.abs(lg - lg_ref))
    assert err <= 1e-4 * rms(lg_ref) + 1e-6, err
    ids_g = ids.cpu().numpy()[rows]
    ntie, nmis = routes_agree(ids_g, lg_ref, wl.k, err)
    same = np.all(ids_g == ids_ref, axis=1)
    assert np.max(np.abs(w.cpu().numpy()[rows][same] - w_ref[same])) <= 1e-5
    print(f"{name}: logit err {err:.2e}, near-tie tokens {ntie}, differing routes {nmis}")


@pytest.mark.parametrize("T,E,k", [(300, 128, 8), (5, 128, 8), (70, 32, 32), (1, 16, 3)])
def test_route_integer_logits_exact(T, E, k, dev):
    """x and W_r hold small integers (times 2^-4), so every partial sum is exact
    in fp32 and the GPU's logits equal the oracle's bit for bit.  Integer
    logits tie often: the lowest-index rule decides many slots."""
    rng = np.random.default_rng(T + E)
    d = 256
    L = Layer.custom(dev, T=T, d=d, E=E, k=k, n=128, group=64, seed=60)
    L.inp["x"] = bf16_bits(rng.integers(-2, 3, (T, d)).astype(np.float32))
    L.inp["w_router"] = bf16_bits(rng.integers(-2, 3, (d, E)).astype(np.float32) / 16)
    L.x = torch.from_numpy(L.inp["x"]).to(dev).view(torch.bfloat16)
    L.w_router = torch.from_numpy(L.inp["w_router"]).to(dev).view(torch.bfloat16)
    ids, w, logits = L.route()
    assert_device_ok()
    lg_ref, ids_ref, w_ref = oracle_routes(L)
    assert np.array_equal(logits.cpu().numpy().astype(np.float64), lg_ref)
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    assert np.max(np.abs(w.cpu().numpy() - w_ref)) <= 1e-6
    if T * k >= 40:
        srt = -np.sort(-lg_ref, axis=1)[:, :k + 1]
        assert np.any(np.diff(srt, axis=1) == 0), "the case should contain exact ties"


def test_route_skewed_chunk(dev):
    L = layer_for("skewed", dev)
    wl = WORKLOADS["skewed"]
    ids, w, logits = L.route(L.x[:6144])
    rows = sample(6144, 512, 8)
    lg_ref, ids_ref, w_ref = oracle_routes(L, rows)
    lg = logits.cpu().numpy().astype(np.float64)[rows]
    err = np.max(np.abs(lg - lg_ref))
    assert err <= 1e-4 * rms(lg_ref) + 1e-6
    routes_agree(ids.cpu().numpy()[rows], lg_ref, wl.k, err)
    # the Zipf bias makes the load skewed: the busiest expert far above the mean
    counts = np.bincount(ids.cpu().numpy().ravel(), minlength=wl.E)
    assert counts.max() > 8 * counts.mean()


# --------------------------------------------------------------------------- permute
def _check_permute(L, ids_np, T):
    ids = torch.from_numpy(ids_np.astype(np.int32)).to(L.device)
    counts, offsets, st, sr = L.permute(ids, T)
    assert_device_ok()
    c_o, o_o, st_o, sr_o = oracle.permute(ids_np, L.dims["E"])
    assert np.array_equal(counts.cpu().numpy(), c_o)
    assert np.array_equal(offsets.cpu().numpy(), o_o)
    assert np.array_equal(st.cpu().numpy(), st_o)
    assert np.array_equal(sr.cpu().numpy(), sr_o)


@pytest.mark.parametrize("name", ["tiny", "default", "large", "verify4", "decode1"])
def test_permute_oracle_routes(name, dev):
    L = layer_for(name, dev)
    _, ids, _ = oracle_routes(L, sample(WORKLOADS[name].T, 2048, 9))
    _check_permute(L, ids, ids.shape[0])


@pytest.mark.parametrize("T,E,k,pattern", [
    (1, 16, 4, "random"), (3000, 64, 4, "random"), (300, 16, 4, "same"),
    (2500, 1024, 32, "random"), (777, 8, 8, "random"), (4097, 5, 1, "skew"),
    (6144, 512, 10, "random")])
def test_permute_patterns(T, E, k, pattern, dev):
    L = Layer.custom(dev, T=1, d=128, E=E, k=k, n=128, group=64, seed=31)
    rng = np.random.default_rng(T + E)
    if pattern == "same":
        ids = np.tile(np.arange(k), (T, 1))
    elif pattern == "skew":
        ids = np.minimum(rng.geometric(0.7, size=(T, k)) - 1, E - 1)
    else:
        ids = np.argsort(rng.random((T, E)), axis=1)[:, :k]
    _check_permute(L, ids.astype(np.int32), T)


def test_permute_flags_out_of_range_ids(dev):
    L = Layer.custom(dev, T=1, d=128, E=8, k=2, n=128, group=64, seed=32)
    ids = np.array([[0, 1], [8, 2], [3, -1]], np.int32)     # 8 and -1 are out of range
    counts, offsets, st, sr = L.permute(torch.from_numpy(ids).to(dev), 3)
    torch.cuda.synchronize()
    assert sm.strata_moe_device_status() == sm.STRATA_ERR_DEVICE_CHECK
    assert sm.strata_moe_device_status() == sm.STRATA_OK        # cleared
    assert int(offsets[-1]) == 6 and sorted(sr.cpu().tolist()) == list(range(6))


# --------------------------------------------------------------------------- expert GEMMs
GEMM_CASES = [("tiny", 10**9), ("default", 10**9), ("large", 384), ("verify4", 10**9),
              ("decode1", 10**9)]


@pytest.mark.parametrize("name,max_rows", GEMM_CASES)
def test_expert_gemms(name, max_rows, dev):
    L = layer_for(name, dev)
    wl = WORKLOADS[name]
    T, S, k = wl.T, wl.S, wl.k
    # routes and grouping from the oracle; both sides get the same
    _, ids, w = oracle_routes(L)
    counts, offsets, st, sr = oracle.permute(ids, wl.E)
    off_d = torch.from_numpy(offsets).to(dev)
    st_d = torch.from_numpy(st).to(dev)
    expert_of_row = np.searchsorted(offsets, np.arange(S), side="right") - 1
    pick = sample(S, max_rows, 11)
    rng = np.random.default_rng(12)

    # gate/up + SwiGLU on the gathered x rows; twice, bit-identical
    h = L.gate_up(L.x, st_d, off_d, T)
    h2 = L.gate_up(L.x, st_d, off_d, T)
    assert_device_ok()
    assert torch.equal(h, h2), int((h != h2).sum())
    h_ref = oracle.gate_up_rows(L.inp["x"][st[pick]], expert_of_row[pick], L.inp, wl.group)
    e_h = gate_error(f16_to_f64(f16_host(h)[pick]), h_ref, "fp16")
    assert e_h <= GATE, e_h

    # down on seeded fp16 rows shaped like h, with and without the row scale
    h_in = (rng.standard_normal((S, wl.n)) * rms(h_ref)).astype(np.float16)
    h_in_d = torch.from_numpy(h_in).to(dev)
    scale = rng.uniform(0.5, 1.5, S).astype(np.float32)
    rows = L.down(h_in_d, off_d, T)
    rows_s = L.down(h_in_d, off_d, T, row_scale=torch.from_numpy(scale).to(dev))
    assert_device_ok()
    hb = h_in.view(np.uint16)[pick]
    o_ref = oracle.down_rows(hb, expert_of_row[pick], L.inp, wl.group, a_fp16=True)
    e_o = gate_error(f16_to_f64(f16_host(rows)[pick]), o_ref, "fp16")
    assert e_o <= GATE, e_o
    o_ref_s = oracle.down_rows(hb, expert_of_row[pick], L.inp, wl.group, scale[pick], a_fp16=True)
    assert gate_error(f16_to_f64(f16_host(rows_s)[pick]), o_ref_s, "fp16") <= GATE

    # combine of seeded fp16 rows with the oracle's weights and slot rows
    rows_in = (rng.standard_normal((S, wl.d)) * 2).astype(np.float16)
    y = L.combine(torch.from_numpy(rows_in).to(dev),
                  torch.from_numpy(w.astype(np.float32)).to(dev),
                  torch.from_numpy(sr).to(dev), T)
    assert_device_ok()
    toks = sample(T, 512, 13)
    y_ref = oracle.combine(rows_in.view(np.uint16), w.astype(np.float32).astype(np.float64),
                           sr, T, k, rows_fp16=True)[toks]
    e_y = gate_error(bf16_to_f64(bf16_host(y))[toks], y_ref, "bf16")
    # combine alone is exact up to fp32 summation and the final rounding
    assert e_y <= 1e-5, e_y
    print(f"{name}: h {e_h:.4f}  rows {e_o:.4f}  combine {e_y:.2e}")


# --------------------------------------------------------------------------- whole layer
FWD_CASES = [("tiny", 64), ("default", 160), ("large", 96), ("verify4", 4), ("decode1", 1)]


def _check_forward(L, y, ids, toks, k, group, label=""):
    """Asserts the gate (computation error beyond one bf16 rounding) and
    prints it beside the literal max-abs error and the distance from the
    correctly rounded oracle (neither of which a correctly rounded exact
    result passes: tests/test_parity_gate.py)."""
    ref = oracle.moe_forward(L.inp, k, group, tokens=toks)
    got = bf16_to_f64(bf16_host(y))[toks]
    err = gate_error(got, ref["y"], "bf16")
    raw = raw_error(got, ref["y"])
    rounded_raw = raw_error(round_to(ref["y"], "bf16"), ref["y"])
    vr, vr_frac = vs_rounded(got, ref["y"], "bf16")
    print(f"{label}: gate {err:.4f}  raw max-abs {raw:.4f} (exactly rounded oracle: "
          f"{rounded_raw:.4f})  vs RNE_bf16(oracle) {vr:.4f}, {100 * vr_frac:.1f}% of "
          f"outputs differ", flush=True)
    assert err <= GATE, (err, raw)
    lg_ref = oracle.router_logits(L.inp["x"][toks], L.inp["w_router"], L.inp.get("bias"))
    ntie, nmis = routes_agree(ids.cpu().numpy()[toks], lg_ref, k, 1e-4 * rms(lg_ref))
    return err, raw, ntie, nmis


@pytest.mark.parametrize("name,ntok", FWD_CASES)
def test_forward(name, ntok, dev):
    L = layer_for(name, dev)
    wl = WORKLOADS[name]
    y, ids, w = L.forward()
    assert_device_ok()
    err, raw, ntie, nmis = _check_forward(L, y, ids, sample(wl.T, ntok, 13), wl.k, wl.group,
                                          name)
    print(f"{name}: near-ties {ntie} differing routes {nmis}")


def test_forward_skewed_chunks(dev):
    """34,000 tokens in chunks of <= 6144 with Zipf-biased routing."""
    L = layer_for("skewed", dev)
    wl = WORKLOADS["skewed"]
    y, ids = L.forward_chunked(wl.chunk)
    assert_device_ok()
    assert y.shape[0] == wl.T
    assert chunk_sizes(wl.T, wl.chunk) == [6144] * 5 + [3280]
    _check_forward(L, y, ids, sample(wl.T, 96, 14), wl.k, wl.group, "skewed")


EDGE = [
    dict(T=1, d=256, E=16, k=4, n=256, group=64),        # single token, streaming path
    dict(T=5, d=256, E=16, k=16, n=128, group=32),       # k = E
    dict(T=8, d=384, E=24, k=3, n=256, group=128),       # largest streaming batch
    dict(T=9, d=256, E=16, k=4, n=256, group=32),        # smallest tensor-core batch
    dict(T=130, d=512, E=128, k=6, n=384, group=64),     # ragged token tile, TC router
    dict(T=300, d=256, E=1, k=1, n=128, group=64),       # one expert: dense SwiGLU FFN
    dict(T=257, d=256, E=4, k=2, n=256, group=128),      # 128+ rows per expert
    dict(T=64, d=128, E=8, k=2, n=128, group=32),        # smallest dims
]


@pytest.mark.parametrize("dims", EDGE, ids=lambda d: "T{T}_d{d}_E{E}_k{k}_n{n}_g{group}".format(**d))
def test_forward_edge_cases(dims, dev):
    L = Layer.custom(dev, seed=40 + dims["T"], **dims)
    y, ids, w = L.forward()
    assert_device_ok()
    _check_forward(L, y, ids, np.arange(dims["T"]), dims["k"], dims["group"], str(dims))


# Batches of at most four tokens with d % 1024 == 0 run as one persistent
# launch (router partials, top-k in two warps per token and merge, grouping,
# both projections, combine); these shapes reach its corners.
FUSED_EDGE = [
    dict(T=1, d=1024, E=8, k=8, n=256, group=32),        # k = E: a half has fewer than k
    dict(T=3, d=1024, E=64, k=32, n=512, group=64),      # k = 32: 64 candidates to merge
    dict(T=4, d=2048, E=1024, k=4, n=1024, group=128),   # E = 1024, group 128
    dict(T=2, d=1024, E=24, k=5, n=512, group=64),       # E not a power of two
]


@pytest.mark.parametrize("dims", FUSED_EDGE,
                         ids=lambda d: "T{T}_d{d}_E{E}_k{k}_n{n}_g{group}".format(**d))
def test_fused_decode_edge_cases(dims, dev):
    import bench
    assert bench.fused_decode(dims["T"], dims["d"], dims["E"], dims["k"], dims["n"],
                              dims["group"])
    L = Layer.custom(dev, seed=45 + dims["E"], **dims)
    y, ids, w = L.forward()
    assert_device_ok()
    _check_forward(L, y, ids, np.arange(dims["T"]), dims["k"], dims["group"], "fused " + str(dims))


def test_fused_decode_exact_ties_go_to_the_lower_index(dev):
    """Integer-valued x and W_r (times 2^-4) make the logits exact in fp32 and
    full of exact ties; the fused kernel's top-k must match the oracle's,
    lowest index first, bit for bit."""
    T, d, E, k = 4, 1024, 64, 8
    L = Layer.custom(dev, T=T, d=d, E=E, k=k, n=512, group=64, seed=61)
    rng = np.random.default_rng(9)
    L.inp["x"] = bf16_bits(rng.integers(-2, 3, (T, d)).astype(np.float32))
    L.inp["w_router"] = bf16_bits(rng.integers(-1, 2, (d, E)).astype(np.float32) / 16)
    L.x = torch.from_numpy(L.inp["x"]).to(dev).view(torch.bfloat16)
    L.w_router = torch.from_numpy(L.inp["w_router"]).to(dev).view(torch.bfloat16)
    y, ids, w = L.forward()
    assert_device_ok()
    lg_ref, ids_ref, w_ref = oracle_routes(L)
    srt = -np.sort(-lg_ref, axis=1)[:, :k + 1]
    assert np.any(np.diff(srt, axis=1) == 0), "the case should contain exact ties"
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    assert np.max(np.abs(w.cpu().numpy() - w_ref)) <= 1e-6


def test_forward_all_tokens_one_expert(dev):
    """A bias that sends every token to the same two experts: 300 rows per
    expert (three row tiles of the tensor-core kernel), the rest empty."""
    L = Layer.custom(dev, T=300, d=256, E=16, k=2, n=256, group=64, seed=50)
    bias = np.zeros(16, np.float32)
    bias[[3, 11]] = 1000.0
    L.inp["bias"] = bias
    L.bias = torch.from_numpy(bias).to(dev)
    y, ids, w = L.forward()
    assert_device_ok()
    assert set(np.unique(ids.cpu().numpy())) == {3, 11}
    _check_forward(L, y, ids, np.arange(300), 2, 64)


def test_zero_scales_give_zero(dev):
    for T in (40, 4):
        L = Layer.custom(dev, T=T, d=256, E=8, k=2, n=128, group=64, seed=51)
        for n in ("gate_s", "up_s", "down_s"):
            L.w[n].zero_()
        y, _, _ = L.forward()
        assert_device_ok()
        assert torch.count_nonzero(y.float()) == 0


def test_out_of_fp16_range_input_is_reported(dev):
    L = Layer.custom(dev, T=16, d=128, E=8, k=2, n=128, group=64, seed=53)
    x = L.x.clone()
    x[3, 5] = 1.0e6
    L.forward(x)
    torch.cuda.synchronize()
    assert sm.strata_moe_device_status() == sm.STRATA_ERR_DEVICE_CHECK
    assert sm.strata_moe_device_status() == sm.STRATA_OK


def _fill(L, name, value):
    """Replace one weight tensor by a constant (codes as a byte, scales as fp16)."""
    a = L.inp[name]
    if name.endswith("_q"):
        arr = np.full(a.shape, value, np.uint8)
    else:
        arr = np.full(a.shape, value, np.float16).view(np.uint16)
    L.inp[name] = arr
    L.w[name] = torch.from_numpy(arr).to(L.device)


def _expect_range_report():
    torch.cuda.synchronize()
    assert sm.strata_moe_device_status() == sm.STRATA_ERR_DEVICE_CHECK
    assert sm.strata_moe_device_status() == sm.STRATA_OK        # cleared


@pytest.mark.parametrize("T", [40, 4])
def test_fp16_overflow_of_h_is_reported(T, dev):
    """x inside the fp16 range, but gate and up sums of 2560 make h = SiLU(g) * u
    about 6.5e6, beyond fp16: the gate/up epilogue reports it (tensor-core path
    at T = 40, decode path at T = 4)."""
    L = Layer.custom(dev, T=T, d=256, E=8, k=2, n=128, group=64, seed=55)
    for nm in ("gate", "up"):
        _fill(L, nm + "_q", 0x11)                         # every code q = 1
        _fill(L, nm + "_s", 0.01)
    L.forward(torch.full_like(L.x, 1000.0))
    _expect_range_report()


@pytest.mark.parametrize("T", [40, 4])
def test_fp16_overflow_of_down_rows_is_reported(T, dev):
    """Finite fp16 h rows of 60000 against codes of 7 and scales of 0.02 give
    per-row outputs near 1.1e6: the down epilogue reports them."""
    L = Layer.custom(dev, T=T, d=256, E=8, k=2, n=128, group=64, seed=56)
    _fill(L, "down_q", 0x77)
    _fill(L, "down_s", 0.02)
    S = T * 2
    ids = np.stack([np.arange(T) % 8, (np.arange(T) + 1) % 8], axis=1).astype(np.int32)
    _, offsets, _, _ = oracle.permute(ids, 8)
    h = torch.full((S, 128), 60000.0, dtype=torch.float16, device=dev)
    L.down(h, torch.from_numpy(offsets).to(dev), T)
    _expect_range_report()


def test_scale_beyond_fp16_weight_range_is_reported(dev):
    """The tensor-core path forms each weight as RNE_fp16(q * s): a scale of
    10000 with codes of 7 gives 70000, beyond fp16.  Scales above 65504 / 8
    are reported."""
    L = Layer.custom(dev, T=40, d=256, E=8, k=2, n=128, group=64, seed=57)
    _fill(L, "gate_q", 0x77)
    _fill(L, "gate_s", 10000.0)
    L.forward()
    _expect_range_report()


def test_token_order_equivariance(dev):
    L = layer_for("default", dev)
    y, ids, _ = L.forward()
    perm = torch.from_numpy(np.random.default_rng(3).permutation(512)).to(dev)
    y_p, ids_p, _ = L.forward(L.x[perm])
    assert torch.equal(ids_p, ids[perm])
    # a token's result depends only on its own row: bit-identical
    assert torch.equal(y_p, y[perm])


def test_chunking_matches_whole_batch(dev):
    L = layer_for("default", dev)
    y, ids, _ = L.forward()
    y1, ids1, _ = L.forward(L.x[:200])
    y2, ids2, _ = L.forward(L.x[200:])
    assert torch.equal(torch.cat([ids1, ids2]), ids)
    d = (torch.cat([y1, y2]).float() - y.float()).abs().max().item()
    assert d <= GATE * y.float().pow(2).mean().sqrt().item()


@pytest.mark.parametrize("name", ["default", "large", "verify4", "decode1"])
def test_deterministic(name, dev):
    # tensor-core path (default, large) and decode path with K split across
    # warps and the split-summed small-batch router (verify4, decode1)
    L = layer_for(name, dev)
    ws = sm.workspace(L.dims, dev)
    y1, i1, w1 = L.forward(ws=ws)
    y2, i2, w2 = L.forward(ws=ws)
    assert torch.equal(y1, y2) and torch.equal(i1, i2) and torch.equal(w1, w2)


@pytest.mark.parametrize("name", ["default", "verify4"])
def test_cuda_graph_replay(name, dev):
    L = layer_for(name, dev)
    ws = sm.workspace(L.dims, dev)
    y_eager, _, _ = L.forward(ws=ws)
    T, d = L.dims["T"], L.dims["d"]
    y = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        st = sm.strata_moe_forward(L.x, L.w_router, L.bias, L.q4("gate"), L.q4("up"),
                                   L.q4("down"), L.dims, y, None, None, ws, stream=s)
        assert st == sm.STRATA_OK
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            sm.strata_moe_forward(L.x, L.w_router, L.bias, L.q4("gate"), L.q4("up"),
                                  L.q4("down"), L.dims, y, None, None, ws, stream=s)
    y.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y, y_eager)
    del g


def test_empty_batch(dev):
    L = Layer.custom(dev, T=4, d=128, E=8, k=2, n=128, group=64, seed=52)
    dims = L.dims_T(0)
    y = torch.empty((0, 128), dtype=torch.bfloat16, device=dev)
    assert sm.strata_moe_forward(L.x[:0], L.w_router, None, L.q4("gate"), L.q4("up"),
                                 L.q4("down"), dims, y, None, None, None, 0) == sm.STRATA_OK
    counts = torch.full((8,), 7, dtype=torch.int32, device=dev)
    offsets = torch.full((9,), 7, dtype=torch.int32, device=dev)
    assert sm.strata_moe_permute(None, dims, counts, offsets, None, None, None, 0) == sm.STRATA_OK
    torch.cuda.synchronize()
    assert int(counts.abs().sum()) == 0 and int(offsets.abs().sum()) == 0
    assert_device_ok()


def test_bad_offsets_are_reported_not_used(dev):
    L = Layer.custom(dev, T=16, d=128, E=8, k=2, n=128, group=64, seed=54)
    dims = L.dims
    offsets = torch.tensor([0, 5, 3, 40, 40, 40, 40, 40, 32], dtype=torch.int32, device=dev)
    st = torch.zeros(32, dtype=torch.int32, device=dev)
    h = torch.full((32, 128), 7.0, dtype=torch.float16, device=dev)
    ws = sm.workspace(dims, dev)
    assert sm.strata_moe_expert_gemm_q4(sm.STRATA_OP_GATE_UP_SWIGLU, L.x, st, offsets,
                                        L.q4("gate"), L.q4("up"), None, dims, h, ws) == sm.STRATA_OK
    torch.cuda.synchronize()
    assert sm.strata_moe_device_status() == sm.STRATA_ERR_DEVICE_CHECK
    assert bool((h == 7.0).all())                    # nothing was written


def test_bounded_waits_give_up_and_leave_the_device_usable(dev):
    """Waits on conditions nothing satisfies (an mbarrier no thread or copy
    arrives on, a grid barrier one CTA never reaches, a count of finished
    work nothing raises) give up after their limit: the kernels return, the
    time-out is reported, tensor memory held during the wait is released,
    and the next forward is correct."""
    out = torch.full((10,), -1, dtype=torch.int32, device=dev)
    sync = torch.zeros(32, dtype=torch.uint8, device=dev)
    assert sm.strata_moe_selftest_wait(out, sync) == sm.STRATA_OK
    torch.cuda.synchronize()
    o = out.cpu().tolist()
    assert o[0:4] == [0, 0, 0, 0], o           # warp 0 gave up, the others saw its abort
    assert 0.9e9 <= o[4] <= 1.9e9, o           # after about the one-second limit
    assert o[5] == 1, o                        # tensor memory released
    assert o[6] == 0 and 0.9e9 <= o[7] <= 1.9e9, o
    assert o[8] == 0 and 0.9e9 <= o[9] <= 1.9e9, o
    assert sm.strata_moe_device_status() == sm.STRATA_ERR_DEVICE_CHECK
    assert sm.strata_moe_device_status() == sm.STRATA_OK
    L = Layer.custom(dev, T=40, d=256, E=8, k=2, n=128, group=64, seed=58)
    y, ids, _ = L.forward()
    assert_device_ok()
    _check_forward(L, y, ids, np.arange(40), 2, 64, "after the self-test")
