"""GPU parity: every step of the layer, through the C ABI, against the fp64
oracle on the same seeded inputs.

Bars (integer work bit-exact, floating point within the output gate):
  * router logits: |gpu - oracle| <= 1e-4 * RMS(logits) (fp32 accumulation);
  * expert ids: identical to the oracle's top-k run on the GPU's own fp32
    logits, and identical to the oracle's fp64 routing except where the
    oracle's own logits are within 1e-4*RMS of a tie (none for these seeds);
  * routing weights: within 1e-6 of the oracle's softmax on the GPU logits;
  * counts, offsets, sorted_token, slot_row: bit-exact;
  * bf16 outputs (h, per-row outputs, y): max |gpu - oracle| <= 1.5e-2 *
    RMS(oracle), the layer's output gate.
Large workloads are checked on seeded samples of rows/tokens (the oracle is
per token, so a sample is exact), in the launch configuration the benchmark
uses.
"""

import gc

import numpy as np
import pytest
import torch

import local_moe_route_b200 as sm
import oracle
from gpu_helpers import (Layer, assert_device_ok, bf16_host, bf16_to_f64, gate_error,
                         near_tie_tokens, rms)
from moe_inputs import WORKLOADS, chunk_sizes

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


def ids_agree(ids_gpu, logits_ref, k):
    """GPU ids equal the oracle's fp64 routing except on near-tie tokens."""
    ids_ref, _ = oracle.topk_softmax(logits_ref, k)
    mism = np.any(ids_gpu != ids_ref, axis=1)
    # a near tie anywhere among the first k+1 sorted logits can reorder picks
    srt = -np.sort(-logits_ref, axis=1)[:, :k + 1]
    gaps = -np.diff(srt, axis=1)
    ties = np.any(gaps < 1e-4 * rms(logits_ref), axis=1)
    assert not np.any(mism & ~ties), np.nonzero(mism & ~ties)[0][:10]
    return int(ties.sum()), int(mism.sum())


# --------------------------------------------------------------------------- route
@pytest.mark.parametrize("name", ["tiny", "default", "large", "verify4", "decode1"])
def test_route(name, dev):
    L = layer_for(name, dev)
    wl = WORKLOADS[name]
    ids, w, logits = L.route()
    assert_device_ok()
    lg = logits.cpu().numpy().astype(np.float64)
    rows = sample(wl.T, 1024, 7)
    ref = oracle.router_logits(L.inp["x"][rows], L.inp["w_router"], L.inp.get("bias"))
    assert np.max(np.abs(lg[rows] - ref)) <= 1e-4 * rms(ref) + 1e-6
    # the same decisions as the oracle's top-k on the GPU's own fp32 logits
    ids_o, w_o = oracle.topk_softmax(lg, wl.k)
    assert np.array_equal(ids.cpu().numpy(), ids_o)
    assert np.max(np.abs(w.cpu().numpy() - w_o)) <= 1e-6
    ntie, nmis = ids_agree(ids.cpu().numpy()[rows], ref, wl.k)
    assert nmis == 0, (ntie, nmis)


def test_route_skewed_chunk(dev):
    L = layer_for("skewed", dev)
    wl = WORKLOADS["skewed"]
    x = L.x[:6144]
    ids, w, logits = L.route(x)
    lg = logits.cpu().numpy().astype(np.float64)
    rows = sample(6144, 512, 8)
    ref = oracle.router_logits(L.inp["x"][rows], L.inp["w_router"], L.inp["bias"])
    assert np.max(np.abs(lg[rows] - ref)) <= 1e-4 * rms(ref) + 1e-6
    ids_o, w_o = oracle.topk_softmax(lg, wl.k)
    assert np.array_equal(ids.cpu().numpy(), ids_o)
    assert np.max(np.abs(w.cpu().numpy() - w_o)) <= 1e-6
    ids_agree(ids.cpu().numpy()[rows], ref, wl.k)
    # the bias makes the load skewed: the busiest expert far above the mean
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
def test_permute_from_route(name, dev):
    L = layer_for(name, dev)
    ids, _, _ = L.route()
    _check_permute(L, ids.cpu().numpy(), WORKLOADS[name].T)


@pytest.mark.parametrize("T,E,k,pattern", [
    (1, 16, 4, "random"), (3000, 64, 4, "random"), (300, 16, 4, "same"),
    (2500, 1024, 32, "random"), (777, 8, 8, "random"), (4097, 5, 1, "skew")])
def test_permute_patterns(T, E, k, pattern, dev):
    L = Layer.custom(dev, T=1, d=128, E=E, k=k, n=128, group=64, seed=31)
    rng = np.random.default_rng(T + E)
    if pattern == "same":
        ids = np.tile(np.arange(k), (T, 1))
    elif pattern == "skew":
        ids = np.minimum(rng.geometric(0.7, size=(T, k)) - 1, E - 1)
    else:
        ids = np.stack([rng.permutation(E)[:k] for _ in range(T)])
    _check_permute(L, ids.astype(np.int32), T)


def test_permute_flags_out_of_range_ids(dev):
    L = Layer.custom(dev, T=1, d=128, E=8, k=2, n=128, group=64, seed=32)
    ids = np.array([[0, 1], [8, 2], [3, -1]], np.int32)     # 8 and -1 are out of range
    t = torch.from_numpy(ids).to(dev)
    counts, offsets, st, sr = L.permute(t, 3)
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
    T, S = wl.T, wl.S
    ids, w, _ = L.route()
    counts, offsets, st, sr = L.permute(ids, T)
    h = L.gate_up(L.x, st, offsets, T)
    scale = torch.linspace(0.5, 1.5, S, device=dev, dtype=torch.float32)
    rows_scaled = L.down(h, offsets, T, row_scale=scale)
    rows = L.down(h, offsets, T)
    assert_device_ok()
    st_np = st.cpu().numpy()
    off_np = offsets.cpu().numpy()
    expert_of_row = np.searchsorted(off_np, np.arange(S), side="right") - 1
    pick = sample(S, max_rows, 11)
    # gate/up + SwiGLU on the gathered x rows
    h_ref = oracle.gate_up_rows(L.inp["x"][st_np[pick]], expert_of_row[pick], L.inp, wl.group)
    h_np = bf16_host(h)
    assert gate_error(bf16_to_f64(h_np[pick]), h_ref) <= GATE
    # down on the GPU's own h rows (bf16), with and without the row scale
    o_ref = oracle.down_rows(h_np[pick], expert_of_row[pick], L.inp, wl.group)
    assert gate_error(bf16_to_f64(bf16_host(rows)[pick]), o_ref) <= GATE
    sc = scale.cpu().numpy()[pick]
    o_ref_s = oracle.down_rows(h_np[pick], expert_of_row[pick], L.inp, wl.group, sc)
    assert gate_error(bf16_to_f64(bf16_host(rows_scaled)[pick]), o_ref_s) <= GATE
    # combine of the GPU rows
    y = L.combine(rows, w, sr, T)
    toks = sample(T, 512, 12)
    y_ref = oracle.combine(bf16_host(rows), w.cpu().numpy().astype(np.float64), sr.cpu().numpy(),
                           T, wl.k)[toks]
    y_np = bf16_to_f64(bf16_host(y))[toks]
    assert np.all(np.abs(y_np - y_ref) <= 2.0 ** -8 * np.abs(y_ref) + 1e-6 * rms(y_ref))


# --------------------------------------------------------------------------- whole layer
FWD_CASES = [("tiny", 64), ("default", 160), ("large", 96), ("verify4", 4), ("decode1", 1)]


@pytest.mark.parametrize("name,ntok", FWD_CASES)
def test_forward(name, ntok, dev):
    L = layer_for(name, dev)
    wl = WORKLOADS[name]
    y, ids, w = L.forward()
    assert_device_ok()
    toks = sample(wl.T, ntok, 13)
    ref = oracle.moe_forward(L.inp, wl.k, wl.group, tokens=toks)
    err = gate_error(bf16_to_f64(bf16_host(y))[toks], ref["y"])
    assert err <= GATE, err
    lg = oracle.router_logits(L.inp["x"][toks], L.inp["w_router"], L.inp.get("bias"))
    ntie, nmis = ids_agree(ids.cpu().numpy()[toks], lg, wl.k)
    assert nmis == 0


def test_forward_skewed_chunks(dev):
    """34,000 tokens in chunks of <= 6144 with Zipf-biased routing."""
    L = layer_for("skewed", dev)
    wl = WORKLOADS["skewed"]
    y, ids = L.forward_chunked(wl.chunk)
    assert_device_ok()
    assert y.shape[0] == wl.T
    assert chunk_sizes(wl.T, wl.chunk) == [6144] * 5 + [3280]
    toks = sample(wl.T, 96, 14)
    ref = oracle.moe_forward(L.inp, wl.k, wl.group, tokens=toks)
    err = gate_error(bf16_to_f64(bf16_host(y))[toks], ref["y"])
    assert err <= GATE, err
    lg = oracle.router_logits(L.inp["x"][toks], L.inp["w_router"], L.inp["bias"])
    ids_agree(ids.cpu().numpy()[toks], lg, wl.k)


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
    ref = oracle.moe_forward(L.inp, dims["k"], dims["group"])
    assert gate_error(bf16_to_f64(bf16_host(y)), ref["y"]) <= GATE
    lg = oracle.router_logits(L.inp["x"], L.inp["w_router"])
    ids_agree(ids.cpu().numpy(), lg, dims["k"])


def test_forward_all_tokens_one_expert(dev):
    """A bias that sends every token to the same experts: 300 rows per expert
    (three row tiles of the tensor-core kernel) and empty experts elsewhere."""
    L = Layer.custom(dev, T=300, d=256, E=16, k=2, n=256, group=64, seed=50)
    bias = np.zeros(16, np.float32)
    bias[[3, 11]] = 1000.0
    L.inp["bias"] = bias
    L.bias = torch.from_numpy(bias).to(dev)
    y, ids, w = L.forward()
    assert_device_ok()
    assert set(np.unique(ids.cpu().numpy())) == {3, 11}
    ref = oracle.moe_forward(L.inp, 2, 64)
    assert gate_error(bf16_to_f64(bf16_host(y)), ref["y"]) <= GATE


def test_zero_scales_give_zero(dev):
    L = Layer.custom(dev, T=40, d=256, E=8, k=2, n=128, group=64, seed=51)
    for n in ("gate_s", "up_s", "down_s"):
        L.w[n].zero_()
    y, _, _ = L.forward()
    assert_device_ok()
    assert torch.count_nonzero(y.float()) == 0


def test_token_order_equivariance(dev):
    L = layer_for("default", dev)
    y, ids, _ = L.forward()
    perm = torch.from_numpy(np.random.default_rng(3).permutation(512)).to(dev)
    y_p, ids_p, _ = L.forward(L.x[perm])
    assert torch.equal(ids_p, ids[perm])
    d = (y_p.float() - y[perm].float()).abs().max().item()
    assert d <= GATE * y.float().pow(2).mean().sqrt().item()


def test_chunking_matches_whole_batch(dev):
    L = layer_for("default", dev)
    y, ids, _ = L.forward()
    y1, ids1, _ = L.forward(L.x[:200])
    y2, ids2, _ = L.forward(L.x[200:])
    assert torch.equal(torch.cat([ids1, ids2]), ids)
    d = (torch.cat([y1, y2]).float() - y.float()).abs().max().item()
    assert d <= GATE * y.float().pow(2).mean().sqrt().item()


def test_deterministic(dev):
    L = layer_for("default", dev)
    ws = sm.workspace(L.dims, dev)
    y1, i1, w1 = L.forward(ws=ws)
    y2, i2, w2 = L.forward(ws=ws)
    assert torch.equal(y1, y2) and torch.equal(i1, i2) and torch.equal(w1, w2)


def test_cuda_graph_replay(dev):
    L = layer_for("default", dev)
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
    dummy = torch.empty(4, dtype=torch.int32, device=dev)
    assert sm.strata_moe_permute(dummy, dims, counts, offsets, dummy, dummy, None, 0) == sm.STRATA_OK
    torch.cuda.synchronize()
    assert int(counts.abs().sum()) == 0 and int(offsets.abs().sum()) == 0
    assert_device_ok()
