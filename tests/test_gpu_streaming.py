"""Layers whose expert weights live in host memory, streamed into a ring of
device slots on a copy stream while the previous layer computes: the output
must be bit-identical to running the same layers with resident weights, and
the uploads must overlap the forwards."""

import numpy as np
import pytest
import torch

import local_moe_route_b200 as sm
from gpu_helpers import assert_device_ok
from moe_inputs import make_custom

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev(cuda_dev):
    from local_moe_route_b200 import build
    build.build()
    return cuda_dev


def _layers(n_layers, dims, seed, **scales):
    """Random layers without normalisation between them grow (or shrink)
    quadratically from one layer to the next; the callers keep the stacks
    short, or the scales small, so that h stays inside the fp16 range."""
    out = []
    for i in range(n_layers):
        inp = make_custom(seed=seed + i, **dims, **scales)
        lay = {k: torch.from_numpy(np.ascontiguousarray(v)) for k, v in inp.items()
               if v is not None and k != "x"}
        out.append(lay)
    return out, make_custom(seed=seed, **dims)["x"]


@pytest.mark.parametrize("T,slots", [(96, 2), (4, 3)])
def test_streamed_layers_equal_resident_layers(T, slots, dev):
    from local_moe_route_b200.streaming import LayerStreamer
    dims = dict(T=T, d=512, E=16, k=4, n=256, group=64)
    layers, x_np = _layers(3, dims, seed=70 + T)
    x = torch.from_numpy(x_np).to(dev).view(torch.bfloat16)
    streamer = LayerStreamer(layers, dims, dev, slots=slots)
    y = streamer.forward(x)
    assert_device_ok()
    # resident reference: the same layers, weights copied to the device up front
    ws = sm.workspace(dims, dev)
    cur = x
    for lay in layers:
        w = {k: v.to(dev) for k, v in lay.items()}
        out = torch.empty_like(cur)
        sm.check(sm.strata_moe_forward(cur, w["w_router"].view(torch.bfloat16), None,
                                       (w["gate_q"], w["gate_s"]), (w["up_q"], w["up_s"]),
                                       (w["down_q"], w["down_s"]), dims, out, None, None, ws))
        cur = out
    assert_device_ok()
    assert torch.equal(y, cur)


def test_uploads_overlap_compute(dev):
    """With several layers queued, the copy stream's uploads run while the
    compute stream works: the whole run takes less than the sum of the
    uploads' and the forwards' times."""
    from local_moe_route_b200.streaming import LayerStreamer
    # about 12.6 MB of weights per layer (~0.25 ms over PCIe) against ~77
    # GFLOP of expert work per layer: uploads and forwards of similar length
    dims = dict(T=4096, d=1024, E=16, k=4, n=512, group=64)
    layers, x_np = _layers(6, dims, seed=80, s_lo=0.002, s_hi=0.006)
    x = torch.from_numpy(x_np).to(dev).view(torch.bfloat16)
    st = LayerStreamer(layers, dims, dev, slots=2)
    st.forward(x)
    torch.cuda.synchronize()
    # time the uploads alone and the forwards alone, then together
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(st.L):
        for n, h in st.host[i].items():
            st.ring[0][n].copy_(h, non_blocking=True)
    t1.record()
    torch.cuda.synchronize()
    upload_ms = t0.elapsed_time(t1)
    ev = []
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record()
    st.forward(x, events=ev)
    a1.record()
    torch.cuda.synchronize()
    total = a0.elapsed_time(a1)
    compute = sum(e0.elapsed_time(e1) for e0, e1 in ev)
    assert_device_ok()
    print(f"uploads {upload_ms:.2f} ms, forwards {compute:.2f} ms, streamed run {total:.2f} ms")
    assert total < 0.9 * (upload_ms + compute)
