"""Attention over indexer-selected KV rows on the GPU, through the C ABI,
against the fp64 oracle (oracle/sparse_attention.py).

Bar: the kernel computes scores, softmax and the weighted sum in fp32 and
rounds the output once to bf16, so beyond that rounding its error is a few
fp32 ulps of the accumulations (about 1e-6 of RMS); the tests allow 1e-3 of
RMS on top of half a bf16 ulp."""

import numpy as np
import pytest
import torch

import local_moe_route_b200 as sm
from gpu_helpers import assert_device_ok, bf16_host, bf16_to_f64
from moe_inputs import ATTN_WORKLOADS, make_attention
from oracle.sparse_attention import sparse_attention
from parity_metrics import gate_error, raw_error

pytestmark = pytest.mark.gpu
BAR = 1e-3


@pytest.fixture(scope="module")
def dev(cuda_dev):
    from local_moe_route_b200 import build
    build.build()
    return cuda_dev


def run(a, dims, dev, scale=0.0):
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(dev)
    out = torch.empty((dims["T"], dims["Hq"], dims["D"]), dtype=torch.bfloat16, device=dev)
    ws = sm.attention_workspace(dims, dev)
    sm.check(sm.strata_sparse_attention(t(a["q"]), t(a["k"]), t(a["v"]), t(a["idx"]), dims,
                                        scale, out, ws), "sparse attention")
    return out


def check(a, out, scale=None):
    ref = sparse_attention(a["q"], a["k"], a["v"], a["idx"], scale)
    got = bf16_to_f64(bf16_host(out))
    err = gate_error(got, ref, "bf16")
    print(f"gate {err:.2e} raw {raw_error(got, ref):.2e}")
    assert err <= BAR, err


@pytest.mark.parametrize("name", ["attn_tiny", "attn_decode1", "attn_verify4"])
def test_sparse_attention_workloads(name, dev):
    w = ATTN_WORKLOADS[name]
    dims = dict(T=w.T, L=w.L, Hq=w.Hq, Hkv=w.Hkv, D=w.D, P=w.P)
    a = make_attention(w.T, w.L, w.Hq, w.Hkv, w.D, w.P, w.seed)
    out = run(a, dims, dev)
    assert_device_ok()
    check(a, out)


def test_padding_ragged_slices_and_empty_queries(dev):
    """-1 slots (fewer selected rows than slots), P not a multiple of the
    128-slot slice, a query with nothing selected, D = 64, groups of 16."""
    T, L, Hq, Hkv, D, P = 4, 5000, 16, 1, 64, 300
    a = make_attention(T, L, Hq, Hkv, D, P, seed=21, n_valid=np.array([300, 129, 1, 0]))
    out = run(a, dict(T=T, L=L, Hq=Hq, Hkv=Hkv, D=D, P=P), dev, scale=0.05)
    assert_device_ok()
    check(a, out, scale=0.05)
    assert not torch.any(out[3].float() != 0)


def test_out_of_range_index_is_reported(dev):
    a = make_attention(1, 100, 4, 2, 64, 16, seed=22)
    a["idx"][0, 3] = 100
    run(a, dict(T=1, L=100, Hq=4, Hkv=2, D=64, P=16), dev)
    torch.cuda.synchronize()
    assert sm.strata_moe_device_status() == sm.STRATA_ERR_DEVICE_CHECK
    assert sm.strata_moe_device_status() == sm.STRATA_OK


def test_rejected_shapes():
    bad = [dict(T=1, L=10, Hq=6, Hkv=4, D=64, P=8), dict(T=1, L=10, Hq=8, Hkv=2, D=96, P=8),
           dict(T=1, L=10, Hq=64, Hkv=2, D=64, P=8)]
    for d in bad:
        assert sm.strata_sparse_attention_workspace_bytes(d) == 0
