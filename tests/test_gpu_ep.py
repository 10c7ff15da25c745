"""The expert-parallel forward on one GPU through the CUDA library (NCCL
process group of one rank, so the all-to-all is local), and the row gather it
uses, against the fp64 oracle.  The multi-rank exchange itself is covered on
the CPU by tests/test_ep.py."""

import datetime
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import local_moe_route_b200 as sm
import oracle
from gpu_helpers import Layer, assert_device_ok, bf16_host, bf16_to_f64
from parity_metrics import gate_error

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev(cuda_dev):
    from local_moe_route_b200 import build
    build.build()
    return cuda_dev


def test_gather_rows(dev):
    src = torch.randint(-30000, 30000, (50, 136), dtype=torch.int16, device=dev)
    idx = torch.tensor([3, 49, 0, 3, 17], dtype=torch.int32, device=dev)
    out = torch.empty((5, 136), dtype=torch.int16, device=dev)
    assert sm.strata_moe_gather_rows(src, idx, 50, 5, 136, out) == sm.STRATA_OK
    assert_device_ok()
    assert torch.equal(out, src[idx.long()])
    bad = torch.tensor([2, 50], dtype=torch.int32, device=dev)
    assert sm.strata_moe_gather_rows(src, bad, 50, 2, 136, out) == sm.STRATA_OK
    torch.cuda.synchronize()
    assert sm.strata_moe_device_status() == sm.STRATA_ERR_DEVICE_CHECK
    assert sm.strata_moe_device_status() == sm.STRATA_OK
    assert sm.strata_moe_gather_rows(src, idx, 50, 5, 130, out) == sm.STRATA_ERR_INVALID_ARG


@pytest.mark.parametrize("T", [40, 6])
def test_expert_parallel_single_rank_matches_oracle(T, dev):
    from local_moe_route_b200.ep import ExpertParallelMoE, LibraryOps
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        L = Layer.custom(dev, T=T, d=256, E=16, k=4, n=256, group=64, seed=90 + T)
        ids, w, _ = L.route()
        ops = LibraryOps(L.w, L.dims, world=1)
        ep = ExpertParallelMoE(16, 4, ops)
        y = ep.forward(L.x, ids, w)
        assert_device_ok()
        toks = np.arange(T)
        ref = oracle.moe_forward(L.inp, 4, 64, tokens=toks, ids=ids.cpu().numpy(),
                                 w=w.cpu().numpy().astype(np.float64))["y"]
        err = gate_error(bf16_to_f64(bf16_host(y)), ref, "bf16")
        assert err <= 1.5e-2, err
    finally:
        dist.destroy_process_group()
