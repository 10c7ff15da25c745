"""Host-side checks of the C ABI (no GPU needed): the library loads, it
exports every entry point the header declares, and argument validation
returns the documented status before anything is launched."""

import os
import re

import pytest

import local_moe_route_b200 as sm
from local_moe_route_b200 import Dims

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "strata_moe.h")


@pytest.fixture(scope="module", autouse=True)
def built_library():
    from local_moe_route_b200 import build
    build.build()
    return sm.lib()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"STRATA_API\s+[\w\s\*]+?\b(strata_\w+)\s*\(", text)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    assert names == {
        "strata_moe_workspace_bytes", "strata_status_string", "strata_moe_route",
        "strata_moe_permute", "strata_moe_permute_static", "strata_moe_expert_gemm_q4",
        "strata_moe_combine",
        "strata_moe_forward", "strata_moe_device_status", "strata_moe_selftest_wait",
        "strata_moe_gather_rows", "strata_sparse_attention",
        "strata_sparse_attention_workspace_bytes"}


def test_library_exports_every_declared_symbol():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", sm.lib_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(sm.lib(), name)


def test_status_strings():
    for code in range(6):
        s = sm.strata_status_string(code)
        assert isinstance(s, str) and s
    assert sm.strata_status_string(0) == "ok"
    assert sm.strata_status_string(99) == "unknown status"


LARGE = dict(T=6144, d=4096, E=512, k=10, n=1024, group=64)


def test_workspace_bytes():
    n = sm.strata_moe_workspace_bytes(LARGE)
    S = 6144 * 10
    # at least the per-row fp16 buffers: grouped x [S][d], h [S][n], rows [S][d]
    rows = S * 4096 * 2 + S * 1024 * 2 + S * 4096 * 2
    assert n >= rows
    assert n < rows + 64 * 2 ** 20
    assert n % 256 == 0
    assert sm.strata_moe_workspace_bytes(dict(LARGE, T=1)) < 4 * 2 ** 20
    assert sm.strata_moe_workspace_bytes(dict(LARGE, T=0)) >= 0
    # rejected dims give 0
    for bad in (dict(LARGE, k=0), dict(LARGE, k=513), dict(LARGE, d=100), dict(LARGE, group=48),
                dict(LARGE, E=2048), dict(LARGE, T=-1), dict(LARGE, n=0)):
        assert sm.strata_moe_workspace_bytes(bad) == 0


FAKE = 1 << 40          # 16-byte aligned, never dereferenced (validation fails first)


def route(**kw):
    args = dict(x=FAKE, w_router=FAKE, bias=None, dims=LARGE, topk_ids=FAKE, topk_w=FAKE,
                logits_out=None, ws=FAKE, ws_bytes=1 << 40, stream=0)
    args.update(kw)
    return sm.strata_moe_route(**args)


def test_route_validation():
    assert route(x=None) == sm.STRATA_ERR_INVALID_ARG
    assert route(w_router=None) == sm.STRATA_ERR_INVALID_ARG
    assert route(topk_ids=None) == sm.STRATA_ERR_INVALID_ARG
    assert route(topk_w=FAKE + 4) == sm.STRATA_ERR_INVALID_ARG          # misaligned
    assert route(bias=FAKE + 8) == sm.STRATA_ERR_INVALID_ARG
    assert route(dims=dict(LARGE, k=600)) == sm.STRATA_ERR_INVALID_ARG   # k > E
    assert route(dims=dict(LARGE, d=4000)) == sm.STRATA_ERR_UNSUPPORTED
    assert route(dims=dict(LARGE, group=16)) == sm.STRATA_ERR_UNSUPPORTED
    assert route(ws=None) == sm.STRATA_ERR_WORKSPACE
    assert route(ws_bytes=16) == sm.STRATA_ERR_WORKSPACE
    assert route(dims=dict(LARGE, T=0), x=None, ws=None, ws_bytes=0) == sm.STRATA_OK   # empty batch


def test_permute_validation():
    def call(**kw):
        args = dict(topk_ids=FAKE, dims=LARGE, counts=FAKE, offsets=FAKE, sorted_token=FAKE,
                    slot_row=FAKE, ws=FAKE, ws_bytes=1 << 40, stream=0)
        args.update(kw)
        return sm.strata_moe_permute(**args)
    assert call(counts=None) == sm.STRATA_ERR_INVALID_ARG
    assert call(slot_row=FAKE + 2) == sm.STRATA_ERR_INVALID_ARG
    assert call(ws_bytes=100) == sm.STRATA_ERR_WORKSPACE
    assert call(dims=dict(LARGE, E=0)) == sm.STRATA_ERR_INVALID_ARG


def test_gemm_validation():
    W = (FAKE, FAKE)

    def call(**kw):
        args = dict(op=sm.STRATA_OP_GATE_UP_SWIGLU, a=FAKE, sorted_token=FAKE, offsets=FAKE,
                    w0=W, w1=W, row_scale=None, dims=LARGE, out=FAKE, ws=FAKE,
                    ws_bytes=1 << 40, stream=0)
        args.update(kw)
        return sm.strata_moe_expert_gemm_q4(**args)
    assert call(op=7) == sm.STRATA_ERR_INVALID_ARG
    assert call(w1=(None, FAKE)) == sm.STRATA_ERR_INVALID_ARG
    assert call(sorted_token=None) == sm.STRATA_ERR_INVALID_ARG
    assert call(row_scale=FAKE) == sm.STRATA_ERR_INVALID_ARG       # only for DOWN
    assert call(op=sm.STRATA_OP_DOWN, w0=(FAKE, FAKE + 1)) == sm.STRATA_ERR_INVALID_ARG
    assert call(ws_bytes=8) == sm.STRATA_ERR_WORKSPACE
    assert call(dims=dict(LARGE, n=96)) == sm.STRATA_ERR_UNSUPPORTED


def test_combine_and_forward_validation():
    assert sm.strata_moe_combine(FAKE, None, FAKE, LARGE, None, stream=0) == sm.STRATA_ERR_INVALID_ARG
    assert sm.strata_moe_combine(FAKE, FAKE + 4, FAKE, LARGE, FAKE, stream=0) == \
        sm.STRATA_ERR_INVALID_ARG
    W = (FAKE, FAKE)

    def fwd(**kw):
        args = dict(x=FAKE, w_router=FAKE, bias=None, gate=W, up=W, down=W, dims=LARGE, y=FAKE,
                    topk_ids_out=None, topk_w_out=None, ws=FAKE, ws_bytes=1 << 40, stream=0)
        args.update(kw)
        return sm.strata_moe_forward(**args)
    assert fwd(down=(FAKE, None)) == sm.STRATA_ERR_INVALID_ARG
    assert fwd(y=None) == sm.STRATA_ERR_INVALID_ARG
    assert fwd(ws_bytes=sm.strata_moe_workspace_bytes(LARGE) - 1) == sm.STRATA_ERR_WORKSPACE
    assert fwd(dims=dict(LARGE, T=0)) == sm.STRATA_OK


def test_dims_marshalling():
    d = Dims.of(LARGE)
    assert (d.T, d.d, d.E, d.k, d.n, d.group) == (6144, 4096, 512, 10, 1024, 64)
    assert Dims.of((1, 2, 3, 4, 5, 6)).group == 6
