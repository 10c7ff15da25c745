"""strata_moe_permute_static: the grouping step with its scratch in a fixed
array inside the library instead of a caller workspace.  It must give
exactly what strata_moe_permute gives, call after call (nothing may carry
over between calls through the shared scratch), and refuse inputs larger
than the fixed scratch before touching the device.

This file is named to be collected last, so that it also runs after every
other test has used the library on the same device."""

import numpy as np
import pytest

import local_moe_route_b200 as sm
import oracle
from local_moe_route_b200 import Dims


@pytest.fixture(scope="module", autouse=True)
def built_library():
    from local_moe_route_b200 import build
    build.build()
    return sm.lib()


def dims(T, E, k):
    return dict(T=T, d=128, E=E, k=k, n=128, group=64)


def scratch_ints(T, E, k):
    return -(-T * k // 1024) * E


def test_oversized_input_is_refused_before_any_device_work():
    # ceil(4200*32/1024) * 1024 = 135168 > 131072 histogram entries
    assert scratch_ints(4200, 1024, 32) > sm.STRATA_PERMUTE_STATIC_SCRATCH_INTS
    fake = 1 << 20          # 16-byte aligned, never dereferenced
    st = sm.lib().strata_moe_permute_static(fake, Dims.of(dims(4200, 1024, 32)), fake, fake,
                                            fake, fake, None)
    assert st == sm.STRATA_ERR_WORKSPACE
    # invalid dims still come first
    st = sm.lib().strata_moe_permute_static(fake, Dims.of(dims(4, 8, 9)), fake, fake, fake,
                                            fake, None)
    assert st == sm.STRATA_ERR_INVALID_ARG


def _routes(T, E, k, seed):
    rng = np.random.default_rng(seed)
    return np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)


def _permute_both(ids, E, dev):
    import torch
    T, k = ids.shape
    S = T * k
    ids_d = torch.from_numpy(ids).to(dev)
    out = {}
    for name in ("workspace", "static"):
        counts = torch.full((E,), -7, dtype=torch.int32, device=dev)
        offsets = torch.full((E + 1,), -7, dtype=torch.int32, device=dev)
        st = torch.full((max(S, 1),), -7, dtype=torch.int32, device=dev)
        sr = torch.full((max(S, 1),), -7, dtype=torch.int32, device=dev)
        dm = dims(T, E, k)
        if name == "workspace":
            ws = sm.workspace(dm, dev)
            sm.check(sm.strata_moe_permute(ids_d, dm, counts, offsets, st, sr, ws), name)
        else:
            sm.check(sm.strata_moe_permute_static(ids_d, dm, counts, offsets, st, sr), name)
        torch.cuda.synchronize()
        sm.check(sm.strata_moe_device_status(), name)
        out[name] = [a.cpu().numpy()[:n] for a, n in
                     ((counts, E), (offsets, E + 1), (st, S), (sr, S))]
    return out


@pytest.mark.gpu
@pytest.mark.parametrize("cases", [
    # two calls in a row on different inputs; the second is smaller, so any
    # histogram entry it did not rewrite would show up as a difference
    [(6144, 512, 10, 1), (3000, 64, 4, 2)],
    # the largest input the scratch holds (131072 entries exactly), then a tiny one
    [(4096, 1024, 32, 3), (5, 16, 2, 4)],
    # an empty batch between two real ones
    [(777, 8, 8, 5), (0, 8, 8, 6), (4097, 5, 1, 7)],
])
def test_matches_workspace_entry_point(cases, cuda_dev):
    for T, E, k, seed in cases:
        assert scratch_ints(T, E, k) <= sm.STRATA_PERMUTE_STATIC_SCRATCH_INTS
        ids = _routes(T, E, k, seed) if T else np.zeros((0, k), np.int32)
        got = _permute_both(ids, E, cuda_dev)
        for a, b, what in zip(got["static"], got["workspace"],
                              ("counts", "offsets", "sorted_token", "slot_row")):
            assert np.array_equal(a, b), (T, E, k, what)
        if T:
            ref = oracle.permute(ids, E)
            for a, b in zip(got["static"], ref):
                assert np.array_equal(a, np.asarray(b))
