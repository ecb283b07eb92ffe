"""moe_load_stats_noalloc: the load-statistics entry point for callers that
cannot allocate device memory (a framework owning the whole memory pool,
fixed-memory real-time code, host callbacks).  It uses the library's fixed
scratch array instead of a caller workspace; its results must equal those
of moe_load_stats with a workspace, call after call.

This file is named to be collected last, so a stop at its first failure
still leaves every other test run."""
import ctypes

import numpy as np
import pytest
import torch

from expert_load_balancing_tcgen05_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from expert_load_balancing_tcgen05_b200 import moe as m
    return m


def _outputs(T, K, n_slots, stats_bytes):
    dev = "cuda"
    return dict(slot=torch.full((T, K), -7, dtype=torch.int32, device=dev),
                counts=torch.full((n_slots,), -7, dtype=torch.int32, device=dev),
                offsets=torch.full((n_slots + 1,), -7, dtype=torch.int32, device=dev),
                rank=torch.full((T, K), -7, dtype=torch.int32, device=dev),
                stats=torch.zeros(stats_bytes, dtype=torch.uint8, device=dev))


def _call_noalloc(moe, idx, T, K, N, rs, n_slots, o, scores=None, fn=1):
    p = lambda t: ctypes.c_void_p(t.data_ptr()) if t is not None else None  # noqa: E731
    st = moe._lib.moe_load_stats_noalloc(p(idx), T, K, N, p(rs), n_slots, p(o["slot"]), p(o["counts"]),
                                         p(o["offsets"]), p(o["rank"]), p(scores), fn, p(o["stats"]),
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


def _call_ws(moe, idx, T, K, N, rs, n_slots, o, scores=None, fn=1):
    ws = moe.workspace(T, K, N, n_slots)
    moe.moe_load_stats(idx, T, K, N, rs, n_slots, o["slot"], o["counts"], o["offsets"], o["rank"], scores, fn,
                       o["stats"], ws)


def _same(moe, a, b):
    for k in ("slot", "counts", "offsets", "rank"):
        assert torch.equal(a[k], b[k]), k
    sa, sb = moe.read_stats(a["stats"]), moe.read_stats(b["stats"])
    assert sa["status"] == 0 and sb["status"] == 0
    for k, v in sa.items():
        if isinstance(v, float) and np.isnan(v):
            assert np.isnan(sb[k])
        else:
            assert abs(v - sb[k]) <= 1e-6 * abs(sb[k]) + 1e-12, k


@pytest.mark.parametrize("T,K,N,R,with_scores", [(5000, 8, 256, 0, True), (131072, 8, 256, 32, False),
                                                 (513, 2, 8, 0, False)])
def test_noalloc_matches_workspace_call_twice(moe, T, K, N, R, with_scores):
    idx = W.make_assignments(T, K, N, seed=T + R, skew=1.1).cuda()
    rs = None
    n_slots = N + R
    if R:
        c = torch.bincount(idx.reshape(-1).long(), minlength=N).to(torch.int32)
        rs = torch.empty(N, dtype=torch.int32, device="cuda")
        moe.moe_replica_plan(c, N, R, rs)
    scores = W.make_scores(T, N, seed=3).cuda() if with_scores else None
    ref = _outputs(T, K, n_slots, moe.STATS_BYTES)
    _call_ws(moe, idx, T, K, N, rs, n_slots, ref, scores)
    # two calls in a row through the fixed scratch array (it keeps the previous
    # call's contents; every call must start clean)
    for _ in range(2):
        got = _outputs(T, K, n_slots, moe.STATS_BYTES)
        assert _call_noalloc(moe, idx, T, K, N, rs, n_slots, got, scores) == moe.MOE_OK
        torch.cuda.synchronize()
        _same(moe, got, ref)


def test_noalloc_rejects_problems_larger_than_its_scratch(moe):
    # a histogram of 2048 slots over 2^30 assignments needs far more than 4 MiB
    T, K, N = 1 << 27, 8, 2048
    assert moe.moe_workspace_bytes(T, K, N) > moe.NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x10000)  # never touched: the size check fails first
    st = moe._lib.moe_load_stats_noalloc(fake, T, K, N, None, N, None, fake, fake, fake, None, 1, None,
                                         None)
    assert st == moe.MOE_ERR_UNSUPPORTED
