"""Host-only checks of the C ABI: the library loads, exports every entry
point the header declares, and rejects bad arguments on the host before any
launch (no GPU needed: the rejected calls never reach CUDA)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_route.h")


@pytest.fixture(scope="module")
def moe():
    from expert_load_balancing_tcgen05_b200 import build
    build.build()
    from expert_load_balancing_tcgen05_b200 import moe as m
    return m


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", text)))


def test_header_declares_the_five_calls():
    names = _declared()
    for n in ("moe_route", "moe_load_stats", "moe_bias_update", "moe_dispatch", "moe_combine"):
        assert n in names


def test_library_exports_every_declared_symbol(moe):
    lib = ctypes.CDLL(moe.LIB_PATH)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(moe.EXPORTS) <= set(_declared())


def test_version_and_status_strings(moe):
    assert "sm_100a" in moe.moe_version()
    assert moe._lib.moe_status_str(moe.MOE_ERR_TIMEOUT).decode() == "bounded device wait timed out"


def test_workspace_bytes(moe):
    a = moe.moe_workspace_bytes(16384, 8, 256)
    b = moe.moe_workspace_bytes(131072, 8, 256, 288)
    assert 0 < a < b < 4 << 20
    assert moe.moe_workspace_bytes(100, 8, 256, 200) == 0   # n_slots < N
    assert moe.moe_workspace_bytes(0, 8, 16) > 0


FAKE = ctypes.c_void_p(0x10000)      # never dereferenced: validation fails first
MISALIGNED = ctypes.c_void_p(0x10008)


def _cfg(moe, **kw):
    c = dict(T=64, d=128, N=256, K=8, score_fn=1, n_groups=8, topk_groups=4, group_topn=2, renorm=1,
             route_scale=2.5, in_dtype=1)
    c.update(kw)
    return moe.RouteCfg(**c)


@pytest.mark.parametrize("kw,status", [
    (dict(K=0), 1), (dict(K=300), 1), (dict(n_groups=3), 1), (dict(topk_groups=0), 1),
    (dict(topk_groups=9), 1), (dict(group_topn=33), 1), (dict(score_fn=5), 1),
    (dict(n_groups=8, topk_groups=1, K=40), 1), (dict(N=96, n_groups=1, K=8), 2),
    (dict(N=256, n_groups=64, topk_groups=8), 1), (dict(N=24, n_groups=2, topk_groups=1, K=4), 2),
    (dict(gate_max_ctas=-1), 1), (dict(bias_mode=3), 1),
])
def test_route_rejects_bad_config(moe, kw, status):
    cfg = _cfg(moe, **kw)
    r = moe._lib.moe_route(ctypes.byref(cfg), None, None, None, None, FAKE, FAKE, FAKE, FAKE, 1 << 20, None)
    assert r == status


def test_route_rejects_null_outputs_and_workspace(moe):
    cfg = _cfg(moe)
    L = moe._lib
    assert L.moe_route(None, None, None, None, None, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == 1
    assert L.moe_route(ctypes.byref(cfg), None, None, None, None, None, FAKE, FAKE, FAKE, 1 << 20, None) == 1
    assert L.moe_route(ctypes.byref(cfg), None, None, None, None, MISALIGNED, FAKE, FAKE, FAKE, 1 << 20, None) == 1
    # gate requested without weights / with a short workspace
    assert L.moe_route(ctypes.byref(cfg), FAKE, None, None, None, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == 1
    assert L.moe_route(ctypes.byref(cfg), FAKE, FAKE, None, None, FAKE, FAKE, FAKE, FAKE, 16, None) == 1


def test_route_bias_mode_validation(moe):
    L = moe._lib
    # unknown mode; the bias in the logits needs the gate input
    assert L.moe_route(ctypes.byref(_cfg(moe, bias_mode=2)), FAKE, FAKE, None, None, FAKE, FAKE, FAKE, FAKE,
                       1 << 20, None) == 1
    assert L.moe_route(ctypes.byref(_cfg(moe, bias_mode=1)), None, None, None, FAKE, FAKE, FAKE, FAKE, FAKE,
                       1 << 20, None) == 1


def test_balanced_and_ema_reject_bad_arguments(moe):
    L = moe._lib
    assert L.moe_route_balanced(-1, 8, 256, 1.0, FAKE, FAKE, None) == 1
    assert L.moe_route_balanced(16, 0, 256, 1.0, FAKE, FAKE, None) == 1
    assert L.moe_route_balanced(16, 300, 256, 1.0, FAKE, FAKE, None) == 1
    assert L.moe_route_balanced(16, 8, 256, 1.0, None, FAKE, None) == 1
    assert L.moe_route_balanced(0, 8, 256, 1.0, None, None, None) == 0  # empty batch: nothing to write
    assert L.moe_bias_update_ema(FAKE, 256, 100, 0.001, 1.0, FAKE, FAKE, None) == 1
    assert L.moe_bias_update_ema(FAKE, 256, 100, 0.001, -0.5, FAKE, FAKE, None) == 1
    assert L.moe_bias_update_ema(FAKE, 256, 0, 0.001, 0.9, FAKE, FAKE, None) == 1
    assert L.moe_bias_update_ema(FAKE, 256, 100, 0.001, 0.9, None, FAKE, None) == 1


def test_route_capacity_rejects_bad_arguments(moe):
    L = moe._lib
    ws = L.moe_capacity_workspace_bytes(64, 8, 256)
    assert ws > L.moe_workspace_bytes(64, 8, 256, 256)
    cfg = _cfg(moe)
    # a negative capacity selects the page's rule; the missing scores are still rejected before any launch
    assert L.moe_route_capacity(ctypes.byref(cfg), None, None, -1, FAKE, FAKE, None, FAKE, ws, None) == 1
    assert L.moe_route_capacity(ctypes.byref(_cfg(moe, K=17, n_groups=1)), FAKE, None, 5, FAKE, FAKE, None, FAKE,
                                ws, None) == 1
    assert L.moe_route_capacity(ctypes.byref(cfg), None, None, 5, FAKE, FAKE, None, FAKE, ws, None) == 1
    assert L.moe_route_capacity(ctypes.byref(cfg), FAKE, None, 5, FAKE, FAKE, None, FAKE, ws - 1, None) == 1
    assert L.moe_route_capacity(ctypes.byref(cfg), MISALIGNED, None, 5, FAKE, FAKE, None, FAKE, ws, None) == 1
    assert L.moe_route_capacity(None, FAKE, None, 5, FAKE, FAKE, None, FAKE, ws, None) == 1


def test_load_stats_rejects_bad_arguments(moe):
    L = moe._lib
    ws = 1 << 24
    assert L.moe_load_stats(FAKE, 64, 8, 256, None, 200, None, FAKE, FAKE, FAKE, None, 1, None, FAKE, ws, None) == 1
    assert L.moe_load_stats(FAKE, 64, 8, 256, None, 288, None, FAKE, FAKE, FAKE, None, 1, None, FAKE, ws, None) == 1
    assert L.moe_load_stats(FAKE, 64, 8, 256, None, 256, None, FAKE, FAKE, FAKE, None, 1, None, FAKE, 8, None) == 1
    assert L.moe_load_stats(None, 64, 8, 256, None, 256, None, FAKE, FAKE, FAKE, None, 1, None, FAKE, ws, None) == 1
    assert L.moe_load_stats(FAKE, 1 << 28, 16, 256, None, 256, None, FAKE, FAKE, FAKE, None, 1, None, FAKE, ws,
                            None) == 1


def test_dispatch_and_combine_reject_bad_arguments(moe):
    L = moe._lib
    # d not a multiple of 8 for bf16; FP8 without scales; FP8 with d % 128 != 0; misaligned rows
    assert L.moe_dispatch(FAKE, 1, 10, 100, 8, FAKE, FAKE, FAKE, FAKE, None, None, None, None, None) == 1
    assert L.moe_dispatch(FAKE, 1, 10, 256, 8, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, None) == 1
    assert L.moe_dispatch(FAKE, 1, 10, 136, 8, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None) == 1
    assert L.moe_dispatch(FAKE, 1, 10, 256, 8, FAKE, FAKE, FAKE, MISALIGNED, None, None, None, None, None) == 1
    assert L.moe_dispatch(FAKE, 7, 10, 256, 8, FAKE, FAKE, FAKE, FAKE, None, None, None, None, None) == 1
    assert L.moe_combine(FAKE, 1, 10, 256, 33, FAKE, FAKE, FAKE, None) == 1
    assert L.moe_combine(FAKE, 1, 10, 256, 8, FAKE, FAKE, MISALIGNED, None) == 1
    assert L.moe_combine(None, 1, 10, 256, 8, FAKE, FAKE, FAKE, None) == 1


def test_bias_update_and_replica_plan_reject_bad_arguments(moe):
    L = moe._lib
    assert L.moe_bias_update(FAKE, 256, 0, 0.001, 0, FAKE, None) == 1
    assert L.moe_bias_update(FAKE, 256, 100, 0.001, 2, FAKE, None) == 1
    assert L.moe_bias_update(None, 256, 100, 0.001, 0, FAKE, None) == 1
    assert L.moe_replica_plan(FAKE, 256, 257, FAKE, None) == 1
    assert L.moe_replica_plan(FAKE, 256, -1, FAKE, None) == 1
    assert L.moe_workspace_status(None, None) == 1


def test_binding_refuses_cpu_tensors(moe):
    import torch
    with pytest.raises(ValueError):
        moe._ptr(torch.zeros(4))


def test_capacity_limit_is_the_pages_rule(moe):
    """moe_capacity_limit computes ceil(1.25*T*K/N) in the library (the entropy
    page's "Production Testing" capacity factor), equal to the pinned oracle rule."""
    import oracle
    L = moe._lib
    for T, K, N in ((16384, 8, 256), (4096, 8, 256), (131072, 8, 256), (65536, 8, 128), (512, 2, 8), (6, 1, 4),
                    (3, 2, 4), (7, 1, 4), (0, 8, 256), (1, 1, 1000), (1 << 27, 8, 2048)):
        assert L.moe_capacity_limit(T, K, N) == oracle.capacity_limit(T, K, N), (T, K, N)
        assert moe.capacity_limit(T, K, N) == oracle.capacity_limit(T, K, N)
    assert L.moe_capacity_limit(-1, 8, 256) == -1 and L.moe_capacity_limit(16, 0, 256) == -1
    assert L.moe_capacity_limit(16, 8, 0) == -1


def test_route_tiles_and_tile_stats_reject_bad_arguments(moe):
    """The fused entry points validate on the host: missing buffers, a shape
    the epilogue cannot select, fp32 inputs, misalignment, a short workspace.
    (Every call here fails before any launch.)"""
    L = moe._lib
    ws = L.moe_workspace_bytes(64, 8, 256, 256)
    cfg = _cfg(moe)
    by = ctypes.byref
    # no tile histogram buffer
    assert L.moe_route_tiles(by(cfg), FAKE, FAKE, None, None, FAKE, FAKE, None, FAKE, ws, None) == 1
    # no x: the fused path needs the gate
    assert L.moe_route_tiles(by(cfg), None, FAKE, None, None, FAKE, FAKE, FAKE, FAKE, ws, None) == 1
    # K > 8, N = 512 and fp32 inputs have no epilogue selection
    assert L.moe_route_tiles(by(_cfg(moe, K=16, n_groups=1)), FAKE, FAKE, None, None, FAKE, FAKE, FAKE, FAKE, ws,
                             None) == 2
    assert L.moe_route_tiles(by(_cfg(moe, N=512, n_groups=16)), FAKE, FAKE, None, None, FAKE, FAKE, FAKE, FAKE,
                             L.moe_workspace_bytes(64, 8, 512, 512), None) == 2
    assert L.moe_route_tiles(by(_cfg(moe, in_dtype=0)), FAKE, FAKE, None, None, FAKE, FAKE, FAKE, FAKE, ws,
                             None) == 2
    assert L.moe_route_tiles(by(cfg), MISALIGNED, FAKE, None, None, FAKE, FAKE, FAKE, FAKE, ws, None) == 1
    assert L.moe_route_tiles(by(cfg), FAKE, FAKE, None, None, FAKE, FAKE, FAKE, FAKE, ws - 1, None) == 1
    # load statistics from tile histograms
    wsl = L.moe_workspace_bytes(64, 8, 256, 256)
    assert L.moe_load_stats_tiles(FAKE, 64, 8, 256, None, None, 256, None, FAKE, FAKE, FAKE, None, FAKE, wsl,
                                  None) == 1
    assert L.moe_load_stats_tiles(FAKE, 64, 8, 256, FAKE, None, 288, None, FAKE, FAKE, FAKE, None, FAKE, wsl,
                                  None) == 1  # replica slots without a replica map
    assert L.moe_load_stats_tiles(FAKE, 64, 8, 256, FAKE, None, 256, None, FAKE, FAKE, FAKE, None, FAKE, wsl - 1,
                                  None) == 1


def test_workspace_must_be_16_byte_aligned(moe):
    """Every call that takes a workspace refuses one that does not start on a
    16-byte boundary, before any launch (all other arguments here are valid)."""
    L = moe._lib
    by = ctypes.byref
    cfg = _cfg(moe)
    ws = L.moe_workspace_bytes(64, 8, 256, 256)
    assert L.moe_route(by(cfg), FAKE, FAKE, None, None, FAKE, FAKE, FAKE, MISALIGNED, ws, None) == 1
    assert L.moe_route_tiles(by(cfg), FAKE, FAKE, None, None, FAKE, FAKE, FAKE, MISALIGNED, ws, None) == 1
    assert L.moe_load_stats(FAKE, 64, 8, 256, None, 256, None, FAKE, FAKE, FAKE, None, 1, None, MISALIGNED, ws,
                            None) == 1
    assert L.moe_load_stats_tiles(FAKE, 64, 8, 256, FAKE, None, 256, None, FAKE, FAKE, FAKE, None, MISALIGNED, ws,
                                  None) == 1
    wsc = L.moe_capacity_workspace_bytes(64, 8, 256)
    assert L.moe_route_capacity(by(cfg), FAKE, None, 5, FAKE, FAKE, None, MISALIGNED, wsc, None) == 1
    assert L.moe_workspace_status(MISALIGNED, None) == 1
    assert L.moe_selftest_wait_timeout(MISALIGNED, 1 << 24, None) == 1
