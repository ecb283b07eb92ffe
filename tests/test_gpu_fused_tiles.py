"""The fused routing path: selection inside the tensor-core gate's epilogue
with the load histogram counted there per 128-token tile (moe_route_tiles),
and the load statistics that take those histograms (moe_load_stats_tiles).

Against the oracle on the same inputs: the indices and weights equal the
oracle's selection on the gate's fp32 scores (taken from moe_route's
scores-only epilogue, which computes the same values); the tile histograms
equal the per-tile bincounts of the oracle's selection split by token
parity; counts, offsets, slots and ranks equal the oracle's positions, with
and without replica slots."""
import numpy as np
import pytest
import torch

from expert_load_balancing_tcgen05_b200 import workloads as W
from gpu_util import assert_stats_close, lib, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")


def _tile_hist_ref(idx, N):
    T, K = idx.shape
    nt = (T + 127) // 128
    ref = np.zeros((nt, 2, N), np.int64)
    t = np.repeat(np.arange(T), K)
    np.add.at(ref, (t // 128, t % 2, idx.reshape(-1)), 1)
    return ref


def _fused(wl, inp, monkeypatch=None):
    moe = lib()
    T, N, K = wl.T, wl.N, wl.K
    idx = torch.full((T, K), -7, dtype=torch.int32, device="cuda")
    w = torch.full((T, K), -7.0, device="cuda")
    tiles = torch.full(moe.tile_counts_shape(T, N), -7, dtype=torch.int32, device="cuda")
    ws = moe.workspace(T, K, N, wl.n_slots)
    cfg = moe.route_cfg(T, wl.d, N, K, wl.fn, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm, wl.scale)
    moe.moe_route_tiles(cfg, inp["x"], inp["W"], inp["off"], inp["bias"], idx, w, tiles, ws)
    torch.cuda.synchronize()
    assert moe.moe_workspace_status(ws) == moe.MOE_OK
    return idx, w, tiles, ws


def _scores_only(wl, inp, monkeypatch):
    moe = lib()
    T, N, K = wl.T, wl.N, wl.K
    monkeypatch.setenv("MOE_FUSED_SELECT", "0")
    scores = torch.empty(T, N, device="cuda")
    idx = torch.empty(T, K, dtype=torch.int32, device="cuda")
    w = torch.empty(T, K, device="cuda")
    ws = moe.workspace(T, K, N)
    cfg = moe.route_cfg(T, wl.d, N, K, wl.fn, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm, wl.scale)
    moe.moe_route(cfg, inp["x"], inp["W"], inp["off"], inp["bias"], scores, idx, w, ws)
    torch.cuda.synchronize()
    return scores


@pytest.mark.parametrize("name,T", [("v3_router", 4096), ("metric", 16384), ("prefill_replicas", 131072),
                                    ("softmax_dispatch", 3001), ("v3_router", 300)])
def test_route_tiles_and_stats_match_oracle(orc, monkeypatch, name, T):
    moe = lib()
    wl = W.WORKLOADS[name].with_(T=T)
    inp = W.make_inputs(wl, device="cuda", seed=31)
    idx, w, tiles, ws = _fused(wl, inp)
    s = _scores_only(wl, inp, monkeypatch)
    b = inp["bias"].cpu().numpy() if inp["bias"] is not None else None
    ri, rw = orc.select(to_np(s), b, wl.K, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm, wl.scale)
    del s
    assert np.array_equal(to_np(idx), ri)
    assert np.array_equal(to_np(w), rw)
    assert np.array_equal(to_np(tiles), _tile_hist_ref(ri, wl.N))
    N, K = wl.N, wl.K
    for R in ([0, wl.n_replicas] if wl.n_replicas else [0]):
        n_slots = N + R
        rs = None
        if R:
            c = torch.from_numpy(orc.histogram(ri, N).astype(np.int32)).cuda()
            rs = torch.empty(N, dtype=torch.int32, device="cuda")
            moe.moe_replica_plan(c, N, R, rs)
            slot_ref = orc.apply_replicas(ri, to_np(rs))
        else:
            slot_ref = ri
        slot = torch.full((T, K), -7, dtype=torch.int32, device="cuda")
        counts = torch.full((n_slots,), -7, dtype=torch.int32, device="cuda")
        offsets = torch.full((n_slots + 1,), -7, dtype=torch.int32, device="cuda")
        rank = torch.full((T, K), -7, dtype=torch.int32, device="cuda")
        stats = moe.empty_stats()
        ws2 = moe.workspace(T, K, N, n_slots)
        moe.moe_load_stats_tiles(idx, T, K, N, tiles, rs, n_slots, slot, counts, offsets, rank, stats, ws2)
        torch.cuda.synchronize()
        c_ref, off_ref, _, rank_ref, _ = orc.positions(slot_ref, n_slots)
        assert np.array_equal(to_np(slot), slot_ref)
        assert np.array_equal(to_np(counts), c_ref)
        assert np.array_equal(to_np(offsets), off_ref)
        assert np.array_equal(to_np(rank), rank_ref)
        assert_stats_close(moe.read_stats(stats), orc.load_stats(c_ref))
        assert moe.moe_workspace_status(ws2) == moe.MOE_OK


def test_inconsistent_tile_histograms_are_reported(orc):
    """A tile histogram that does not match the indices (here one count
    moved between experts in the last block's tiles) is reported as an
    invalid argument by the call's status and by the workspace status."""
    moe = lib()
    T, K, N = 4096, 8, 256
    idx = W.make_assignments(T, K, N, seed=3).cuda()
    ref = _tile_hist_ref(to_np(idx), N)
    bad = ref.copy()
    j = ref.shape[0] - 1
    e_from = int(np.nonzero(bad[j, 0])[0][0])
    bad[j, 0, e_from] -= 1
    bad[j, 0, (e_from + 1) % N] += 1
    out = {}
    for name, tc in (("good", ref), ("bad", bad)):
        tiles = torch.from_numpy(tc.astype(np.int32)).cuda()
        counts = torch.empty(N, dtype=torch.int32, device="cuda")
        offsets = torch.empty(N + 1, dtype=torch.int32, device="cuda")
        rank = torch.empty(T, K, dtype=torch.int32, device="cuda")
        stats = moe.empty_stats()
        ws = moe.workspace(T, K, N)
        moe.moe_load_stats_tiles(idx, T, K, N, tiles, None, N, None, counts, offsets, rank, stats, ws)
        torch.cuda.synchronize()
        out[name] = (moe.read_stats(stats)["status"], moe.moe_workspace_status(ws))
    assert out["good"] == (moe.MOE_OK, moe.MOE_OK)
    assert out["bad"] == (moe.MOE_ERR_INVALID, moe.MOE_ERR_INVALID)


def test_route_tiles_rejects_what_the_epilogue_cannot_select():
    moe = lib()
    wl = W.WORKLOADS["v3_router"].with_(T=64)
    inp = W.make_inputs(wl, device="cuda", seed=1)
    idx = torch.empty(wl.T, 16, dtype=torch.int32, device="cuda")
    w = torch.empty(wl.T, 16, device="cuda")
    tiles = torch.empty(moe.tile_counts_shape(wl.T, wl.N), dtype=torch.int32, device="cuda")
    ws = moe.workspace(wl.T, 16, wl.N)
    cfg = moe.route_cfg(wl.T, wl.d, wl.N, 16, wl.fn, wl.n_groups, wl.topk_groups, wl.group_topn, True, 1.0)
    with pytest.raises(moe.MoeError) as e:
        moe.moe_route_tiles(cfg, inp["x"], inp["W"], None, inp["bias"], idx, w, tiles, ws)  # K = 16 > 8
    assert e.value.status == moe.MOE_ERR_UNSUPPORTED


@pytest.mark.parametrize("kind", ["zero_gate", "twin_experts", "quad_experts_topn1"])
def test_route_tiles_with_ties_match_oracle(orc, monkeypatch, kind):
    """Tied keys inside and across groups: the epilogue's candidate bound
    admits keys equal to it and the choice keeps (key desc, index asc).
    zero_gate: every score is 0.5 and every key equal without bias;
    twin_experts / quad_experts: experts share their gate row (and bias)
    in pairs or fours, so every key has equal partners."""
    wl = W.WORKLOADS["v3_router"].with_(T=1500, d=512)
    if kind == "quad_experts_topn1":
        wl = wl.with_(group_topn=1)
    inp = W.make_inputs(wl, device="cuda", seed=41)
    if kind == "zero_gate":
        inp["W"] = torch.zeros_like(inp["W"])
        inp["bias"] = None
    else:
        m = 2 if kind == "twin_experts" else 4
        src = torch.arange(wl.N, device="cuda") // m * m
        inp["W"] = inp["W"][src].contiguous()
        inp["bias"] = inp["bias"][src].contiguous()
    idx, w, tiles, _ = _fused(wl, inp)
    s = _scores_only(wl, inp, monkeypatch)
    b = inp["bias"].cpu().numpy() if inp["bias"] is not None else None
    ri, rw = orc.select(to_np(s), b, wl.K, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm, wl.scale)
    assert np.array_equal(to_np(idx), ri)
    assert np.array_equal(to_np(w), rw)
    assert np.array_equal(to_np(tiles), _tile_hist_ref(ri, wl.N))
    if kind == "zero_gate":
        assert np.array_equal(ri, np.broadcast_to(np.arange(wl.K, dtype=ri.dtype), ri.shape))


@pytest.mark.parametrize("kind", ["softmax_n128", "softmax_zero_gate", "sigmoid_one_group", "softmax_twins"])
def test_route_tiles_one_group_match_oracle(orc, monkeypatch, kind):
    """One group (every expert a candidate): the epilogue's bound comes from
    the 8-column pieces' second-largest keys of both row halves.  Random
    scores, a zero gate (every key equal: the lowest experts win) and experts
    sharing their gate rows in pairs (ties at and around the bound)."""
    if kind == "sigmoid_one_group":
        wl = W.Workload("sig1", 0, 900, 1024, 256, 8, fn=1, scale=2.5, has_bias=True)
    else:
        wl = W.Workload("sm128", 0, 900, 1024, 128, 8, fn=0, scale=1.0, has_bias=kind == "softmax_twins")
    inp = W.make_inputs(wl, device="cuda", seed=43)
    if kind == "softmax_zero_gate":
        inp["W"] = torch.zeros_like(inp["W"])
    if kind == "softmax_twins":
        src = torch.arange(wl.N, device="cuda") // 2 * 2
        inp["W"] = inp["W"][src].contiguous()
        inp["bias"] = inp["bias"][src].contiguous()
    idx, w, tiles, _ = _fused(wl, inp)
    s = _scores_only(wl, inp, monkeypatch)
    b = inp["bias"].cpu().numpy() if inp["bias"] is not None else None
    ri, rw = orc.select(to_np(s), b, wl.K, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm, wl.scale)
    assert np.array_equal(to_np(idx), ri)
    assert np.array_equal(to_np(w), rw)
    assert np.array_equal(to_np(tiles), _tile_hist_ref(ri, wl.N))
    if kind == "softmax_zero_gate":
        assert np.array_equal(ri, np.broadcast_to(np.arange(wl.K, dtype=ri.dtype), ri.shape))
