"""GPU parity of capacity-limited routing (a hard per-expert capacity, the
excess moved to each token's next ranked candidates, the rest dropped)
against the oracle on the same fp32 scores: indices, weights and counters
bit-exact; then the dropped assignments through histogram, offsets,
dispatch and combine."""
import numpy as np
import pytest
import torch

from expert_load_balancing_tcgen05_b200 import workloads as W
from gpu_util import assert_stats_close, lib, load_stats_gpu, route_gpu, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")


def _capacity_gpu(wl, scores, bias, C, bias_mode=0):
    moe = lib()
    T, N, K = wl.T, wl.N, wl.K
    idx = torch.full((T, K), -7, dtype=torch.int32, device="cuda")
    w = torch.full((T, K), -7.0, device="cuda")
    info = moe.empty_capacity_info()
    ws = moe.capacity_workspace(T, K, N)
    cfg = moe.route_cfg(T, wl.d, N, K, wl.fn, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm, wl.scale,
                        bias_in_logits=bool(bias_mode))
    moe.moe_route_capacity(cfg, scores, bias, C, idx, w, info, ws)
    torch.cuda.synchronize()
    return idx, w, moe.read_capacity_info(info), ws


def _gpu_scores(wl, seed):
    inp = W.make_inputs(wl, seed=seed)
    off = inp["off"].cuda() if inp["off"] is not None else None
    b = inp["bias"].cuda() if inp["bias"] is not None else None
    s, _, _, _ = route_gpu(wl, inp["x"].cuda(), inp["W"].cuda(), off, b)
    return s, b


def _check(orc, wl, s, b, C):
    idx, w, info, _ = _capacity_gpu(wl, s, b, C)
    ri, rw, rinfo = orc.route_capacity(to_np(s), to_np(b) if b is not None else None, wl.K, wl.n_groups,
                                       wl.topk_groups, wl.group_topn, wl.renorm, wl.scale, capacity=C)
    assert np.array_equal(to_np(idx), ri)
    assert np.array_equal(to_np(w), rw)
    assert info == rinfo
    return idx, w, info


@pytest.mark.parametrize("name,T", [("collapse", 16384), ("v3_router", 1000), ("softmax_dispatch", 3001)])
def test_capacity_matches_oracle(orc, name, T):
    wl = W.WORKLOADS[name].with_(T=T)
    s, b = _gpu_scores(wl, seed=41)
    C = lib().capacity_limit(T, wl.K, wl.N)
    idx, w, info = _check(orc, wl, s, b, C)
    if name == "collapse":
        assert info["overflow"] > 0 and info["rerouted"] > 0  # the celebrity experts overflow


@pytest.mark.parametrize("C", [0, 1, 5, 10 ** 9])
def test_capacity_edge_values(orc, C):
    wl = W.WORKLOADS["v3_router"].with_(T=257)
    s, b = _gpu_scores(wl, seed=3)
    idx, w, info = _check(orc, wl, s, b, C)
    if C == 0:
        assert (to_np(idx) == -1).all() and (to_np(w) == 0).all()
    if C == 10 ** 9:
        # no limit: exactly moe_route's selection
        _, ri, rw, _ = route_gpu(wl, None, None, None, b, scores_in=s)
        assert torch.equal(idx, ri) and torch.equal(w, rw)


def test_capacity_small_groups_and_ragged(orc):
    # fp32 scores drawn directly; N=64 in 8 groups, K=6, several candidate
    # exhaustions with topk_groups=1 (8 candidates for 12 ranks)
    T, N, K = 999, 64, 6
    wl = W.Workload("cap_small", 0, T, 64, N, K, 1, n_groups=8, topk_groups=1, group_topn=2, renorm=True,
                    scale=1.5)
    s = (W.make_scores(T, N, seed=5) * torch.linspace(1.0, 0.3, N)[None, :]).contiguous()
    b = torch.from_numpy(np.random.default_rng(2).uniform(-0.01, 0.01, N).astype(np.float32))
    _check(orc, wl, s.cuda(), b.cuda(), lib().capacity_limit(T, K, N))


def test_capacity_bias_in_logits_ignores_bias(orc):
    wl = W.WORKLOADS["v3_router"].with_(T=500)
    s, b = _gpu_scores(wl, seed=9)
    C = 40
    i1, w1, _, _ = _capacity_gpu(wl, s, b, C, bias_mode=1)
    i2, w2, _, _ = _capacity_gpu(wl, s, None, C)
    assert torch.equal(i1, i2) and torch.equal(w1, w2)


def test_capacity_empty_batch():
    moe = lib()
    wl = W.WORKLOADS["v3_router"].with_(T=0)
    info = moe.empty_capacity_info()
    ws = moe.capacity_workspace(1, wl.K, wl.N)
    cfg = moe.route_cfg(0, wl.d, wl.N, wl.K, wl.fn, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm, wl.scale)
    moe._check(moe._lib.moe_route_capacity(moe.ctypes.byref(cfg), None, None, 5, None, None, moe._ptr(info),
                                           moe._ptr(ws), ws.numel(), None), "moe_route_capacity")
    torch.cuda.synchronize()
    assert moe.read_capacity_info(info) == dict(capacity=5, overflow=0, rerouted=0, dropped=0)


def test_dropped_assignments_through_dispatch_and_combine(orc):
    """Capacity output -> histogram/offsets/ranks -> dispatch (bf16 + FP8) ->
    combine, each against the oracle; dropped slots get no row."""
    moe = lib()
    wl = W.WORKLOADS["collapse"].with_(T=3000, d=512)
    s, b = _gpu_scores(wl, seed=13)
    T, N, K, d = wl.T, wl.N, wl.K, wl.d
    C = moe.capacity_limit(T, K, N)
    idx, w, info = _check(orc, wl, s, b, C)
    assert info["dropped"] > 0
    ri = to_np(idx)
    slot, counts, offsets, rank, stats, _ = load_stats_gpu(idx, T, K, N)
    torch.cuda.synchronize()
    c_ref, off_ref, pos_ref, rank_ref, src_ref = orc.positions(ri, N)
    assert np.array_equal(to_np(counts), c_ref)
    assert np.array_equal(to_np(offsets), off_ref)
    assert np.array_equal(to_np(rank), rank_ref)
    assert np.array_equal(to_np(slot), np.where(ri < 0, -1, ri))
    assert to_np(counts).max() <= C
    kept = T * K - info["dropped"]
    assert int(to_np(offsets)[-1]) == kept
    assert_stats_close(moe.read_stats(stats), orc.load_stats(c_ref))
    assert moe.read_stats(stats)["status"] == 0
    x = torch.randn(T, d, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    rows = torch.zeros(T * K, d, dtype=torch.bfloat16, device="cuda")
    q = torch.zeros(T * K, d, dtype=torch.uint8, device="cuda")
    sc = torch.zeros(T * K, d // 128, dtype=torch.float32, device="cuda")
    pos = torch.empty(T, K, dtype=torch.int32, device="cuda")
    row_src = torch.full((T * K,), -5, dtype=torch.int32, device="cuda")
    moe.moe_dispatch(x.cuda(), T, d, K, slot, offsets, rank, rows, q, sc, pos, row_src)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(pos), pos_ref)
    assert np.array_equal(to_np(row_src)[:kept], src_ref[:kept])
    assert (to_np(row_src)[kept:] == -5).all()  # nothing written past the kept rows
    # the kept rows; rows past them are scratch (dropped copies land in the last one)
    rows_ref = orc.dispatch_rows(x.view(torch.int16).numpy(), pos_ref)
    assert np.array_equal(rows.view(torch.int16).cpu().numpy()[:kept], rows_ref[:kept])
    assert not rows.view(torch.int16)[kept:T * K - 1].any()
    q_ref, sc_ref = orc.fp8_rows(orc.dispatch_rows(x.float().numpy(), pos_ref))
    assert np.array_equal(to_np(q)[:kept], q_ref[:kept]) and np.array_equal(to_np(sc)[:kept], sc_ref[:kept])
    out = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(rows, T, d, K, pos, w, out)
    ref = orc.combine(rows.float().cpu().numpy(), pos_ref, to_np(w))
    got = to_np(out).astype(np.float64)
    assert (np.abs(got - ref) <= np.maximum(2e-2, np.abs(ref) * 2.0 ** -8)).all()


@pytest.mark.parametrize("name", ["v3_router", "metric"])
def test_negative_capacity_is_the_pages_rule(orc, name):
    """capacity < 0: the library applies ceil(1.25*T*K/N) itself (entropy page,
    "Production Testing"); the result equals the oracle run at that capacity."""
    wl = W.WORKLOADS[name]
    s, b = _gpu_scores(wl, seed=17)
    idx, w, info, _ = _capacity_gpu(wl, s, b, -1)
    C = orc.capacity_limit(wl.T, wl.K, wl.N)
    assert info["capacity"] == C
    ri, rw, rinfo = orc.route_capacity(to_np(s), to_np(b), wl.K, wl.n_groups, wl.topk_groups, wl.group_topn,
                                       wl.renorm, wl.scale, capacity=C)
    assert np.array_equal(to_np(idx), ri) and np.array_equal(to_np(w), rw)
    assert info == rinfo
