"""Edge cases and maximum sizes through the C ABI, against the oracle:
selection with K = N, K = 32, all-tied scores and all groups kept; load
statistics at the largest slot count (2048, with replicas) and K = 32, and
at a million tokens; dispatch with K = 32 and the FP8 copy; the gate at the
smallest hidden size; every call on an empty batch."""
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


def _wl(N, K, G, TG, T, topn=2, renorm=True, scale=1.0, fn=1):
    return W.Workload("edge", 0, T, 64, N, K, fn, n_groups=G, topk_groups=TG, group_topn=topn, renorm=renorm,
                      scale=scale)


@pytest.mark.parametrize("N,K,G,TG", [(8, 8, 1, 1), (32, 32, 1, 1), (64, 32, 2, 2), (256, 32, 8, 8),
                                      (128, 16, 4, 4), (512, 32, 1, 1)])
def test_selection_large_k(orc, N, K, G, TG):
    T = 333
    s = W.make_scores(T, N, seed=N + K)
    b = W.make_bias(N, seed=K)
    _, idx, w, _ = route_gpu(_wl(N, K, G, TG, T, scale=2.5), None, None, None, b.cuda(), scores_in=s.cuda())
    ri, rw = orc.select(s.numpy(), b.numpy(), K, G, TG, 2, True, 2.5)
    assert np.array_equal(to_np(idx), ri)
    assert np.array_equal(to_np(w), rw)


@pytest.mark.parametrize("N,K,G,TG", [(256, 8, 8, 4), (128, 8, 1, 1), (64, 6, 4, 2), (8, 2, 1, 1)])
def test_selection_all_tied(orc, N, K, G, TG):
    # every key equal: the lowest groups, then the lowest experts, win
    T = 100
    s = torch.full((T, N), 0.25)
    _, idx, w, _ = route_gpu(_wl(N, K, G, TG, T), None, None, None, None, scores_in=s.cuda())
    ri, rw = orc.select(s.numpy(), None, K, G, TG, 2, True, 1.0)
    assert np.array_equal(to_np(idx), ri)
    assert np.array_equal(to_np(w), rw)
    assert (ri == np.arange(K)[None, :]).all()
    assert (rw == np.float32(1.0 / K)).all()


def test_load_stats_largest_slot_count_and_k(orc):
    # 1024 experts, 1024 replicas: 2048 slots; K = 32
    T, K, N, R = 3001, 32, 1024, 1024
    idx = W.make_assignments(T, K, N, seed=4, skew=0.7)
    slot, counts, offsets, rank, stats, ws = load_stats_gpu(idx.cuda(), T, K, N)
    c_ref = orc.histogram(idx.numpy(), N)
    assert np.array_equal(to_np(counts), c_ref)
    rs = torch.empty(N, dtype=torch.int32, device="cuda")
    lib().moe_replica_plan(counts, N, R, rs)
    rs_ref = orc.replica_plan(c_ref, R)
    assert np.array_equal(to_np(rs), rs_ref)
    slot2, counts2, offsets2, rank2, stats2, _ = load_stats_gpu(idx.cuda(), T, K, N, n_slots=N + R, replica_slot=rs)
    s_ref = orc.apply_replicas(idx.numpy(), rs_ref)
    c2, o2, p2, r2, _ = orc.positions(s_ref, N + R)
    assert np.array_equal(to_np(slot2), s_ref)
    assert np.array_equal(to_np(counts2), c2)
    assert np.array_equal(to_np(offsets2), o2)
    assert np.array_equal(to_np(rank2), r2)
    assert_stats_close(lib().read_stats(stats2), orc.load_stats(c2))


def test_load_stats_million_tokens(orc):
    T, K, N = 1 << 20, 8, 256
    idx = W.make_assignments(T, K, N, seed=12, device="cuda", skew=1.1)
    slot, counts, offsets, rank, stats, ws = load_stats_gpu(idx, T, K, N)
    i_np = to_np(idx)
    c_ref, off_ref, _, rank_ref, _ = orc.positions(i_np, N)
    assert np.array_equal(to_np(counts), c_ref)
    assert np.array_equal(to_np(offsets), off_ref)
    assert np.array_equal(to_np(rank), rank_ref)
    assert_stats_close(lib().read_stats(stats), orc.load_stats(c_ref))
    assert lib().moe_workspace_status(ws) == 0


def test_dispatch_k32_with_fp8(orc):
    T, d, K, N = 200, 256, 32, 64
    x = torch.randn(T, d, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    idx = W.make_assignments(T, K, N, seed=2)
    slot, counts, offsets, rank, _, _ = load_stats_gpu(idx.cuda(), T, K, N)
    rows = torch.empty(T * K, d, dtype=torch.bfloat16, device="cuda")
    q = torch.empty(T * K, d, dtype=torch.uint8, device="cuda")
    sc = torch.empty(T * K, d // 128, device="cuda")
    pos = torch.empty(T, K, dtype=torch.int32, device="cuda")
    lib().moe_dispatch(x.cuda(), T, d, K, slot, offsets, rank, rows, q, sc, pos, None)
    _, _, pos_ref, _, _ = orc.positions(idx.numpy(), N)
    assert np.array_equal(to_np(pos), pos_ref)
    assert np.array_equal(rows.view(torch.int16).cpu().numpy(), orc.dispatch_rows(x.view(torch.int16).numpy(), pos_ref))
    q_ref, sc_ref = orc.fp8_rows(orc.dispatch_rows(x.float().numpy(), pos_ref))
    assert np.array_equal(to_np(q), q_ref) and np.array_equal(to_np(sc), sc_ref)


@pytest.mark.parametrize("d", [8, 72])
def test_gate_smallest_hidden_sizes(orc, d):
    wl = W.WORKLOADS["v3_router"].with_(T=130, d=d)
    inp = W.make_inputs(wl, seed=3)
    s, idx, w, ws = route_gpu(wl, inp["x"].cuda(), inp["W"].cuda(), None, inp["bias"].cuda())
    assert lib().moe_workspace_status(ws) == 0
    h = orc.logits(inp["x"].float().numpy(), inp["W"].float().numpy())
    s_ref = orc.scores(h, wl.fn)
    err = np.abs(to_np(s).astype(np.float64) - s_ref)
    assert (err <= 1e-3 * np.abs(s_ref) + 1e-7).all()
    ri, rw = orc.select(to_np(s), inp["bias"].numpy(), wl.K, wl.n_groups, wl.topk_groups, wl.group_topn, True,
                        wl.scale)
    assert np.array_equal(to_np(idx), ri) and np.array_equal(to_np(w), rw)


def test_every_call_accepts_an_empty_batch():
    moe = lib()
    wl = W.WORKLOADS["v3_router"].with_(T=0)
    N, K, d = wl.N, wl.K, wl.d
    e_f = torch.empty(0, device="cuda")
    x = torch.empty(0, d, dtype=torch.bfloat16, device="cuda")
    Wg = torch.randn(N, d, device="cuda").to(torch.bfloat16)
    ws = moe.workspace(1, K, N)
    cfg = moe.route_cfg(0, d, N, K, wl.fn, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm, wl.scale)
    L = moe._lib
    P = moe.ctypes.c_void_p
    # route with the gate and from scores: nothing to do
    assert L.moe_route(moe.ctypes.byref(cfg), P(x.data_ptr() or Wg.data_ptr()), P(Wg.data_ptr()), None, None,
                       P(ws.data_ptr()), P(ws.data_ptr()), P(ws.data_ptr()), P(ws.data_ptr()), ws.numel(),
                       None) == 0
    counts = torch.full((N,), 7, dtype=torch.int32, device="cuda")
    offsets = torch.full((N + 1,), 7, dtype=torch.int32, device="cuda")
    stats = moe.empty_stats()
    moe.moe_load_stats(None, 0, K, N, None, N, None, counts, offsets, None, None, wl.fn, stats, ws)
    torch.cuda.synchronize()
    assert not counts.any() and not offsets.any()
    assert moe.read_stats(stats)["total"] == 0
    assert L.moe_dispatch(None, 1, 0, d, K, None, None, None, None, None, None, None, None, None) == 0
    assert L.moe_combine(None, 1, 0, d, K, None, None, None, None) == 0
    assert L.moe_route_balanced(0, K, N, 1.0, None, None, None) == 0
    del e_f


@pytest.mark.parametrize("N,K,G,TG,fn", [(512, 8, 16, 4, 1), (32, 4, 4, 2, 1), (512, 16, 1, 1, 0), (16, 3, 1, 1, 0)])
def test_route_with_gate_outside_the_tensor_core_shapes(orc, N, K, G, TG, fn):
    # bf16 inputs whose N has no tensor-core tile run the CUDA-core gate, then the general selection kernel
    T, d = 333, 256
    wl = W.Workload("edge_gate", 0, T, d, N, K, fn, n_groups=G, topk_groups=TG, group_topn=2, renorm=True,
                    scale=2.5, has_bias=True)
    inp = W.make_inputs(wl, seed=N + K)
    s, idx, w, ws = route_gpu(wl, inp["x"].cuda(), inp["W"].cuda(), None, inp["bias"].cuda())
    assert lib().moe_workspace_status(ws) == 0
    h = orc.logits(inp["x"].float().numpy(), inp["W"].float().numpy())
    s_ref = orc.scores(h, fn)
    err = np.abs(to_np(s).astype(np.float64) - s_ref)
    assert (err <= 1e-3 * np.abs(s_ref) + 1e-7).all()
    ri, rw = orc.select(to_np(s), inp["bias"].numpy(), K, G, TG, 2, True, 2.5)
    assert np.array_equal(to_np(idx), ri) and np.array_equal(to_np(w), rw)


def test_load_stats_kernels_share_one_workspace(orc):
    """Problems above and below the chain-free kernel's limit (~2.6M
    assignments: look-back kernel vs tagged-count kernel, one and several
    blocks) alternate on one workspace; each call's counts, offsets and
    ranks equal the oracle's, so neither kernel's left-over words (look-back
    flags, tagged counts, prefixes) are ever read as this call's."""
    N, K = 64, 8
    sizes = [400000, 16384, 100, 131072, 400000, 70000, 100, 16384]
    moe = lib()
    ws = moe.workspace(max(sizes), K, N)
    for i, T in enumerate(sizes):
        idx = W.make_assignments(T, K, N, seed=50 + i, device="cuda", skew=0.6)
        slot, counts, offsets, rank, stats, _ = load_stats_gpu(idx, T, K, N, ws=ws)
        c_ref, off_ref, _, rank_ref, _ = orc.positions(to_np(idx), N)
        assert np.array_equal(to_np(counts), c_ref), T
        assert np.array_equal(to_np(offsets), off_ref), T
        assert np.array_equal(to_np(rank), rank_ref), T
        assert_stats_close(moe.read_stats(stats), orc.load_stats(c_ref))
    assert moe.moe_workspace_status(ws) == 0
