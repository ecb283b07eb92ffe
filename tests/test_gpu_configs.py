"""The five routing workloads at their full sizes, in the launch
configuration the benchmark uses, against the oracle: everything integer
bit-exact over the whole batch, floating-point outputs on sampled tokens
(the fp64 gate for the sample, combine for the sample), and the invariants
that hold at any size."""
import numpy as np
import pytest
import torch

from expert_load_balancing_tcgen05_b200 import workloads as W
from gpu_util import assert_stats_close, gap_ok, lib, load_stats_gpu, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")


def _sample(T, n, seed):
    g = np.random.default_rng(seed)
    s = np.unique(np.concatenate([g.choice(T, size=min(n, T), replace=False), [0, T - 1]]))
    return s


def _route(wl, inp):
    moe = lib()
    T, N, K = wl.T, wl.N, wl.K
    scores = torch.empty(T, N, device="cuda")
    idx = torch.empty(T, K, dtype=torch.int32, device="cuda")
    w = torch.empty(T, K, device="cuda")
    ws = moe.workspace(T, K, N, wl.n_slots)
    cfg = moe.route_cfg(T, wl.d, N, K, wl.fn, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm, wl.scale,
                        moe.MOE_BF16 if wl.dtype == torch.bfloat16 else moe.MOE_F32)
    moe.moe_route(cfg, inp["x"], inp["W"], inp["off"], inp["bias"], scores, idx, w, ws)
    torch.cuda.synchronize()
    assert moe.moe_workspace_status(ws) == 0
    return scores, idx, w, ws


def _check_gate_sample(orc, wl, inp, scores, idx, sample):
    x = inp["x"][torch.from_numpy(sample).cuda()].float().cpu().numpy()
    Wg = inp["W"].float().cpu().numpy()
    off = inp["off"].cpu().numpy() if inp["off"] is not None else None
    s_ref = orc.scores(orc.logits(x, Wg, off), wl.fn)
    s_gpu = to_np(scores)[sample]
    err = np.abs(s_gpu.astype(np.float64) - s_ref)
    assert (err <= 1e-3 * np.abs(s_ref) + 1e-7).all()
    b = inp["bias"].cpu().numpy() if inp["bias"] is not None else None
    ri, _ = orc.select(s_ref, b, wl.K, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm, wl.scale)
    _, bad = gap_ok(s_ref, b, to_np(idx)[sample], ri, wl.K, wl.n_groups, wl.topk_groups, wl.group_topn)
    assert not bad


def _check_selection_full(orc, wl, inp, scores, idx, w):
    b = inp["bias"].cpu().numpy() if inp["bias"] is not None else None
    ri, rw = orc.select(to_np(scores), b, wl.K, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm, wl.scale)
    assert np.array_equal(to_np(idx), ri)
    assert np.array_equal(to_np(w), rw)
    return ri


def _dispatch(x, T, d, K, slot, offsets, rank, fp8=False):
    moe = lib()
    rows = torch.empty(T * K, d, dtype=x.dtype, device="cuda")
    q = torch.empty(T * K, d, dtype=torch.uint8, device="cuda") if fp8 else None
    sc = torch.empty(T * K, d // 128, dtype=torch.float32, device="cuda") if fp8 else None
    pos = torch.empty(T, K, dtype=torch.int32, device="cuda")
    row_src = torch.empty(T * K, dtype=torch.int32, device="cuda")
    moe.moe_dispatch(x, T, d, K, slot, offsets, rank, rows, q, sc, pos, row_src)
    return rows, q, sc, pos, row_src


def _check_dispatch_sample(orc, x, rows, q, sc, pos, sample):
    p = to_np(pos)[sample]                      # [S, K]
    xs = x[torch.from_numpy(sample).cuda()]
    pr = torch.from_numpy(p.reshape(-1).astype(np.int64)).cuda()
    got = rows[pr].view(len(sample), -1, x.shape[1])
    assert torch.equal(got, xs[:, None, :].expand_as(got))
    if q is not None:
        q_ref, sc_ref = orc.fp8_rows(xs.float().cpu().numpy())
        K = p.shape[1]
        assert np.array_equal(to_np(q[pr]).reshape(len(sample), K, -1), np.repeat(q_ref[:, None], K, 1))
        assert np.array_equal(to_np(sc[pr]).reshape(len(sample), K, -1), np.repeat(sc_ref[:, None], K, 1))


def test_tiny_softmax_router_full(orc):
    wl = W.WORKLOADS["tiny_softmax"]
    inp = W.make_inputs(wl, device="cuda")
    scores, idx, w, ws = _route(wl, inp)
    x = inp["x"].cpu().numpy()
    s_ref = orc.scores(orc.logits(x, inp["W"].cpu().numpy()), 0)
    assert (np.abs(to_np(scores) - s_ref) <= 1e-3 * np.abs(s_ref) + 1e-7).all()
    ri = _check_selection_full(orc, wl, inp, scores, idx, w)
    slot, counts, offsets, rank, stats, _ = load_stats_gpu(idx, wl.T, wl.K, wl.N, scores=scores, score_fn=0)
    c_ref, off_ref, pos_ref, rank_ref, src_ref = orc.positions(ri, wl.N)
    assert np.array_equal(to_np(counts), c_ref) and np.array_equal(to_np(rank), rank_ref)
    st = lib().read_stats(stats)
    assert_stats_close(st, orc.load_stats(c_ref))
    assert abs(st["entropy_score_bits"] - orc.score_entropy(to_np(scores), 0)) <= 1e-6 * 3
    rows, q, sc, pos, row_src = _dispatch(inp["x"], wl.T, wl.d, wl.K, slot, offsets, rank, fp8=True)
    assert np.array_equal(to_np(rows), orc.dispatch_rows(x, pos_ref))
    assert np.array_equal(to_np(row_src), src_ref)
    q_ref, sc_ref = orc.fp8_rows(orc.dispatch_rows(x, pos_ref))
    assert np.array_equal(to_np(q), q_ref) and np.array_equal(to_np(sc), sc_ref)
    out = torch.empty_like(inp["x"])
    lib().moe_combine(rows, wl.T, wl.d, wl.K, pos, w, out)
    ref = orc.combine(to_np(rows), pos_ref, to_np(w))
    assert (np.abs(to_np(out) - ref) <= 1e-5 * np.maximum(1, np.abs(ref))).all()
    assert (np.abs(to_np(out) - x) <= 1e-5 * np.maximum(1, np.abs(x))).all()  # round trip


def test_v3_router_full(orc):
    wl = W.WORKLOADS["v3_router"]
    inp = W.make_inputs(wl, device="cuda")
    scores, idx, w, ws = _route(wl, inp)
    _check_gate_sample(orc, wl, inp, scores, idx, _sample(wl.T, 384, 1))
    ri = _check_selection_full(orc, wl, inp, scores, idx, w)
    slot, counts, offsets, rank, stats, _ = load_stats_gpu(idx, wl.T, wl.K, wl.N, scores=scores, score_fn=1)
    c_ref, off_ref, pos_ref, rank_ref, _ = orc.positions(ri, wl.N)
    assert np.array_equal(to_np(counts), c_ref) and np.array_equal(to_np(offsets), off_ref)
    assert np.array_equal(to_np(rank), rank_ref)
    assert_stats_close(lib().read_stats(stats), orc.load_stats(c_ref))
    rows, _, _, pos, row_src = _dispatch(inp["x"], wl.T, wl.d, wl.K, slot, offsets, rank)
    assert np.array_equal(to_np(pos), pos_ref)
    _check_dispatch_sample(orc, inp["x"], rows, None, None, pos, _sample(wl.T, 512, 2))
    # every row of the dispatch buffer is some token's row: row_src is a valid inverse
    rs = to_np(row_src)
    assert np.array_equal(np.sort(to_np(pos).reshape(-1)), np.arange(wl.T * wl.K))
    assert np.array_equal(rs[to_np(pos).reshape(-1)], np.repeat(np.arange(wl.T), wl.K))


def test_collapse_and_bias_balancing_100_steps(orc):
    """Celebrity experts collapse the routing; 100 sign-rule bias steps on
    that batch, each step's stats and the final bias replayed by the oracle
    on the same (GPU) scores, bit for bit."""
    moe = lib()
    wl = W.WORKLOADS["collapse"]
    inp = W.make_inputs(wl, device="cuda")
    scores, idx, w, ws = _route(wl, inp)
    _check_gate_sample(orc, wl, inp, scores, idx, _sample(wl.T, 256, 3))
    T, N, K = wl.T, wl.N, wl.K
    s_np = to_np(scores)
    bias = inp["bias"].clone()
    b_ref = inp["bias"].cpu().numpy().copy()
    cfg = moe.route_cfg(T, wl.d, N, K, wl.fn, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm, wl.scale)
    counts = torch.empty(N, dtype=torch.int32, device="cuda")
    offsets = torch.empty(N + 1, dtype=torch.int32, device="cuda")
    rank = torch.empty(T, K, dtype=torch.int32, device="cuda")
    stats = moe.empty_stats()
    imb = []
    for step in range(wl.bias_steps + 1):
        moe.moe_route(cfg, None, None, None, bias, scores, idx, w, ws)
        moe.moe_load_stats(idx, T, K, N, None, N, None, counts, offsets, rank, None, wl.fn, stats, ws)
        if step < wl.bias_steps:
            moe.moe_bias_update(counts, N, T * K, 0.001, 0, bias)
        ri, _ = orc.select(s_np, b_ref, K, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm, wl.scale)
        c_ref = orc.histogram(ri, N)
        st = moe.read_stats(stats)
        ref = orc.load_stats(c_ref)
        assert np.array_equal(to_np(counts), c_ref), step
        assert_stats_close(st, ref)
        imb.append(st["imbalance"])
        if step < wl.bias_steps:
            b_ref = orc.bias_update(c_ref, T * K, b_ref, 0.001, 0)
    assert np.array_equal(to_np(bias), b_ref)
    assert imb[-1] < imb[0]          # the bias steps move load off the celebrity experts


def test_softmax_dispatch_combine_full(orc):
    wl = W.WORKLOADS["softmax_dispatch"]
    inp = W.make_inputs(wl, device="cuda", with_y=True)
    scores, idx, w, ws = _route(wl, inp)
    _check_gate_sample(orc, wl, inp, scores, idx, _sample(wl.T, 256, 4))
    ri = _check_selection_full(orc, wl, inp, scores, idx, w)
    slot, counts, offsets, rank, stats, _ = load_stats_gpu(idx, wl.T, wl.K, wl.N, scores=scores, score_fn=0)
    c_ref, off_ref, pos_ref, rank_ref, _ = orc.positions(ri, wl.N)
    assert np.array_equal(to_np(counts), c_ref) and np.array_equal(to_np(rank), rank_ref)
    rows, q, sc, pos, _ = _dispatch(inp["x"], wl.T, wl.d, wl.K, slot, offsets, rank, fp8=True)
    assert np.array_equal(to_np(pos), pos_ref)
    sample = _sample(wl.T, 256, 5)
    _check_dispatch_sample(orc, inp["x"], rows, q, sc, pos, sample)
    del rows, q, sc
    out = torch.empty(wl.T, wl.d, dtype=torch.bfloat16, device="cuda")
    lib().moe_combine(inp["y"], wl.T, wl.d, wl.K, pos, w, out)
    p = pos_ref[sample]
    y_rows = inp["y"][torch.from_numpy(p.reshape(-1)).cuda()].float().cpu().numpy()
    ref = orc.combine(y_rows, np.arange(p.size).reshape(p.shape), to_np(w)[sample])
    got = to_np(out)[sample].astype(np.float64)
    assert (np.abs(got - ref) <= np.maximum(2e-2, np.abs(ref) * 2.0 ** -8)).all()


def test_prefill_with_replicas_full(orc):
    moe = lib()
    wl = W.WORKLOADS["prefill_replicas"]
    inp = W.make_inputs(wl, device="cuda")
    scores, idx, w, ws = _route(wl, inp)
    _check_gate_sample(orc, wl, inp, scores, idx, _sample(wl.T, 256, 6))
    ri = _check_selection_full(orc, wl, inp, scores, idx, w)
    del scores
    T, N, K, R = wl.T, wl.N, wl.K, wl.n_replicas
    _, counts, _, _, stats, _ = load_stats_gpu(idx, T, K, N)
    c_ref = orc.histogram(ri, N)
    assert np.array_equal(to_np(counts), c_ref)
    before = moe.read_stats(stats)
    rs = torch.empty(N, dtype=torch.int32, device="cuda")
    moe.moe_replica_plan(counts, N, R, rs)
    rs_ref = orc.replica_plan(c_ref, R)
    assert np.array_equal(to_np(rs), rs_ref)
    slot, counts2, offsets2, rank2, stats2, _ = load_stats_gpu(idx, T, K, N, n_slots=N + R, replica_slot=rs)
    s_ref = orc.apply_replicas(ri, rs_ref)
    c2, o2, p2, r2, _ = orc.positions(s_ref, N + R)
    assert np.array_equal(to_np(slot), s_ref)
    assert np.array_equal(to_np(counts2), c2) and np.array_equal(to_np(offsets2), o2)
    assert np.array_equal(to_np(rank2), r2)
    after = moe.read_stats(stats2)
    assert_stats_close(after, orc.load_stats(c2))
    assert after["max_load"] < before["max_load"]
    rows, _, _, pos, _ = _dispatch(inp["x"], T, wl.d, K, slot, offsets2, rank2)
    assert np.array_equal(to_np(pos), p2)
    _check_dispatch_sample(orc, inp["x"], rows, None, None, pos, _sample(T, 256, 7))
