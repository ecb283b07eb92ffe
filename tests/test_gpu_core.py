"""GPU parity: selection, histogram / offsets / ranks / stats, replica plan,
bias update, dispatch (bf16, fp32, FP8) and combine against the CPU oracle,
on the same seeded inputs, through the C ABI.  Integer and index outputs are
compared bit for bit."""
import math

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


def _sel_wl(N, K, G, TG, T, scale=2.5, renorm=True, topn=2):
    return W.Workload("sel", 0, T, 64, N, K, fn=1, n_groups=G, topk_groups=TG, group_topn=topn, renorm=renorm,
                      scale=scale)


SEL_CASES = [
    # N, K, G, TG, quantum, with bias
    (8, 2, 1, 1, 0.0, False),       # tiny softmax router shape
    (8, 2, 2, 1, 0.125, True),
    (32, 3, 4, 2, 0.0625, True),
    (64, 6, 4, 2, 0.0, True),
    (128, 8, 1, 1, 0.0, False),     # softmax top-8 of 128
    (128, 8, 1, 1, 1 / 64, True),
    (256, 8, 8, 4, 0.0, True),      # V3 routing
    (256, 8, 8, 4, 1 / 32, True),   # with many ties
    (256, 1, 8, 1, 0.0, True),
    (512, 8, 16, 4, 0.0, True),
]


@pytest.mark.parametrize("N,K,G,TG,q,with_bias", SEL_CASES)
def test_selection_bit_exact_from_scores(orc, N, K, G, TG, q, with_bias):
    T = 2053  # ragged against the 8 tokens per block
    s = W.make_scores(T, N, seed=N * 7 + K, quantum=q)
    b = W.make_bias(N, seed=N + 3) if with_bias else None
    if b is not None and q:
        b = torch.round(b / q) * q
    wl = _sel_wl(N, K, G, TG, T)
    _, idx, w, _ = route_gpu(wl, None, None, None, b.cuda() if b is not None else None, scores_in=s.cuda())
    ri, rw = orc.select(s.numpy(), b.numpy() if b is not None else None, K, G, TG, 2, True, 2.5)
    assert np.array_equal(to_np(idx), ri)
    assert np.array_equal(to_np(w), rw)  # same fp32 operations in the same order


def test_selection_unnormalised_and_topn(orc):
    T, N = 777, 256
    s = W.make_scores(T, N, seed=5)
    b = W.make_bias(N, seed=6)
    wl = _sel_wl(N, 8, 8, 3, T, scale=1.0, renorm=False, topn=3)
    _, idx, w, _ = route_gpu(wl, None, None, None, b.cuda(), scores_in=s.cuda())
    ri, rw = orc.select(s.numpy(), b.numpy(), 8, 8, 3, 3, False, 1.0)
    assert np.array_equal(to_np(idx), ri) and np.array_equal(to_np(w), rw)


@pytest.mark.parametrize("T,K,N,skew,R", [(5000, 8, 256, 0.0, 0), (5000, 8, 256, 1.1, 32), (513, 2, 8, 0.0, 0),
                                           (131072, 8, 256, 1.1, 32), (4096, 8, 128, 0.5, 0),
                                           (65536, 8, 128, 0.3, 16), (40961, 8, 256, 0.9, 0),
                                           (327681, 8, 256, 0.2, 0)])
def test_histogram_offsets_ranks_stats(orc, T, K, N, skew, R):
    idx = W.make_assignments(T, K, N, seed=T + K, skew=skew)
    slot_i, counts, offsets, rank, stats, ws = load_stats_gpu(idx.cuda(), T, K, N)
    i_np = idx.numpy()
    c_ref, off_ref, pos_ref, rank_ref, _ = orc.positions(i_np, N)
    assert np.array_equal(to_np(counts), c_ref)
    assert np.array_equal(to_np(offsets), off_ref)
    assert np.array_equal(to_np(rank), rank_ref)
    assert np.array_equal(to_np(slot_i), i_np)
    assert_stats_close(lib().read_stats(stats), orc.load_stats(c_ref))
    assert lib().moe_workspace_status(ws) == 0
    if R:
        rs = torch.empty(N, dtype=torch.int32, device="cuda")
        lib().moe_replica_plan(counts, N, R, rs)
        rs_ref = orc.replica_plan(c_ref, R)
        assert np.array_equal(to_np(rs), rs_ref)
        slot2, counts2, offsets2, rank2, stats2, ws2 = load_stats_gpu(idx.cuda(), T, K, N, n_slots=N + R,
                                                                      replica_slot=rs)
        s_ref = orc.apply_replicas(i_np, rs_ref)
        c2, o2, p2, r2, _ = orc.positions(s_ref, N + R)
        assert np.array_equal(to_np(slot2), s_ref)
        assert np.array_equal(to_np(counts2), c2)
        assert np.array_equal(to_np(offsets2), o2)
        assert np.array_equal(to_np(rank2), r2)
        st2 = lib().read_stats(stats2)
        assert_stats_close(st2, orc.load_stats(c2))
        assert st2["max_load"] <= lib().read_stats(stats)["max_load"]


@pytest.mark.parametrize("case", ["balanced", "skewed", "concentrated"])
def test_printed_imbalance_example_on_gpu(case):
    """The four-expert, 64-assignment cases of "A minimal experiment in
    expert-load imbalance" (Expected output), through the GPU histogram."""
    loads = {"balanced": [16, 16, 16, 16], "skewed": [40, 8, 8, 8], "concentrated": [64, 0, 0, 0]}[case]
    expect = {"balanced": (16, 1.0, 64), "skewed": (40, 2.5, 160), "concentrated": (64, 4.0, 256)}[case]
    idx = torch.tensor([e for e, c in enumerate(loads) for _ in range(c)], dtype=torch.int32)[:, None]
    _, counts, _, _, stats, _ = load_stats_gpu(idx.cuda(), 64, 1, 4)
    st = lib().read_stats(stats)
    assert to_np(counts).tolist() == loads
    assert st["total"] == 64 and st["max_load"] == expect[0]
    assert st["imbalance"] == expect[1] and st["capacity_fixed"] == expect[2]


def test_empty_batch_stats():
    idx = torch.empty(0, 8, dtype=torch.int32, device="cuda")
    _, counts, offsets, _, stats, _ = load_stats_gpu(idx, 0, 8, 16)
    st = lib().read_stats(stats)
    assert to_np(counts).tolist() == [0] * 16 and to_np(offsets).tolist() == [0] * 17
    assert st["total"] == 0 and st["imbalance"] == 0.0 and st["std_over_mean"] == 0.0


def test_stats_are_deterministic():
    T, K, N = 20000, 8, 256
    idx = W.make_assignments(T, K, N, seed=9, skew=0.7).cuda()
    outs = [load_stats_gpu(idx, T, K, N) for _ in range(3)]
    for o in outs[1:]:
        for a, b in zip(outs[0][:5], o[:5]):
            assert torch.equal(a, b)


@pytest.mark.parametrize("fn,N", [(1, 256), (0, 128), (0, 8)])
def test_score_entropy(orc, fn, N):
    T = 3001
    s = W.make_scores(T, N, seed=fn + N)
    idx = W.make_assignments(T, 2, N, seed=1)
    _, _, _, _, stats, _ = load_stats_gpu(idx.cuda(), T, 2, N, scores=s.cuda(), score_fn=fn)
    hs = lib().read_stats(stats)["entropy_score_bits"]
    ref = orc.score_entropy(s.numpy(), fn)
    assert abs(hs - ref) <= 1e-6 * abs(ref)


def test_score_entropy_uniform_is_log2_n():
    T, N = 1000, 256
    s = torch.full((T, N), 0.5, device="cuda")
    idx = W.make_assignments(T, 8, N, seed=2).cuda()
    _, _, _, _, stats, _ = load_stats_gpu(idx, T, 8, N, scores=s, score_fn=1)
    assert abs(lib().read_stats(stats)["entropy_score_bits"] - math.log2(N)) < 1e-9


@pytest.mark.parametrize("mode,u", [(0, 0.001), (1, 0.05)])
def test_bias_update_bit_exact(orc, mode, u):
    N, T, K = 256, 4096, 8
    idx = W.make_assignments(T, K, N, seed=mode + 40, skew=1.0)
    counts = orc.histogram(idx.numpy(), N)
    b0 = W.make_bias(N, seed=77)
    bias = b0.clone().cuda()
    lib().moe_bias_update(torch.from_numpy(counts.astype(np.int32)).cuda(), N, T * K, u, mode, bias)
    ref = orc.bias_update(counts, T * K, b0.numpy(), u, mode)
    assert np.array_equal(to_np(bias), ref)


DISPATCH_CASES = [
    # T, d, K, N, dtype, fp8
    (1000, 512, 8, 256, torch.bfloat16, True),
    (777, 7168, 8, 256, torch.bfloat16, True),
    (300, 4096, 8, 128, torch.bfloat16, False),
    (512, 128, 2, 8, torch.float32, True),
    (129, 136, 3, 16, torch.bfloat16, False),  # d not a multiple of 128 or 256
    (64, 1024, 20, 64, torch.bfloat16, True),  # K > 8
]


@pytest.mark.parametrize("T,d,K,N,dtype,fp8", DISPATCH_CASES)
def test_dispatch_bit_exact(orc, T, d, K, N, dtype, fp8):
    g = torch.Generator().manual_seed(T + d)
    x = torch.randn(T, d, generator=g).to(dtype)
    x[min(5, T - 1), : min(128, d)] = 0.0  # an all-zero FP8 block
    idx = W.make_assignments(T, K, N, seed=d + K, skew=0.8)
    xc = x.cuda()
    slot, counts, offsets, rank, _, _ = load_stats_gpu(idx.cuda(), T, K, N)
    rows = torch.empty(T * K, d, dtype=dtype, device="cuda")
    q = torch.empty(T * K, d, dtype=torch.uint8, device="cuda") if fp8 else None
    sc = torch.empty(T * K, d // 128, dtype=torch.float32, device="cuda") if fp8 else None
    pos = torch.empty(T, K, dtype=torch.int32, device="cuda")
    row_src = torch.empty(T * K, dtype=torch.int32, device="cuda")
    lib().moe_dispatch(xc, T, d, K, slot, offsets, rank, rows, q, sc, pos, row_src)
    _, _, pos_ref, _, src_ref = orc.positions(idx.numpy(), N)
    assert np.array_equal(to_np(pos), pos_ref)
    assert np.array_equal(to_np(row_src), src_ref)
    x_np = x.view(torch.int16).numpy() if dtype == torch.bfloat16 else x.numpy()
    rows_np = rows.view(torch.int16).cpu().numpy() if dtype == torch.bfloat16 else to_np(rows)
    assert np.array_equal(rows_np, orc.dispatch_rows(x_np, pos_ref))
    if fp8:
        q_ref, sc_ref = orc.fp8_rows(orc.dispatch_rows(x.float().numpy(), pos_ref))
        assert np.array_equal(to_np(sc), sc_ref)
        assert np.array_equal(to_np(q), q_ref)


def test_dispatch_fp8_only_buffer(orc):
    T, d, K, N = 200, 256, 4, 32
    x = torch.randn(T, d, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    idx = W.make_assignments(T, K, N, seed=4)
    slot, counts, offsets, rank, _, _ = load_stats_gpu(idx.cuda(), T, K, N)
    q = torch.empty(T * K, d, dtype=torch.uint8, device="cuda")
    sc = torch.empty(T * K, d // 128, dtype=torch.float32, device="cuda")
    lib().moe_dispatch(x.cuda(), T, d, K, slot, offsets, rank, None, q, sc, None, None)
    _, _, pos_ref, _, _ = orc.positions(idx.numpy(), N)
    q_ref, sc_ref = orc.fp8_rows(orc.dispatch_rows(x.float().numpy(), pos_ref))
    assert np.array_equal(to_np(q), q_ref) and np.array_equal(to_np(sc), sc_ref)


@pytest.mark.parametrize("T,d,K,dtype", [(1000, 512, 8, torch.bfloat16), (333, 4096, 8, torch.bfloat16),
                                         (512, 128, 2, torch.float32), (100, 264, 5, torch.float32),
                                         (64, 1024, 20, torch.bfloat16)])
def test_combine(orc, T, d, K, dtype):
    N = 64
    g = torch.Generator().manual_seed(d + K)
    y = torch.randn(T * K, d, generator=g).to(dtype)
    s = W.make_scores(T, N, seed=d)
    idx, w = orc.select(s.numpy(), None, K, 1, 1, 2, True, 1.0)
    _, _, pos, _, _ = orc.positions(idx, N)
    out = torch.empty(T, d, dtype=dtype, device="cuda")
    lib().moe_combine(y.cuda(), T, d, K, torch.from_numpy(pos.astype(np.int32)).cuda(), torch.from_numpy(w).cuda(),
                      out)
    ref = orc.combine(y.float().numpy(), pos, w)
    got = to_np(out).astype(np.float64)
    if dtype == torch.bfloat16:
        # bf16 output: 2e-2 absolute, widened by half a bf16 ulp for |out| >= 4
        tol = np.maximum(2e-2, np.abs(ref) * 2.0 ** -8)
    else:
        tol = 1e-5 * np.maximum(1.0, np.abs(ref))
    assert (np.abs(got - ref) <= tol).all()


def test_dispatch_combine_round_trip():
    """combine(dispatch(x)) with renormalised weights (scale 1) returns x."""
    T, d, K, N = 2000, 1024, 8, 128
    x = torch.randn(T, d, device="cuda").to(torch.bfloat16)
    s = W.make_scores(T, N, seed=8).cuda()
    wl = _sel_wl(N, K, 1, 1, T, scale=1.0)
    _, idx, w, _ = route_gpu(wl, None, None, None, None, scores_in=s)
    slot, counts, offsets, rank, _, _ = load_stats_gpu(idx, T, K, N)
    rows = torch.empty(T * K, d, dtype=torch.bfloat16, device="cuda")
    pos = torch.empty(T, K, dtype=torch.int32, device="cuda")
    lib().moe_dispatch(x, T, d, K, slot, offsets, rank, rows, None, None, pos, None)
    out = torch.empty_like(x)
    lib().moe_combine(rows, T, d, K, pos, w, out)
    diff = (out.float() - x.float()).abs()
    assert (diff <= x.float().abs() * 2.0 ** -7 + 1e-6).all()


def test_launch_count_counts_kernels():
    moe = lib()
    T, K, N = 100, 2, 8
    idx = W.make_assignments(T, K, N, seed=1).cuda()
    moe.moe_launch_count(reset=True)
    load_stats_gpu(idx, T, K, N)
    assert moe.moe_launch_count() == 1  # one single-pass kernel


def test_bounded_wait_times_out_and_context_survives():
    """The look-back wait of the offsets pass, run on a flag nothing sets,
    gives up after about a second with a timeout status; the context stays
    usable for the next call."""
    import time
    moe = lib()
    ws = moe.workspace(4096, 1, 8)
    t0 = time.time()
    assert moe.moe_selftest_wait_timeout(ws) == moe.MOE_ERR_TIMEOUT
    assert 0.5 < time.time() - t0 < 30
    T, K, N = 300, 4, 16
    idx = W.make_assignments(T, K, N, seed=5).cuda()
    _, counts, _, _, stats, ws2 = load_stats_gpu(idx, T, K, N)
    assert lib().read_stats(stats)["status"] == 0
    assert int(counts.sum()) == T * K
