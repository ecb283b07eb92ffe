"""GPU parity of the gate GEMM + score nonlinearity (tcgen05 tensor-core
kernel for bf16, CUDA-core kernel for fp32) against the fp64 oracle on the
same inputs: scores within 1e-3 relative; the selection made from the GPU's
own scores bit-exact against the oracle's selection on those scores; and
against the oracle's own scores, differing only on near ties (gap < 1e-3)."""
import numpy as np
import pytest
import torch

from expert_load_balancing_tcgen05_b200 import workloads as W
from gpu_util import gap_ok, lib, route_gpu, to_np

pytestmark = pytest.mark.gpu

RTOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")


def _check_scores(s_gpu, s_ref):
    err = np.abs(s_gpu.astype(np.float64) - s_ref.astype(np.float64))
    bad = err > RTOL * np.abs(s_ref) + 1e-7
    assert not bad.any(), (int(bad.sum()), float(err.max()))


@pytest.fixture(params=["separate", "fused"], autouse=True)
def select_path(request, monkeypatch):
    """Run every case with the selection in its own kernel and inside the
    GEMM epilogue (where the configuration allows it)."""
    monkeypatch.setenv("MOE_FUSED_SELECT", "0" if request.param == "separate" else "1")
    return request.param


def _run_and_check(orc, wl, T, d, seed, check_gap=True):
    wl = wl.with_(T=T, d=d)
    inp = W.make_inputs(wl, seed=seed)
    x, Wg, b, off = inp["x"], inp["W"], inp["bias"], inp["off"]
    s_gpu, idx, w, ws = route_gpu(wl, x.cuda(), Wg.cuda(), off.cuda() if off is not None else None,
                                  b.cuda() if b is not None else None)
    assert lib().moe_workspace_status(ws) == 0
    h = orc.logits(x.float().numpy(), Wg.float().numpy(), off.numpy() if off is not None else None)
    s_ref = orc.scores(h, wl.fn)
    sg = to_np(s_gpu)
    _check_scores(sg, s_ref)
    bn = b.numpy() if b is not None else None
    # selection on the GPU's own scores: bit-exact
    ri, rw = orc.select(sg, bn, wl.K, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm, wl.scale)
    assert np.array_equal(to_np(idx), ri)
    assert np.array_equal(to_np(w), rw)
    if check_gap:
        ri2, _ = orc.select(s_ref, bn, wl.K, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm, wl.scale)
        diff, bad = gap_ok(s_ref, bn, to_np(idx), ri2, wl.K, wl.n_groups, wl.topk_groups, wl.group_topn)
        assert not bad, bad[:10]
    return sg, s_ref


TC_CASES = [
    # workload, T, d
    ("v3_router", 421, 7168),        # 4 tiles, ragged token tail, 112 k-steps
    ("v3_router", 128, 1000),        # ragged k tail (1000 = 15*64 + 40)
    ("v3_router", 1, 64),            # one token, one k-step
    ("collapse", 300, 7168),         # celebrity logit offsets
    ("prefill_replicas", 260, 7168),  # Zipf logit offsets
    ("softmax_dispatch", 389, 4096),  # N=128 softmax
    # odd k-block counts: the last ring slot holds one k-block of two
    ("v3_router", 300, 936),         # 15 k-blocks (14*64 + 40), pair kernel
    ("softmax_dispatch", 257, 264),  # 5 k-blocks, N=128 one-SM kernel
]


@pytest.mark.parametrize("name,T,d", TC_CASES)
def test_gate_tc_against_oracle(orc, name, T, d):
    _run_and_check(orc, W.WORKLOADS[name], T, d, seed=T + d)


def test_gate_tc_n256_softmax_small_batch(orc):
    """N = 256 with the row softmax, at batch sizes where the pair kernel
    splits each tile's k-blocks over several CTA pairs (the softmax epilogue
    then runs on the added partial sums) and where it does not."""
    wl = W.Workload("n256sm", 0, 0, 0, 256, 8, fn=0, scale=1.0, has_bias=True)
    _run_and_check(orc, wl, 600, 2048, seed=11)   # 3 tiles: split over 4 pairs
    _run_and_check(orc, wl, 97, 1000, seed=12)    # 1 ragged tile, 16 k-blocks: split
    _run_and_check(orc, wl, 700, 128, seed=13)    # 2 k-blocks: too few to split


def test_gate_tc_n64_sigmoid(orc):
    wl = W.Workload("n64", 0, 0, 0, 64, 6, fn=1, n_groups=4, topk_groups=2, scale=1.0, has_bias=True)
    _run_and_check(orc, wl, 700, 512, seed=3)
    _run_and_check(orc, wl, 333, 192, seed=4)  # 3 k-blocks: an odd count


def test_gate_tc_many_tiles_per_cta(orc):
    """More tiles than SMs: every CTA runs 2-3 tiles, so both TMEM
    accumulators and every ring-slot phase are exercised."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    T = sms * 128 * 2 + 77
    wl = W.WORKLOADS["softmax_dispatch"]
    _run_and_check(orc, wl, T, 256, seed=11)


def test_gate_simt_fp32_tiny_router(orc):
    """The tiny softmax top-2 router of 8 experts, fp32, end to end."""
    wl = W.WORKLOADS["tiny_softmax"]
    _run_and_check(orc, wl, wl.T, wl.d, seed=wl.seed)


def test_gate_simt_bf16_small_n(orc):
    wl = W.Workload("n8bf16", 0, 0, 0, 8, 2, fn=0)
    _run_and_check(orc, wl, 333, 256, seed=5)


def test_zero_gate_gives_uniform_scores():
    wl = W.WORKLOADS["v3_router"].with_(T=256, d=512)
    x = torch.randn(256, 512, device="cuda").to(torch.bfloat16)
    Wg = torch.zeros(256, 512, device="cuda", dtype=torch.bfloat16)
    s, idx, _, _ = route_gpu(wl, x, Wg, None, None)
    assert torch.all(s == 0.5)
    # all-equal scores select the lowest experts (ties to the lower index)
    assert torch.equal(idx.cpu(), torch.arange(8, dtype=torch.int32).expand(256, 8))


def test_fused_selection_without_scores_output():
    """With the selection inside the GEMM epilogue the scores output is
    optional; the choice and weights are the same with or without it."""
    moe = lib()
    wl = W.WORKLOADS["v3_router"].with_(T=777, d=1024)
    inp = W.make_inputs(wl, seed=9)
    x, Wg, b = inp["x"].cuda(), inp["W"].cuda(), inp["bias"].cuda()
    s1, i1, w1, _ = route_gpu(wl, x, Wg, None, b)
    i2 = torch.empty_like(i1)
    w2 = torch.empty_like(w1)
    ws = moe.workspace(wl.T, wl.K, wl.N)
    cfg = moe.route_cfg(wl.T, wl.d, wl.N, wl.K, wl.fn, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm,
                        wl.scale)
    moe.moe_route(cfg, x, Wg, None, b, None, i2, w2, ws)
    assert torch.equal(i1, i2) and torch.equal(w1, w2)
    # the non-fused configuration (groups of 16) refuses a missing scores buffer
    cfg16 = moe.route_cfg(wl.T, wl.d, wl.N, wl.K, wl.fn, 16, 4, 2, True, 2.5)
    with pytest.raises(moe.MoeError):
        moe.moe_route(cfg16, x, Wg, None, b, None, i2, w2, ws)


def test_gate_pair_many_tiles_per_cluster(orc):
    """N = 256 runs on CTA pairs (2-SM MMA); with more 256-token tiles than
    pairs, every pair runs several tiles and a ragged last tile."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    T = (sms // 2) * 256 * 2 + 300
    _run_and_check(orc, W.WORKLOADS["v3_router"], T, 256, seed=12)


@pytest.mark.parametrize("pair", ["0", "1"])
def test_gate_one_sm_and_pair_agree(pair, monkeypatch):
    """The 1-SM and 2-SM kernels compute the same scores up to fp32
    accumulation order, and the same selection from them."""
    monkeypatch.setenv("MOE_GATE_PAIR", pair)
    wl = W.WORKLOADS["v3_router"].with_(T=1000, d=2048)
    inp = W.make_inputs(wl, seed=13)
    s, idx, w, ws = route_gpu(wl, inp["x"].cuda(), inp["W"].cuda(), None, inp["bias"].cuda())
    assert lib().moe_workspace_status(ws) == 0
    ref = inp["x"].cuda().float() @ inp["W"].cuda().float().t()
    assert torch.allclose(s, torch.sigmoid(ref), rtol=1e-3, atol=1e-6)


@pytest.mark.parametrize("T,d", [(4096, 7168), (300, 7168), (700, 936), (1, 2048)])
def test_gate_split_k_matches_unsplit(monkeypatch, T, d):
    """With fewer 256-token tiles than half the CTA pairs the pair kernel
    splits each tile's k-blocks over up to four pairs of one cluster and adds
    their partial sums in pair order.  The scores equal the unsplit kernel's
    up to fp32 summation order, and repeated runs are bit-identical (the
    order of the additions does not depend on timing)."""
    wl = W.WORKLOADS["v3_router"].with_(T=T, d=d)
    inp = W.make_inputs(wl, seed=T + d)
    x, Wg, b = inp["x"].cuda(), inp["W"].cuda(), inp["bias"].cuda()
    s1, i1, w1, ws1 = route_gpu(wl, x, Wg, None, b)
    s2, i2, w2, ws2 = route_gpu(wl, x, Wg, None, b)
    monkeypatch.setenv("MOE_GATE_SPLIT", "0")
    s0, _, _, ws0 = route_gpu(wl, x, Wg, None, b)
    torch.cuda.synchronize()
    for ws in (ws0, ws1, ws2):
        assert lib().moe_workspace_status(ws) == 0
    assert torch.equal(s1, s2) and torch.equal(i1, i2) and torch.equal(w1, w2)
    assert torch.allclose(s1, s0, rtol=1e-4, atol=1e-6)
    ref = torch.sigmoid(x.float() @ Wg.float().t())
    assert torch.allclose(s1, ref, rtol=1e-3, atol=1e-6)


@pytest.mark.parametrize("T,d", [(255, 7168), (256, 640), (257, 704), (511, 1088), (2049, 2048), (3841, 1024),
                                 (3840, 7168), (4097, 4096), (7000, 1536), (9472, 1024), (9473, 1024)])
def test_gate_split_k_sweep(monkeypatch, T, d):
    """Batch sizes around the thresholds of the small-batch split (tile
    edges; S = 4, 3, 2 pairs; the largest batch that still splits and the
    first that does not) and k-block counts that do not divide evenly:
    scores equal the unsplit kernel's up to fp32 summation order, and a
    second run gives bit-identical scores and choices (with the selection in
    its own kernel and in the epilogue)."""
    wl = W.WORKLOADS["v3_router"].with_(T=T, d=d)
    inp = W.make_inputs(wl, seed=T * 7 + d)
    x, Wg, b = inp["x"].cuda(), inp["W"].cuda(), inp["bias"].cuda()
    s1, i1, w1, ws1 = route_gpu(wl, x, Wg, None, b)
    s2, i2, _, _ = route_gpu(wl, x, Wg, None, b)
    monkeypatch.setenv("MOE_GATE_SPLIT", "0")
    s0, _, _, ws0 = route_gpu(wl, x, Wg, None, b)
    torch.cuda.synchronize()
    assert lib().moe_workspace_status(ws1) == 0 and lib().moe_workspace_status(ws0) == 0
    assert torch.equal(s1, s2) and torch.equal(i1, i2)
    assert torch.allclose(s1, s0, rtol=1e-4, atol=1e-6)
