"""GPU parity of the routing variants against the oracle: the bias added to
the logits before the nonlinearity (so it shapes the combine weights too),
the forcible round-robin balance, and the bias step on a smoothed load."""
import numpy as np
import pytest
import torch

from expert_load_balancing_tcgen05_b200 import workloads as W
from gpu_util import assert_stats_close, gap_ok, lib, load_stats_gpu, to_np

pytestmark = pytest.mark.gpu

RTOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")


@pytest.mark.parametrize("path", ["separate", "fused"])
@pytest.mark.parametrize("name,T,dtype", [
    ("v3_router", 1000, torch.bfloat16), ("softmax_dispatch", 777, torch.bfloat16),
    ("tiny_softmax", 333, torch.float32), ("v3_router", 129, torch.float32),
])
def test_bias_in_logits(orc, monkeypatch, path, name, T, dtype):
    monkeypatch.setenv("MOE_FUSED_SELECT", "0" if path == "separate" else "1")
    moe = lib()
    wl = W.WORKLOADS[name].with_(T=T, d=512, dtype=dtype)
    inp = W.make_inputs(wl, seed=11)
    g = np.random.default_rng(5)
    bias = torch.from_numpy(g.normal(0.0, 0.5, wl.N).astype(np.float32))
    x, Wg, off = inp["x"], inp["W"], inp["off"]
    N, K = wl.N, wl.K
    scores = torch.empty(T, N, device="cuda")
    idx = torch.empty(T, K, dtype=torch.int32, device="cuda")
    w = torch.empty(T, K, device="cuda")
    ws = moe.workspace(T, K, N, N)
    cfg = moe.route_cfg(T, wl.d, N, K, wl.fn, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm, wl.scale,
                        moe.MOE_BF16 if dtype == torch.bfloat16 else moe.MOE_F32, bias_in_logits=True)
    moe.moe_route(cfg, x.cuda(), Wg.cuda(), off.cuda() if off is not None else None, bias.cuda(), scores, idx, w,
                  ws)
    torch.cuda.synchronize()
    assert moe.moe_workspace_status(ws) == 0
    h, s_ref, ri_ref, _ = orc.route(x.float().numpy(), Wg.float().numpy(), off.numpy() if off is not None else None,
                                   bias.numpy(), wl.fn, K, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm,
                                   wl.scale, bias_in_logits=True)
    sg = to_np(scores)
    err = np.abs(sg.astype(np.float64) - s_ref)
    assert not (err > RTOL * np.abs(s_ref) + 1e-7).any(), float(err.max())
    # the selection on the GPU's own scores, with no bias in the key: bit-exact
    ri, rw = orc.select(sg, None, K, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm, wl.scale)
    assert np.array_equal(to_np(idx), ri)
    assert np.array_equal(to_np(w), rw)
    _, bad = gap_ok(s_ref, None, to_np(idx), ri_ref, K, wl.n_groups, wl.topk_groups, wl.group_topn)
    assert not bad, bad[:10]


@pytest.mark.parametrize("T,K,N,scale", [(16384, 8, 256, 2.5), (1, 8, 256, 1.0), (4099, 6, 64, 1.0),
                                         (3, 1, 7, 0.5)])
def test_route_balanced(orc, T, K, N, scale):
    moe = lib()
    idx = torch.full((T, K), -1, dtype=torch.int32, device="cuda")
    w = torch.zeros(T, K, device="cuda")
    moe.moe_route_balanced(T, K, N, scale, idx, w)
    torch.cuda.synchronize()
    ri, rw = orc.route_balanced(T, K, N, scale)
    assert np.array_equal(to_np(idx), ri)
    assert np.array_equal(to_np(w), rw)
    # the histogram of the forced assignment: every expert within one of the mean
    _, counts, _, _, stats, ws = load_stats_gpu(idx, T, K, N)
    torch.cuda.synchronize()
    c = to_np(counts)
    assert c.max() - c.min() <= 1 and int(c.sum()) == T * K
    assert_stats_close(moe.read_stats(stats), orc.load_stats(orc.histogram(ri, N)))


@pytest.mark.parametrize("alpha", [0.0, 0.5, 0.9, 0.99])
def test_bias_update_ema_bit_exact(orc, alpha):
    moe = lib()
    N, steps = 256, 20
    g = np.random.default_rng(17)
    bias = np.zeros(N, np.float32)
    ema = np.zeros(N, np.float32)
    b_d = torch.zeros(N, device="cuda")
    e_d = torch.zeros(N, device="cuda")
    for s in range(steps):
        c = g.multinomial(131072, g.dirichlet(np.full(N, 0.3))).astype(np.int32)
        moe.moe_bias_update_ema(torch.from_numpy(c).cuda(), N, int(c.sum()), 0.001, alpha, e_d, b_d)
        bias, ema = orc.bias_update_ema(c, int(c.sum()), bias, ema, 0.001, alpha)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(e_d), ema)
    assert np.array_equal(to_np(b_d), bias)


def test_bias_update_ema_alpha_zero_is_sign_rule(orc):
    """alpha = 0 keeps no memory: the step equals the plain sign rule."""
    moe = lib()
    N = 160
    g = np.random.default_rng(3)
    c = g.integers(0, 900, N).astype(np.int32)
    b0 = g.normal(0, 0.01, N).astype(np.float32)
    b1 = torch.from_numpy(b0.copy()).cuda()
    b2 = torch.from_numpy(b0.copy()).cuda()
    e = torch.from_numpy(g.normal(0, 50, N).astype(np.float32)).cuda()
    cd = torch.from_numpy(c).cuda()
    moe.moe_bias_update_ema(cd, N, int(c.sum()), 0.002, 0.0, e, b1)
    moe.moe_bias_update(cd, N, int(c.sum()), 0.002, 0, b2)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(b1), to_np(b2))
