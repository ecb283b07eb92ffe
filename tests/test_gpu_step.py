"""The pipelined routing step (routing of batch i+1 beside the dispatch of
batch i, double-buffered load-statistics outputs) produces exactly what the
serial schedule produces: the same bias after the last step, the same
routing, offsets, ranks, statistics and dispatched rows for the last batch.
(Intermediate biases are not compared: the routing stream may already be
updating the next batch's bias while the caller's stream runs.)"""
import pytest
import torch

from expert_load_balancing_tcgen05_b200 import workloads as W
from expert_load_balancing_tcgen05_b200.step import RoutingStep

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")


@pytest.mark.parametrize("name,T,steps", [("metric", 4096, 7), ("collapse", 3000, 6), ("softmax_dispatch", 2500, 5)])
def test_pipelined_equals_serial(name, T, steps):
    wl = W.WORKLOADS[name].with_(T=T)
    inp = W.make_inputs(wl, device="cuda", seed=5)
    bias0 = inp["bias"] if inp["bias"] is not None else torch.zeros(wl.N, device="cuda")
    runs = {}
    for pipelined in (False, True):
        S = RoutingStep(wl, inp["x"], inp["W"], bias0.clone(), inp["off"], "cuda", pipelined=pipelined)
        for _ in range(steps):
            S.step()
        torch.cuda.synchronize()
        last = S.last()
        runs[pipelined] = dict(bias=S.bias.clone(), idx=S.idx.clone(), w=S.w.clone(), rows=S.rows.clone(), pos=S.pos.clone(),
                               **{k: last[k].clone() for k in ("slot", "counts", "offsets", "rank", "stats")})
    a, b = runs[False], runs[True]
    assert torch.equal(a["bias"], b["bias"])
    for k in ("idx", "w", "pos", "slot", "counts", "offsets", "rank", "stats"):
        assert torch.equal(a[k], b[k]), k
    assert torch.equal(a["rows"].view(torch.int16), b["rows"].view(torch.int16))


def test_pipelined_with_host_copies_equals_serial():
    """Tokens copied from pinned host memory on a copy stream (two device
    buffers) and routing results copied back to host: the last batch's host
    results equal the serial schedule's device results."""
    wl = W.WORKLOADS["metric"].with_(T=2048)
    inp = W.make_inputs(wl, device="cuda", seed=9)
    S = RoutingStep(wl, inp["x"], inp["W"], inp["bias"].clone(), inp["off"], "cuda", pipelined=False)
    P = RoutingStep(wl, inp["x"], inp["W"], inp["bias"].clone(), inp["off"], "cuda", pipelined=True)
    x_host = inp["x"].cpu().pin_memory()
    x_dev = [torch.empty_like(inp["x"]) for _ in range(2)]
    host = [torch.empty(r.shape, dtype=r.dtype, pin_memory=True) for r in P.results(P.sets[0])]
    cs = torch.cuda.Stream()
    main = torch.cuda.current_stream()
    ev_copied = [torch.cuda.Event() for _ in range(2)]
    ev_free = [torch.cuda.Event() for _ in range(2)]
    steps = 5
    cs.wait_stream(main)
    for i in range(steps):
        b = i % 2
        if i >= 2:
            cs.wait_event(ev_free[b])
        with torch.cuda.stream(cs):
            x_dev[b].copy_(x_host, non_blocking=True)
        ev_copied[b].record(cs)
        P.step(x_dev[b], ready=ev_copied[b], host_out=host)
        ev_free[b].record(main)
        S.step()
    torch.cuda.synchronize()
    for h, d in zip(host, S.results(S.last())):
        assert torch.equal(h, d.cpu())
    assert torch.equal(P.rows.view(torch.int16), S.rows.view(torch.int16))
    assert torch.equal(P.bias, S.bias)


@pytest.mark.parametrize("name,T,steps,fused", [("metric", 2048, 6, False), ("softmax_dispatch", 1500, 5, False),
                                                ("metric", 2048, 6, True), ("softmax_dispatch", 1500, 5, True)])
def test_every_batch_with_combine_equals_serial(name, T, steps, fused):
    """Each batch's indices, weights, offsets, counts and stats (copied to the
    host on the routing stream right after its routing) and its combine
    output (identity experts, on the caller's stream after its dispatch) are
    the same in both schedules, for every batch: with the routing outputs
    double-buffered, batch i+1's routing never overwrites what batch i's
    dispatch and combine still read."""
    wl = W.WORKLOADS[name].with_(T=T)
    xs = [W.make_inputs(wl, device="cuda", seed=20 + j)["x"] for j in range(3)]
    inp = W.make_inputs(wl, device="cuda", seed=19)
    bias0 = inp["bias"] if inp["bias"] is not None else torch.zeros(wl.N, device="cuda")
    got = {}
    for pipelined in (False, True):
        # the serial reference always takes the unfused path: both paths route identically
        S = RoutingStep(wl, xs, inp["W"], bias0.clone(), inp["off"], "cuda", pipelined=pipelined,
                        fused=fused and pipelined)
        host, outs = [], []
        for i in range(steps):
            h = [torch.empty(r.shape, dtype=r.dtype, pin_memory=True) for r in S.results(S.sets[0])]
            o = torch.empty(wl.T, wl.d, dtype=xs[0].dtype, device="cuda")
            S.step(host_out=h, combine_out=o)
            host.append(h)
            outs.append(o)
        torch.cuda.synchronize()
        got[pipelined] = (host, outs)
    for i in range(steps):
        for a, b in zip(got[False][0][i], got[True][0][i]):
            assert torch.equal(a, b), i
        assert torch.equal(got[False][1][i].view(torch.int16), got[True][1][i].view(torch.int16)), i
        # identity experts with weights summing to the route scale: out = scale * x up to rounding
        x = xs[i % len(xs)].float()
        scale = wl.scale if wl.renorm else None
        if scale is not None:
            diff = (got[True][1][i].float() - scale * x).abs()
            assert (diff <= (scale * x).abs() * 2.0 ** -6 + 1e-5).all(), i
