"""Pins for the CPU oracle: every check here is fixed by something other
than the oracle itself -- values printed on the pages, closed forms,
library routines, brute-force enumeration and invariants.  No GPU."""
import itertools
import math
import os

import numpy as np
import pytest
import torch

HERE = os.path.dirname(os.path.abspath(__file__))


def _p4_cases():
    rows = []
    with open(os.path.join(HERE, "golden", "p4_expert_load.txt")) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            name, loads, total, mx, imb, cap = line.split()
            rows.append((name, [int(v) for v in loads.split(",")], int(total), int(mx), imb,
                         int(cap)))
    assert len(rows) == 3
    return rows


def _idx_from_loads(loads):
    """K=1 assignment array whose histogram is `loads` (tokens in expert order)."""
    return np.array([e for e, c in enumerate(loads) for _ in range(c)], dtype=np.int32)[:, None]


# --------------------------------------------------------------------------------------
# "A minimal experiment in expert-load imbalance", Expected output
# --------------------------------------------------------------------------------------
@pytest.mark.parametrize("case", _p4_cases(), ids=lambda c: c[0])
def test_p4_printed_example(orc, case):
    name, loads, total, mx, imb_printed, cap = case
    idx = _idx_from_loads(loads)
    counts = orc.histogram(idx, 4)
    assert counts.tolist() == loads
    st = orc.load_stats(counts)
    assert st["total"] == total
    assert st["max"] == mx
    assert f"{st['imbalance']:.1f}" == imb_printed
    assert st["imbalance"] == float(imb_printed)
    assert st["capacity_fixed"] == cap


# closed forms for the same three histograms
@pytest.mark.parametrize("loads,H,som", [
    ([16, 16, 16, 16], 2.0, 0.0),
    # p = (5/8, 1/8, 1/8, 1/8): H = 5/8 log2(8/5) + 3/8 * 3
    ([40, 8, 8, 8], 0.625 * (3.0 - math.log2(5.0)) + 1.125, math.sqrt(3.0) / 2.0),
    ([64, 0, 0, 0], 0.0, math.sqrt(3.0)),
])
def test_load_entropy_and_spread_closed_forms(orc, loads, H, som):
    st = orc.load_stats(np.array(loads))
    assert st["entropy_load_bits"] == pytest.approx(H, rel=1e-12, abs=1e-15)
    assert st["std_over_mean"] == pytest.approx(som, rel=1e-12, abs=1e-15)
    assert st["capacity_125"] == pytest.approx(1.25 * 16)
    assert st["mean"] == 16.0


def test_empty_histogram_stats(orc):
    st = orc.load_stats(np.zeros(4, dtype=np.int64))
    assert st["imbalance"] == 0.0 and st["std_over_mean"] == 0.0 and st["entropy_load_bits"] == 0.0


def test_uniform_histogram_entropy_is_log2_n(orc):
    for N in (8, 128, 256, 288):
        st = orc.load_stats(np.full(N, 7))
        assert st["entropy_load_bits"] == pytest.approx(math.log2(N), rel=1e-12)


# --------------------------------------------------------------------------------------
# logits and scores
# --------------------------------------------------------------------------------------
def test_logits_integer_inputs_exact(orc):
    rng = np.random.default_rng(1)
    x = rng.integers(-8, 9, size=(37, 65)).astype(np.float32)
    W = rng.integers(-8, 9, size=(11, 65)).astype(np.float32)
    off = rng.integers(-3, 4, size=11).astype(np.float32)
    h = orc.logits(x, W, off)
    ref = x.astype(np.int64) @ W.astype(np.int64).T + off.astype(np.int64)
    assert np.array_equal(h, ref.astype(np.float64))


def test_logits_match_library_matmul(orc):
    rng = np.random.default_rng(2)
    x = rng.standard_normal((64, 300)).astype(np.float32)
    W = rng.standard_normal((24, 300)).astype(np.float32)
    h = orc.logits(x, W)
    ref = x.astype(np.float64) @ W.astype(np.float64).T
    np.testing.assert_allclose(h, ref, rtol=1e-12, atol=1e-12)


def test_sigmoid_and_softmax_against_library(orc):
    import scipy.special as sp
    rng = np.random.default_rng(3)
    h = rng.standard_normal((50, 40)) * 4
    s1 = orc.scores(h, 1)
    np.testing.assert_array_max_ulp(s1, sp.expit(h).astype(np.float32), maxulp=1)
    s0 = orc.scores(h, 0)
    np.testing.assert_array_max_ulp(s0, sp.softmax(h, axis=1).astype(np.float32), maxulp=1)
    np.testing.assert_allclose(s0.astype(np.float64).sum(1), 1.0, rtol=0, atol=4e-7)


def test_score_special_values(orc):
    h = np.array([[0.0, math.log(3.0)]])
    assert orc.scores(h, 0).tolist()[0] == pytest.approx([0.25, 0.75], rel=1e-7)
    assert orc.scores(np.zeros((1, 5)), 1).tolist()[0] == [0.5] * 5
    assert orc.scores(np.zeros((1, 5)), 0).tolist()[0] == [np.float32(0.2)] * 5


def test_score_entropy_uniform_is_log2_n(orc):
    """H = log2 N for uniform routing ("The Mathematics", high-entropy case):
    a zero gate gives uniform scores for both nonlinearities."""
    for N, fn in ((8, 0), (128, 0), (256, 1), (64, 1)):
        x = np.random.default_rng(N).standard_normal((40, 16)).astype(np.float32)
        s = orc.scores(orc.logits(x, np.zeros((N, 16), np.float32)), fn)
        assert orc.score_entropy(s, fn) == pytest.approx(math.log2(N), rel=1e-6)


def test_score_entropy_hand_example(orc):
    # sigmoid rows normalised per token: [.2,.6] -> [.25,.75]; [.5,.5] -> [.5,.5]
    s = np.array([[0.2, 0.6], [0.5, 0.5]], np.float32)
    m = np.array([0.375, 0.625])
    assert orc.score_entropy(s, 1) == pytest.approx(float(-(m * np.log2(m)).sum()), rel=1e-6)
    # softmax rows are used as they are
    s0 = np.array([[0.25, 0.75], [0.75, 0.25]], np.float32)
    assert orc.score_entropy(s0, 0) == pytest.approx(1.0, rel=1e-12)


# --------------------------------------------------------------------------------------
# selection
# --------------------------------------------------------------------------------------
def test_all_equal_scores_pick_lowest_indices(orc):
    for (N, G, TG, K) in ((8, 1, 1, 2), (256, 8, 4, 8), (128, 1, 1, 8), (64, 4, 2, 5)):
        s = np.full((10, N), 0.5, np.float32)
        idx, w = orc.select(s, None, K, G, TG, 2, True, 2.5)
        assert (idx == np.arange(K)).all()
        counts = orc.histogram(idx, N)
        assert counts.tolist() == [10] * K + [0] * (N - K)
        assert orc.load_stats(counts)["imbalance"] == pytest.approx(N / K)


def _brute_force(key, N, K, G, TG, n):
    """Enumerate group subsets and K-subsets; return the unique sets such
    that every chosen element beats every unchosen one."""
    gsize = N // G

    def better(a, b, vals):  # (value desc, index asc)
        return vals[a] > vals[b] or (vals[a] == vals[b] and a < b)

    if G > 1:
        gsc = []
        for g in range(G):
            top = sorted(key[g * gsize:(g + 1) * gsize], reverse=True)[:n]
            acc = np.float32(top[0])
            for v in top[1:]:
                acc = np.float32(acc + np.float32(v))
            gsc.append(acc)
        kept = [set(c) for c in itertools.combinations(range(G), TG)
                if all(better(a, b, gsc) for a in c for b in range(G) if b not in c)]
        assert len(kept) == 1
        cand = [e for e in range(N) if e // gsize in kept[0]]
    else:
        cand = list(range(N))
    sets = [c for c in itertools.combinations(cand, K)
            if all(better(a, b, key) for a in c for b in cand if b not in c)]
    assert len(sets) == 1
    return sorted(sets[0], key=lambda e: (-key[e], e))


@pytest.mark.parametrize("G,TG,K,quant", [
    (1, 1, 1, 0.0), (1, 1, 3, 0.25), (2, 1, 2, 0.0), (2, 1, 4, 0.25), (4, 2, 3, 0.0),
    (4, 2, 4, 0.125), (4, 1, 2, 0.25), (2, 2, 4, 0.0)])
def test_selection_brute_force(orc, G, TG, K, quant):
    from expert_load_balancing_tcgen05_b200 import workloads as wl
    N, T = 8, 400
    s = wl.make_scores(T, N, seed=17 + G * 10 + K, quantum=quant).numpy()
    b = wl.make_bias(N, seed=99 + K, amplitude=0.05).numpy()
    if quant:
        b = np.round(b / quant) * quant  # keep ties after the bias add
    idx, _ = orc.select(s, b, K, G, TG, 2, True, 1.0)
    key = (s + b).astype(np.float32)
    for t in range(T):
        assert idx[t].tolist() == _brute_force(key[t], N, K, G, TG, 2), t


def test_masked_groups_are_excluded_not_zeroed(orc):
    # group 0 keys negative but kept (its top-2 sum beats group 1's); group 1
    # is dropped: a zeroed group-1 expert (key 0) must not beat group 0's -0.1.
    s = np.array([[0.0, 0.0, 0.0, 0.0]], np.float32)
    b = np.array([-0.1, -0.1, -0.3, -0.3], np.float32)
    idx, _ = orc.select(s, b, 2, 2, 1, 2, True, 1.0)
    assert idx.tolist() == [[0, 1]]


def test_weights_use_unbiased_scores(orc):
    s = np.array([[0.5, 0.25, 0.125, 0.125]], np.float32)
    b = np.array([0.0, 0.0, 0.5, 0.0], np.float32)   # bias promotes expert 2
    idx, w = orc.select(s, b, 2, 1, 1, 2, True, 2.5)
    assert idx.tolist() == [[2, 0]]
    # weights: 0.125/0.625 = 0.2, 0.5/0.625 = 0.8, times 2.5
    assert w[0].tolist() == pytest.approx([0.5, 2.0], rel=1e-7)
    idx, w = orc.select(s, None, 2, 1, 1, 2, False, 1.0)
    assert idx.tolist() == [[0, 1]] and w[0].tolist() == [0.5, 0.25]


def test_weights_sum_to_scale(orc):
    from expert_load_balancing_tcgen05_b200 import workloads as wl
    s = wl.make_scores(300, 256, seed=5).numpy()
    b = wl.make_bias(256, seed=6).numpy()
    idx, w = orc.select(s, b, 8, 8, 4, 2, True, 2.5)
    np.testing.assert_allclose(w.astype(np.float64).sum(1), 2.5, rtol=2e-6)
    assert all(len(set(r)) == 8 for r in idx.tolist())
    # chosen experts come from exactly <= 4 groups
    assert max(len({e // 32 for e in r}) for r in idx.tolist()) <= 4


# --------------------------------------------------------------------------------------
# histogram, offsets, positions, dispatch, replicas
# --------------------------------------------------------------------------------------
def test_positions_hand_example(orc):
    slot = np.array([[1, 0], [1, 2], [0, 1]], np.int32)
    counts, offsets, pos, rank, row_src = orc.positions(slot, 3)
    assert counts.tolist() == [2, 3, 1]
    assert offsets.tolist() == [0, 2, 5, 6]
    assert pos.tolist() == [[2, 0], [3, 5], [1, 4]]
    assert rank.tolist() == [[0, 0], [1, 0], [1, 2]]
    assert row_src.tolist() == [0, 2, 0, 1, 2, 1]


def test_positions_invariants(orc):
    from expert_load_balancing_tcgen05_b200 import workloads as wl
    T, K, N = 3000, 8, 64
    idx = wl.make_assignments(T, K, N, seed=3, skew=1.1).numpy()
    counts, offsets, pos, rank, row_src = orc.positions(idx, N)
    assert counts.sum() == T * K and offsets[-1] == T * K
    assert np.array_equal(np.sort(pos.reshape(-1)), np.arange(T * K))
    flat = idx.reshape(-1)
    assert np.array_equal(pos.reshape(-1), offsets[flat] + rank.reshape(-1))
    for e in range(N):
        seg = row_src[offsets[e]:offsets[e + 1]]
        assert (np.diff(seg) >= 0).all()
        assert np.array_equal(np.sort(rank.reshape(-1)[flat == e]), np.arange(counts[e]))


def test_dispatch_rows_follow_row_src(orc):
    rng = np.random.default_rng(7)
    T, K, N, d = 50, 3, 7, 16
    x = rng.standard_normal((T, d)).astype(np.float32)
    idx = np.stack([rng.choice(N, K, replace=False) for _ in range(T)]).astype(np.int32)
    _, _, pos, _, row_src = orc.positions(idx, N)
    rows = orc.dispatch_rows(x, pos)
    assert np.array_equal(rows, x[row_src])


def test_replica_plan_hand_example(orc):
    r = orc.replica_plan(np.array([5, 9, 9, 1]), 2)
    assert r.tolist() == [-1, 4, 5, -1]
    idx = np.array([[1, 0], [1, 2], [3, 2], [2, 1]], np.int32)
    slot = orc.apply_replicas(idx, r)
    assert slot.tolist() == [[1, 0], [4, 5], [3, 2], [5, 4]]


def test_replica_pairs_sum_to_original_load(orc):
    from expert_load_balancing_tcgen05_b200 import workloads as wl
    T, K, N, R = 2001, 8, 256, 32
    idx = wl.make_assignments(T, K, N, seed=11, skew=1.1).numpy()
    c = orc.histogram(idx, N)
    r = orc.replica_plan(c, R)
    hot = np.argsort(-c, kind="stable")[:R]
    assert sorted(np.nonzero(r >= 0)[0].tolist()) == sorted(hot.tolist())
    assert [r[e] for e in hot] == list(range(N, N + R))
    c2 = orc.histogram(orc.apply_replicas(idx, r), N + R)
    for e in range(N):
        if r[e] >= 0:
            assert c2[e] + c2[r[e]] == c[e]
        else:
            assert c2[e] == c[e]
    assert c2.sum() == T * K
    assert orc.load_stats(c2)["max"] <= orc.load_stats(c)["max"]


# --------------------------------------------------------------------------------------
# FP8 e4m3
# --------------------------------------------------------------------------------------
def test_e4m3_known_codes(orc):
    cases = {448.0: 0x7E, -448.0: 0xFE, 1.0: 0x38, 2.0 ** -9: 0x01, 2.0 ** -6: 0x08,
             7 * 2.0 ** -9: 0x07, 1.0625: 0x38, 1.1875: 0x3A, 500.0: 0x7E, -1e6: 0xFE,
             0.0: 0x00, 464.0: 0x7E, 240.0: 0x77, 2.0 ** -10: 0x00, 3 * 2.0 ** -11: 0x01}
    for v, code in cases.items():
        assert orc.e4m3_encode(v) == code, (v, hex(orc.e4m3_encode(v)))
    assert orc.e4m3_encode(float("nan")) == 0x7F
    assert orc.e4m3_encode(-0.0) == 0x80


def test_e4m3_decode_matches_library(orc):
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).float().numpy()
    ours = np.array([orc.e4m3_decode(c) for c in range(256)], np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_e4m3_encode_matches_library_in_range(orc):
    rng = np.random.default_rng(8)
    v = np.concatenate([rng.uniform(-448, 448, 20000), rng.standard_normal(20000),
                        rng.standard_normal(5000) * 1e-2, rng.standard_normal(5000) * 1e-3,
                        # every code value and every midpoint between neighbours
                        np.array([orc.e4m3_decode(c) for c in range(0, 0x7F)])]).astype(np.float32)
    mids = []
    pos_vals = [orc.e4m3_decode(c) for c in range(0, 0x7F)]
    for a, b in zip(pos_vals[:-1], pos_vals[1:]):
        mids += [(a + b) / 2, -(a + b) / 2]
    v = np.concatenate([v, np.array(mids, np.float32)])
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([orc.e4m3_encode(float(a)) for a in v], np.uint8)
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, [(float(v[i]), hex(ours[i]), hex(ref[i])) for i in bad[:5]]


def test_fp8_rows_block_max_and_error_bound(orc):
    rng = np.random.default_rng(9)
    rows = rng.standard_normal((20, 512)).astype(np.float32)
    rows[3, 128:256] = 0.0                      # an all-zero block
    rows[4] *= 1e-4
    q, sc = orc.fp8_rows(rows)
    assert sc[3, 1] == 0.0 and (q[3, 128:256] == 0).all()
    dec = np.vectorize(orc.e4m3_decode, otypes=[np.float32])(q)
    for r in range(20):
        for b in range(4):
            blk = rows[r, b * 128:(b + 1) * 128]
            if not np.abs(blk).max():
                continue
            j = int(np.argmax(np.abs(blk)))
            assert q[r, b * 128 + j] in (0x7E, 0xFE)
            assert sc[r, b] == np.float32(np.abs(blk).max() / np.float32(448.0))
            d = dec[r, b * 128:(b + 1) * 128]
            # |q - v*inv| <= half the e4m3 spacing at q (subnormal spacing 2^-9)
            a = np.maximum(np.abs(d), 2.0 ** -6)
            half_ulp = 2.0 ** (np.floor(np.log2(a)) - 4)
            inv = np.float32(448.0) / np.float32(np.abs(blk).max())
            assert (np.abs(d - blk * inv) <= half_ulp * (1 + 1e-6)).all()


# --------------------------------------------------------------------------------------
# combine and bias update
# --------------------------------------------------------------------------------------
def test_combine_hand_example(orc):
    y = np.array([[1.0, 2.0], [10.0, 20.0], [100.0, 200.0]], np.float32)
    pos = np.array([[2, 0], [1, 1]], np.int64)
    w = np.array([[0.5, 0.25], [1.0, -1.0]], np.float32)
    out = orc.combine(y, pos, w)
    assert out.tolist() == [[50.25, 100.5], [0.0, 0.0]]


def test_dispatch_combine_round_trip(orc):
    from expert_load_balancing_tcgen05_b200 import workloads as wl
    T, K, N, d = 200, 4, 16, 32
    x = np.random.default_rng(4).standard_normal((T, d)).astype(np.float32)
    s = wl.make_scores(T, N, seed=4).numpy()
    idx, w = orc.select(s, None, K, 1, 1, 2, True, 1.0)
    _, _, pos, _, _ = orc.positions(idx, N)
    rows = orc.dispatch_rows(x, pos)
    out = orc.combine(rows, pos, w)
    np.testing.assert_allclose(out, x, rtol=1e-6, atol=1e-6)


def test_bias_update_sign_rule(orc):
    counts = np.array([10, 6, 8, 8])
    b = orc.bias_update(counts, 32, np.zeros(4, np.float32), 0.001, 0)
    assert b.tolist() == [-np.float32(0.001), np.float32(0.001), 0.0, 0.0]
    b0 = np.array([0.25, -0.5, 0.125, 1.0], np.float32)
    b1 = orc.bias_update(counts, 32, b0, 0.001, 0)
    # each bias moves by 0 or by one step of 0.001 in the right direction
    assert b1[0] < b0[0] and b1[1] > b0[1] and b1[2] == b0[2] and b1[3] == b0[3]
    assert abs(float(b1[0]) - 0.249) < 1e-7 and abs(float(b1[1]) + 0.499) < 1e-7


def test_bias_update_proportional_rule(orc):
    # "Concrete Implementation": target 8, errors (2, -2, 0, 0), decay 0.05
    counts = np.array([10, 6, 8, 8])
    b = orc.bias_update(counts, 32, np.zeros(4, np.float32), 0.05, 1)
    q = np.float32(0.05) * np.float32(0.25)
    assert b.tolist() == [-q, q, 0.0, 0.0]


# --------------------------------------------------------------------------------------
# forcible balancing, bias in the logits, smoothed-load bias update
# --------------------------------------------------------------------------------------
def test_forcible_balance_is_exactly_balanced(orc):
    for T, K, N in ((64, 1, 4), (1000, 8, 256), (513, 2, 8), (7, 3, 5)):
        idx, w = orc.route_balanced(T, K, N, 2.5)
        assert all(len(set(r)) == K for r in idx.tolist())        # distinct experts per token
        c = orc.histogram(idx, N)
        assert c.max() - c.min() <= 1 and c.sum() == T * K
        np.testing.assert_allclose(w.astype(np.float64).sum(1), 2.5, rtol=1e-6)
    # the page's four experts and 64 assignments: the balanced case of the worked example
    idx, _ = orc.route_balanced(64, 1, 4)
    st = orc.load_stats(orc.histogram(idx, 4))
    assert st["imbalance"] == 1.0 and st["capacity_fixed"] == 64


def test_bias_in_logits_softmax_shift_invariance(orc):
    # a bias equal on every expert cancels in the softmax
    rng = np.random.default_rng(21)
    x = rng.standard_normal((30, 16)).astype(np.float32)
    W = rng.standard_normal((8, 16)).astype(np.float32)
    _, s0, i0, w0 = orc.route(x, W, None, None, 0, 2)
    _, s1, i1, w1 = orc.route(x, W, None, np.full(8, 0.75, np.float32), 0, 2, bias_in_logits=True)
    np.testing.assert_allclose(s1, s0, rtol=1e-6)
    assert np.array_equal(i0, i1)


def test_bias_in_logits_shapes_weights(orc):
    # one token, equal logits: a logit bias of ln 3 on expert 2 makes it three
    # times as likely as the others; selection-only bias would leave weights equal
    x = np.zeros((1, 4), np.float32)
    W = np.zeros((4, 4), np.float32)
    b = np.array([0, 0, np.log(3.0), 0], np.float32)
    _, s, idx, w = orc.route(x, W, None, b, 0, 2, bias_in_logits=True)
    assert idx.tolist() == [[2, 0]]
    assert w[0].tolist() == pytest.approx([0.75, 0.25], rel=1e-6)
    _, s2, idx2, w2 = orc.route(x, W, None, b, 0, 2)
    assert idx2.tolist() == [[2, 0]] and w2[0].tolist() == [0.5, 0.5]


def test_bias_update_ema_reduces_to_sign_rule(orc):
    counts = np.array([10, 6, 8, 8])
    b0 = np.zeros(4, np.float32)
    b, e = orc.bias_update_ema(counts, 32, b0, np.zeros(4, np.float32), 0.001, 0.0)
    assert b.tolist() == orc.bias_update(counts, 32, b0, 0.001, 0).tolist()
    assert e.tolist() == [10.0, 6.0, 8.0, 8.0]


def test_bias_update_ema_smooths(orc):
    # alpha = 0.5: the moving average moves halfway to the new load each step
    counts = np.array([16, 0, 8, 8])
    b, e = orc.bias_update_ema(counts, 32, np.zeros(4, np.float32), np.full(4, 8, np.float32), 0.001, 0.5)
    assert e.tolist() == [12.0, 4.0, 8.0, 8.0]
    assert b.tolist() == [-np.float32(0.001), np.float32(0.001), 0.0, 0.0]
    # a load that stays constant: the average converges to it geometrically
    e = np.zeros(4, np.float32)
    for _ in range(40):
        _, e = orc.bias_update_ema(counts, 32, np.zeros(4, np.float32), e, 0.001, 0.5)
    np.testing.assert_allclose(e, counts, atol=1e-5)


# --- dropped assignments and capacity-limited routing ("Production Testing") ---

def test_dropped_assignments_take_no_slot(orc):
    # hand example: token 1's second slot is dropped (-1)
    slot = np.array([[0, 1], [1, -1], [0, 1]], np.int32)
    counts, offsets, pos, rank, row_src = orc.positions(slot, 2)
    assert counts.tolist() == [2, 3]
    assert offsets.tolist() == [0, 2, 5]
    assert pos.tolist() == [[0, 2], [3, -1], [1, 4]]
    assert rank.tolist() == [[0, 0], [1, -1], [1, 2]]
    assert row_src[:5].tolist() == [0, 2, 0, 1, 2]
    x = np.arange(6, dtype=np.float32).reshape(3, 2)
    rows = orc.dispatch_rows(x, pos)
    assert rows[:5].tolist() == [[0, 1], [4, 5], [0, 1], [2, 3], [4, 5]]
    # combine skips the dropped slot even with a nonzero weight
    w = np.array([[1, 1], [1, 7], [1, 1]], np.float32)
    out = orc.combine(rows[:5], pos, w)
    assert out.tolist() == [[0, 2], [2, 3], [8, 10]]
    assert orc.histogram(slot, 2).tolist() == [2, 3]
    with pytest.raises(ValueError):
        orc.histogram(np.array([[2]], np.int32), 2)


def test_capacity_limit_value(orc):
    # 1.25 * T*K/N, rounded up: 1.25 * 16384*8/256 = 640 exactly; 1.875 -> 2
    assert orc.capacity_limit(16384, 8, 256) == 640
    assert orc.capacity_limit(6, 1, 4) == 2
    assert orc.capacity_limit(3, 2, 4) == 2
    assert orc.capacity_limit(7, 1, 4) == 3  # 2.1875


def test_capacity_hand_example_single_slot(orc):
    # six tokens all preferring expert 0 then 1; capacity 2: tokens 0, 1 keep
    # expert 0, tokens 2, 3 move to expert 1, tokens 4, 5 find it full
    s = np.tile(np.array([0.9, 0.5, 0.3, 0.1], np.float32), (6, 1))
    idx, w, info = orc.route_capacity(s, None, 1)
    assert info == dict(capacity=2, overflow=4, rerouted=2, dropped=2)
    assert idx[:, 0].tolist() == [0, 0, 1, 1, -1, -1]
    assert w[:, 0].tolist() == [1, 1, 1, 1, 0, 0]


def test_capacity_hand_example_two_slots(orc):
    # both slots of token 2 overflow; its 1st overflow takes candidate 3 (rank
    # K+0), the 2nd candidate 4 (rank K+1); weights renormalise over them
    s = np.array([[0.9, 0.8, 0.2, 0.1], [0.9, 0.8, 0.2, 0.1], [0.9, 0.8, 0.3, 0.2]], np.float32)
    idx, w, info = orc.route_capacity(s, None, 2, scale=2.0)
    assert info == dict(capacity=2, overflow=2, rerouted=2, dropped=0)
    assert idx.tolist() == [[0, 1], [0, 1], [2, 3]]
    den = np.float32(0.3) + np.float32(0.2)
    assert w[2].tolist() == [np.float32(np.float32(0.3) / den) * np.float32(2.0),
                             np.float32(np.float32(0.2) / den) * np.float32(2.0)]


def test_capacity_primaries_before_reroutes(orc):
    # the primary pass finishes before any reroute: token 2's primary on
    # expert 1 wins over token 1's reroute there, which is dropped
    s = np.array([[0.9, 0.5, 0.1], [0.9, 0.5, 0.1], [0.1, 0.9, 0.5]], np.float32)
    idx, w, info = orc.route_capacity(s, None, 1, capacity=1)
    assert idx[:, 0].tolist() == [0, -1, 1]
    assert info == dict(capacity=1, overflow=1, rerouted=0, dropped=1)


def test_capacity_unbounded_is_plain_selection(orc):
    g = np.random.default_rng(8)
    s = g.random((300, 64)).astype(np.float32)
    b = g.uniform(-0.05, 0.05, 64).astype(np.float32)
    for kw in (dict(), dict(n_groups=8, topk_groups=3, group_topn=2)):
        ri, rw = orc.select(s, b, 6, renorm=True, scale=2.5, **kw)
        ci, cw, info = orc.route_capacity(s, b, 6, renorm=True, scale=2.5, capacity=300 * 6, **kw)
        assert np.array_equal(ci, ri) and np.array_equal(cw, rw)
        assert info["overflow"] == 0


def test_capacity_zero_drops_everything(orc):
    s = np.random.default_rng(1).random((10, 16)).astype(np.float32)
    idx, w, info = orc.route_capacity(s, None, 4, capacity=0)
    assert (idx == -1).all() and (w == 0).all()
    assert info == dict(capacity=0, overflow=40, rerouted=0, dropped=40)


@pytest.mark.parametrize("grouped", [False, True])
def test_capacity_invariants(orc, grouped):
    """Against the pinned selection and positions: primaries kept exactly when
    their stable in-expert rank is below C; the j-th overflowed slot of a
    token moves to its (K+j)-th ranked candidate (selection with 2K) or is
    dropped; no expert exceeds C; kept weights renormalise to the scale."""
    g = np.random.default_rng(21)
    T, N, K = 700, 64, 4
    kw = dict(n_groups=8, topk_groups=4, group_topn=2) if grouped else dict()
    # skewed scores so that the capacity binds
    s = (g.random((T, N)) * np.linspace(1.0, 0.2, N)[None, :]).astype(np.float32)
    b = g.uniform(-0.01, 0.01, N).astype(np.float32)
    idx, w, info = orc.route_capacity(s, b, K, scale=2.5, **kw)
    C = info["capacity"]
    prim, _ = orc.select(s, b, K, **kw)
    wide, _ = orc.select(s, b, 2 * K, **kw)
    assert np.array_equal(wide[:, :K], prim)
    _, _, _, rank, _ = orc.positions(prim, N)
    keep = rank < C
    assert info["overflow"] == int((~keep).sum()) > 0
    assert np.array_equal(idx[keep], prim[keep])
    for t in range(T):
        j = 0
        for k in range(K):
            if keep[t, k]:
                continue
            assert idx[t, k] in (-1, wide[t, K + j])
            j += 1
    assert info["rerouted"] + info["dropped"] == info["overflow"]
    assert int((idx == -1).sum()) == info["dropped"]
    assert orc.histogram(idx, N).max() <= C
    for t in range(T):
        row = idx[t]
        kept = row[row >= 0]
        assert len(set(kept.tolist())) == len(kept)
        if len(kept):
            assert float(w[t][row >= 0].sum()) == pytest.approx(2.5, rel=1e-5)
        assert (w[t][row < 0] == 0).all()


def test_bias_update_ema_sign_follows_the_average_not_the_batch(orc):
    # ema0 = [20, 0, 8, 4], this batch [4, 12, 8, 8] (mean 8), alpha = 0.5:
    # ema = [12, 6, 8, 6] -> signs (+, -, 0, -) although the batch alone
    # says (-, +, 0, 0)
    counts = np.array([4, 12, 8, 8])
    b, e = orc.bias_update_ema(counts, 32, np.zeros(4, np.float32), np.array([20, 0, 8, 4], np.float32), 0.001, 0.5)
    assert e.tolist() == [12.0, 6.0, 8.0, 6.0]
    u = np.float32(0.001)
    assert b.tolist() == [-u, u, 0.0, u]


def test_bias_in_logits_selects_on_the_scores_alone(orc):
    # sigmoid, two experts, K = 1: h = (3, 2), b = (0, 0.5).  With the bias in
    # the logits the scores are sigma(3) > sigma(2.5), so expert 0 wins; adding
    # the bias to the key as well would pick expert 1 (sigma(2.5) + 0.5 larger)
    x = np.array([[1.0]], np.float32)
    W = np.array([[3.0], [2.0]], np.float32)
    b = np.array([0.0, 0.5], np.float32)
    _, s, idx, w = orc.route(x, W, None, b, 1, 1, bias_in_logits=True)
    assert idx.tolist() == [[0]] and w.tolist() == [[1.0]]
    assert s[0, 0] > s[0, 1] and s[0, 1] + b[1] > s[0, 0]
