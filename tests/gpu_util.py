"""Shared helpers of the GPU parity tests: run the library through its
binding and bring results back as numpy for comparison with the oracle."""
import numpy as np
import torch


def lib():
    from expert_load_balancing_tcgen05_b200 import moe
    return moe


def to_np(t):
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy()
    return t.cpu().numpy()


def route_gpu(wl, x, W, off, bias, scores_in=None):
    """moe_route on device tensors; returns (scores, idx, w, ws)."""
    moe = lib()
    dev = "cuda"
    T, N, K = wl.T, wl.N, wl.K
    scores = scores_in if scores_in is not None else torch.empty(T, N, dtype=torch.float32, device=dev)
    idx = torch.empty(T, K, dtype=torch.int32, device=dev)
    w = torch.empty(T, K, dtype=torch.float32, device=dev)
    ws = moe.workspace(T, K, N, wl.n_slots)
    cfg = moe.route_cfg(T, wl.d, N, K, wl.fn, wl.n_groups, wl.topk_groups, wl.group_topn, wl.renorm, wl.scale,
                        moe.MOE_BF16 if (x is not None and x.dtype == torch.bfloat16) else moe.MOE_F32)
    moe.moe_route(cfg, x if scores_in is None else None, W if scores_in is None else None, off, bias, scores,
                  idx, w, ws)
    return scores, idx, w, ws


def load_stats_gpu(idx, T, K, N, n_slots=None, replica_slot=None, scores=None, score_fn=1, ws=None):
    moe = lib()
    n_slots = N if n_slots is None else n_slots
    dev = "cuda"
    slot = torch.empty(T, K, dtype=torch.int32, device=dev)
    counts = torch.empty(n_slots, dtype=torch.int32, device=dev)
    offsets = torch.empty(n_slots + 1, dtype=torch.int32, device=dev)
    rank = torch.empty(T, K, dtype=torch.int32, device=dev)
    stats = moe.empty_stats(dev)
    if ws is None:
        ws = moe.workspace(T, K, N, n_slots)
    moe.moe_load_stats(idx, T, K, N, replica_slot, n_slots, slot, counts, offsets, rank, scores, score_fn, stats,
                       ws)
    return slot, counts, offsets, rank, stats, ws


def assert_stats_close(gpu: dict, ref: dict, rel=1e-6):
    assert gpu["status"] == 0
    assert gpu["total"] == int(ref["total"])
    assert gpu["max_load"] == int(ref["max"])
    for g, r in (("mean", "mean"), ("imbalance", "imbalance"), ("std_over_mean", "std_over_mean"),
                 ("entropy_load_bits", "entropy_load_bits"), ("capacity_fixed", "capacity_fixed"),
                 ("capacity_125", "capacity_125")):
        assert abs(gpu[g] - ref[r]) <= rel * abs(ref[r]) + 1e-12, (g, gpu[g], ref[r])


def gap_ok(s_ref: np.ndarray, bias, idx_gpu: np.ndarray, idx_ref: np.ndarray, K: int, n_groups=1,
           topk_groups=1, group_topn=2, tol=1e-3):
    """Tokens whose GPU choice differs from the oracle's (each side on its own
    scores) must sit on a near tie of the oracle's keys: the K-th / (K+1)-th
    key gap among the oracle's candidates, or the topk_groups-th /
    (topk_groups+1)-th group-score gap, below tol.  Returns (differing, bad)."""
    diff = np.nonzero((np.sort(idx_gpu, 1) != np.sort(idx_ref, 1)).any(1))[0]
    key = (s_ref + (bias if bias is not None else 0)).astype(np.float32)
    N = key.shape[1]
    bad = []
    for t in diff:
        cand = np.ones(N, bool)
        if n_groups > 1:
            gk = key[t].reshape(n_groups, -1)
            gs = np.sort(gk, 1)[:, ::-1][:, :group_topn].sum(1)
            order = np.argsort(-gs, kind="stable")
            srt = gs[order]
            if srt[topk_groups - 1] - srt[topk_groups] < tol:
                continue
            keep = np.zeros(n_groups, bool)
            keep[order[:topk_groups]] = True
            cand = np.repeat(keep, N // n_groups)
        srt = np.sort(key[t][cand])[::-1]
        if srt[K - 1] - srt[K] >= tol:
            bad.append(t)
    return diff, bad
