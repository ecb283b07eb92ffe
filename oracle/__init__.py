"""CPU oracle for the MoE routing hot path -- TEST INFRASTRUCTURE ONLY.

A plain, slow, double-precision restatement of what the routing path
computes, used to check the CUDA library.  Only the tests, the smoke check
and the benchmark's CPU-baseline / reference leg may import it; the product
path never does.  It shares no code with the CUDA library: the arithmetic
lives in ``moe_oracle.c`` (plain C, built with gcc by :func:`build`), and
this module only marshals numpy arrays into it.

Each wrapper names the passage it follows; the C file states each
definition in full.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

# -ffp-contract=off: fp32 steps (keys, weights, bias step, FP8 products) must
# be single rounded operations, never fused multiply-adds.
CFLAGS = ["-O3", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
          "-fno-fast-math", "-Wall", "-Wno-unused-label"]


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into libmoe_oracle.so next to it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", _LIB, "-lm"])
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i64, i32, f32 = ctypes.c_int64, ctypes.c_int, ctypes.c_float
        L.oracle_num_threads.restype = i32
        L.oracle_set_num_threads.argtypes = [i32]
        L.oracle_logits.argtypes = [P, P, P, i64, i64, i64, P]
        L.oracle_scores.argtypes = [P, i64, i64, i32, P]
        L.oracle_select.argtypes = [P, P, i64, i32, i32, i32, i32, i32, i32, f32, P, P]
        L.oracle_select.restype = i32
        L.oracle_histogram.argtypes = [P, i64, i32, P]
        L.oracle_histogram.restype = i32
        L.oracle_load_stats.argtypes = [P, i32, P]
        L.oracle_score_entropy.argtypes = [P, i64, i32, i32]
        L.oracle_score_entropy.restype = ctypes.c_double
        L.oracle_replica_plan.argtypes = [P, i32, i32, P]
        L.oracle_apply_replicas.argtypes = [P, i64, i32, P, P]
        L.oracle_positions.argtypes = [P, i64, i32, P, i32, P, P, P, P]
        L.oracle_dispatch_rows.argtypes = [P, i64, i64, i32, P, P]
        L.oracle_e4m3_encode.argtypes = [f32]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_decode.restype = f32
        L.oracle_fp8_rows.argtypes = [P, i64, i64, P, P]
        L.oracle_combine.argtypes = [P, P, P, i64, i32, i64, P]
        L.oracle_bias_update.argtypes = [P, i32, i64, f32, i32, P]
        L.oracle_route_balanced.argtypes = [i64, i32, i32, f32, P, P]
        L.oracle_bias_update_ema.argtypes = [P, i32, i64, f32, f32, P, P]
        L.oracle_route_capacity.argtypes = [P, P, i64, i32, i32, i32, i32, i32, i32, f32, i64, P, P, P]
        L.oracle_route_capacity.restype = i32
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def set_num_threads(n: int) -> None:
    lib().oracle_set_num_threads(int(n))


def logits(x, W, off=None) -> np.ndarray:
    """h = x . W^T (+ off), fp64 sums of the exact input values.

    "MoE Routing Entropy vs Expert Saturation", section "The Mathematics"
    (h = x . W_g) with the nn.Linear(hidden, N, bias=False) gate of section
    "Concrete Implementation".
    """
    x, W = _f32(x), _f32(W)
    T, d = x.shape
    N = W.shape[0]
    assert W.shape[1] == d
    h = np.empty((T, N), dtype=np.float64)
    o = _f32(off) if off is not None else None
    lib().oracle_logits(_p(x), _p(W), _p(o) if o is not None else None, T, d, N, _p(h))
    return h


def scores(h, fn: int) -> np.ndarray:
    """fn 0 = softmax ("The Mathematics", softmax equation), fn 1 = sigmoid
    ("DeepSeek V4 MoE load balancing", token routing section); double, then
    one rounding to fp32."""
    h = np.ascontiguousarray(h, dtype=np.float64)
    T, N = h.shape
    s = np.empty((T, N), dtype=np.float32)
    lib().oracle_scores(_p(h), T, N, int(fn), _p(s))
    return s


def select(s, bias, K, n_groups=1, topk_groups=1, group_topn=2, renorm=True, scale=1.0):
    """Bias-adjusted, group-limited top-K and combine weights.

    Group-limited routing: "DeepSeek-V3 Group-Limited Expert Routing",
    sections 1 and 3; bias for selection only: "DeepSeek V4 MoE load
    balancing", aux-loss-free section; renormalised weights: "MoE Routing
    Entropy vs Expert Saturation", section "Concrete Implementation".
    """
    s = _f32(s)
    T, N = s.shape
    b = _f32(bias) if bias is not None else None
    idx = np.empty((T, K), dtype=np.int32)
    w = np.empty((T, K), dtype=np.float32)
    rc = lib().oracle_select(_p(s), _p(b) if b is not None else None, T, N, K, n_groups,
                             topk_groups, group_topn, int(bool(renorm)), float(scale),
                             _p(idx), _p(w))
    if rc != 0:
        raise ValueError("oracle_select: invalid configuration")
    return idx, w


def histogram(slot, n_slots) -> np.ndarray:
    """bincount of the chosen slots ("Concrete Implementation")."""
    slot = np.ascontiguousarray(slot, dtype=np.int32).reshape(-1)
    c = np.empty(n_slots, dtype=np.int64)
    if lib().oracle_histogram(_p(slot), slot.size, n_slots, _p(c)) != 0:
        raise ValueError("slot index out of range")
    return c


STAT_KEYS = ("total", "max", "mean", "imbalance", "std_over_mean", "entropy_load_bits",
             "capacity_fixed", "capacity_125")


def load_stats(counts) -> dict:
    """Total / max / mean / max-over-mean / capacity ("A minimal experiment in
    expert-load imbalance"), std/mean (hotdry monitoring section), load
    entropy in bits ("The Mathematics"), 1.25 capacity ("Production
    Testing")."""
    c = np.ascontiguousarray(counts, dtype=np.int64)
    out = np.empty(8, dtype=np.float64)
    lib().oracle_load_stats(_p(c), c.size, _p(out))
    return dict(zip(STAT_KEYS, out.tolist()))


def score_entropy(s, fn: int) -> float:
    """Entropy of the batch-mean routing distribution ("Concrete
    Implementation", compute_routing_entropy), in bits."""
    s = _f32(s)
    T, N = s.shape
    return float(lib().oracle_score_entropy(_p(s), T, N, int(fn)))


def replica_plan(counts, n_rep: int) -> np.ndarray:
    """Replica slots N.. for the n_rep hottest experts (count desc, index asc)."""
    c = np.ascontiguousarray(counts, dtype=np.int64)
    r = np.empty(c.size, dtype=np.int32)
    lib().oracle_replica_plan(_p(c), c.size, int(n_rep), _p(r))
    return r


def apply_replicas(idx, replica_slot) -> np.ndarray:
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, K = idx.shape
    out = np.empty_like(idx)
    r = np.ascontiguousarray(replica_slot, dtype=np.int32) if replica_slot is not None else None
    lib().oracle_apply_replicas(_p(idx), T, K, _p(r) if r is not None else None, _p(out))
    return out


def positions(slot, n_slots):
    """offsets (exclusive prefix of counts), pos, in-expert rank, row_src."""
    slot = np.ascontiguousarray(slot, dtype=np.int32)
    T, K = slot.shape
    counts = histogram(slot, n_slots)
    offsets = np.empty(n_slots + 1, dtype=np.int64)
    pos = np.empty((T, K), dtype=np.int64)
    rank = np.empty((T, K), dtype=np.int64)
    row_src = np.empty(T * K, dtype=np.int64)
    lib().oracle_positions(_p(slot), T, K, _p(counts), n_slots, _p(offsets), _p(pos),
                           _p(rank), _p(row_src))
    return counts, offsets, pos, rank, row_src


def dispatch_rows(x: np.ndarray, pos) -> np.ndarray:
    """rows[pos[t,k]] = x[t] (byte copy)."""
    x = np.ascontiguousarray(x)
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    T, K = pos.shape
    rows = np.zeros((T * K,) + x.shape[1:], dtype=x.dtype)
    row_bytes = x.strides[0]
    lib().oracle_dispatch_rows(_p(x), T, row_bytes, K, _p(pos), _p(rows))
    return rows


def e4m3_encode(v: float) -> int:
    return int(lib().oracle_e4m3_encode(float(v)))


def e4m3_decode(c: int) -> float:
    return float(lib().oracle_e4m3_decode(int(c)))


def fp8_rows(rows):
    """Per-row, per-128-channel e4m3 quantisation with fp32 scale amax/448."""
    r = _f32(rows)
    R, d = r.shape
    assert d % 128 == 0
    q = np.empty((R, d), dtype=np.uint8)
    sc = np.empty((R, d // 128), dtype=np.float32)
    lib().oracle_fp8_rows(_p(r), R, d, _p(q), _p(sc))
    return q, sc


def combine(y, pos, w) -> np.ndarray:
    """out[t] = sum_k w[t,k] y[pos[t,k]] in double."""
    y = _f32(y)
    pos = np.ascontiguousarray(pos, dtype=np.int64)
    w = _f32(w)
    T, K = pos.shape
    d = y.shape[1]
    out = np.empty((T, d), dtype=np.float64)
    lib().oracle_combine(_p(y), _p(pos), _p(w), T, K, d, _p(out))
    return out


def bias_update(counts, total, bias, u=0.001, mode=0) -> np.ndarray:
    """mode 0: b -= u * sign(c - total/N) (hotdry aux-loss-free section, sign
    reading); mode 1: the DynamicEntropyMoERouter proportional rule."""
    c = np.ascontiguousarray(counts, dtype=np.int64)
    b = _f32(bias).copy()
    lib().oracle_bias_update(_p(c), c.size, int(total), float(u), int(mode), _p(b))
    return b


def route(x, W, off, bias, fn, K, n_groups=1, topk_groups=1, group_topn=2, renorm=True,
          scale=1.0, bias_in_logits=False):
    """Gate -> scores -> selection, end to end on the CPU.

    bias_in_logits: the bias joins the logits before the nonlinearity, as in
    the DynamicEntropyMoERouter of "MoE Routing Entropy vs Expert
    Saturation" ("Concrete Implementation": the router adds its expert biases
    to the raw logits), so it shapes the weights too and selection uses the
    scores themselves; otherwise it only shifts the selection key."""
    h = logits(x, W, off)
    if bias_in_logits and bias is not None:
        h = h + np.asarray(bias, dtype=np.float64)[None, :]
    s = scores(h, fn)
    idx, w = select(s, None if bias_in_logits else bias, K, n_groups, topk_groups, group_topn, renorm, scale)
    return h, s, idx, w


def route_balanced(T, K, N, scale=1.0):
    """Round-robin expert (t*K + k) mod N with equal weights scale/K: the
    "forcible load balancing" upper bound of the MindIE load-balancer page."""
    idx = np.empty((T, K), dtype=np.int32)
    w = np.empty((T, K), dtype=np.float32)
    lib().oracle_route_balanced(T, K, N, float(scale), _p(idx), _p(w))
    return idx, w


def bias_update_ema(counts, total, bias, ema, u=0.001, alpha=0.9):
    """Sign-rule bias step on an exponential moving average of the load
    (hotdry aux-loss-free section: smoothed load statistics).  Returns
    (new_bias, new_ema)."""
    c = np.ascontiguousarray(counts, dtype=np.int64)
    b = _f32(bias).copy()
    e = _f32(ema).copy()
    lib().oracle_bias_update_ema(_p(c), c.size, int(total), float(u), float(alpha), _p(e), _p(b))
    return b, e


def capacity_limit(T, K, N, factor_quarters=5):
    """ceil(1.25 * T*K/N) in integers: the per-expert token capacity of the
    "Production Testing" section of the entropy page."""
    return (factor_quarters * T * K + 4 * N - 1) // (4 * N)


def route_capacity(s, bias, K, n_groups=1, topk_groups=1, group_topn=2, renorm=True, scale=1.0,
                   capacity=None):
    """Capacity-limited selection on fp32 scores: primaries accepted in flat
    (t, k) order up to the capacity, each token's overflowed slots moved to
    its next ranked candidates, the rest dropped (idx -1, weight 0).
    Returns (idx, w, info) with info = {capacity, overflow, rerouted, dropped}."""
    s = _f32(s)
    T, N = s.shape
    C = capacity_limit(T, K, N) if capacity is None else int(capacity)
    b = _f32(bias) if bias is not None else None
    idx = np.empty((T, K), dtype=np.int32)
    w = np.empty((T, K), dtype=np.float32)
    info = np.zeros(3, dtype=np.int64)
    rc = lib().oracle_route_capacity(_p(s), _p(b) if b is not None else None, T, N, K, n_groups,
                                     topk_groups, group_topn, 1 if renorm else 0, float(scale), C,
                                     _p(idx), _p(w), _p(info))
    if rc != 0:
        raise ValueError("oracle_route_capacity: invalid configuration")
    return idx, w, dict(capacity=C, overflow=int(info[0]), rerouted=int(info[1]), dropped=int(info[2]))
