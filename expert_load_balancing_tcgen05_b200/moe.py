"""Python binding of libmoeroute.so (ctypes): argument marshalling only.

Every function here has the name and meaning of the C entry point it wraps
(see include/moe_route.h).  Tensors are passed by device pointer together
with torch's current CUDA stream; every step runs in the library's kernels.
Importing this module loads the library and raises if it is missing -- there
is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# MOEROUTE_LIB names another build of the library (for side-by-side timing)
LIB_PATH = os.environ.get("MOEROUTE_LIB") or os.path.join(_HERE, "libmoeroute.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} not found: build it with `python -m expert_load_balancing_tcgen05_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

MOE_OK, MOE_ERR_INVALID, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_TIMEOUT = range(5)
MOE_SOFTMAX, MOE_SIGMOID = 0, 1
MOE_F32, MOE_BF16 = 0, 1

EXPORTS = ("moe_workspace_bytes", "moe_route", "moe_load_stats", "moe_replica_plan", "moe_bias_update",
           "moe_dispatch", "moe_combine", "moe_workspace_status", "moe_launch_count", "moe_status_str",
           "moe_version", "moe_load_stats_noalloc", "moe_selftest_wait_timeout", "moe_route_balanced",
           "moe_bias_update_ema", "moe_route_capacity", "moe_capacity_workspace_bytes", "moe_capacity_limit",
           "moe_route_tiles", "moe_load_stats_tiles")


class RouteCfg(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("N", ctypes.c_int32), ("K", ctypes.c_int32),
                ("score_fn", ctypes.c_int32), ("n_groups", ctypes.c_int32), ("topk_groups", ctypes.c_int32),
                ("group_topn", ctypes.c_int32), ("renorm", ctypes.c_int32), ("route_scale", ctypes.c_float),
                ("in_dtype", ctypes.c_int32), ("bias_mode", ctypes.c_int32), ("gate_max_ctas", ctypes.c_int32)]


class Stats(ctypes.Structure):
    _fields_ = [("status", ctypes.c_int32), ("n_slots", ctypes.c_int32), ("total", ctypes.c_int64),
                ("max_load", ctypes.c_int64), ("mean", ctypes.c_double), ("imbalance", ctypes.c_double),
                ("std_over_mean", ctypes.c_double), ("entropy_load_bits", ctypes.c_double),
                ("entropy_score_bits", ctypes.c_double), ("capacity_fixed", ctypes.c_double),
                ("capacity_125", ctypes.c_double)]


STATS_BYTES = ctypes.sizeof(Stats)

_P, _I32, _I64, _F32, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
_lib.moe_workspace_bytes.argtypes = [_I64, _I32, _I32, _I32]
_lib.moe_workspace_bytes.restype = _SZ
_lib.moe_route.argtypes = [ctypes.POINTER(RouteCfg), _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
_lib.moe_load_stats.argtypes = [_P, _I64, _I32, _I32, _P, _I32, _P, _P, _P, _P, _P, _I32, _P, _P, _SZ, _P]
_lib.moe_replica_plan.argtypes = [_P, _I32, _I32, _P, _P]
_lib.moe_bias_update.argtypes = [_P, _I32, _I64, _F32, _I32, _P, _P]
_lib.moe_dispatch.argtypes = [_P, _I32, _I64, _I32, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _P]
_lib.moe_combine.argtypes = [_P, _I32, _I64, _I32, _I32, _P, _P, _P, _P]
_lib.moe_workspace_status.argtypes = [_P, _P]
_lib.moe_launch_count.argtypes = [_I32]
_lib.moe_launch_count.restype = _I64
_lib.moe_status_str.argtypes = [_I32]
_lib.moe_status_str.restype = ctypes.c_char_p
_lib.moe_version.restype = ctypes.c_char_p
for _n in ("moe_route", "moe_load_stats", "moe_replica_plan", "moe_bias_update", "moe_dispatch", "moe_combine",
           "moe_workspace_status"):
    getattr(_lib, _n).restype = _I32


class MoeError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        super().__init__(f"{call}: {_lib.moe_status_str(status).decode()} (status {status})")


def _check(status: int, call: str) -> None:
    if status != MOE_OK:
        raise MoeError(status, call)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("expected a contiguous CUDA tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return MOE_BF16
    if t.dtype == torch.float32:
        return MOE_F32
    raise ValueError(f"unsupported dtype {t.dtype}")


def moe_workspace_bytes(T: int, K: int, N: int, n_slots: Optional[int] = None) -> int:
    return int(_lib.moe_workspace_bytes(T, K, N, N if n_slots is None else n_slots))


def moe_route(cfg: RouteCfg, x, w_gate, logit_offset, bias, scores, topk_idx, topk_w, ws, stream=None):
    _check(_lib.moe_route(ctypes.byref(cfg), _ptr(x), _ptr(w_gate), _ptr(logit_offset), _ptr(bias), _ptr(scores),
                          _ptr(topk_idx), _ptr(topk_w), _ptr(ws), ws.numel() * ws.element_size() if ws is not None else 0,
                          _stream(stream)), "moe_route")


def moe_load_stats(topk_idx, T, K, N, replica_slot, n_slots, slot_idx, counts, offsets, rank, scores, score_fn,
                   stats, ws, stream=None):
    _check(_lib.moe_load_stats(_ptr(topk_idx), T, K, N, _ptr(replica_slot), n_slots, _ptr(slot_idx), _ptr(counts),
                               _ptr(offsets), _ptr(rank), _ptr(scores), score_fn, _ptr(stats), _ptr(ws),
                               ws.numel() * ws.element_size(), _stream(stream)), "moe_load_stats")


_lib.moe_load_stats_noalloc.argtypes = [_P, _I64, _I32, _I32, _P, _I32, _P, _P, _P, _P, _P, _I32, _P, _P]
_lib.moe_load_stats_noalloc.restype = _I32
NOALLOC_SCRATCH_BYTES = 4 << 20


def moe_load_stats_noalloc(topk_idx, T, K, N, replica_slot, n_slots, slot_idx, counts, offsets, rank, scores,
                           score_fn, stats, stream=None):
    """moe_load_stats with the library's fixed scratch array (for callers that cannot allocate)."""
    _check(_lib.moe_load_stats_noalloc(_ptr(topk_idx), T, K, N, _ptr(replica_slot), n_slots, _ptr(slot_idx),
                                       _ptr(counts), _ptr(offsets), _ptr(rank), _ptr(scores), score_fn,
                                       _ptr(stats), _stream(stream)), "moe_load_stats_noalloc")


_lib.moe_route_tiles.argtypes = [ctypes.POINTER(RouteCfg), _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
_lib.moe_route_tiles.restype = _I32
_lib.moe_load_stats_tiles.argtypes = [_P, _I64, _I32, _I32, _P, _P, _I32, _P, _P, _P, _P, _P, _P, _SZ, _P]
_lib.moe_load_stats_tiles.restype = _I32


def tile_counts_shape(T, N):
    """Shape of the per-tile histograms of moe_route_tiles: [ceil(T/128), 2, N]."""
    return ((T + 127) // 128, 2, N)


def moe_route_tiles(cfg, x, w_gate, logit_offset, bias, topk_idx, topk_w, tile_counts, ws, stream=None):
    _check(_lib.moe_route_tiles(ctypes.byref(cfg), _ptr(x), _ptr(w_gate), _ptr(logit_offset), _ptr(bias),
                                _ptr(topk_idx), _ptr(topk_w), _ptr(tile_counts), _ptr(ws),
                                ws.numel() * ws.element_size(), _stream(stream)), "moe_route_tiles")


def moe_load_stats_tiles(topk_idx, T, K, N, tile_counts, replica_slot, n_slots, slot_idx, counts, offsets, rank,
                         stats, ws, stream=None):
    _check(_lib.moe_load_stats_tiles(_ptr(topk_idx), T, K, N, _ptr(tile_counts), _ptr(replica_slot), n_slots,
                                     _ptr(slot_idx), _ptr(counts), _ptr(offsets), _ptr(rank), _ptr(stats), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream)), "moe_load_stats_tiles")


_lib.moe_route_balanced.argtypes = [_I64, _I32, _I32, _F32, _P, _P, _P]
_lib.moe_route_balanced.restype = _I32
_lib.moe_bias_update_ema.argtypes = [_P, _I32, _I64, _F32, _F32, _P, _P, _P]
_lib.moe_bias_update_ema.restype = _I32


_lib.moe_capacity_workspace_bytes.argtypes = [_I64, _I32, _I32]
_lib.moe_capacity_workspace_bytes.restype = ctypes.c_size_t
_lib.moe_route_capacity.argtypes = [ctypes.POINTER(RouteCfg), _P, _P, _I64, _P, _P, _P, _P, ctypes.c_size_t, _P]
_lib.moe_route_capacity.restype = _I32


_lib.moe_capacity_limit.argtypes = [_I64, _I32, _I32]
_lib.moe_capacity_limit.restype = _I64


def capacity_limit(T, K, N):
    """The library's per-expert token capacity, ceil(1.25 * T*K/N) (the
    "Production Testing" section of the entropy page); moe_route_capacity
    applies the same rule when given a negative capacity."""
    return int(_lib.moe_capacity_limit(T, K, N))


def capacity_workspace(T, K, N, device="cuda"):
    """Zero-filled workspace for moe_route_capacity (reuse it across calls)."""
    n = _lib.moe_capacity_workspace_bytes(T, K, N)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def empty_capacity_info(device="cuda"):
    return torch.zeros(4, dtype=torch.int64, device=device)


def read_capacity_info(info) -> dict:
    v = info.cpu().tolist()
    return dict(capacity=v[0], overflow=v[1], rerouted=v[2], dropped=v[3])


def moe_route_capacity(cfg, scores, bias, capacity, topk_idx, topk_w, info, ws, stream=None):
    _check(_lib.moe_route_capacity(ctypes.byref(cfg), _ptr(scores), _ptr(bias), int(capacity), _ptr(topk_idx),
                                   _ptr(topk_w), _ptr(info), _ptr(ws), ws.numel() * ws.element_size(),
                                   _stream(stream)), "moe_route_capacity")


def moe_route_balanced(T, K, N, route_scale, topk_idx, topk_w, stream=None):
    _check(_lib.moe_route_balanced(T, K, N, float(route_scale), _ptr(topk_idx), _ptr(topk_w), _stream(stream)),
           "moe_route_balanced")


def moe_bias_update_ema(counts, N, total_assignments, u, alpha, load_ema, bias, stream=None):
    _check(_lib.moe_bias_update_ema(_ptr(counts), N, total_assignments, float(u), float(alpha), _ptr(load_ema),
                                    _ptr(bias), _stream(stream)), "moe_bias_update_ema")


def moe_replica_plan(counts, N, n_replicas, replica_slot, stream=None):
    _check(_lib.moe_replica_plan(_ptr(counts), N, n_replicas, _ptr(replica_slot), _stream(stream)),
           "moe_replica_plan")


def moe_bias_update(counts, N, total_assignments, u, mode, bias, stream=None):
    _check(_lib.moe_bias_update(_ptr(counts), N, total_assignments, u, mode, _ptr(bias), _stream(stream)),
           "moe_bias_update")


def moe_dispatch(x, T, d, K, slot_idx, offsets, rank, rows, rows_fp8, scales, pos, row_src, stream=None):
    _check(_lib.moe_dispatch(_ptr(x), _dtype_code(x), T, d, K, _ptr(slot_idx), _ptr(offsets), _ptr(rank),
                             _ptr(rows), _ptr(rows_fp8), _ptr(scales), _ptr(pos), _ptr(row_src), _stream(stream)),
           "moe_dispatch")


def moe_combine(y, T, d, K, pos, w, out, stream=None):
    _check(_lib.moe_combine(_ptr(y), _dtype_code(y), T, d, K, _ptr(pos), _ptr(w), _ptr(out), _stream(stream)),
           "moe_combine")


_lib.moe_selftest_wait_timeout.argtypes = [_P, _SZ, _P]
_lib.moe_selftest_wait_timeout.restype = _I32


def moe_selftest_wait_timeout(ws, stream=None) -> int:
    return int(_lib.moe_selftest_wait_timeout(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def moe_workspace_status(ws, stream=None) -> int:
    return int(_lib.moe_workspace_status(_ptr(ws), _stream(stream)))


def moe_launch_count(reset: bool = False) -> int:
    return int(_lib.moe_launch_count(1 if reset else 0))


def moe_version() -> str:
    return _lib.moe_version().decode()


# --------------------------------------------------------------------------------------
# small conveniences (allocation of caller-owned buffers, decoding the stats struct)
# --------------------------------------------------------------------------------------
def route_cfg(T, d, N, K, score_fn, n_groups=1, topk_groups=1, group_topn=2, renorm=True, route_scale=1.0,
              in_dtype=MOE_BF16, bias_in_logits=False, gate_max_ctas=0) -> RouteCfg:
    return RouteCfg(T, d, N, K, score_fn, n_groups, topk_groups, group_topn, 1 if renorm else 0,
                    float(route_scale), in_dtype, 1 if bias_in_logits else 0, int(gate_max_ctas))


def empty_stats(device="cuda") -> torch.Tensor:
    return torch.zeros(STATS_BYTES, dtype=torch.uint8, device=device)


def read_stats(stats: torch.Tensor) -> dict:
    raw = bytes(stats.cpu().numpy().tobytes())
    s = Stats.from_buffer_copy(raw)
    return {name: getattr(s, name) for name, _ in Stats._fields_}


def workspace(T, K, N, n_slots=None, device="cuda") -> torch.Tensor:
    return torch.zeros(moe_workspace_bytes(T, K, N, n_slots), dtype=torch.uint8, device=device)
