"""ctypes binding of libmoe (include/moe.h): argument marshalling only.

Each function has the C entry point's name and takes torch tensors (device
memory) in place of pointers. Every step of the layer runs in libmoe's CUDA
kernels; this module computes nothing. If libmoe.so has not been built the
import fails loudly: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_TIMEOUT = range(6)
MOE_F32, MOE_BF16 = 0, 1

# Every symbol include/moe.h declares.
EXPORTED = (
    "moe_workspace_size", "moe_router_topk", "moe_topk_from_logits", "moe_topk_from_logits_noisy",
    "moe_dispatch", "moe_layer_forward_noisy",
    "moe_grouped_ffn", "moe_combine", "moe_layer_forward", "moe_layer_forward_profiled",
    "moe_expert_stats", "moe_bias_update",
    "moe_check_status", "moe_status_string", "moe_kernel_launch_count", "moe_dispatch_noalloc",
    "moe_expert_gemms", "moe_gather_rows", "moe_ep_local_order",
)


class MoELayerDesc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("T", "H", "E", "K", "D", "Ds", "dtype", "cf_num", "cf_den")]


class MoELayerWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("w_router", "w1", "w2", "ws1", "ws2", "expert_bias")]


class MoERouting(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("topk_idx", "topk_w", "counts", "offsets", "perm", "inv", "logits")]


class MoEStats(ctypes.Structure):
    _fields_ = [("num_copies", ctypes.c_int64), ("overflow", ctypes.c_int64),
                ("capacity", ctypes.c_int32), ("max_load", ctypes.c_int32),
                ("min_load", ctypes.c_int32), ("num_stragglers", ctypes.c_int32),
                ("skew_ratio", ctypes.c_double), ("gini", ctypes.c_double),
                ("overflow_rate", ctypes.c_double), ("max_over_mean", ctypes.c_double)]

    def as_dict(self):
        return {n: getattr(self, n) for n, _ in self._fields_}


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libmoe.so is not built ({LIB_PATH}); run `python -m fine_grained_moe_router_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, S = ctypes.c_void_p, ctypes.c_size_t
    D = ctypes.POINTER(MoELayerDesc)
    sig = {
        "moe_workspace_size": (S, [D]),
        "moe_router_topk": (ctypes.c_int, [D, P, P, P, P, P, P, P, S, P]),
        "moe_topk_from_logits": (ctypes.c_int, [D, P, P, P, P, P]),
        "moe_topk_from_logits_noisy": (ctypes.c_int, [D, P, P, P, P, P, P]),
        "moe_layer_forward_noisy": (ctypes.c_int, [D, ctypes.POINTER(MoELayerWeights), P, P, P,
                                                   ctypes.POINTER(MoERouting), P, S, P]),
        "moe_dispatch": (ctypes.c_int, [D, P, P, P, P, P, P, S, P]),
        "moe_grouped_ffn": (ctypes.c_int, [D, P, P, P, P, P, P, P, P, P, P, S, P]),
        "moe_combine": (ctypes.c_int, [D, P, P, P, P, P, P]),
        "moe_layer_forward": (ctypes.c_int, [D, ctypes.POINTER(MoELayerWeights), P, P,
                                             ctypes.POINTER(MoERouting), P, S, P]),
        "moe_layer_forward_profiled": (ctypes.c_int, [D, ctypes.POINTER(MoELayerWeights), P, P,
                                                      ctypes.POINTER(MoERouting), P, S, P,
                                                      ctypes.POINTER(ctypes.c_void_p), ctypes.c_int]),
        "moe_expert_stats": (ctypes.c_int, [D, P, P, ctypes.POINTER(MoEStats), P, S, P]),
        "moe_bias_update": (ctypes.c_int, [D, P, P, ctypes.c_float, P]),
        "moe_check_status": (ctypes.c_int, [P, S, P]),
        "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "moe_kernel_launch_count": (ctypes.c_uint64, []),
        "moe_dispatch_noalloc": (ctypes.c_int, [D, P, P, P, P, P, P]),
        "moe_expert_gemms": (ctypes.c_int, [D, ctypes.POINTER(MoELayerWeights), P, P, S, P]),
        "moe_gather_rows": (ctypes.c_int, [P, ctypes.c_int64, P, ctypes.c_int32, ctypes.c_int64,
                                           ctypes.c_int64, P, P]),
        "moe_ep_local_order": (ctypes.c_int, [P, ctypes.c_int32, ctypes.c_int32, P, P, P,
                                              ctypes.c_int64, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


lib = _load()


def status_string(status: int) -> str:
    return lib.moe_status_string(int(status)).decode()


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoEError(status, where)


def make_desc(T: int, H: int, E: int, K: int, D: int, Ds: int = 0, dtype: int = MOE_BF16,
              cf: tuple = (5, 4)) -> MoELayerDesc:
    return MoELayerDesc(T, H, E, K, D, Ds, dtype, cf[0], cf[1])


def dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return MOE_BF16
    if dt == torch.float32:
        return MOE_F32
    raise ValueError(f"unsupported layer dtype {dt}")


def moe_workspace_size(desc: MoELayerDesc) -> int:
    return int(lib.moe_workspace_size(ctypes.byref(desc)))


def alloc_workspace(desc: MoELayerDesc, device="cuda") -> torch.Tensor:
    """A zero-filled workspace of moe_workspace_size(desc) bytes."""
    n = moe_workspace_size(desc)
    if n == 0:
        raise MoEError(MOE_ERR_INVALID_ARG, "moe_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def moe_router_topk(desc, x, w_router, bias, logits, topk_idx, topk_w, ws, stream=None):
    _check(lib.moe_router_topk(ctypes.byref(desc), _p(x), _p(w_router), _p(bias), _p(logits),
                               _p(topk_idx), _p(topk_w), _p(ws), ws.numel() if ws is not None else 0,
                               _stream(stream)), "moe_router_topk")


def moe_topk_from_logits(desc, logits, bias, topk_idx, topk_w, stream=None):
    _check(lib.moe_topk_from_logits(ctypes.byref(desc), _p(logits), _p(bias), _p(topk_idx),
                                    _p(topk_w), _stream(stream)), "moe_topk_from_logits")


def moe_topk_from_logits_noisy(desc, logits, bias, gumbel_noise, topk_idx, topk_w, stream=None):
    """Selection on (logits + bias) + gumbel_noise [T, E] fp32 (noisy routing)."""
    _check(lib.moe_topk_from_logits_noisy(ctypes.byref(desc), _p(logits), _p(bias),
                                          _p(gumbel_noise), _p(topk_idx), _p(topk_w),
                                          _stream(stream)), "moe_topk_from_logits_noisy")


def moe_dispatch(desc, topk_idx, counts, offsets, perm, inv, ws, stream=None):
    _check(lib.moe_dispatch(ctypes.byref(desc), _p(topk_idx), _p(counts), _p(offsets), _p(perm),
                            _p(inv), _p(ws), ws.numel() if ws is not None else 0, _stream(stream)),
           "moe_dispatch")


def moe_dispatch_noalloc(desc, topk_idx, counts, offsets, perm, inv, stream=None):
    """moe_dispatch without a workspace, for callers that cannot allocate device
    memory: its scratch is a fixed array inside libmoe (T*K <= 65536). Calls that
    overlap on the GPU share that array and race."""
    _check(lib.moe_dispatch_noalloc(ctypes.byref(desc), _p(topk_idx), _p(counts), _p(offsets),
                                    _p(perm), _p(inv), _stream(stream)), "moe_dispatch_noalloc")


def moe_grouped_ffn(desc, x, perm, offsets, w1, w2, ws1, ws2, y_rows, y_shared, ws, stream=None):
    _check(lib.moe_grouped_ffn(ctypes.byref(desc), _p(x), _p(perm), _p(offsets), _p(w1), _p(w2),
                               _p(ws1), _p(ws2), _p(y_rows), _p(y_shared), _p(ws),
                               ws.numel() if ws is not None else 0, _stream(stream)),
           "moe_grouped_ffn")


def moe_combine(desc, y_rows, topk_w, inv, y_shared, y, stream=None):
    _check(lib.moe_combine(ctypes.byref(desc), _p(y_rows), _p(topk_w), _p(inv), _p(y_shared),
                           _p(y), _stream(stream)), "moe_combine")


def make_weights(w_router, w1, w2, ws1=None, ws2=None, bias=None) -> MoELayerWeights:
    return MoELayerWeights(*(t.data_ptr() if t is not None else None
                             for t in (w_router, w1, w2, ws1, ws2, bias)))


def make_routing(topk_idx=None, topk_w=None, counts=None, offsets=None, perm=None, inv=None,
                 logits=None) -> MoERouting:
    return MoERouting(*(t.data_ptr() if t is not None else None
                        for t in (topk_idx, topk_w, counts, offsets, perm, inv, logits)))


def moe_layer_forward(desc, weights: MoELayerWeights, x, y, routing: Optional[MoERouting], ws,
                      stream=None):
    _check(lib.moe_layer_forward(ctypes.byref(desc), ctypes.byref(weights), _p(x), _p(y),
                                 ctypes.byref(routing) if routing is not None else None, _p(ws),
                                 ws.numel() if ws is not None else 0, _stream(stream)),
           "moe_layer_forward")


def moe_layer_forward_noisy(desc, weights: MoELayerWeights, x, gumbel_noise, y,
                            routing: Optional[MoERouting], ws, stream=None):
    """moe_layer_forward with Gumbel noise [T, E] fp32 added to the selection scores."""
    _check(lib.moe_layer_forward_noisy(ctypes.byref(desc), ctypes.byref(weights), _p(x),
                                       _p(gumbel_noise), _p(y),
                                       ctypes.byref(routing) if routing is not None else None,
                                       _p(ws), ws.numel() if ws is not None else 0,
                                       _stream(stream)), "moe_layer_forward_noisy")


FORWARD_STAGES = ("router", "dispatch", "gemm1", "gemm2", "combine")


def moe_layer_forward_profiled(desc, weights: MoELayerWeights, x, y, routing: Optional[MoERouting],
                               ws, events, stream=None):
    """moe_layer_forward recording torch.cuda.Event objects (6, timing-enabled)
    between its stages on the launching stream."""
    for e in events:                 # torch creates the CUDA event on its first record
        if not e.cuda_event:
            e.record()
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    _check(lib.moe_layer_forward_profiled(ctypes.byref(desc), ctypes.byref(weights), _p(x), _p(y),
                                          ctypes.byref(routing) if routing is not None else None,
                                          _p(ws), ws.numel() if ws is not None else 0,
                                          _stream(stream), arr, len(events)),
           "moe_layer_forward_profiled")


def moe_expert_gemms(desc, weights: MoELayerWeights, x, ws, stream=None) -> None:
    """The expert-GEMM launches of the last moe_layer_forward on `ws` again (timing)."""
    _check(lib.moe_expert_gemms(ctypes.byref(desc), ctypes.byref(weights), _p(x), _p(ws),
                                ws.numel() if ws is not None else 0, _stream(stream)),
           "moe_expert_gemms")


def moe_gather_rows(src, idx, divisor: int, dst, stream=None) -> None:
    """dst[r] = src[idx[r] // divisor] for every row of dst (row-major 2-D tensors)."""
    row_bytes = dst[0].numel() * dst.element_size() if dst.shape[0] else 16
    _check(lib.moe_gather_rows(_p(src), src.shape[0], _p(idx), int(divisor), dst.shape[0],
                               row_bytes, _p(dst), _stream(stream)), "moe_gather_rows")


def moe_ep_local_order(recv_counts, offsets, perm, inv, stream=None) -> None:
    """Expert-major order of the rows received from G ranks (recv_counts [G, El] int32)."""
    G, El = recv_counts.shape
    _check(lib.moe_ep_local_order(_p(recv_counts), G, El, _p(offsets),
                                  _p(perm) if perm.numel() else None,
                                  _p(inv) if inv.numel() else None, perm.numel(),
                                  _stream(stream)), "moe_ep_local_order")


def moe_expert_stats(desc, counts, straggler_mask, ws, stream=None) -> dict:
    out = MoEStats()
    _check(lib.moe_expert_stats(ctypes.byref(desc), _p(counts), _p(straggler_mask),
                                ctypes.byref(out), _p(ws), ws.numel() if ws is not None else 0,
                                _stream(stream)), "moe_expert_stats")
    return out.as_dict()


def moe_bias_update(desc, counts, bias, gamma: float, stream=None) -> None:
    """Updates `bias` [E] fp32 in place from the accumulated `counts` [E] int32."""
    _check(lib.moe_bias_update(ctypes.byref(desc), _p(counts), _p(bias), ctypes.c_float(gamma),
                               _stream(stream)), "moe_bias_update")


def moe_kernel_launch_count() -> int:
    return int(lib.moe_kernel_launch_count())


def moe_check_status(ws, stream=None) -> int:
    return int(lib.moe_check_status(_p(ws), ws.numel(), _stream(stream)))
