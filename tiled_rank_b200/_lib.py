"""ctypes binding of libtileq.so (include/tileq.h).

Argument marshalling only: every step of the forward runs in the library's
CUDA kernels.  PyTorch supplies device memory and the stream.  Importing this
module fails loudly when the library has not been built; there is no CPU
fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libtileq.so")

TILEQ_OK = 0
TILEQ_ERR_INVALID_ARG = -1
TILEQ_ERR_UNSUPPORTED = -2
TILEQ_ERR_WORKSPACE = -3
TILEQ_ERR_CUDA = -4
TILEQ_ERR_TIMEOUT = -5
TILEQ_ERR_RANGE = -6
TILEQ_LINEAR = 0
TILEQ_SWIGLU = 1
TILEQ_ROUTE_TOPK_SOFTMAX = 0
TILEQ_ROUTE_FULL_SOFTMAX = 1

# every symbol include/tileq.h declares
EXPORTS = (
    "tileq_status_string", "tileq_packed_size", "tileq_pack", "tileq_workspace_size",
    "tileq_moe_forward", "tileq_packed_per_expert_size", "tileq_pack_per_expert",
    "tileq_moe_forward_unfused", "tileq_route", "tileq_route_static", "tileq_device_status",
    "tileq_selftest_bounded_wait", "tileq_set_stage_events", "tileq_launch_count",
    "tileq_sketch_workspace_size", "tileq_sketch_lowrank",
    "tileq_place_workspace_size", "tileq_place_experts",
)
TILEQ_SKETCH_MAX_L = 160
TILEQ_PLACE_MAX_R0 = 256


class TileQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


class tileq_proj(ctypes.Structure):
    _fields_ = [
        ("d_in", ctypes.c_int), ("d_out", ctypes.c_int), ("rank", ctypes.c_int),
        ("group", ctypes.c_int),
        ("grid_assign", ctypes.POINTER(ctypes.c_int32)),
        ("U", ctypes.c_void_p), ("Sigma", ctypes.c_void_p), ("V", ctypes.c_void_p),
        ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("zeros", ctypes.c_void_p),
        ("bits", ctypes.c_int), ("codes_hi", ctypes.c_void_p),
    ]


class tileq_layer(ctypes.Structure):
    _fields_ = [
        ("kind", ctypes.c_int), ("K", ctypes.c_int), ("M", ctypes.c_int), ("N", ctypes.c_int),
        ("d_model", ctypes.c_int), ("d_ff", ctypes.c_int),
        ("proj", tileq_proj * 3),
        ("shared_d_ff", ctypes.c_int),
        ("shared_w", ctypes.c_void_p * 3),
        ("route_mode", ctypes.c_int),
    ]


class tileq_route_out(ctypes.Structure):
    _fields_ = [("topk_idx", ctypes.c_void_p), ("topk_w", ctypes.c_void_p),
                ("expert_offsets", ctypes.c_void_p), ("sorted_pairs", ctypes.c_void_p)]


class tileq_wbig(ctypes.Structure):
    _fields_ = [
        ("K", ctypes.c_int), ("M", ctypes.c_int), ("N", ctypes.c_int),
        ("d_out", ctypes.c_int), ("d_in", ctypes.c_int),
        ("w", ctypes.c_void_p), ("grid_assign", ctypes.POINTER(ctypes.c_int32)),
    ]


class tileq_place_in(ctypes.Structure):
    _fields_ = [
        ("K", ctypes.c_int), ("M", ctypes.c_int), ("N", ctypes.c_int),
        ("d_u", ctypes.c_int), ("d_v", ctypes.c_int), ("r0", ctypes.c_int),
        ("u", ctypes.c_void_p), ("v", ctypes.c_void_p), ("max_iter", ctypes.c_int),
    ]


class tileq_place_out(ctypes.Structure):
    _fields_ = [("grid_assign", ctypes.c_void_p), ("ideal", ctypes.c_void_p),
                ("iterations", ctypes.c_void_p)]


class tileq_per_expert_lr(ctypes.Structure):
    _fields_ = [("U_pe", ctypes.c_void_p * 3), ("V_pe", ctypes.c_void_p * 3)]


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m tiled_rank_b200.build`")
    lib = ctypes.CDLL(path)
    c_int, c_size, vp = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
    P = ctypes.POINTER
    sigs = {
        "tileq_status_string": ([c_int], ctypes.c_char_p),
        "tileq_packed_size": ([P(tileq_layer), P(c_size)], c_int),
        "tileq_pack": ([P(tileq_layer), vp, c_size, vp], c_int),
        "tileq_workspace_size": ([P(tileq_layer), c_int, c_int, P(c_size)], c_int),
        "tileq_moe_forward": ([P(tileq_layer), vp, vp, c_int, vp, c_int, vp, vp, c_size,
                               P(tileq_route_out), vp], c_int),
        "tileq_packed_per_expert_size": ([P(tileq_layer), P(c_size)], c_int),
        "tileq_pack_per_expert": ([P(tileq_layer), P(tileq_per_expert_lr), vp, c_size, vp], c_int),
        "tileq_moe_forward_unfused": ([P(tileq_layer), vp, vp, vp, c_int, vp, c_int, vp, vp,
                                       c_size, P(tileq_route_out), vp], c_int),
        "tileq_route": ([vp, c_int, c_int, c_int, P(tileq_route_out), vp, c_size, vp], c_int),
        "tileq_route_static": ([vp, c_int, c_int, c_int, P(tileq_route_out), vp], c_int),
        "tileq_device_status": ([vp, P(c_int), vp], c_int),
        "tileq_selftest_bounded_wait": ([vp, c_size, c_int, vp], c_int),
        "tileq_set_stage_events": ([P(vp), c_int], c_int),
        "tileq_launch_count": ([P(ctypes.c_ulonglong)], c_int),
        "tileq_sketch_workspace_size": ([P(tileq_wbig), c_int, c_int, P(c_size)], c_int),
        "tileq_sketch_lowrank": ([P(tileq_wbig), vp, c_int, c_int, vp, vp, vp, vp, c_size, vp], c_int),
        "tileq_place_workspace_size": ([P(tileq_place_in), P(c_size)], c_int),
        "tileq_place_experts": ([P(tileq_place_in), P(tileq_place_out), vp, c_size, vp], c_int),
    }
    for name, (argtypes, restype) in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = argtypes
        fn.restype = restype
    return lib


_LIB: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        _LIB = load()
    return _LIB


def status_string(status: int) -> str:
    return lib().tileq_status_string(status).decode()


def _check(status: int, where: str):
    if status != TILEQ_OK:
        raise TileQError(status, where)


def _ptr(t) -> Optional[int]:
    """Device pointer of a torch tensor (None passes NULL)."""
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ---------------------------------------------------------------------------
# the ABI calls, same names as include/tileq.h
# ---------------------------------------------------------------------------
def tileq_packed_size(layer: tileq_layer) -> int:
    n = ctypes.c_size_t()
    _check(lib().tileq_packed_size(ctypes.byref(layer), ctypes.byref(n)), "tileq_packed_size")
    return n.value


def tileq_pack(layer: tileq_layer, packed, stream=None):
    _check(lib().tileq_pack(ctypes.byref(layer), _ptr(packed), packed.numel() * packed.element_size(),
                            _stream(stream)), "tileq_pack")


def tileq_workspace_size(layer: tileq_layer, T: int, top_k: int) -> int:
    n = ctypes.c_size_t()
    _check(lib().tileq_workspace_size(ctypes.byref(layer), T, top_k, ctypes.byref(n)),
           "tileq_workspace_size")
    return n.value


def _route_struct(route: Optional[dict]):
    if route is None:
        return None
    r = tileq_route_out(_ptr(route.get("topk_idx")), _ptr(route.get("topk_w")),
                        _ptr(route.get("expert_offsets")), _ptr(route.get("sorted_pairs")))
    return ctypes.byref(r)


def tileq_moe_forward(layer: tileq_layer, packed, x, T: int, router_logits, top_k: int, out, ws,
                      route: Optional[dict] = None, stream=None):
    _check(lib().tileq_moe_forward(ctypes.byref(layer), _ptr(packed), _ptr(x), T,
                                   _ptr(router_logits), top_k, _ptr(out), _ptr(ws),
                                   ws.numel() * ws.element_size(), _route_struct(route),
                                   _stream(stream)), "tileq_moe_forward")


def tileq_packed_per_expert_size(layer: tileq_layer) -> int:
    n = ctypes.c_size_t()
    _check(lib().tileq_packed_per_expert_size(ctypes.byref(layer), ctypes.byref(n)),
           "tileq_packed_per_expert_size")
    return n.value


def tileq_pack_per_expert(layer: tileq_layer, pe: tileq_per_expert_lr, packed_pe, stream=None):
    _check(lib().tileq_pack_per_expert(ctypes.byref(layer), ctypes.byref(pe), _ptr(packed_pe),
                                       packed_pe.numel() * packed_pe.element_size(),
                                       _stream(stream)), "tileq_pack_per_expert")


def tileq_moe_forward_unfused(layer: tileq_layer, packed, packed_pe, x, T: int, router_logits,
                              top_k: int, out, ws, route: Optional[dict] = None, stream=None):
    _check(lib().tileq_moe_forward_unfused(ctypes.byref(layer), _ptr(packed), _ptr(packed_pe),
                                           _ptr(x), T, _ptr(router_logits), top_k, _ptr(out),
                                           _ptr(ws), ws.numel() * ws.element_size(),
                                           _route_struct(route), _stream(stream)),
           "tileq_moe_forward_unfused")


def tileq_route(router_logits, T: int, K: int, top_k: int, route: dict, ws, stream=None):
    _check(lib().tileq_route(_ptr(router_logits), T, K, top_k, _route_struct(route), _ptr(ws),
                             ws.numel() * ws.element_size(), _stream(stream)), "tileq_route")


def tileq_route_static(router_logits, T: int, K: int, top_k: int, route: dict, stream=None):
    _check(lib().tileq_route_static(_ptr(router_logits), T, K, top_k, _route_struct(route),
                                    _stream(stream)), "tileq_route_static")


def tileq_device_status(ws, stream=None) -> int:
    s = ctypes.c_int()
    _check(lib().tileq_device_status(_ptr(ws), ctypes.byref(s), _stream(stream)),
           "tileq_device_status")
    return s.value


def tileq_selftest_bounded_wait(ws, max_polls: int, stream=None):
    _check(lib().tileq_selftest_bounded_wait(_ptr(ws), ws.numel() * ws.element_size(), max_polls,
                                             _stream(stream)), "tileq_selftest_bounded_wait")


def tileq_set_stage_events(events):
    """events: a list of torch.cuda.Event (created with enable_timing) or None to switch off."""
    if not events:
        _check(lib().tileq_set_stage_events(None, 0), "tileq_set_stage_events")
        return
    for e in events:
        if e.cuda_event == 0:  # torch creates the CUDA event on its first record
            e.record()
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    _check(lib().tileq_set_stage_events(arr, len(events)), "tileq_set_stage_events")


def tileq_launch_count() -> int:
    n = ctypes.c_ulonglong()
    _check(lib().tileq_launch_count(ctypes.byref(n)), "tileq_launch_count")
    return n.value


def tileq_sketch_workspace_size(wbig: tileq_wbig, l: int, r: int) -> int:
    n = ctypes.c_size_t()
    _check(lib().tileq_sketch_workspace_size(ctypes.byref(wbig), l, r, ctypes.byref(n)),
           "tileq_sketch_workspace_size")
    return n.value


def tileq_sketch_lowrank(wbig: tileq_wbig, omega, l: int, r: int, U, sigma, V, ws, stream=None):
    _check(lib().tileq_sketch_lowrank(ctypes.byref(wbig), _ptr(omega), l, r, _ptr(U), _ptr(sigma),
                                      _ptr(V), _ptr(ws), ws.numel() * ws.element_size(),
                                      _stream(stream)), "tileq_sketch_lowrank")


def place_in(u, v, M: int, N: int, max_iter: int = 100) -> tileq_place_in:
    """The placement input for device fp32 factors u [K, d_u, r0], v [K, d_v, r0]."""
    K, d_u, r0 = (int(x) for x in u.shape)
    if tuple(v.shape[::2]) != (K, r0):
        raise ValueError("u and v must share K and r0")
    c = tileq_place_in()
    c.K, c.M, c.N, c.d_u, c.d_v, c.r0 = K, M, N, d_u, int(v.shape[1]), r0
    c.u, c.v, c.max_iter = _ptr(u), _ptr(v), max_iter
    return c


def tileq_place_workspace_size(pin: tileq_place_in) -> int:
    n = ctypes.c_size_t()
    _check(lib().tileq_place_workspace_size(ctypes.byref(pin), ctypes.byref(n)), "tileq_place_workspace_size")
    return n.value


def tileq_place_experts(pin: tileq_place_in, grid_assign, ws, ideal=None, iterations=None, stream=None):
    out = tileq_place_out(_ptr(grid_assign), _ptr(ideal), _ptr(iterations))
    _check(lib().tileq_place_experts(ctypes.byref(pin), ctypes.byref(out), _ptr(ws),
                                     ws.numel() * ws.element_size() if ws is not None else 0,
                                     _stream(stream)), "tileq_place_experts")
