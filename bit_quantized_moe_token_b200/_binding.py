"""ctypes binding of libmoe_w4a8.so — argument marshalling only.

Every function has the name of the C entry point it calls.  Tensors are torch CUDA tensors;
their data pointers go straight to the library, which runs every step on the GPU.  There is
no CPU or PyTorch fallback: if the library cannot be loaded, the import fails.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

from . import build as _build

MOE_OK = 0
STATUS = {0: "MOE_OK", -1: "MOE_ERR_INVALID_ARG", -2: "MOE_ERR_UNSUPPORTED_SHAPE",
          -3: "MOE_ERR_MISALIGNED", -4: "MOE_ERR_WORKSPACE", -5: "MOE_ERR_CUDA",
          -6: "MOE_ERR_TIMEOUT", -7: "MOE_ERR_NO_DEVICE"}


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({moe_status_string(status)})")


class _CLayer(ctypes.Structure):
    _fields_ = [("E", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int),
                ("group", ctypes.c_int),
                ("gate_packed", ctypes.c_void_p), ("up_packed", ctypes.c_void_p),
                ("down_packed", ctypes.c_void_p),
                ("gate_scales", ctypes.c_void_p), ("up_scales", ctypes.c_void_p),
                ("down_scales", ctypes.c_void_p),
                ("n_shared", ctypes.c_int), ("shared_N", ctypes.c_int),
                ("sh_gate", ctypes.c_void_p), ("sh_up", ctypes.c_void_p),
                ("sh_down", ctypes.c_void_p)]


class _CLayer8(ctypes.Structure):
    _fields_ = [("E", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int),
                ("gate_w8", ctypes.c_void_p), ("up_w8", ctypes.c_void_p),
                ("down_w8", ctypes.c_void_p),
                ("gate_rs", ctypes.c_void_p), ("up_rs", ctypes.c_void_p),
                ("down_rs", ctypes.c_void_p),
                ("n_shared", ctypes.c_int), ("shared_N", ctypes.c_int),
                ("sh_gate", ctypes.c_void_p), ("sh_up", ctypes.c_void_p),
                ("sh_down", ctypes.c_void_p)]


class _CLayer4(ctypes.Structure):
    _fields_ = [("E", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int),
                ("gate_f4", ctypes.c_void_p), ("up_f4", ctypes.c_void_p), ("down_f4", ctypes.c_void_p),
                ("gate_bs", ctypes.c_void_p), ("up_bs", ctypes.c_void_p), ("down_bs", ctypes.c_void_p),
                ("gate_s2", ctypes.c_void_p), ("up_s2", ctypes.c_void_p), ("down_s2", ctypes.c_void_p),
                ("n_shared", ctypes.c_int), ("shared_N", ctypes.c_int),
                ("sh_gate", ctypes.c_void_p), ("sh_up", ctypes.c_void_p),
                ("sh_down", ctypes.c_void_p)]


class _CLayerH(ctypes.Structure):
    _fields_ = [("E", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int),
                ("n_hot", ctypes.c_int), ("n_cold", ctypes.c_int),
                ("hot_ids", ctypes.c_void_p), ("cold_ids", ctypes.c_void_p),
                ("hot_gate_f4", ctypes.c_void_p), ("hot_up_f4", ctypes.c_void_p), ("hot_down_f4", ctypes.c_void_p),
                ("hot_gate_bs", ctypes.c_void_p), ("hot_up_bs", ctypes.c_void_p), ("hot_down_bs", ctypes.c_void_p),
                ("hot_gate_s2", ctypes.c_void_p), ("hot_up_s2", ctypes.c_void_p), ("hot_down_s2", ctypes.c_void_p),
                ("cold_gate_packed", ctypes.c_void_p), ("cold_up_packed", ctypes.c_void_p),
                ("cold_down_packed", ctypes.c_void_p),
                ("cold_gate_scales", ctypes.c_void_p), ("cold_up_scales", ctypes.c_void_p),
                ("cold_down_scales", ctypes.c_void_p),
                ("n_shared", ctypes.c_int), ("shared_N", ctypes.c_int),
                ("sh_gate", ctypes.c_void_p), ("sh_up", ctypes.c_void_p),
                ("sh_down", ctypes.c_void_p)]


class _CLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in
                ("topk_ids", "topk_w", "expert_offsets", "sorted_pairs", "row_of_pair",
                 "xq", "s_x", "hq", "s_h", "total", "act_order")]


_lib = None


def lib() -> ctypes.CDLL:
    """Load (building first if the sources are newer) libmoe_w4a8.so."""
    global _lib
    if _lib is None:
        path = _build.LIB
        try:
            if _build.stale():
                _build.build()
        except Exception:
            if not os.path.exists(path):
                raise
        L = ctypes.CDLL(path)
        vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        L.w4a8_pack_weights.argtypes = [vp, i64, i64, i32, vp, vp, vp]
        L.fp8_quant_tokens.argtypes = [vp, i64, i64, vp, vp, vp]
        L.moe_route_workspace_bytes.argtypes = [i64, i32, i32]
        L.moe_route_workspace_bytes.restype = sz
        L.moe_route_topk.argtypes = [vp, i64, i32, i32, vp, vp, vp, vp, vp, vp, sz, vp]
        L.moe_router_logits.argtypes = [vp, vp, i64, i32, i32, vp, vp]
        L.moe_w4a8_workspace_bytes.argtypes = [ctypes.POINTER(_CLayer), i64, i32]
        L.moe_w4a8_workspace_bytes.restype = sz
        L.moe_w4a8_workspace_layout.argtypes = [ctypes.POINTER(_CLayer), i64, i32,
                                                ctypes.POINTER(_CLayout)]
        L.moe_w4a8_forward.argtypes = [ctypes.POINTER(_CLayer), vp, vp, i64, i32, vp, vp, sz, vp]
        L.moe_w4a8_forward_profiled.argtypes = [ctypes.POINTER(_CLayer), vp, vp, i64, i32, vp, vp,
                                                sz, vp, vp, i32, ctypes.POINTER(ctypes.c_int)]
        L.w8a8_quant_weights.argtypes = [vp, i64, i64, vp, vp, vp]
        L.moe_w8a8_workspace_bytes.argtypes = [ctypes.POINTER(_CLayer8), i64, i32]
        L.moe_w8a8_workspace_bytes.restype = sz
        L.moe_w8a8_workspace_layout.argtypes = [ctypes.POINTER(_CLayer8), i64, i32,
                                                ctypes.POINTER(_CLayout)]
        L.moe_w8a8_forward.argtypes = [ctypes.POINTER(_CLayer8), vp, vp, i64, i32, vp, vp, sz, vp]
        L.moe_w8a8_forward_profiled.argtypes = [ctypes.POINTER(_CLayer8), vp, vp, i64, i32, vp, vp,
                                                sz, vp, vp, i32, vp]
        L.nvfp4_quant_weights.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp]
        L.moe_nvfp4_workspace_bytes.argtypes = [ctypes.POINTER(_CLayer4), i64, i32]
        L.moe_nvfp4_workspace_bytes.restype = sz
        L.moe_nvfp4_workspace_layout.argtypes = [ctypes.POINTER(_CLayer4), i64, i32,
                                                 ctypes.POINTER(_CLayout)]
        L.moe_nvfp4_forward.argtypes = [ctypes.POINTER(_CLayer4), vp, vp, i64, i32, vp, vp, sz, vp]
        L.moe_nvfp4_forward_profiled.argtypes = [ctypes.POINTER(_CLayer4), vp, vp, i64, i32, vp, vp,
                                                 sz, vp, vp, i32, vp]
        L.moe_hybrid_workspace_bytes.argtypes = [ctypes.POINTER(_CLayerH), i64, i32]
        L.moe_hybrid_workspace_bytes.restype = sz
        L.moe_hybrid_workspace_layout.argtypes = [ctypes.POINTER(_CLayerH), i64, i32,
                                                  ctypes.POINTER(_CLayout)]
        L.moe_hybrid_forward.argtypes = [ctypes.POINTER(_CLayerH), vp, vp, i64, i32, vp, vp, sz, vp]
        L.moe_hybrid_forward_profiled.argtypes = [ctypes.POINTER(_CLayerH), vp, vp, i64, i32, vp, vp,
                                                  sz, vp, vp, i32, vp]
        L.moe_router_topk_workspace_bytes.argtypes = [i64, i32, i32]
        L.moe_router_topk_workspace_bytes.restype = sz
        L.moe_router_topk.argtypes = [vp, vp, i64, i32, i32, i32, vp, vp, vp, vp, sz, vp]
        L.moe_w4a8_forward_router.argtypes = [ctypes.POINTER(_CLayer), vp, vp, i64, i32, vp, vp, sz, vp]
        L.moe_w8a8_forward_router.argtypes = [ctypes.POINTER(_CLayer8), vp, vp, i64, i32, vp, vp, sz, vp]
        L.moe_nvfp4_forward_router.argtypes = [ctypes.POINTER(_CLayer4), vp, vp, i64, i32, vp, vp, sz, vp]
        L.moe_ep_dispatch_workspace_bytes.argtypes = [ctypes.POINTER(_CLayer), i64, i32]
        L.moe_ep_dispatch_workspace_bytes.restype = sz
        L.moe_ep_dispatch.argtypes = [ctypes.POINTER(_CLayer), vp, vp, i64, i32, i32, vp, vp, vp, sz, vp]
        L.moe_ep_experts_workspace_bytes.argtypes = [ctypes.POINTER(_CLayer), i64]
        L.moe_ep_experts_workspace_bytes.restype = sz
        L.moe_ep_experts_forward.argtypes = [ctypes.POINTER(_CLayer), vp, i64, vp, vp, sz, vp]
        L.moe_ep_combine.argtypes = [ctypes.POINTER(_CLayer), vp, vp, i64, i32, vp, vp, sz, vp]
        L.moe_last_device_status.argtypes = [vp]
        L.moe_selftest_bounded_wait.argtypes = [i64, vp]
        L.moe_status_string.argtypes = [i32]
        L.moe_status_string.restype = ctypes.c_char_p
        for f in (L.w4a8_pack_weights, L.fp8_quant_tokens, L.moe_route_topk, L.moe_router_logits,
                  L.moe_w4a8_workspace_layout, L.moe_w4a8_forward, L.moe_w4a8_forward_profiled,
                  L.moe_last_device_status, L.moe_selftest_bounded_wait, L.moe_ep_dispatch,
                  L.moe_ep_experts_forward, L.moe_ep_combine):
            f.restype = i32
        _lib = L
    return _lib


def moe_status_string(status: int) -> str:
    return lib().moe_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != MOE_OK:
        raise MoeError(status, where)


def _ptr(t) -> Optional[ctypes.c_void_p]:
    """Device pointer of a torch tensor (or pass an int / None through)."""
    if t is None:
        return None
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


# ----------------------------------------------------------------------------------------------
# entry points
# ----------------------------------------------------------------------------------------------

def w4a8_pack_weights(w, packed, scales, group: int = 128, stream=None) -> None:
    """w bf16 [rows, K] -> packed int32 [rows, K/8], scales bf16 [rows, K/group]."""
    rows, K = w.shape[-2] if w.dim() > 1 else 1, w.shape[-1]
    rows = w.numel() // K
    _check(lib().w4a8_pack_weights(_ptr(w), rows, K, group, _ptr(packed), _ptr(scales),
                                   _stream(stream)), "w4a8_pack_weights")


def fp8_quant_tokens(x, q, scale, stream=None) -> None:
    """x bf16 [T, H] -> q uint8 (E4M3 codes) [T, H], scale fp32 [T]."""
    T, H = x.shape
    _check(lib().fp8_quant_tokens(_ptr(x), T, H, _ptr(q), _ptr(scale), _stream(stream)),
           "fp8_quant_tokens")


def moe_router_logits(x, wr, logits, stream=None) -> None:
    """x bf16 [T, H], router weight wr bf16 [E, H] -> logits fp32 [T, E]."""
    T, H = x.shape
    E = wr.shape[0]
    _check(lib().moe_router_logits(_ptr(x), _ptr(wr), T, H, E, _ptr(logits), _stream(stream)),
           "moe_router_logits")


def moe_router_topk_workspace_bytes(T: int, E: int, k: int) -> int:
    return int(lib().moe_router_topk_workspace_bytes(T, E, k))


def moe_router_topk(x, wr, k: int, logits, topk_ids, topk_w, ws, stream=None) -> None:
    """x bf16 [T, H], router weight wr bf16 [E, H] -> logits fp32 [T, E], top-k ids int32 [T, k]
    and gates fp32 [T, k] (router and top-k fused)."""
    T, H = x.shape
    E = wr.shape[0]
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib().moe_router_topk(_ptr(x), _ptr(wr), T, H, E, k, _ptr(logits), _ptr(topk_ids),
                                 _ptr(topk_w), _ptr(ws), nbytes, _stream(stream)), "moe_router_topk")


def moe_route_workspace_bytes(T: int, E: int, k: int) -> int:
    return int(lib().moe_route_workspace_bytes(T, E, k))


def moe_route_topk(logits, k: int, topk_ids, topk_w, expert_offsets, sorted_pairs, row_of_pair,
                   ws, stream=None) -> None:
    T, E = logits.shape
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib().moe_route_topk(_ptr(logits), T, E, k, _ptr(topk_ids), _ptr(topk_w),
                                _ptr(expert_offsets), _ptr(sorted_pairs), _ptr(row_of_pair),
                                _ptr(ws), nbytes, _stream(stream)), "moe_route_topk")


@dataclass
class Layer:
    """Device tensors of one layer (see moe_w4a8_layer in include/moe_w4a8.h)."""
    E: int
    H: int
    N: int
    gate_packed: object
    up_packed: object
    down_packed: object
    gate_scales: object
    up_scales: object
    down_scales: object
    group: int = 128
    sh_gate: object = None
    sh_up: object = None
    sh_down: object = None

    @property
    def n_shared(self) -> int:
        return 0 if self.sh_gate is None else int(self.sh_gate.shape[0])

    @property
    def shared_N(self) -> int:
        return 0 if self.sh_gate is None else int(self.sh_gate.shape[1])

    def c_struct(self) -> _CLayer:
        return _CLayer(self.E, self.H, self.N, self.group,
                       _ptr(self.gate_packed), _ptr(self.up_packed), _ptr(self.down_packed),
                       _ptr(self.gate_scales), _ptr(self.up_scales), _ptr(self.down_scales),
                       self.n_shared, self.shared_N,
                       _ptr(self.sh_gate), _ptr(self.sh_up), _ptr(self.sh_down))

    def shape_struct(self) -> _CLayer:
        """The same struct with null pointers: enough for the size/layout queries."""
        return _CLayer(self.E, self.H, self.N, self.group, None, None, None, None, None, None,
                       self.n_shared, self.shared_N, None, None, None)


def layer_struct(E, H, N, group=128, n_shared=0, shared_N=0) -> _CLayer:
    return _CLayer(E, H, N, group, None, None, None, None, None, None, n_shared, shared_N,
                   None, None, None)


def moe_w4a8_workspace_bytes(layer, T: int, k: int) -> int:
    s = layer if isinstance(layer, _CLayer) else layer.shape_struct()
    return int(lib().moe_w4a8_workspace_bytes(ctypes.byref(s), T, k))


def moe_w4a8_workspace_layout(layer, T: int, k: int) -> dict:
    s = layer if isinstance(layer, _CLayer) else layer.shape_struct()
    out = _CLayout()
    _check(lib().moe_w4a8_workspace_layout(ctypes.byref(s), T, k, ctypes.byref(out)),
           "moe_w4a8_workspace_layout")
    return {n: int(getattr(out, n)) for n, _ in _CLayout._fields_}


def moe_w4a8_forward(layer: Layer, x, logits, k: int, out, ws, stream=None) -> None:
    """out bf16 [T, H] = the routed W4A8 MoE layer (+ shared experts) applied to x."""
    T = x.shape[0]
    s = layer.c_struct()
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib().moe_w4a8_forward(ctypes.byref(s), _ptr(x), _ptr(logits), T, k, _ptr(out),
                                  _ptr(ws), nbytes, _stream(stream)), "moe_w4a8_forward")


N_STAGE_EVENTS = 8
STAGES = ("route", "quant", "shared", "gateup_gemm", "swiglu_requant", "down_gemm", "combine")


def moe_w4a8_forward_profiled(layer: Layer, x, logits, k: int, out, ws, events, stream=None) -> int:
    """moe_w4a8_forward that also records `events` (8 entries: torch.cuda.Event with timing, or
    None to skip that boundary) at the stage boundaries; returns the number of kernels launched."""
    T = x.shape[0]
    s = layer.c_struct()
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    arr = (ctypes.c_void_p * len(events))(
        *[ctypes.c_void_p(e.cuda_event if e is not None else 0) for e in events])
    n = ctypes.c_int(0)
    _check(lib().moe_w4a8_forward_profiled(ctypes.byref(s), _ptr(x), _ptr(logits), T, k, _ptr(out),
                                           _ptr(ws), nbytes, _stream(stream), arr, len(events),
                                           ctypes.byref(n)), "moe_w4a8_forward_profiled")
    return int(n.value)


# ---- expert parallelism ---------------------------------------------------------------------

def ep_record_bytes(H: int) -> int:
    """Bytes of one dispatch record (MOE_EP_RECORD_BYTES): H FP8 codes, scale, expert, padding."""
    return int(H) + 16


def _shape_or_struct(layer) -> _CLayer:
    return layer if isinstance(layer, _CLayer) else layer.c_struct()


def moe_ep_dispatch_workspace_bytes(layer, T: int, k: int) -> int:
    s = layer if isinstance(layer, _CLayer) else layer.shape_struct()
    return int(lib().moe_ep_dispatch_workspace_bytes(ctypes.byref(s), T, k))


def moe_ep_dispatch(layer, x, logits, k: int, n_ranks: int, send_counts, send_records, ws,
                    stream=None) -> None:
    """x bf16 [T, H], logits fp32 [T, E] -> send_counts int32 [n_ranks], send_records uint8
    [T*k, ep_record_bytes(H)] (owner-major); ws keeps what moe_ep_combine needs."""
    T = x.shape[0]
    s = _shape_or_struct(layer)
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib().moe_ep_dispatch(ctypes.byref(s), _ptr(x), _ptr(logits), T, k, n_ranks,
                                 _ptr(send_counts), _ptr(send_records), _ptr(ws), nbytes,
                                 _stream(stream)), "moe_ep_dispatch")


def moe_ep_experts_workspace_bytes(local_layer, R: int) -> int:
    s = local_layer if isinstance(local_layer, _CLayer) else local_layer.shape_struct()
    return int(lib().moe_ep_experts_workspace_bytes(ctypes.byref(s), R))


def moe_ep_experts_forward(local_layer: Layer, records, y_rows, ws, stream=None) -> None:
    """records uint8 [R, ep_record_bytes(H)] received for this GPU's experts -> y_rows fp32 [R, H]."""
    R = records.shape[0]
    s = local_layer.c_struct()
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib().moe_ep_experts_forward(ctypes.byref(s), _ptr(records) if R else None, R,
                                        _ptr(y_rows) if R else None, _ptr(ws), nbytes,
                                        _stream(stream)), "moe_ep_experts_forward")


def moe_ep_combine(layer, x, y_back, k: int, out, ws, stream=None) -> None:
    """y_back fp32 [T*k, H] (rows returned for this GPU's records, record order) -> out bf16 [T, H]."""
    T = x.shape[0]
    s = _shape_or_struct(layer)
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib().moe_ep_combine(ctypes.byref(s), _ptr(x), _ptr(y_back), T, k, _ptr(out), _ptr(ws),
                                nbytes, _stream(stream)), "moe_ep_combine")


def moe_last_device_status(stream=None) -> int:
    return int(lib().moe_last_device_status(_stream(stream)))


def moe_selftest_bounded_wait(limit_ns: int, stream=None) -> None:
    _check(lib().moe_selftest_bounded_wait(int(limit_ns), _stream(stream)),
           "moe_selftest_bounded_wait")


# ---- row-scaled FP8 (W8A8) experts -------------------------------------------------------------

def w8a8_quant_weights(w, q, row_scale, stream=None) -> None:
    """w bf16 [..., rows, K] -> q uint8 (E4M3 codes) [..., rows, K], row_scale fp32 [..., rows]."""
    K = w.shape[-1]
    rows = w.numel() // K
    _check(lib().w8a8_quant_weights(_ptr(w), rows, K, _ptr(q), _ptr(row_scale), _stream(stream)),
           "w8a8_quant_weights")


@dataclass
class Layer8:
    """Device tensors of one layer with row-scaled FP8 experts (moe_w8a8_layer)."""
    E: int
    H: int
    N: int
    gate_w8: object
    up_w8: object
    down_w8: object
    gate_rs: object
    up_rs: object
    down_rs: object
    sh_gate: object = None
    sh_up: object = None
    sh_down: object = None

    @property
    def n_shared(self) -> int:
        return 0 if self.sh_gate is None else int(self.sh_gate.shape[0])

    @property
    def shared_N(self) -> int:
        return 0 if self.sh_gate is None else int(self.sh_gate.shape[1])

    def c_struct(self) -> _CLayer8:
        return _CLayer8(self.E, self.H, self.N,
                        _ptr(self.gate_w8), _ptr(self.up_w8), _ptr(self.down_w8),
                        _ptr(self.gate_rs), _ptr(self.up_rs), _ptr(self.down_rs),
                        self.n_shared, self.shared_N,
                        _ptr(self.sh_gate), _ptr(self.sh_up), _ptr(self.sh_down))

    def shape_struct(self) -> _CLayer8:
        return _CLayer8(self.E, self.H, self.N, None, None, None, None, None, None,
                        self.n_shared, self.shared_N, None, None, None)


def layer8_struct(E, H, N, n_shared=0, shared_N=0) -> _CLayer8:
    return _CLayer8(E, H, N, None, None, None, None, None, None, n_shared, shared_N,
                    None, None, None)


def moe_w8a8_workspace_bytes(layer, T: int, k: int) -> int:
    s = layer if isinstance(layer, _CLayer8) else layer.shape_struct()
    return int(lib().moe_w8a8_workspace_bytes(ctypes.byref(s), T, k))


def moe_w8a8_workspace_layout(layer, T: int, k: int) -> dict:
    s = layer if isinstance(layer, _CLayer8) else layer.shape_struct()
    out = _CLayout()
    _check(lib().moe_w8a8_workspace_layout(ctypes.byref(s), T, k, ctypes.byref(out)),
           "moe_w8a8_workspace_layout")
    return {n: int(getattr(out, n)) for n, _ in _CLayout._fields_}


def moe_w8a8_forward(layer: Layer8, x, logits, k: int, out, ws, stream=None) -> None:
    """out bf16 [T, H] = the routed MoE layer with row-scaled FP8 experts applied to x."""
    T = x.shape[0]
    s = layer.c_struct()
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib().moe_w8a8_forward(ctypes.byref(s), _ptr(x), _ptr(logits), T, k, _ptr(out),
                                  _ptr(ws), nbytes, _stream(stream)), "moe_w8a8_forward")


def moe_w8a8_forward_profiled(layer: Layer8, x, logits, k: int, out, ws, events, stream=None) -> int:
    T = x.shape[0]
    s = layer.c_struct()
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    arr = (ctypes.c_void_p * len(events))(
        *[ctypes.c_void_p(e.cuda_event if e is not None else 0) for e in events])
    n = ctypes.c_int(0)
    _check(lib().moe_w8a8_forward_profiled(ctypes.byref(s), _ptr(x), _ptr(logits), T, k, _ptr(out),
                                           _ptr(ws), nbytes, _stream(stream), arr, len(events),
                                           ctypes.byref(n)), "moe_w8a8_forward_profiled")
    return int(n.value)


def moe_w4a8_forward_router(layer: Layer, x, wr, k: int, out, ws, stream=None) -> None:
    """The W4A8 layer fed by the router weight wr bf16 [E, H] (logits computed inside)."""
    T = x.shape[0]
    s = layer.c_struct()
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib().moe_w4a8_forward_router(ctypes.byref(s), _ptr(x), _ptr(wr), T, k, _ptr(out), _ptr(ws),
                                         nbytes, _stream(stream)), "moe_w4a8_forward_router")


def moe_w8a8_forward_router(layer: Layer8, x, wr, k: int, out, ws, stream=None) -> None:
    """The row-scaled FP8 layer fed by the router weight wr bf16 [E, H]."""
    T = x.shape[0]
    s = layer.c_struct()
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib().moe_w8a8_forward_router(ctypes.byref(s), _ptr(x), _ptr(wr), T, k, _ptr(out), _ptr(ws),
                                         nbytes, _stream(stream)), "moe_w8a8_forward_router")


# ---- NVFP4 experts ------------------------------------------------------------------------------

def nvfp4_quant_weights(w, codes, scales, scale2, stream=None) -> None:
    """w bf16 [experts, rows, K] -> codes uint8 [experts, rows, K/2], E4M3 block scales uint8
    [experts, rows, K/16], fp32 scale2 [experts]."""
    E, rows, K = w.shape
    _check(lib().nvfp4_quant_weights(_ptr(w), E, rows, K, _ptr(codes), _ptr(scales), _ptr(scale2),
                                     _stream(stream)), "nvfp4_quant_weights")


@dataclass
class Layer4:
    """Device tensors of one layer with NVFP4 experts (moe_nvfp4_layer)."""
    E: int
    H: int
    N: int
    gate_f4: object
    up_f4: object
    down_f4: object
    gate_bs: object
    up_bs: object
    down_bs: object
    gate_s2: object
    up_s2: object
    down_s2: object
    sh_gate: object = None
    sh_up: object = None
    sh_down: object = None

    @property
    def n_shared(self) -> int:
        return 0 if self.sh_gate is None else int(self.sh_gate.shape[0])

    @property
    def shared_N(self) -> int:
        return 0 if self.sh_gate is None else int(self.sh_gate.shape[1])

    def c_struct(self) -> _CLayer4:
        return _CLayer4(self.E, self.H, self.N, _ptr(self.gate_f4), _ptr(self.up_f4), _ptr(self.down_f4),
                        _ptr(self.gate_bs), _ptr(self.up_bs), _ptr(self.down_bs),
                        _ptr(self.gate_s2), _ptr(self.up_s2), _ptr(self.down_s2),
                        self.n_shared, self.shared_N, _ptr(self.sh_gate), _ptr(self.sh_up),
                        _ptr(self.sh_down))

    def shape_struct(self) -> _CLayer4:
        return _CLayer4(self.E, self.H, self.N, None, None, None, None, None, None, None, None, None,
                        self.n_shared, self.shared_N, None, None, None)


def layer4_struct(E, H, N, n_shared=0, shared_N=0) -> _CLayer4:
    return _CLayer4(E, H, N, None, None, None, None, None, None, None, None, None, n_shared, shared_N,
                    None, None, None)


def moe_nvfp4_workspace_bytes(layer, T: int, k: int) -> int:
    s = layer if isinstance(layer, _CLayer4) else layer.shape_struct()
    return int(lib().moe_nvfp4_workspace_bytes(ctypes.byref(s), T, k))


def moe_nvfp4_workspace_layout(layer, T: int, k: int) -> dict:
    s = layer if isinstance(layer, _CLayer4) else layer.shape_struct()
    out = _CLayout()
    _check(lib().moe_nvfp4_workspace_layout(ctypes.byref(s), T, k, ctypes.byref(out)),
           "moe_nvfp4_workspace_layout")
    return {n: int(getattr(out, n)) for n, _ in _CLayout._fields_}


def moe_nvfp4_forward(layer: Layer4, x, logits, k: int, out, ws, stream=None) -> None:
    """out bf16 [T, H] = the routed MoE layer with NVFP4 experts applied to x."""
    T = x.shape[0]
    s = layer.c_struct()
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib().moe_nvfp4_forward(ctypes.byref(s), _ptr(x), _ptr(logits), T, k, _ptr(out),
                                   _ptr(ws), nbytes, _stream(stream)), "moe_nvfp4_forward")


def moe_nvfp4_forward_profiled(layer: Layer4, x, logits, k: int, out, ws, events, stream=None) -> int:
    T = x.shape[0]
    s = layer.c_struct()
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    arr = (ctypes.c_void_p * len(events))(
        *[ctypes.c_void_p(e.cuda_event if e is not None else 0) for e in events])
    n = ctypes.c_int(0)
    _check(lib().moe_nvfp4_forward_profiled(ctypes.byref(s), _ptr(x), _ptr(logits), T, k, _ptr(out),
                                            _ptr(ws), nbytes, _stream(stream), arr, len(events),
                                            ctypes.byref(n)), "moe_nvfp4_forward_profiled")
    return int(n.value)


def moe_nvfp4_forward_router(layer: Layer4, x, wr, k: int, out, ws, stream=None) -> None:
    """The NVFP4 layer fed by the router weight wr bf16 [E, H]."""
    T = x.shape[0]
    s = layer.c_struct()
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib().moe_nvfp4_forward_router(ctypes.byref(s), _ptr(x), _ptr(wr), T, k, _ptr(out), _ptr(ws),
                                          nbytes, _stream(stream)), "moe_nvfp4_forward_router")


# ---- hybrid layers: NVFP4 hot experts, W4A8 cold experts ---------------------------------------

@dataclass
class LayerH:
    """Device tensors of a hybrid layer (moe_hybrid_layer): `hot` (a Layer4 of the hot slabs),
    `cold` (a Layer of the cold slabs), and the int32 slab -> expert lists."""
    E: int
    hot: Layer4
    cold: Layer
    hot_ids: object
    cold_ids: object

    @property
    def H(self) -> int:
        return self.cold.H

    @property
    def N(self) -> int:
        return self.cold.N

    def c_struct(self) -> _CLayerH:
        h, c = self.hot, self.cold
        return _CLayerH(self.E, c.H, c.N, int(self.hot_ids.numel()), int(self.cold_ids.numel()),
                        _ptr(self.hot_ids), _ptr(self.cold_ids),
                        _ptr(h.gate_f4), _ptr(h.up_f4), _ptr(h.down_f4), _ptr(h.gate_bs), _ptr(h.up_bs),
                        _ptr(h.down_bs), _ptr(h.gate_s2), _ptr(h.up_s2), _ptr(h.down_s2),
                        _ptr(c.gate_packed), _ptr(c.up_packed), _ptr(c.down_packed), _ptr(c.gate_scales),
                        _ptr(c.up_scales), _ptr(c.down_scales), c.n_shared, c.shared_N,
                        _ptr(c.sh_gate), _ptr(c.sh_up), _ptr(c.sh_down))

    def shape_struct(self) -> _CLayerH:
        """Shapes and slab counts, null pointers: enough for the size/layout queries."""
        c = self.cold
        return _CLayerH(self.E, c.H, c.N, int(self.hot_ids.numel()), int(self.cold_ids.numel()), None, None,
                        None, None, None, None, None, None, None, None, None, None, None, None, None, None, None,
                        c.n_shared, c.shared_N, None, None, None)


def moe_hybrid_workspace_bytes(layer, T: int, k: int) -> int:
    s = layer if isinstance(layer, _CLayerH) else layer.shape_struct()
    return int(lib().moe_hybrid_workspace_bytes(ctypes.byref(s), T, k))


def moe_hybrid_workspace_layout(layer, T: int, k: int) -> dict:
    s = layer if isinstance(layer, _CLayerH) else layer.shape_struct()
    out = _CLayout()
    _check(lib().moe_hybrid_workspace_layout(ctypes.byref(s), T, k, ctypes.byref(out)),
           "moe_hybrid_workspace_layout")
    return {n: int(getattr(out, n)) for n, _ in _CLayout._fields_}


def moe_hybrid_forward(layer: LayerH, x, logits, k: int, out, ws, stream=None) -> None:
    """out bf16 [T, H] = the routed MoE layer with NVFP4 hot and W4A8 cold experts."""
    T = x.shape[0]
    s = layer.c_struct()
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib().moe_hybrid_forward(ctypes.byref(s), _ptr(x), _ptr(logits), T, k, _ptr(out),
                                    _ptr(ws), nbytes, _stream(stream)), "moe_hybrid_forward")


def moe_hybrid_forward_profiled(layer: LayerH, x, logits, k: int, out, ws, events, stream=None) -> int:
    T = x.shape[0]
    s = layer.c_struct()
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    arr = (ctypes.c_void_p * len(events))(
        *[ctypes.c_void_p(e.cuda_event if e is not None else 0) for e in events])
    n = ctypes.c_int(0)
    _check(lib().moe_hybrid_forward_profiled(ctypes.byref(s), _ptr(x), _ptr(logits), T, k, _ptr(out),
                                             _ptr(ws), nbytes, _stream(stream), arr, len(events),
                                             ctypes.byref(n)), "moe_hybrid_forward_profiled")
    return int(n.value)
