"""CPU oracle of the W4A8-FP8 routed MoE layer (plain C, fp32), with numpy wrappers.

TEST INFRASTRUCTURE ONLY: imported by tests/, ``__graft_entry__.smoke()`` and
the cpu_baseline / reference leg of ``bench.py``.  The CUDA library never
imports, links or calls it, and it shares no code with the CUDA library.

Every function cites, in ``oracle.c``, the page passage it follows.  Parity of
the fp32 accumulation order inside the GPU's tensor-core sums (and of expf's
last ulp) is not pinned by any page: those differences are covered only by
the layer's stated tolerances (see tests/).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_SRC = os.path.join(_HERE, "oracle.c")


def build(verbose: bool = False) -> None:
    if os.path.exists(_SO) and os.path.getmtime(_SO) >= os.path.getmtime(_SRC):
        return
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", _SRC, "-o", _SO, "-lm"]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)


class _Layer(ctypes.Structure):
    _fields_ = [("E", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int),
                ("group", ctypes.c_int),
                ("gate_packed", ctypes.c_void_p), ("up_packed", ctypes.c_void_p),
                ("down_packed", ctypes.c_void_p),
                ("gate_scales", ctypes.c_void_p), ("up_scales", ctypes.c_void_p),
                ("down_scales", ctypes.c_void_p),
                ("n_shared", ctypes.c_int), ("shared_N", ctypes.c_int),
                ("sh_gate", ctypes.c_void_p), ("sh_up", ctypes.c_void_p),
                ("sh_down", ctypes.c_void_p),
                ("fmt", ctypes.c_int),
                ("gate_w8", ctypes.c_void_p), ("up_w8", ctypes.c_void_p),
                ("down_w8", ctypes.c_void_p),
                ("gate_rs", ctypes.c_void_p), ("up_rs", ctypes.c_void_p),
                ("down_rs", ctypes.c_void_p),
                ("gate_f4", ctypes.c_void_p), ("up_f4", ctypes.c_void_p),
                ("down_f4", ctypes.c_void_p),
                ("gate_bs", ctypes.c_void_p), ("up_bs", ctypes.c_void_p),
                ("down_bs", ctypes.c_void_p),
                ("gate_s2", ctypes.c_void_p), ("up_s2", ctypes.c_void_p),
                ("down_s2", ctypes.c_void_p),
                ("hot_ids", ctypes.c_void_p), ("cold_ids", ctypes.c_void_p),
                ("n_hot", ctypes.c_int), ("n_cold", ctypes.c_int)]

FMT_W4A8 = 0
FMT_W8A8 = 1
FMT_NVFP4 = 2
FMT_HYBRID = 3


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        L.or_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.or_bf16_to_f32.restype = ctypes.c_float
        L.or_f32_to_bf16.argtypes = [ctypes.c_float]
        L.or_f32_to_bf16.restype = ctypes.c_uint16
        L.or_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.or_e4m3_decode.restype = ctypes.c_float
        L.or_e4m3_encode.argtypes = [ctypes.c_float]
        L.or_e4m3_encode.restype = ctypes.c_uint8
        L.or_rtn_pack.argtypes = [vp, i64, i64, i32, vp, vp, vp]
        L.or_rtn_pack.restype = i32
        L.or_unpack.argtypes = [vp, i64, i64, vp]
        L.or_unpack.restype = None
        L.or_quant_tokens.argtypes = [vp, i64, i64, vp, vp]
        L.or_quant_tokens.restype = None
        L.or_quant_rows.argtypes = [vp, i64, i64, vp, vp]
        L.or_quant_rows.restype = None
        L.or_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.or_e2m1_decode.restype = ctypes.c_float
        L.or_e2m1_encode.argtypes = [ctypes.c_float]
        L.or_e2m1_encode.restype = ctypes.c_uint8
        L.or_nvfp4_quant.argtypes = [vp, i64, i64, vp, vp, vp]
        L.or_nvfp4_quant.restype = i32
        L.or_route_topk.argtypes = [vp, i64, i32, i32, vp, vp]
        L.or_router_logits.argtypes = [vp, vp, i64, i64, i32, vp]
        L.or_route_topk.restype = None
        L.or_permute.argtypes = [vp, i64, i32, i32, vp, vp, vp]
        L.or_permute.restype = None
        L.or_moe_forward.argtypes = [ctypes.POINTER(_Layer), vp, vp, i64, i32, vp] + [vp] * 11
        L.or_moe_forward.restype = i32
        L.or_moe_forward_dense.argtypes = [ctypes.POINTER(_Layer), vp, vp, i64, i32, vp, vp, vp,
                                           vp, vp]
        L.or_moe_forward_given_h.argtypes = [ctypes.POINTER(_Layer), vp, vp, i64, i32, vp, vp, vp, vp]
        L.or_moe_forward_given_h.restype = i32
        L.or_moe_forward_dense.restype = i32
        L.or_expert_rows.argtypes = [ctypes.POINTER(_Layer), vp, vp, vp, i64, vp]
        L.or_expert_rows.restype = i32
        L.or_combine.argtypes = [ctypes.POINTER(_Layer), vp, vp, vp, i64, i32, vp]
        L.or_combine.restype = i32
        L.or_set_threads.argtypes = [i32]
        L.or_set_threads.restype = None
        L.or_max_threads.argtypes = []
        L.or_max_threads.restype = i32
        _lib = L
    return _lib


def set_threads(n: int) -> None:
    """Threads the oracle's OpenMP loops use from now on (timing only: results do not change)."""
    lib().or_set_threads(int(n))


def max_threads() -> int:
    return int(lib().or_max_threads())


def _p(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "arrays passed to the oracle must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


# ---- scalars --------------------------------------------------------------------------------

def bf16_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, np.uint16).astype(np.uint32) << 16).view(np.float32)


def e4m3_decode(c: int) -> float:
    return float(lib().or_e4m3_decode(int(c)))


def e4m3_encode(x: float) -> int:
    return int(lib().or_e4m3_encode(float(x)))


def e4m3_decode_table() -> np.ndarray:
    return np.array([e4m3_decode(c) for c in range(256)], np.float32)


# ---- S0..S3 ---------------------------------------------------------------------------------

def rtn_pack(w_bf16: np.ndarray, group: int = 128):
    """bf16 bits [rows, K] -> (packed int32 [rows, K/8], scales bf16 bits [rows, K/g], codes int8)."""
    w = np.ascontiguousarray(w_bf16, np.uint16)
    rows, K = w.shape
    packed = np.zeros((rows, K // 8), np.int32)
    scales = np.zeros((rows, K // group), np.uint16)
    codes = np.zeros((rows, K), np.int8)
    rc = lib().or_rtn_pack(_p(w), rows, K, group, _p(packed), _p(scales), _p(codes))
    if rc != 0:
        raise ValueError("or_rtn_pack: bad shape or code out of range")
    return packed, scales, codes


def unpack(packed: np.ndarray, K: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, np.int32)
    rows = packed.shape[0]
    codes = np.zeros((rows, K), np.int8)
    lib().or_unpack(_p(packed), rows, K, _p(codes))
    return codes


def quant_tokens(x_bf16: np.ndarray):
    x = np.ascontiguousarray(x_bf16, np.uint16)
    T, H = x.shape
    q = np.zeros((T, H), np.uint8)
    s = np.zeros(T, np.float32)
    lib().or_quant_tokens(_p(x), T, H, _p(q), _p(s))
    return q, s


def quant_rows(w_bf16: np.ndarray):
    """Row-scaled FP8 weights: bf16 bits [rows, K] -> (E4M3 codes [rows, K], fp32 scale [rows])."""
    w = np.ascontiguousarray(w_bf16, np.uint16)
    rows, K = w.shape
    q = np.zeros((rows, K), np.uint8)
    s = np.zeros(rows, np.float32)
    lib().or_quant_rows(_p(w), rows, K, _p(q), _p(s))
    return q, s


def e2m1_decode(c: int) -> float:
    return float(lib().or_e2m1_decode(int(c)))


def e2m1_encode(x: float) -> int:
    return int(lib().or_e2m1_encode(float(x)))


def nvfp4_quant(w_bf16: np.ndarray):
    """NVFP4 of one projection: bf16 bits [rows, K] -> (codes uint8 [rows, K/2], E4M3 block
    scales uint8 [rows, K/16], fp32 scale2)."""
    w = np.ascontiguousarray(w_bf16, np.uint16)
    rows, K = w.shape
    codes = np.zeros((rows, K // 2), np.uint8)
    scales = np.zeros((rows, K // 16), np.uint8)
    s2 = ctypes.c_float(0.0)
    if lib().or_nvfp4_quant(_p(w), rows, K, _p(codes), _p(scales), ctypes.byref(s2)) != 0:
        raise ValueError("or_nvfp4_quant: K must be a multiple of 16")
    return codes, scales, np.float32(s2.value)


def router_logits(x_bf16: np.ndarray, wr_bf16: np.ndarray) -> np.ndarray:
    """[T, E] fp32 logits of bf16 tokens [T, H] against the bf16 router weight [E, H]."""
    x = np.ascontiguousarray(x_bf16, np.uint16)
    w = np.ascontiguousarray(wr_bf16, np.uint16)
    T, H = x.shape
    E = w.shape[0]
    assert w.shape[1] == H
    out = np.zeros((T, E), np.float32)
    lib().or_router_logits(_p(x), _p(w), T, H, E, _p(out))
    return out


def route_topk(logits: np.ndarray, k: int):
    l = np.ascontiguousarray(logits, np.float32)
    T, E = l.shape
    ids = np.zeros((T, k), np.int32)
    gates = np.zeros((T, k), np.float32)
    lib().or_route_topk(_p(l), T, E, k, _p(ids), _p(gates))
    return ids, gates


def permute(ids: np.ndarray, E: int):
    ids = np.ascontiguousarray(ids, np.int32)
    T, k = ids.shape
    P = T * k
    offsets = np.zeros(E + 1, np.int32)
    sorted_pairs = np.zeros(P, np.int32)
    row_of_pair = np.zeros(P, np.int32)
    lib().or_permute(_p(ids), T, k, E, _p(offsets), _p(sorted_pairs), _p(row_of_pair))
    return offsets, sorted_pairs, row_of_pair


# ---- the layer ------------------------------------------------------------------------------

class Layer:
    """Host copy of one layer's packed weights (numpy), laid out like the C ABI's layer.

    The default format is W4A8 (packed INT4 + bf16 group scales); ``Layer.w8a8`` builds the
    row-scaled FP8 format (E4M3 codes + one fp32 scale per output row)."""

    def __init__(self, E, H, N, gate_packed, up_packed, down_packed, gate_scales, up_scales,
                 down_scales, group=128, sh_gate=None, sh_up=None, sh_down=None):
        self.E, self.H, self.N, self.group = E, H, N, group
        self.fmt = FMT_W4A8
        self.gate_packed = None if gate_packed is None else np.ascontiguousarray(gate_packed, np.int32)
        self.up_packed = None if up_packed is None else np.ascontiguousarray(up_packed, np.int32)
        self.down_packed = None if down_packed is None else np.ascontiguousarray(down_packed, np.int32)
        self.gate_scales = None if gate_scales is None else np.ascontiguousarray(gate_scales, np.uint16)
        self.up_scales = None if up_scales is None else np.ascontiguousarray(up_scales, np.uint16)
        self.down_scales = None if down_scales is None else np.ascontiguousarray(down_scales, np.uint16)
        self.gate_w8 = self.up_w8 = self.down_w8 = None
        self.gate_rs = self.up_rs = self.down_rs = None
        self.gate_f4 = self.up_f4 = self.down_f4 = None
        self.gate_bs = self.up_bs = self.down_bs = None
        self.gate_s2 = self.up_s2 = self.down_s2 = None
        self.hot_ids = self.cold_ids = None
        self.sh_gate = None if sh_gate is None else np.ascontiguousarray(sh_gate, np.uint16)
        self.sh_up = None if sh_up is None else np.ascontiguousarray(sh_up, np.uint16)
        self.sh_down = None if sh_down is None else np.ascontiguousarray(sh_down, np.uint16)
        self.n_shared = 0 if sh_gate is None else sh_gate.shape[0]
        self.shared_N = 0 if sh_gate is None else sh_gate.shape[1]

    @classmethod
    def w8a8(cls, E, H, N, gate_w8, up_w8, down_w8, gate_rs, up_rs, down_rs, group=128,
             sh_gate=None, sh_up=None, sh_down=None):
        """Row-scaled FP8 layer: codes [E,N,H], [E,N,H], [E,H,N]; scales [E,N], [E,N], [E,H]."""
        L = cls(E, H, N, None, None, None, None, None, None, group=group, sh_gate=sh_gate,
                sh_up=sh_up, sh_down=sh_down)
        L.fmt = FMT_W8A8
        L.gate_w8 = np.ascontiguousarray(gate_w8, np.uint8)
        L.up_w8 = np.ascontiguousarray(up_w8, np.uint8)
        L.down_w8 = np.ascontiguousarray(down_w8, np.uint8)
        L.gate_rs = np.ascontiguousarray(gate_rs, np.float32)
        L.up_rs = np.ascontiguousarray(up_rs, np.float32)
        L.down_rs = np.ascontiguousarray(down_rs, np.float32)
        assert L.gate_w8.shape == (E, N, H) and L.down_w8.shape == (E, H, N)
        assert L.gate_rs.shape == (E, N) and L.down_rs.shape == (E, H)
        return L

    @classmethod
    def nvfp4(cls, E, H, N, gate_f4, up_f4, down_f4, gate_bs, up_bs, down_bs, gate_s2, up_s2,
              down_s2, group=128, sh_gate=None, sh_up=None, sh_down=None):
        """NVFP4 layer: codes [E,N,H/2], [E,N,H/2], [E,H,N/2]; E4M3 block scales [E,N,H/16],
        [E,N,H/16], [E,H,N/16]; fp32 scale2 [E] per projection."""
        L = cls(E, H, N, None, None, None, None, None, None, group=group, sh_gate=sh_gate,
                sh_up=sh_up, sh_down=sh_down)
        L.fmt = FMT_NVFP4
        L.gate_f4, L.up_f4, L.down_f4 = (np.ascontiguousarray(a, np.uint8) for a in (gate_f4, up_f4, down_f4))
        L.gate_bs, L.up_bs, L.down_bs = (np.ascontiguousarray(a, np.uint8) for a in (gate_bs, up_bs, down_bs))
        L.gate_s2, L.up_s2, L.down_s2 = (np.ascontiguousarray(a, np.float32) for a in (gate_s2, up_s2, down_s2))
        assert L.gate_f4.shape == (E, N, H // 2) and L.down_f4.shape == (E, H, N // 2)
        assert L.gate_bs.shape == (E, N, H // 16) and L.down_bs.shape == (E, H, N // 16)
        assert L.gate_s2.shape == (E,)
        return L

    @classmethod
    def hybrid(cls, cold: "Layer", hot: "Layer", hot_ids, cold_ids):
        """Hot experts in NVFP4 (the slabs of `hot`, slab i = expert hot_ids[i]) and cold experts
        in W4A8 (the slabs of `cold`, slab j = expert cold_ids[j]); the lists partition 0..E-1."""
        hot_ids = np.ascontiguousarray(hot_ids, np.int32)
        cold_ids = np.ascontiguousarray(cold_ids, np.int32)
        E = len(hot_ids) + len(cold_ids)
        assert np.array_equal(np.sort(np.concatenate([hot_ids, cold_ids])), np.arange(E))
        L = cls(E, cold.H, cold.N, cold.gate_packed, cold.up_packed, cold.down_packed, cold.gate_scales,
                cold.up_scales, cold.down_scales, group=cold.group, sh_gate=cold.sh_gate,
                sh_up=cold.sh_up, sh_down=cold.sh_down)
        L.fmt = FMT_HYBRID
        for a in ("gate_f4", "up_f4", "down_f4", "gate_bs", "up_bs", "down_bs", "gate_s2", "up_s2", "down_s2"):
            setattr(L, a, getattr(hot, a))
        L.hot_ids, L.cold_ids = hot_ids, cold_ids
        return L

    def _c(self):
        return _Layer(self.E, self.H, self.N, self.group,
                      _p(self.gate_packed), _p(self.up_packed), _p(self.down_packed),
                      _p(self.gate_scales), _p(self.up_scales), _p(self.down_scales),
                      self.n_shared, self.shared_N,
                      _p(self.sh_gate), _p(self.sh_up), _p(self.sh_down),
                      self.fmt, _p(self.gate_w8), _p(self.up_w8), _p(self.down_w8),
                      _p(self.gate_rs), _p(self.up_rs), _p(self.down_rs),
                      _p(self.gate_f4), _p(self.up_f4), _p(self.down_f4),
                      _p(self.gate_bs), _p(self.up_bs), _p(self.down_bs),
                      _p(self.gate_s2), _p(self.up_s2), _p(self.down_s2),
                      _p(self.hot_ids), _p(self.cold_ids),
                      0 if self.hot_ids is None else len(self.hot_ids),
                      0 if self.cold_ids is None else len(self.cold_ids))


def moe_forward(layer: Layer, x_bf16: np.ndarray, logits: np.ndarray, k: int):
    """Run the layer; returns a dict with out (bf16 bits) and every intermediate."""
    x = np.ascontiguousarray(x_bf16, np.uint16)
    l = np.ascontiguousarray(logits, np.float32)
    T, H = x.shape
    E, N = layer.E, layer.N
    P = T * k
    r = dict(out=np.zeros((T, H), np.uint16), ids=np.zeros((T, k), np.int32),
             gates=np.zeros((T, k), np.float32), offsets=np.zeros(E + 1, np.int32),
             sorted_pairs=np.zeros(P, np.int32), row_of_pair=np.zeros(P, np.int32),
             xq=np.zeros((T, H), np.uint8), s_x=np.zeros(T, np.float32),
             hq=np.zeros((P, N), np.uint8), s_h=np.zeros(P, np.float32),
             y=np.zeros((P, H), np.float32), out_f32=np.zeros((T, H), np.float32))
    L = layer._c()
    rc = lib().or_moe_forward(ctypes.byref(L), _p(x), _p(l), T, k, _p(r["out"]), _p(r["ids"]),
                              _p(r["gates"]), _p(r["offsets"]), _p(r["sorted_pairs"]),
                              _p(r["row_of_pair"]), _p(r["xq"]), _p(r["s_x"]), _p(r["hq"]),
                              _p(r["s_h"]), _p(r["y"]), _p(r["out_f32"]))
    if rc != 0:
        raise ValueError("or_moe_forward: bad shape")
    return r


def moe_forward_given_h(layer: Layer, x_bf16: np.ndarray, logits: np.ndarray, k: int,
                        hq_pairs: np.ndarray, sh_pairs: np.ndarray):
    """The layer's output with the requantized SwiGLU activations given in pair order
    (hq_pairs [T*k, N] E4M3, sh_pairs [T*k]): S6-S8 on them.  Returns (out bf16, out_f32)."""
    x = np.ascontiguousarray(x_bf16, np.uint16)
    l = np.ascontiguousarray(logits, np.float32)
    hq = np.ascontiguousarray(hq_pairs, np.uint8)
    sh = np.ascontiguousarray(sh_pairs, np.float32)
    T, H = x.shape
    out = np.zeros((T, H), np.uint16)
    out_f32 = np.zeros((T, H), np.float32)
    L = layer._c()
    if lib().or_moe_forward_given_h(ctypes.byref(L), _p(x), _p(l), T, k, _p(hq), _p(sh), _p(out),
                                    _p(out_f32)) != 0:
        raise ValueError("or_moe_forward_given_h: bad shape")
    return out, out_f32


def moe_forward_dense(layer: Layer, x_bf16: np.ndarray, logits: np.ndarray, k: int):
    x = np.ascontiguousarray(x_bf16, np.uint16)
    l = np.ascontiguousarray(logits, np.float32)
    T, H = x.shape
    E, N = layer.E, layer.N
    r = dict(out=np.zeros((T, H), np.uint16), out_f32=np.zeros((T, H), np.float32),
             hq=np.zeros((T, E, N), np.uint8), s_h=np.zeros((T, E), np.float32),
             y=np.zeros((T, E, H), np.float32))
    L = layer._c()
    rc = lib().or_moe_forward_dense(ctypes.byref(L), _p(x), _p(l), T, k, _p(r["out"]),
                                    _p(r["out_f32"]), _p(r["hq"]), _p(r["s_h"]), _p(r["y"]))
    if rc != 0:
        raise ValueError("or_moe_forward_dense: bad shape")
    return r


def expert_slice(layer: Layer, e0: int, e1: int) -> Layer:
    """Experts e0..e1-1 of a W4A8 layer as a layer of their own (no shared experts)."""
    assert layer.fmt == FMT_W4A8 and 0 <= e0 < e1 <= layer.E
    return Layer(e1 - e0, layer.H, layer.N, layer.gate_packed[e0:e1], layer.up_packed[e0:e1],
                 layer.down_packed[e0:e1], layer.gate_scales[e0:e1], layer.up_scales[e0:e1],
                 layer.down_scales[e0:e1], group=layer.group)


def expert_rows(layer: Layer, q: np.ndarray, s_x: np.ndarray, expert: np.ndarray) -> np.ndarray:
    """S4-S6 for given FP8 rows: q [R,H] E4M3 codes, s_x [R], expert [R] -> y [R,H] fp32."""
    q = np.ascontiguousarray(q, np.uint8)
    s = np.ascontiguousarray(s_x, np.float32)
    e = np.ascontiguousarray(expert, np.int32)
    R = q.shape[0]
    y = np.zeros((R, layer.H), np.float32)
    L = layer._c()
    if lib().or_expert_rows(ctypes.byref(L), _p(q), _p(s), _p(e), R, _p(y)) != 0:
        raise ValueError("or_expert_rows: bad shape or expert index")
    return y


def combine(layer: Layer, x_bf16: np.ndarray, gates: np.ndarray, y_pairs: np.ndarray, k: int) -> np.ndarray:
    """S7 (+ S8) alone: bf16 out [T,H] from routed rows y_pairs [T*k, H] in pair order."""
    x = np.ascontiguousarray(x_bf16, np.uint16)
    g = np.ascontiguousarray(gates, np.float32)
    y = np.ascontiguousarray(y_pairs, np.float32)
    T = g.shape[0]
    out = np.zeros((T, layer.H), np.uint16)
    L = layer._c()
    if lib().or_combine(ctypes.byref(L), _p(x), _p(g), _p(y), T, k, _p(out)) != 0:
        raise ValueError("or_combine: bad shape")
    return out


def _each_expert(fn, experts):
    """fn(e) for every expert, on a pool of host threads (the C routines release the GIL; each
    expert writes only its own slabs, so the result does not depend on the order)."""
    from concurrent.futures import ThreadPoolExecutor
    experts = list(experts)
    n = min(len(experts), os.cpu_count() or 1)
    if n <= 1:
        for e in experts:
            fn(e)
        return
    with ThreadPoolExecutor(n) as ex:
        list(ex.map(fn, experts))


def pack_workload_layer(wl, experts=None, with_shared=True, into=None):
    """Pack (RTN, oracle side) the seeded weights of workload `wl`.

    Only experts in `experts` (default: all) are drawn and packed; the others stay zero,
    which is enough when the caller knows which experts its tokens route to.  With `into` (a
    Layer of this workload's shapes) the experts are packed into its arrays and it is returned.
    """
    import synth
    E, H, N, g = wl.E, wl.H, wl.N, wl.group
    if into is not None:
        gp, up, dp = into.gate_packed, into.up_packed, into.down_packed
        gs, us, ds = into.gate_scales, into.up_scales, into.down_scales
    else:
        gp = np.zeros((E, N, H // 8), np.int32)
        up = np.zeros((E, N, H // 8), np.int32)
        dp = np.zeros((E, H, N // 8), np.int32)
        gs = np.zeros((E, N, H // g), np.uint16)
        us = np.zeros((E, N, H // g), np.uint16)
        ds = np.zeros((E, H, N // g), np.uint16)
    def one(e):
        gp[e], gs[e], _ = rtn_pack(synth.expert_weight(wl, e, "gate"), g)
        up[e], us[e], _ = rtn_pack(synth.expert_weight(wl, e, "up"), g)
        dp[e], ds[e], _ = rtn_pack(synth.expert_weight(wl, e, "down"), g)
    _each_expert(one, range(E) if experts is None else experts)
    if into is not None:
        return into
    sh = {}
    if with_shared and wl.n_shared:
        sh = dict(sh_gate=np.stack([synth.shared_weight(wl, s, "gate") for s in range(wl.n_shared)]),
                  sh_up=np.stack([synth.shared_weight(wl, s, "up") for s in range(wl.n_shared)]),
                  sh_down=np.stack([synth.shared_weight(wl, s, "down") for s in range(wl.n_shared)]))
    return Layer(E, H, N, gp, up, dp, gs, us, ds, group=g, **sh)


def quant_workload_layer_w8a8(wl, experts=None, with_shared=True, into=None):
    """Row-quantize (oracle side) the seeded weights of workload `wl` to the row-scaled FP8
    format; experts outside `experts` stay zero, and `into` fills a given layer, as in
    ``pack_workload_layer``."""
    import synth
    E, H, N = wl.E, wl.H, wl.N
    if into is not None:
        gq, uq, dq, gs, us, ds = into.gate_w8, into.up_w8, into.down_w8, into.gate_rs, into.up_rs, into.down_rs
    else:
        gq = np.zeros((E, N, H), np.uint8)
        uq = np.zeros((E, N, H), np.uint8)
        dq = np.zeros((E, H, N), np.uint8)
        gs = np.zeros((E, N), np.float32)
        us = np.zeros((E, N), np.float32)
        ds = np.zeros((E, H), np.float32)
    def one(e):
        gq[e], gs[e] = quant_rows(synth.expert_weight(wl, e, "gate"))
        uq[e], us[e] = quant_rows(synth.expert_weight(wl, e, "up"))
        dq[e], ds[e] = quant_rows(synth.expert_weight(wl, e, "down"))
    _each_expert(one, range(E) if experts is None else experts)
    if into is not None:
        return into
    sh = {}
    if with_shared and wl.n_shared:
        sh = dict(sh_gate=np.stack([synth.shared_weight(wl, s, "gate") for s in range(wl.n_shared)]),
                  sh_up=np.stack([synth.shared_weight(wl, s, "up") for s in range(wl.n_shared)]),
                  sh_down=np.stack([synth.shared_weight(wl, s, "down") for s in range(wl.n_shared)]))
    return Layer.w8a8(E, H, N, gq, uq, dq, gs, us, ds, group=wl.group, **sh)


def quant_workload_layer_nvfp4(wl, experts=None, with_shared=True, into=None):
    """NVFP4-quantize (oracle side) the seeded weights of workload `wl`; experts outside
    `experts` stay zero, and `into` fills a given layer, as in ``pack_workload_layer``."""
    import synth
    E, H, N = wl.E, wl.H, wl.N
    if into is not None:
        c = {"gate": into.gate_f4, "up": into.up_f4, "down": into.down_f4}
        b = {"gate": into.gate_bs, "up": into.up_bs, "down": into.down_bs}
        s2 = {"gate": into.gate_s2, "up": into.up_s2, "down": into.down_s2}
    else:
        c = {p: np.zeros((E, *synth.weight_shape(wl, p)[:1], synth.weight_shape(wl, p)[1] // 2), np.uint8)
             for p in ("gate", "up", "down")}
        b = {p: np.zeros((E, *synth.weight_shape(wl, p)[:1], synth.weight_shape(wl, p)[1] // 16), np.uint8)
             for p in ("gate", "up", "down")}
        s2 = {p: np.zeros(E, np.float32) for p in ("gate", "up", "down")}
    def one(e):
        for p in ("gate", "up", "down"):
            c[p][e], b[p][e], s2[p][e] = nvfp4_quant(synth.expert_weight(wl, e, p))
    _each_expert(one, range(E) if experts is None else experts)
    if into is not None:
        return into
    sh = {}
    if with_shared and wl.n_shared:
        sh = dict(sh_gate=np.stack([synth.shared_weight(wl, s, "gate") for s in range(wl.n_shared)]),
                  sh_up=np.stack([synth.shared_weight(wl, s, "up") for s in range(wl.n_shared)]),
                  sh_down=np.stack([synth.shared_weight(wl, s, "down") for s in range(wl.n_shared)]))
    return Layer.nvfp4(E, H, N, c["gate"], c["up"], c["down"], b["gate"], b["up"], b["down"],
                       s2["gate"], s2["up"], s2["down"], group=wl.group, **sh)
