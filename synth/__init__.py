"""Seeded synthetic workloads for the W4A8-FP8 routed MoE layer.

This module only draws inputs; it holds none of the layer's arithmetic.  Both
the CPU oracle (``oracle/``) and the CUDA path read the same bytes from it:
the host filler (``synth_host.c``) and the device filler (``synth_dev.cu``)
evaluate the same counter-based definition (``synth_core.h``) and agree bit
for bit, so a full-size weight set can be drawn directly in HBM while the
oracle regenerates just the slices it checks.

Workloads follow the five layer configurations of the Inkling-Small W4A8-G128
model card (section 1 "What is being created?": hidden 4096, expert width 2048,
256 routed experts; top-6 from the opening paragraph of the Inkling-512k hybrid
card), with synthetic values:

* hidden states bf16 ~ N(0,1); where ``outliers`` is set, round(0.01*H)
  channels drawn once per workload (same for every token) are scaled x20;
* router logits fp32 ~ N(0,1); ``zipf`` routing adds -1.1*ln(rank_e) with
  rank a seeded permutation of 1..E (Zipf(s=1.1) prior on expert mass);
* expert and shared-expert weights bf16 ~ N(0, 0.02).

Stream numbering: X=1, logits=2, outlier channels=3, expert ranks=4, routed
expert e projection p (0 gate, 1 up, 2 down) = 100 + 3e + p, shared expert s
projection p = 1_000_000 + 3s + p.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_HOST_SO = os.path.join(_HERE, "libsynth_host.so")
_DEV_SO = os.path.join(_HERE, "libsynth_cuda.so")

S_X, S_LOGITS, S_OUTLIERS, S_RANKS = 1, 2, 3, 4
WEIGHT_SIGMA = 0.02
OUTLIER_GAIN = 20.0
ZIPF_S = 1.1
PROJ = {"gate": 0, "up": 1, "down": 2}


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    N: int
    E: int
    k: int
    outliers: bool
    routing: str  # "uniform" | "zipf"
    n_shared: int = 0
    shared_N: int = 0
    seed: int = 0
    group: int = 128

    @property
    def P(self) -> int:
        return self.T * self.k

    def describe(self) -> str:
        s = (f"T={self.T} H={self.H} N={self.N} E={self.E} top-{self.k} "
             f"routing={self.routing} outliers={'1%x20' if self.outliers else 'none'}")
        if self.n_shared:
            s += f" shared={self.n_shared}x{self.shared_N} bf16"
        return s + f" seed={self.seed}"


WORKLOADS = {
    "tiny": Workload("tiny", T=16, H=256, N=128, E=8, k=2, outliers=False, routing="uniform"),
    "decode_t8": Workload("decode_t8", T=8, H=4096, N=2048, E=256, k=6, outliers=True,
                          routing="uniform"),
    "decode_t64": Workload("decode_t64", T=64, H=4096, N=2048, E=256, k=6, outliers=False,
                           routing="uniform"),
    "prefill_t2048_zipf": Workload("prefill_t2048_zipf", T=2048, H=4096, N=2048, E=256, k=6,
                                   outliers=True, routing="zipf"),
    "prefill_t16384_shared": Workload("prefill_t16384_shared", T=16384, H=4096, N=2048, E=256,
                                      k=6, outliers=False, routing="uniform", n_shared=2,
                                      shared_N=2048),
    # The same layer shape with 64 experts: profiler captures that replay each launch many times
    # stay within a few GB of device memory (the full 256-expert row-scaled FP8 layer is 6.4 GB).
    "decode_t8_e64": Workload("decode_t8_e64", T=8, H=4096, N=2048, E=64, k=6, outliers=True,
                              routing="uniform"),
    "prefill_t512_e64_zipf": Workload("prefill_t512_e64_zipf", T=512, H=4096, N=2048, E=64, k=6,
                                      outliers=True, routing="zipf"),
    "prefill_t4096_e64": Workload("prefill_t4096_e64", T=4096, H=4096, N=2048, E=64, k=6,
                                  outliers=False, routing="uniform"),
}


def weight_stream(e: int, proj: str) -> int:
    return 100 + 3 * e + PROJ[proj]


def shared_stream(s: int, proj: str) -> int:
    return 1_000_000 + 3 * s + PROJ[proj]


def weight_shape(wl: Workload, proj: str, shared: bool = False):
    n = wl.shared_N if shared else wl.N
    return (n, wl.H) if proj in ("gate", "up") else (wl.H, n)


# ----------------------------------------------------------------------------------------------
# build + load
# ----------------------------------------------------------------------------------------------

def build(verbose: bool = False) -> None:
    """Compile the host filler (gcc) and, when nvcc is present, the device filler."""
    core = os.path.join(_HERE, "synth_core.h")
    src = os.path.join(_HERE, "synth_host.c")
    if _stale(_HOST_SO, [src, core]):
        _run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
              "-fno-fast-math", src, "-o", _HOST_SO, "-lm"], verbose)
    dsrc = os.path.join(_HERE, "synth_dev.cu")
    nvcc = _nvcc()
    if nvcc and _stale(_DEV_SO, [dsrc, core]):
        _run([nvcc, "-O2", "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-fmad=false",
              "-gencode", "arch=compute_100a,code=sm_100a", dsrc, "-o", _DEV_SO], verbose)


def _nvcc():
    for c in (os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc"),):
        if os.path.exists(c):
            return c
    return None


def _stale(out, srcs):
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(s) > t for s in srcs)


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)


_host = None
_dev = None


def host_lib():
    global _host
    if _host is None:
        build()
        L = ctypes.CDLL(_HOST_SO)
        u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        L.syn_fill_normal_bf16.argtypes = [u64, u64, i64, i64, dbl, vp]
        L.syn_fill_normal_f32.argtypes = [u64, u64, i64, i64, dbl, vp]
        L.syn_fill_tokens_bf16.argtypes = [u64, u64, i64, i64, i64, vp, dbl, vp]
        L.syn_fill_logits.argtypes = [u64, u64, i64, i64, i64, vp, vp]
        L.syn_permutation.argtypes = [u64, u64, i64, vp]
        L.syn_zipf_bias.argtypes = [vp, i64, dbl, vp]
        L.syn_normal_at.argtypes = [u64, u64, u64]
        L.syn_normal_at.restype = dbl
        L.syn_log_at.argtypes = [dbl]
        L.syn_log_at.restype = dbl
        L.syn_cossin_at.argtypes = [dbl, vp, vp]
        for f in (L.syn_fill_normal_bf16, L.syn_fill_normal_f32, L.syn_fill_tokens_bf16,
                  L.syn_fill_logits, L.syn_permutation, L.syn_zipf_bias):
            f.restype = None
        _host = L
    return _host


def dev_lib():
    global _dev
    if _dev is None:
        build()
        if not os.path.exists(_DEV_SO):
            raise RuntimeError("device filler not built (nvcc missing)")
        L = ctypes.CDLL(_DEV_SO)
        u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        L.syn_dev_fill_normal_bf16.argtypes = [u64, u64, i64, i64, dbl, vp, vp]
        L.syn_dev_fill_tokens_bf16.argtypes = [u64, u64, i64, i64, i64, vp, dbl, vp, vp]
        L.syn_dev_fill_logits.argtypes = [u64, u64, i64, i64, i64, vp, vp, vp]
        for f in (L.syn_dev_fill_normal_bf16, L.syn_dev_fill_tokens_bf16, L.syn_dev_fill_logits):
            f.restype = ctypes.c_int
        _dev = L
    return _dev


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


# ----------------------------------------------------------------------------------------------
# host arrays
# ----------------------------------------------------------------------------------------------

def outlier_mask(wl: Workload) -> np.ndarray | None:
    """uint8[H]: 1 on the round(0.01*H) seeded outlier channels, or None."""
    if not wl.outliers:
        return None
    perm = permutation(wl.seed, S_OUTLIERS, wl.H)
    m = np.zeros(wl.H, np.uint8)
    m[perm[: int(round(0.01 * wl.H))]] = 1
    return m


def expert_ranks(wl: Workload) -> np.ndarray:
    """int32[E]: the seeded popularity rank (1..E) of each expert."""
    return (permutation(wl.seed, S_RANKS, wl.E) + 1).astype(np.int32)


HOT_FRACTION = 0.148   # the NVFP4 share of expert slots in the hybrid card's 512k tier


def hot_experts(wl: Workload) -> np.ndarray:
    """int32[round(0.148 * E)]: the hot (NVFP4) experts of a hybrid layer of workload `wl`, in
    slab order: the most popular experts under Zipf routing, a seeded choice otherwise."""
    n = int(round(HOT_FRACTION * wl.E))
    if wl.routing == "zipf":
        return np.argsort(expert_ranks(wl), kind="stable")[:n].astype(np.int32)
    return np.sort(permutation(wl.seed, S_RANKS + 1, wl.E)[:n]).astype(np.int32)


def logit_bias(wl: Workload) -> np.ndarray | None:
    """float64[E]: -1.1*ln(rank_e) for zipf routing, else None."""
    if wl.routing != "zipf":
        return None
    b = np.zeros(wl.E, np.float64)
    ranks = expert_ranks(wl)          # keep a reference while C reads it
    host_lib().syn_zipf_bias(_p(ranks), wl.E, ZIPF_S, _p(b))
    return b


def permutation(seed: int, stream: int, n: int) -> np.ndarray:
    out = np.zeros(n, np.int32)
    host_lib().syn_permutation(seed, stream, n, _p(out))
    return out


def tokens(wl: Workload, t0: int = 0, nt: int | None = None) -> np.ndarray:
    """bf16 bits uint16[nt, H]: rows t0..t0+nt of the hidden states."""
    nt = wl.T - t0 if nt is None else nt
    out = np.zeros((nt, wl.H), np.uint16)
    m = outlier_mask(wl)
    host_lib().syn_fill_tokens_bf16(wl.seed, S_X, t0, nt, wl.H,
                                    _p(m) if m is not None else None, OUTLIER_GAIN, _p(out))
    return out


def logits(wl: Workload, t0: int = 0, nt: int | None = None) -> np.ndarray:
    """float32[nt, E]: rows t0..t0+nt of the router logits."""
    nt = wl.T - t0 if nt is None else nt
    out = np.zeros((nt, wl.E), np.float32)
    b = logit_bias(wl)
    host_lib().syn_fill_logits(wl.seed, S_LOGITS, t0, nt, wl.E,
                               _p(b) if b is not None else None, _p(out))
    return out


def expert_weight(wl: Workload, e: int, proj: str) -> np.ndarray:
    """bf16 bits uint16[rows, K] of routed expert e's projection (gate/up [N,H], down [H,N])."""
    shape = weight_shape(wl, proj)
    out = np.zeros(shape, np.uint16)
    host_lib().syn_fill_normal_bf16(wl.seed, weight_stream(e, proj), 0, out.size, WEIGHT_SIGMA,
                                    _p(out))
    return out


def shared_weight(wl: Workload, s: int, proj: str) -> np.ndarray:
    shape = weight_shape(wl, proj, shared=True)
    out = np.zeros(shape, np.uint16)
    host_lib().syn_fill_normal_bf16(wl.seed, shared_stream(s, proj), 0, out.size, WEIGHT_SIGMA,
                                    _p(out))
    return out


ROUTER_STREAM = 2_000_000


def router_weight(wl: Workload) -> np.ndarray:
    """bf16 router weight [E, H] ~ N(0, 1/sqrt(H)): with N(0,1) tokens the logits are ~N(0,1),
    the spread the workloads' given logits have."""
    out = np.zeros((wl.E, wl.H), np.uint16)
    host_lib().syn_fill_normal_bf16(wl.seed, ROUTER_STREAM, 0, out.size, 1.0 / np.sqrt(wl.H), _p(out))
    return out


def normal_f32(seed: int, stream: int, n: int, sigma: float = 1.0, start: int = 0) -> np.ndarray:
    out = np.zeros(n, np.float32)
    host_lib().syn_fill_normal_f32(seed, stream, start, n, sigma, _p(out))
    return out


def normal_bf16(seed: int, stream: int, n: int, sigma: float = 1.0, start: int = 0) -> np.ndarray:
    out = np.zeros(n, np.uint16)
    host_lib().syn_fill_normal_bf16(seed, stream, start, n, sigma, _p(out))
    return out


# ----------------------------------------------------------------------------------------------
# device tensors (torch is imported lazily: the host side never needs it)
# ----------------------------------------------------------------------------------------------

def _stream_handle(torch, device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(rc):
    if rc != 0:
        raise RuntimeError(f"device filler failed: cuda error {rc}")


def dev_tokens(wl: Workload, out, t0: int = 0):
    """Fill a CUDA int16/uint16 tensor [nt, H] with hidden-state rows t0.. (bf16 bits)."""
    import torch
    m = outlier_mask(wl)
    md = torch.from_numpy(m).to(out.device) if m is not None else None
    nt = out.shape[0]
    _check(dev_lib().syn_dev_fill_tokens_bf16(
        wl.seed, S_X, t0, nt, wl.H, ctypes.c_void_p(md.data_ptr()) if md is not None else None,
        OUTLIER_GAIN, ctypes.c_void_p(out.data_ptr()), _stream_handle(torch, out.device)))
    torch.cuda.current_stream(out.device).synchronize()
    return out


def dev_logits(wl: Workload, out, t0: int = 0):
    import torch
    b = logit_bias(wl)
    bd = torch.from_numpy(b).to(out.device) if b is not None else None
    nt = out.shape[0]
    _check(dev_lib().syn_dev_fill_logits(
        wl.seed, S_LOGITS, t0, nt, wl.E, ctypes.c_void_p(bd.data_ptr()) if bd is not None else None,
        ctypes.c_void_p(out.data_ptr()), _stream_handle(torch, out.device)))
    torch.cuda.current_stream(out.device).synchronize()
    return out


def dev_weight(seed: int, stream: int, out, sigma: float = WEIGHT_SIGMA):
    """Fill a contiguous CUDA 16-bit tensor with bf16 N(0, sigma) draws of `stream`."""
    import torch
    _check(dev_lib().syn_dev_fill_normal_bf16(seed, stream, 0, out.numel(), sigma,
                                              ctypes.c_void_p(out.data_ptr()),
                                              _stream_handle(torch, out.device)))
    return out
