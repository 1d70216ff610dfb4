"""Seeded synthetic layers and batches in HBM (for tests, smoke and the benchmark).

Weights are drawn on the GPU by the seeded generator (``synth``), bit-identical to the host
draws the CPU oracle makes, then quantized and packed by ``w4a8_pack_weights`` (or, for the
row-scaled FP8 format, quantized by ``w8a8_quant_weights``).
"""
from __future__ import annotations

import synth

from ._binding import Layer, Layer4, Layer8
from .layer import pack_expert_weights, quant_expert_weights_nvfp4, quant_expert_weights_w8a8


def _expert_tensors(wl, device, experts_per_chunk, w8=False, f4=False):
    import torch
    E = wl.E
    out = {}
    for proj in ("gate", "up", "down"):
        rows, K = synth.weight_shape(wl, proj)
        if f4:
            p = torch.empty(E, rows, K // 2, dtype=torch.uint8, device=device)
            s = torch.empty(E, rows, K // 16, dtype=torch.uint8, device=device)
            s2 = torch.empty(E, dtype=torch.float32, device=device)
        elif w8:
            p = torch.empty(E, rows, K, dtype=torch.uint8, device=device)
            s = torch.empty(E, rows, dtype=torch.float32, device=device)
        else:
            p = torch.empty(E, rows, K // 8, dtype=torch.int32, device=device)
            s = torch.empty(E, rows, K // wl.group, dtype=torch.bfloat16, device=device)
        buf = torch.empty(min(E, experts_per_chunk), rows, K, dtype=torch.bfloat16, device=device)
        for e0 in range(0, E, experts_per_chunk):
            n = min(experts_per_chunk, E - e0)
            for i in range(n):
                synth.dev_weight(wl.seed, synth.weight_stream(e0 + i, proj), buf[i])
            if f4:
                pp, ss, s22 = quant_expert_weights_nvfp4(buf[:n])
                s2[e0:e0 + n].copy_(s22)
            else:
                pp, ss = (quant_expert_weights_w8a8 if w8 else pack_expert_weights)(buf[:n])
            p[e0:e0 + n].copy_(pp)
            s[e0:e0 + n].copy_(ss)
        out[proj] = (p, s, s2) if f4 else (p, s)
        del buf
    return out


def _shared_tensors(wl, device):
    import torch
    sh = {}
    if wl.n_shared:
        for proj, key in (("gate", "sh_gate"), ("up", "sh_up"), ("down", "sh_down")):
            rows, K = synth.weight_shape(wl, proj, shared=True)
            t = torch.empty(wl.n_shared, rows, K, dtype=torch.bfloat16, device=device)
            for s_ in range(wl.n_shared):
                synth.dev_weight(wl.seed, synth.shared_stream(s_, proj), t[s_])
            sh[key] = t
    return sh


def device_layer(wl: synth.Workload, device="cuda", experts_per_chunk: int = 32) -> Layer:
    """The packed routed experts (and bf16 shared experts) of workload `wl` on `device`."""
    import torch
    packed = _expert_tensors(wl, device, experts_per_chunk, w8=False)
    sh = _shared_tensors(wl, device)
    torch.cuda.synchronize()
    return Layer(wl.E, wl.H, wl.N, packed["gate"][0], packed["up"][0], packed["down"][0],
                 packed["gate"][1], packed["up"][1], packed["down"][1], group=wl.group, **sh)


def device_layer_w8a8(wl: synth.Workload, device="cuda", experts_per_chunk: int = 32) -> Layer8:
    """The same seeded experts of workload `wl` in the row-scaled FP8 format."""
    import torch
    q = _expert_tensors(wl, device, experts_per_chunk, w8=True)
    sh = _shared_tensors(wl, device)
    torch.cuda.synchronize()
    return Layer8(wl.E, wl.H, wl.N, q["gate"][0], q["up"][0], q["down"][0],
                  q["gate"][1], q["up"][1], q["down"][1], **sh)


def device_layer_nvfp4(wl: synth.Workload, device="cuda", experts_per_chunk: int = 32) -> Layer4:
    """The same seeded experts of workload `wl` in the NVFP4 format."""
    import torch
    q = _expert_tensors(wl, device, experts_per_chunk, f4=True)
    sh = _shared_tensors(wl, device)
    torch.cuda.synchronize()
    return Layer4(wl.E, wl.H, wl.N, q["gate"][0], q["up"][0], q["down"][0], q["gate"][1], q["up"][1],
                  q["down"][1], q["gate"][2], q["up"][2], q["down"][2], **sh)


def device_inputs(wl: synth.Workload, device="cuda", t0: int = 0, T: int | None = None):
    """(x bf16 [T, H], logits fp32 [T, E]) of workload `wl`, rows t0.. on `device`."""
    import torch
    T = wl.T if T is None else T
    x = torch.empty(T, wl.H, dtype=torch.bfloat16, device=device)
    lg = torch.empty(T, wl.E, dtype=torch.float32, device=device)
    if T:
        synth.dev_tokens(wl, x, t0)
        synth.dev_logits(wl, lg, t0)
    return x, lg
