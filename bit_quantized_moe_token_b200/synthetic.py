"""Seeded synthetic layers and batches in HBM (for tests, smoke and the benchmark).

Weights are drawn on the GPU by the seeded generator (``synth``), bit-identical to the host
draws the CPU oracle makes, then quantized and packed by ``w4a8_pack_weights``.
"""
from __future__ import annotations

import synth

from ._binding import Layer
from .layer import pack_expert_weights


def device_layer(wl: synth.Workload, device="cuda", experts_per_chunk: int = 32) -> Layer:
    """The packed routed experts (and bf16 shared experts) of workload `wl` on `device`."""
    import torch
    E, H, N = wl.E, wl.H, wl.N
    packed = {}
    for proj in ("gate", "up", "down"):
        rows, K = synth.weight_shape(wl, proj)
        p = torch.empty(E, rows, K // 8, dtype=torch.int32, device=device)
        s = torch.empty(E, rows, K // wl.group, dtype=torch.bfloat16, device=device)
        buf = torch.empty(min(E, experts_per_chunk), rows, K, dtype=torch.bfloat16, device=device)
        for e0 in range(0, E, experts_per_chunk):
            n = min(experts_per_chunk, E - e0)
            for i in range(n):
                synth.dev_weight(wl.seed, synth.weight_stream(e0 + i, proj), buf[i])
            pp, ss = pack_expert_weights(buf[:n])
            p[e0:e0 + n].copy_(pp)
            s[e0:e0 + n].copy_(ss)
        packed[proj] = (p, s)
        del buf
    sh = {}
    if wl.n_shared:
        for proj, key in (("gate", "sh_gate"), ("up", "sh_up"), ("down", "sh_down")):
            rows, K = synth.weight_shape(wl, proj, shared=True)
            t = torch.empty(wl.n_shared, rows, K, dtype=torch.bfloat16, device=device)
            for s_ in range(wl.n_shared):
                synth.dev_weight(wl.seed, synth.shared_stream(s_, proj), t[s_])
            sh[key] = t
    torch.cuda.synchronize()
    return Layer(E, H, N, packed["gate"][0], packed["up"][0], packed["down"][0],
                 packed["gate"][1], packed["up"][1], packed["down"][1], group=wl.group, **sh)


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
