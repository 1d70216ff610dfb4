"""Convenience wrappers: torch allocation around the C entry points."""
from __future__ import annotations

from ._binding import (Layer, Layer4, Layer8, LayerH, moe_hybrid_forward, moe_hybrid_workspace_bytes,
                       moe_nvfp4_forward, moe_nvfp4_workspace_bytes,
                       moe_w4a8_forward, moe_w4a8_workspace_bytes, moe_w8a8_forward,
                       moe_w8a8_workspace_bytes, nvfp4_quant_weights, w4a8_pack_weights,
                       w8a8_quant_weights)


def pack_expert_weights(w, group: int = 128, stream=None):
    """bf16 weights [..., rows, K] on the GPU -> (int32 packed [..., rows, K/8],
    bf16 scales [..., rows, K/group]) in pack-quantized storage."""
    import torch
    *lead, rows, K = w.shape
    packed = torch.empty(*lead, rows, K // 8, dtype=torch.int32, device=w.device)
    scales = torch.empty(*lead, rows, K // group, dtype=torch.bfloat16, device=w.device)
    w4a8_pack_weights(w.contiguous(), packed, scales, group=group, stream=stream)
    return packed, scales


def make_layer(gate_w, up_w, down_w, sh_gate=None, sh_up=None, sh_down=None,
               stream=None) -> Layer:
    """Quantize and pack bf16 expert weights gate/up [E, N, H], down [E, H, N]."""
    E, N, H = gate_w.shape
    gp, gs = pack_expert_weights(gate_w, stream=stream)
    up, us = pack_expert_weights(up_w, stream=stream)
    dp, ds = pack_expert_weights(down_w, stream=stream)
    return Layer(E, H, N, gp, up, dp, gs, us, ds, sh_gate=sh_gate, sh_up=sh_up, sh_down=sh_down)


def quant_expert_weights_w8a8(w, stream=None):
    """bf16 weights [..., rows, K] on the GPU -> (E4M3 codes uint8 [..., rows, K],
    fp32 row scales [..., rows])."""
    import torch
    *lead, rows, K = w.shape
    q = torch.empty(*lead, rows, K, dtype=torch.uint8, device=w.device)
    s = torch.empty(*lead, rows, dtype=torch.float32, device=w.device)
    w8a8_quant_weights(w.contiguous(), q, s, stream=stream)
    return q, s


def make_layer_w8a8(gate_w, up_w, down_w, sh_gate=None, sh_up=None, sh_down=None,
                    stream=None) -> Layer8:
    """Row-quantize bf16 expert weights gate/up [E, N, H], down [E, H, N] to FP8."""
    E, N, H = gate_w.shape
    gq, gs = quant_expert_weights_w8a8(gate_w, stream=stream)
    uq, us = quant_expert_weights_w8a8(up_w, stream=stream)
    dq, ds = quant_expert_weights_w8a8(down_w, stream=stream)
    return Layer8(E, H, N, gq, uq, dq, gs, us, ds, sh_gate=sh_gate, sh_up=sh_up, sh_down=sh_down)


def quant_expert_weights_nvfp4(w, stream=None):
    """bf16 weights [experts, rows, K] on the GPU -> (E2M1 codes uint8 [experts, rows, K/2],
    E4M3 block scales uint8 [experts, rows, K/16], fp32 scale2 [experts])."""
    import torch
    E, rows, K = w.shape
    codes = torch.empty(E, rows, K // 2, dtype=torch.uint8, device=w.device)
    scales = torch.empty(E, rows, K // 16, dtype=torch.uint8, device=w.device)
    s2 = torch.empty(E, dtype=torch.float32, device=w.device)
    nvfp4_quant_weights(w.contiguous(), codes, scales, s2, stream=stream)
    return codes, scales, s2


def make_layer_nvfp4(gate_w, up_w, down_w, sh_gate=None, sh_up=None, sh_down=None,
                     stream=None) -> Layer4:
    """NVFP4-quantize bf16 expert weights gate/up [E, N, H], down [E, H, N]."""
    E, N, H = gate_w.shape
    g = quant_expert_weights_nvfp4(gate_w, stream=stream)
    u = quant_expert_weights_nvfp4(up_w, stream=stream)
    d = quant_expert_weights_nvfp4(down_w, stream=stream)
    return Layer4(E, H, N, g[0], u[0], d[0], g[1], u[1], d[1], g[2], u[2], d[2],
                  sh_gate=sh_gate, sh_up=sh_up, sh_down=sh_down)


def hybrid_from(w4: Layer, f4: Layer4, hot_ids) -> LayerH:
    """A hybrid layer from a W4A8 layer and an NVFP4 layer of the same experts: the hot experts
    (hot_ids, in slab order) take their NVFP4 slabs, the others their W4A8 slabs."""
    import torch
    dev = w4.gate_packed.device
    hot = torch.as_tensor(hot_ids, dtype=torch.int32).to(dev)
    mask = torch.ones(w4.E, dtype=torch.bool, device=dev)
    mask[hot.long()] = False
    cold = torch.arange(w4.E, dtype=torch.int32, device=dev)[mask]
    hi, ci = hot.long(), cold.long()
    h = Layer4(len(hot_ids), f4.H, f4.N, f4.gate_f4[hi].contiguous(), f4.up_f4[hi].contiguous(),
               f4.down_f4[hi].contiguous(), f4.gate_bs[hi].contiguous(), f4.up_bs[hi].contiguous(),
               f4.down_bs[hi].contiguous(), f4.gate_s2[hi].contiguous(), f4.up_s2[hi].contiguous(),
               f4.down_s2[hi].contiguous())
    c = Layer(int(cold.numel()), w4.H, w4.N, w4.gate_packed[ci].contiguous(), w4.up_packed[ci].contiguous(),
              w4.down_packed[ci].contiguous(), w4.gate_scales[ci].contiguous(), w4.up_scales[ci].contiguous(),
              w4.down_scales[ci].contiguous(), group=w4.group, sh_gate=w4.sh_gate, sh_up=w4.sh_up,
              sh_down=w4.sh_down)
    return LayerH(w4.E, h, c, hot.contiguous(), cold.contiguous())


def alloc_workspace(layer, T: int, k: int, device=None):
    import torch
    if isinstance(layer, LayerH):
        n, ref = moe_hybrid_workspace_bytes(layer, T, k), layer.hot_ids
    elif isinstance(layer, Layer8):
        n, ref = moe_w8a8_workspace_bytes(layer, T, k), layer.gate_w8
    elif isinstance(layer, Layer4):
        n, ref = moe_nvfp4_workspace_bytes(layer, T, k), layer.gate_f4
    else:
        n, ref = moe_w4a8_workspace_bytes(layer, T, k), layer.gate_packed
    if n == 0 and T > 0:
        raise ValueError("unsupported layer shape for the MoE forward")
    dev = device if device is not None else ref.device
    return torch.empty(max(n, 256), dtype=torch.uint8, device=dev)


def forward(layer, x, logits, k: int, out=None, ws=None, stream=None):
    """The layer on x for any expert format (Layer: W4A8, Layer8: row-scaled FP8, Layer4: NVFP4)."""
    import torch
    if out is None:
        out = torch.empty_like(x)
    if ws is None:
        ws = alloc_workspace(layer, x.shape[0], k, x.device)
    if isinstance(layer, LayerH):
        moe_hybrid_forward(layer, x, logits, k, out, ws, stream=stream)
    elif isinstance(layer, Layer8):
        moe_w8a8_forward(layer, x, logits, k, out, ws, stream=stream)
    elif isinstance(layer, Layer4):
        moe_nvfp4_forward(layer, x, logits, k, out, ws, stream=stream)
    else:
        moe_w4a8_forward(layer, x, logits, k, out, ws, stream=stream)
    return out
