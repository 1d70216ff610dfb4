"""Host-side checks of the C ABI: the library loads, exports every declared entry point, and
rejects bad arguments before touching the GPU (no compute call is made here)."""
import ctypes
import glob
import os
import re

import pytest

import bit_quantized_moe_token_b200 as moe
from conftest import ROOT


def _declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", src,
                             flags=re.M):
            name = m.group(1)
            if name not in ("if", "while", "for", "sizeof"):
                names.append(name)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ("w4a8_pack_weights", "fp8_quant_tokens", "moe_route_topk", "moe_w4a8_forward",
              "moe_router_logits", "w8a8_quant_weights", "moe_w8a8_forward",
              "moe_w8a8_workspace_bytes", "moe_w8a8_forward_profiled", "moe_router_topk",
              "moe_router_topk_workspace_bytes", "moe_w4a8_forward_router", "moe_w8a8_forward_router",
              "nvfp4_quant_weights", "moe_nvfp4_forward", "moe_nvfp4_workspace_bytes",
              "moe_nvfp4_forward_profiled", "moe_nvfp4_forward_router", "moe_hybrid_forward",
              "moe_hybrid_workspace_bytes", "moe_hybrid_forward_profiled",
              "moe_w4a8_workspace_bytes", "moe_last_device_status", "moe_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol():
    L = moe.lib()
    for n in _declared_functions():
        assert hasattr(L, n), n
        assert ctypes.cast(getattr(L, n), ctypes.c_void_p).value


def test_selftest_rejects_bad_limits():
    L = _L()
    assert L.moe_selftest_bounded_wait(10, None) == -1
    assert L.moe_selftest_bounded_wait(2_000_000_000, None) == -1


def test_status_strings():
    assert moe.moe_status_string(0) == "ok"
    assert "workspace" in moe.moe_status_string(-4)
    assert moe.moe_status_string(12345) == "unknown status"


def _L():
    return moe.lib()


def test_pack_rejects_bad_args():
    L = _L()
    p = ctypes.c_void_p(4096)
    assert L.w4a8_pack_weights(p, 10, 100, 128, p, p, None) == -2      # K not multiple of 128
    assert L.w4a8_pack_weights(p, 10, 256, 64, p, p, None) == -2       # group != 128
    assert L.w4a8_pack_weights(p, -1, 256, 128, p, p, None) == -1
    assert L.w4a8_pack_weights(None, 10, 256, 128, p, p, None) == -1
    assert L.w4a8_pack_weights(ctypes.c_void_p(4100), 10, 256, 128, p, p, None) == -3
    assert L.w4a8_pack_weights(p, 0, 256, 128, p, p, None) == 0          # no-op


def test_quant_rejects_bad_args():
    L = _L()
    p = ctypes.c_void_p(4096)
    assert L.fp8_quant_tokens(p, 4, 12, p, p, None) == -2                # H % 8
    assert L.fp8_quant_tokens(None, 4, 16, p, p, None) == -1
    assert L.fp8_quant_tokens(ctypes.c_void_p(4104), 4, 16, p, p, None) == -3
    assert L.fp8_quant_tokens(p, 0, 16, p, p, None) == 0


def test_route_rejects_bad_args():
    L = _L()
    p = ctypes.c_void_p(4096)
    ws = moe.moe_route_workspace_bytes(64, 256, 6)
    assert ws >= 256 and ws % 256 == 0
    assert moe.moe_route_workspace_bytes(64, 256, 9) == 0                # k > 8
    assert L.moe_route_topk(p, 64, 256, 9, p, p, p, p, p, p, ws, None) == -2
    assert L.moe_route_topk(p, 64, 4, 6, p, p, p, p, p, p, ws, None) == -2   # k > E
    assert L.moe_route_topk(p, 64, 2048, 6, p, p, p, p, p, p, ws, None) == -2
    assert L.moe_route_topk(p, 64, 256, 6, p, p, p, p, p, p, ws - 1, None) == -4
    assert L.moe_route_topk(p, 64, 256, 6, p, p, p, p, p, None, ws, None) == -4
    assert L.moe_route_topk(p, 64, 256, 6, p, p, p, p, p, ctypes.c_void_p(4096 + 16), ws, None) == -3
    assert L.moe_route_topk(None, 64, 256, 6, p, p, p, p, p, p, ws, None) == -1


def test_router_rejects_bad_args():
    L = _L()
    p = ctypes.c_void_p(4096)
    assert L.moe_router_logits(p, p, 4, 100, 8, p, None) == -2          # H % 8
    assert L.moe_router_logits(p, p, 4, 256, 2000, p, None) == -2       # E > 1024
    assert L.moe_router_logits(p, p, 4, 32768, 8, p, None) == -2        # H > 16384
    assert L.moe_router_logits(p, p, -1, 256, 8, p, None) == -1
    assert L.moe_router_logits(None, p, 4, 256, 8, p, None) == -1
    assert L.moe_router_logits(ctypes.c_void_p(4104), p, 4, 256, 8, p, None) == -3
    assert L.moe_router_logits(p, p, 0, 256, 8, p, None) == 0            # no-op


def test_forward_workspace_and_layout():
    s = moe.layer_struct(256, 4096, 2048)
    n8 = moe.moe_w4a8_workspace_bytes(s, 8, 6)
    n64 = moe.moe_w4a8_workspace_bytes(s, 64, 6)
    assert 0 < n8 < n64
    lay = moe.moe_w4a8_workspace_layout(s, 8, 6)
    assert lay["total"] == n8
    offs = [lay[k] for k in ("topk_ids", "topk_w", "expert_offsets", "sorted_pairs", "row_of_pair",
                             "xq", "s_x", "hq", "s_h")]
    assert all(o % 256 == 0 for o in offs) and len(set(offs)) == len(offs)
    assert max(offs) < n8
    assert moe.moe_w4a8_workspace_bytes(moe.layer_struct(256, 4000, 2048), 8, 6) == 0  # H % 128
    assert moe.moe_w4a8_workspace_bytes(moe.layer_struct(256, 4096, 2048, group=64), 8, 6) == 0
    shared = moe.layer_struct(256, 4096, 2048, n_shared=2, shared_N=2048)
    assert moe.moe_w4a8_workspace_bytes(shared, 8, 6) > n8


def test_forward_rejects_bad_args():
    L = _L()
    s = moe.layer_struct(8, 256, 128)
    p = ctypes.c_void_p(4096)
    # null weights
    assert L.moe_w4a8_forward(ctypes.byref(s), p, p, 4, 2, p, p, 1 << 20, None) == -1
    full = moe._binding._CLayer(8, 256, 128, 128, p, p, p, p, p, p, 0, 0, None, None, None)
    need = moe.moe_w4a8_workspace_bytes(full, 4, 2)
    assert L.moe_w4a8_forward(ctypes.byref(full), p, p, 4, 2, p, p, need - 1, None) == -4
    assert L.moe_w4a8_forward(ctypes.byref(full), p, p, 4, 2, p, ctypes.c_void_p(4096 + 128),
                              need, None) == -3
    assert L.moe_w4a8_forward(ctypes.byref(full), p, p, 4, 0, p, p, need, None) == -1
    assert L.moe_w4a8_forward(ctypes.byref(full), p, p, 0, 2, p, p, need, None) == 0
    assert L.moe_w4a8_forward(None, p, p, 4, 2, p, p, need, None) == -1


def test_router_topk_rejects_bad_args():
    L = _L()
    p = ctypes.c_void_p(4096)
    ws = moe.moe_router_topk_workspace_bytes(8, 256, 6)
    assert ws >= 256 and ws % 256 == 0
    assert moe.moe_router_topk_workspace_bytes(8, 256, 9) == 0          # k > 8
    assert L.moe_router_topk(p, p, 8, 100, 256, 6, p, p, p, p, ws, None) == -2     # H % 8
    assert L.moe_router_topk(p, p, 8, 256, 4, 6, p, p, p, p, ws, None) == -2       # k > E
    assert L.moe_router_topk(p, p, 8, 256, 256, 6, p, p, p, p, ws - 1, None) == -4
    assert L.moe_router_topk(p, p, 8, 256, 256, 6, None, p, p, p, ws, None) == -1
    assert L.moe_router_topk(p, p, 8, 256, 256, 6, p, p, p, ctypes.c_void_p(4096 + 64), ws, None) == -3
    assert L.moe_router_topk(p, p, 0, 256, 256, 6, p, p, p, p, ws, None) == 0
    full = moe._binding._CLayer(8, 256, 128, 128, p, p, p, p, p, p, 0, 0, None, None, None)
    need = moe.moe_w4a8_workspace_bytes(full, 4, 2)
    assert L.moe_w4a8_forward_router(ctypes.byref(full), p, None, 4, 2, p, p, need, None) == -1
    assert L.moe_w4a8_forward_router(ctypes.byref(full), p, ctypes.c_void_p(4098), 4, 2, p, p, need,
                                     None) == -3
    assert L.moe_w4a8_forward_router(ctypes.byref(full), p, p, 4, 2, p, p, need - 1, None) == -4


def test_w8a8_rejects_bad_args():
    L = _L()
    p = ctypes.c_void_p(4096)
    assert L.w8a8_quant_weights(p, 4, 12, p, p, None) == -2              # K % 8
    assert L.w8a8_quant_weights(None, 4, 16, p, p, None) == -1
    assert L.w8a8_quant_weights(p, 0, 16, p, p, None) == 0
    s8 = moe.layer8_struct(256, 4096, 2048)
    s4 = moe.layer_struct(256, 4096, 2048)
    assert moe.moe_w8a8_workspace_bytes(s8, 8, 6) == moe.moe_w4a8_workspace_bytes(s4, 8, 6) > 0
    l8, l4 = moe.moe_w8a8_workspace_layout(s8, 8, 6), moe.moe_w4a8_workspace_layout(s4, 8, 6)
    # the same plan; only the W4A8 layer's narrow (decode) tiles keep their codes in the
    # even/odd-nibble K order
    assert l8["act_order"] == 0 and l4["act_order"] == 1
    assert {k: v for k, v in l8.items() if k != "act_order"} == {k: v for k, v in l4.items() if k != "act_order"}
    assert moe.moe_w8a8_workspace_bytes(moe.layer8_struct(256, 4000, 2048), 8, 6) == 0
    assert L.moe_w8a8_forward(ctypes.byref(s8), p, p, 4, 2, p, p, 1 << 24, None) == -1   # null weights
    full = moe._binding._CLayer8(8, 256, 128, p, p, p, p, p, p, 0, 0, None, None, None)
    need = moe.moe_w8a8_workspace_bytes(full, 4, 2)
    assert L.moe_w8a8_forward(ctypes.byref(full), p, p, 4, 2, p, p, need - 1, None) == -4
    odd = moe._binding._CLayer8(8, 256, 128, p, p, p, ctypes.c_void_p(4098), p, p, 0, 0, None, None,
                                None)                                     # fp32 scales need 4 bytes
    assert L.moe_w8a8_forward(ctypes.byref(odd), p, p, 4, 2, p, p, need, None) == -3
    assert L.moe_w8a8_forward(ctypes.byref(full), p, p, 0, 2, p, p, need, None) == 0
    assert L.moe_w8a8_forward(None, p, p, 4, 2, p, p, need, None) == -1


def test_nvfp4_rejects_bad_args():
    L = _L()
    p = ctypes.c_void_p(4096)
    assert L.nvfp4_quant_weights(p, 2, 4, 24, p, p, p, None) == -2        # K % 16
    assert L.nvfp4_quant_weights(None, 2, 4, 32, p, p, p, None) == -1
    assert L.nvfp4_quant_weights(p, 0, 4, 32, p, p, p, None) == 0
    assert L.nvfp4_quant_weights(p, 2, 4, 32, ctypes.c_void_p(4100), p, p, None) == -3
    s4 = moe.layer4_struct(256, 4096, 2048)
    n4 = moe.moe_nvfp4_workspace_bytes(s4, 64, 6)
    assert n4 > moe.moe_w4a8_workspace_bytes(moe.layer_struct(256, 4096, 2048), 64, 6)
    assert moe.moe_nvfp4_workspace_layout(s4, 64, 6)["total"] == n4
    full = moe._binding._CLayer4(8, 256, 128, p, p, p, p, p, p, p, p, p, 0, 0, None, None, None)
    need = moe.moe_nvfp4_workspace_bytes(full, 4, 2)
    assert L.moe_nvfp4_forward(ctypes.byref(full), p, p, 4, 2, p, p, need - 1, None) == -4
    odd = moe._binding._CLayer4(8, 256, 128, p, p, p, ctypes.c_void_p(4100), p, p, p, p, p, 0, 0, None,
                                None, None)                           # block scales need 8 bytes
    assert L.moe_nvfp4_forward(ctypes.byref(odd), p, p, 4, 2, p, p, need, None) == -3
    nos2 = moe._binding._CLayer4(8, 256, 128, p, p, p, p, p, p, None, p, p, 0, 0, None, None, None)
    assert L.moe_nvfp4_forward(ctypes.byref(nos2), p, p, 4, 2, p, p, need, None) == -1
    assert L.moe_nvfp4_forward(ctypes.byref(full), p, p, 0, 2, p, p, need, None) == 0


def test_hybrid_rejects_bad_args():
    L = _L()
    p = ctypes.c_void_p(4096)
    H = moe._binding._CLayerH
    full = H(8, 256, 128, 2, 6, p, p, *([p] * 15), 0, 0, None, None, None)
    need = moe.moe_hybrid_workspace_bytes(full, 4, 2)
    assert need > 0
    assert L.moe_hybrid_forward(ctypes.byref(full), p, p, 4, 2, p, p, need - 1, None) == -4
    no_ids = H(8, 256, 128, 2, 6, None, p, *([p] * 15), 0, 0, None, None, None)
    assert L.moe_hybrid_forward(ctypes.byref(no_ids), p, p, 4, 2, p, p, need, None) == -1
    all_hot = H(8, 256, 128, 8, 0, p, None, *([p] * 9), *([None] * 6), 0, 0, None, None, None)
    assert L.moe_hybrid_forward(ctypes.byref(all_hot), p, p, 0, 2, p, p, need, None) == 0
    odd = H(8, 256, 128, 2, 6, p, p, *([p] * 3), ctypes.c_void_p(4100), p, p, *([p] * 9), 0, 0, None,
            None, None)                                               # hot block scales need 8 bytes
    assert L.moe_hybrid_forward(ctypes.byref(odd), p, p, 4, 2, p, p, need, None) == -3


def test_binding_has_no_fallback():
    src = open(os.path.join(ROOT, "bit_quantized_moe_token_b200", "_binding.py")).read()
    assert "oracle" not in src and "numpy" not in src
    for f in glob.glob(os.path.join(ROOT, "bit_quantized_moe_token_b200", "*.py")):
        assert "import oracle" not in open(f).read(), f


def test_ep_entry_points_reject_bad_args():
    L = _L()
    p = ctypes.c_void_p(4096)
    full = moe._binding._CLayer(8, 256, 128, 128, p, p, p, p, p, p, 0, 0, None, None, None)
    nd = moe.moe_ep_dispatch_workspace_bytes(full, 4, 2)
    assert 0 < nd < moe.moe_w4a8_workspace_bytes(full, 4, 2)
    assert moe.moe_ep_dispatch_workspace_bytes(full, 4, 9) == 0                    # k > E
    assert moe.moe_ep_experts_workspace_bytes(full, 40) == moe.moe_w4a8_workspace_bytes(full, 40, 1)
    assert moe.ep_record_bytes(256) == 272
    d = L.moe_ep_dispatch
    assert d(ctypes.byref(full), p, p, 4, 2, 3, p, p, p, nd, None) == -2            # 8 % 3 != 0
    assert d(ctypes.byref(full), p, p, 4, 2, 0, p, p, p, nd, None) == -1            # no ranks
    assert d(ctypes.byref(full), p, p, 4, 2, 16, p, p, p, nd, None) == -1           # more ranks than experts
    assert d(ctypes.byref(full), p, p, 4, 2, 2, None, p, p, nd, None) == -1         # no counts
    assert d(ctypes.byref(full), p, p, 4, 2, 2, p, None, p, nd, None) == -1         # no records
    assert d(ctypes.byref(full), p, p, 4, 2, 2, p, p, p, nd - 1, None) == -4
    assert d(ctypes.byref(full), p, p, 4, 2, 2, p, ctypes.c_void_p(4104), p, nd, None) == -3
    f = L.moe_ep_experts_forward
    ne = moe.moe_ep_experts_workspace_bytes(full, 40)
    assert f(ctypes.byref(full), p, 0, p, p, ne, None) == 0                          # no records: no-op
    assert f(ctypes.byref(full), None, 40, p, p, ne, None) == -1
    assert f(ctypes.byref(full), p, 40, p, p, ne - 1, None) == -4
    assert f(ctypes.byref(full), ctypes.c_void_p(4104), 40, p, p, ne, None) == -3   # records below 16 B
    assert f(ctypes.byref(moe.layer_struct(8, 256, 128)), p, 40, p, p, ne, None) == -1   # no weights
    c = L.moe_ep_combine
    assert c(ctypes.byref(full), p, p, 0, 2, p, p, nd, None) == 0                    # no tokens: no-op
    assert c(ctypes.byref(full), p, None, 4, 2, p, p, nd, None) == -1
    assert c(ctypes.byref(full), p, p, 4, 2, p, p, nd - 1, None) == -4
    assert c(ctypes.byref(full), p, p, 4, 2, ctypes.c_void_p(4104), p, nd, None) == -3
