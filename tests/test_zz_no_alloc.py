"""The allocation-free routing entry point (moe_route_topk_noalloc) against the allocating one.

Callers that cannot allocate device memory use moe_route_topk_noalloc, whose permutation scratch
lives in a fixed array inside the library.  This file runs last (pytest collects files in name
order), so a failure here leaves every other test already run; it also passes on its own in a
fresh process.
"""
import ctypes

import numpy as np
import pytest

import synth
from conftest import cuda_ok

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not cuda_ok():
        pytest.skip("no CUDA device")


def _outputs(T, E, k):
    import torch
    P = T * k
    return dict(ids=torch.empty(T, k, dtype=torch.int32, device="cuda"),
                w=torch.empty(T, k, dtype=torch.float32, device="cuda"),
                off=torch.empty(E + 1, dtype=torch.int32, device="cuda"),
                sp=torch.empty(P, dtype=torch.int32, device="cuda"),
                rop=torch.empty(P, dtype=torch.int32, device="cuda"))


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _call_noalloc(L, logits, k, o, stream):
    T, E = logits.shape
    return L.moe_route_topk_noalloc(_p(logits), T, E, k, _p(o["ids"]), _p(o["w"]), _p(o["off"]),
                                    _p(o["sp"]), _p(o["rop"]), stream)


@pytest.mark.parametrize("T,E,k", [(2048, 256, 6), (8, 256, 6), (1500, 64, 4), (16384, 256, 6)])
def test_noalloc_route_matches_allocating_route_twice(T, E, k):
    import torch
    import bit_quantized_moe_token_b200 as moe
    L = moe.lib()
    L.moe_route_topk_noalloc.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_int] + \
        [ctypes.c_void_p] * 6
    L.moe_route_topk_noalloc.restype = ctypes.c_int
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):                  # two calls in a row, different inputs
        logits = torch.from_numpy(synth.normal_f32(call, 424242 + T + E, T * E).reshape(T, E)).cuda()
        ref = _outputs(T, E, k)
        ws = torch.empty(moe.moe_route_workspace_bytes(T, E, k), dtype=torch.uint8, device="cuda")
        moe.moe_route_topk(logits, k, ref["ids"], ref["w"], ref["off"], ref["sp"], ref["rop"], ws)
        got = _outputs(T, E, k)
        assert _call_noalloc(L, logits, k, got, stream) == 0
        torch.cuda.synchronize()
        for key in ("ids", "off", "sp", "rop"):          # integer outputs: bit-exact
            assert torch.equal(got[key], ref[key]), key
        np.testing.assert_allclose(got["w"].cpu().numpy(), ref["w"].cpu().numpy(), rtol=1e-6, atol=0)
    assert moe.moe_last_device_status() == 0


def test_noalloc_route_rejects_sizes_beyond_its_scratch():
    import torch
    import bit_quantized_moe_token_b200 as moe
    L = moe.lib()
    L.moe_route_noalloc_max_scratch_bytes.restype = ctypes.c_size_t
    cap = L.moe_route_noalloc_max_scratch_bytes()
    T, E, k = 100_000, 1024, 8                         # 782 chunks x 1024 experts of counts
    assert moe.moe_route_workspace_bytes(T, E, k) > cap
    L.moe_route_topk_noalloc.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_int] + \
        [ctypes.c_void_p] * 6
    p = ctypes.c_void_p(1 << 20)
    assert L.moe_route_topk_noalloc(p, T, E, k, p, p, p, p, p, None) == -2   # MOE_ERR_UNSUPPORTED_SHAPE
