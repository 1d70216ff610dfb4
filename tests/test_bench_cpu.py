"""The measurement arithmetic of bench.py on CPU: algorithmic bytes and FLOPs per launch, the
choice between the HBM and the tensor bound, the fractions against the peaks, and the rule that
an ncu summary only supplies `traffic` while the kernel sources it was taken on are unchanged.

Expected values are worked by hand from the layer shapes (H = 4096, N = 2048, K-groups of 128,
top-6 of 256 experts), not from bench.py's own formulas."""
import hashlib
import os
import re
from types import SimpleNamespace

import pytest

from conftest import ROOT


@pytest.fixture(scope="module")
def bench():
    import sys
    sys.path.insert(0, ROOT)
    import bench as b
    return b


@pytest.fixture(scope="module")
def wls():
    import synth
    return synth.WORKLOADS


def test_expert_bytes_by_format(bench, wls):
    wl = wls["decode_t8"]
    # W4A8: 2048 x 4096 nibbles = 4,194,304 B of codes per matrix, plus 2048 rows x 32 groups x
    # 2 B = 131,072 B of bf16 scales; gate and up together, down transposed (4096 rows x 16 groups)
    assert bench.expert_bytes(wl, "w4a8") == (2 * (4_194_304 + 131_072), 4_194_304 + 131_072)
    # W8A8: one byte per weight plus an fp32 scale per output row
    assert bench.expert_bytes(wl, "w8a8") == (2 * (8_388_608 + 8_192), 8_388_608 + 16_384)
    # NVFP4: half a byte per weight, one E4M3 scale per 16 weights, one fp32 scale2 per matrix
    assert bench.expert_bytes(wl, "nvfp4") == (2 * (4_194_304 + 524_288 + 4), 4_194_304 + 524_288 + 4)


def test_flops_per_pair(bench, wls):
    # gate and up: 2 x (2 FLOP x 4096 x 2048); down: 2 FLOP x 2048 x 4096
    assert bench.flops_per_pair(wls["decode_t8"]) == 2 * 2 * 4096 * 2048 + 2 * 2048 * 4096


def _roofline(bench, wl, touched, ms):
    fx = SimpleNamespace(fmt="w4a8", kname="test")
    return bench.gateup_roofline(wl, fx, [touched] * bench.N_BATCHES, [0] * bench.N_BATCHES, 4, ms,
                                 6546.6, 1662.9, "measured")


def test_decode_is_scored_against_hbm(bench, wls):
    r, layer_bytes = _roofline(bench, wls["decode_t8"], 40, 0.1)
    # 40 experts x 8,650,752 B in 0.1 ms = 3,460.3 GB/s of 6,546.6
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["algorithmic_bytes_per_launch"] == 346_030_080
    assert r["achieved"] == pytest.approx(3460.3, abs=0.05)
    assert r["frac"] == pytest.approx(3460.3008 / 6546.6, abs=1e-4)
    assert r["other_bound"]["bound"] == "tensor"
    # 48 pairs x 33,554,432 FLOP = 1,610,612,736 FLOP; ideal 52.9 us on HBM, 0.5 us on the FP8 peak
    assert r["other_bound"]["algorithmic_flops_per_launch"] == 1_610_612_736
    assert r["ideal_us"]["hbm"] == pytest.approx(52.9, abs=0.05)
    assert r["ideal_us"]["tensor"] == pytest.approx(0.5, abs=0.05)
    assert layer_bytes == pytest.approx(40 * (8_650_752 + 4_325_376))


def test_prefill_is_scored_against_the_fp8_peak(bench, wls):
    r, _ = _roofline(bench, wls["prefill_t16384_shared"], 256, 4.0)
    # 98,304 pairs x 33,554,432 FLOP = 3.2985e12 FLOP in 4 ms = 824.6 TFLOP/s of 2 x 1662.9
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["algorithmic_flops_per_launch"] == 98_304 * 33_554_432
    assert r["peak"] == pytest.approx(3325.8)
    assert r["achieved"] == pytest.approx(824.6, abs=0.05)
    assert r["frac"] == pytest.approx(824.634 / 3325.8, abs=1e-4)
    assert r["other_bound"]["bound"] == "hbm"


def _sources_sha(bench, fmt):
    h = hashlib.sha256()
    for f in bench.KERNEL_SOURCES[fmt]:
        with open(os.path.join(ROOT, "bit_quantized_moe_token_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


@pytest.mark.parametrize("fmt,workload", [("w4a8", "decode_t8"), ("w4a8", "prefill_t2048_zipf"),
                                          ("w4a8", "prefill_t16384_shared"), ("w8a8", "decode_t8"),
                                          ("nvfp4", "prefill_t2048_zipf")])
def test_profile_traffic_only_for_unchanged_sources(bench, fmt, workload):
    name = bench.PROFILE_FOR[(fmt, workload)]
    text = open(os.path.join(ROOT, "profiles", name)).read()
    recorded = re.search(r"^\s*sources_sha256:\s*(\S+)", text, flags=re.M).group(1)
    got = bench.ncu_traffic(workload, fmt, 1_000_000_000)
    if recorded == _sources_sha(bench, fmt):
        assert isinstance(got, int) and got > 0
    else:
        assert got is None


def test_profile_traffic_none_when_sources_differ(bench, monkeypatch):
    assert bench.ncu_traffic("no_such_workload", "w4a8", 1) is None
    monkeypatch.setitem(bench.KERNEL_SOURCES, "w4a8", bench.KERNEL_SOURCES["w4a8"] + ("quant.cuh",))
    assert bench.ncu_traffic("decode_t8", "w4a8", 1_000_000_000) is None
