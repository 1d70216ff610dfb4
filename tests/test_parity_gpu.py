"""GPU parity: every entry point of libmoe_w4a8 (called through the C ABI) against the CPU
oracle on the same seeded inputs, under the layer's three rules (tests/parity.py)."""
import json
import os

import numpy as np
import pytest

import oracle
import synth
from conftest import cuda_ok
from parity import bf16_to_f32, check_fp8_codes, check_output_explained, output_errors

pytestmark = pytest.mark.gpu

if cuda_ok():
    import torch
    import bit_quantized_moe_token_b200 as moe
    from bit_quantized_moe_token_b200.synthetic import (device_inputs, device_layer, device_layer_nvfp4,
                                                        device_layer_w8a8)


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not cuda_ok():
        pytest.skip("no CUDA device")


# ---- host <-> device helpers -------------------------------------------------------------------

def to_dev_bf16(a_u16):
    return torch.from_numpy(np.ascontiguousarray(a_u16).view(np.int16)).cuda().view(torch.bfloat16)


def bits(t):
    """bf16 tensor -> uint16 numpy bits."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


# stored position p of an 8-column block holds column (0,2,4,6,1,3,5,7)[p]; this gathers them back
_UNPERM8 = np.argsort(np.array([0, 2, 4, 6, 1, 3, 5, 7]))


def ws_views(layer, ws, T, k):
    layout = (moe.moe_w8a8_workspace_layout if isinstance(layer, moe.Layer8) else
              moe.moe_nvfp4_workspace_layout if isinstance(layer, moe.Layer4) else
              moe.moe_hybrid_workspace_layout if isinstance(layer, moe.LayerH) else moe.moe_w4a8_workspace_layout)
    lay = layout(layer, T, k)
    P = T * k
    b = ws.cpu().numpy()
    def arr(off, dtype, n):
        return np.frombuffer(b[off:off + n * np.dtype(dtype).itemsize].tobytes(), dtype=dtype).copy()
    offsets = arr(lay["expert_offsets"], np.int32, layer.E + 1)
    def codes(off, rows, cols, which):
        c = arr(off, np.uint8, rows * cols).reshape(rows, cols)
        # which rows hold columns 0,2,4,6,1,3,5,7 of every 8-column block: all (act_order 1), or
        # for hq the rows of segments of at most 32 rows (act_order 2)
        if lay["act_order"] == 1:
            sel = np.ones(rows, bool)
        elif lay["act_order"] == 2 and which == "hq":
            seg = np.diff(offsets)
            sel = np.repeat(seg <= 32, seg)
        else:
            sel = np.zeros(rows, bool)
        c[sel] = c[sel].reshape(-1, cols // 8, 8)[:, :, _UNPERM8].reshape(-1, cols)
        return c
    return dict(ids=arr(lay["topk_ids"], np.int32, P).reshape(T, k),
                gates=arr(lay["topk_w"], np.float32, P).reshape(T, k),
                offsets=offsets,
                sorted_pairs=arr(lay["sorted_pairs"], np.int32, P),
                row_of_pair=arr(lay["row_of_pair"], np.int32, P),
                xq=codes(lay["xq"], T, layer.H, "xq"),
                s_x=arr(lay["s_x"], np.float32, T),
                hq=codes(lay["hq"], P, layer.N, "hq"),
                s_h=arr(lay["s_h"], np.float32, P))


# ---- generator -----------------------------------------------------------------------------------

def test_device_generator_matches_host():
    for name in ("tiny", "decode_t8", "prefill_t2048_zipf"):
        wl = synth.WORKLOADS[name]
        n = min(wl.T, 64)
        x, lg = device_inputs(wl, T=n)
        assert np.array_equal(bits(x), synth.tokens(wl, 0, n)), name
        assert np.array_equal(lg.cpu().numpy(), synth.logits(wl, 0, n)), name
    wl = synth.WORKLOADS["decode_t8"]
    w = torch.empty(wl.N, wl.H, dtype=torch.bfloat16, device="cuda")
    synth.dev_weight(wl.seed, synth.weight_stream(5, "gate"), w)
    torch.cuda.synchronize()
    assert np.array_equal(bits(w), synth.expert_weight(wl, 5, "gate"))


# ---- S0 ----------------------------------------------------------------------------------------

def _f32_to_bf16_bits(x):
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def test_pack_bitexact_random_and_edge_groups():
    rng = np.random.default_rng(11)
    w = (rng.standard_normal((300, 1024)) * 0.02).astype(np.float32)
    w[0, :128] = 0.0                                   # zero group -> scale 0, codes 0
    w[1, :128] = 0.0
    w[1, 5] = 1e-40                                    # subnormal amax: bf16(amax/7) rounds to 0
    w[2, 128:256] *= 1e30                              # huge values
    w[3, :128] = -0.0                                  # negative zeros
    w[4, :8] = np.array([0.4375, 0.21875, 0.15625, -0.03125, -0.4375, 0, 0, 0])  # exact ties
    w[4, 8:128] = 0
    w[5, :128] = rng.choice([-1.0, 1.0], 128) * 7 * 2.0 ** -8   # all codes +-7
    wb = _f32_to_bf16_bits(w)
    packed_ref, scales_ref, _ = oracle.rtn_pack(wb)
    wd = to_dev_bf16(wb)
    packed, scales = moe.pack_expert_weights(wd)
    torch.cuda.synchronize()
    assert np.array_equal(packed.cpu().numpy(), packed_ref)
    assert np.array_equal(bits(scales), scales_ref)


def test_pack_bitexact_seeded_expert():
    wl = synth.WORKLOADS["decode_t8"]
    for proj in ("gate", "down"):
        wb = synth.expert_weight(wl, 17, proj)
        p_ref, s_ref, _ = oracle.rtn_pack(wb)
        p, s = moe.pack_expert_weights(to_dev_bf16(wb))
        assert np.array_equal(p.cpu().numpy(), p_ref)
        assert np.array_equal(bits(s), s_ref)


# ---- S1 ----------------------------------------------------------------------------------------

def test_quant_tokens_bitexact():
    wl = synth.WORKLOADS["decode_t64"]
    x = synth.tokens(wl)
    xo = synth.tokens(synth.WORKLOADS["decode_t8"])
    extra = np.zeros((4, wl.H), np.float32)
    extra[1, :] = 1e-30                                # tiny row
    extra[2, :] = np.linspace(-3, 3, wl.H)
    extra[3, ::2] = 1.0
    extra[3, 1::2] = 2.0 ** -12                        # values that underflow to +-0 codes
    extra[3, 3] = -(2.0 ** -12)
    xs = np.concatenate([x, xo, _f32_to_bf16_bits(extra)])
    q_ref, s_ref = oracle.quant_tokens(xs)
    xd = to_dev_bf16(xs)
    q = torch.empty(xs.shape, dtype=torch.uint8, device="cuda")
    s = torch.empty(xs.shape[0], dtype=torch.float32, device="cuda")
    moe.fp8_quant_tokens(xd, q, s)
    assert np.array_equal(s.cpu().numpy(), s_ref)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    tiny = synth.tokens(synth.WORKLOADS["tiny"])
    q_ref, s_ref = oracle.quant_tokens(tiny)
    q = torch.empty(tiny.shape, dtype=torch.uint8, device="cuda")
    s = torch.empty(tiny.shape[0], dtype=torch.float32, device="cuda")
    moe.fp8_quant_tokens(to_dev_bf16(tiny), q, s)
    assert np.array_equal(q.cpu().numpy(), q_ref) and np.array_equal(s.cpu().numpy(), s_ref)


# ---- S2 + S3 -----------------------------------------------------------------------------------

ROUTE_CASES = [(16, 8, 2, None), (8, 256, 6, None), (64, 256, 6, None), (700, 256, 6, None),
               (2048, 256, 6, "prefill_t2048_zipf"), (3, 1, 1, None), (5, 1024, 8, None),
               (1000, 33, 3, None), (1, 256, 6, None), (4097, 7, 1, None)]


@pytest.mark.parametrize("T,E,k,wlname", ROUTE_CASES)
def test_route_bitexact(T, E, k, wlname):
    if wlname:
        logits = synth.logits(synth.WORKLOADS[wlname])
    else:
        logits = synth.normal_f32(0, 9000 + T * 7 + E, T * E).reshape(T, E)
        if E >= 4:
            logits[: T // 2, 1] = logits[: T // 2, 3]     # ties, lower index first
    ids_ref, g_ref = oracle.route_topk(logits, k)
    off_ref, sp_ref, rop_ref = oracle.permute(ids_ref, E)
    ld = torch.from_numpy(logits).cuda()
    P = T * k
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    g = torch.empty(T, k, dtype=torch.float32, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    sp = torch.empty(P, dtype=torch.int32, device="cuda")
    rop = torch.empty(P, dtype=torch.int32, device="cuda")
    ws = torch.empty(moe.moe_route_workspace_bytes(T, E, k), dtype=torch.uint8, device="cuda")
    moe.moe_route_topk(ld, k, ids, g, off, sp, rop, ws)
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    assert np.array_equal(off.cpu().numpy(), off_ref)
    assert np.array_equal(sp.cpu().numpy(), sp_ref)
    assert np.array_equal(rop.cpu().numpy(), rop_ref)
    np.testing.assert_allclose(g.cpu().numpy(), g_ref, rtol=1e-6, atol=0)


# ---- the layer: small shapes, everything compared ------------------------------------------------

def _host_layer_and_dev(E, H, N, seed, n_shared=0, shared_N=0):
    """Seeded random layer: packed on the host by the oracle and on the GPU by the library."""
    rng_stream = 50_000 + seed * 10
    gw = synth.normal_bf16(seed, rng_stream + 0, E * N * H, 0.02).reshape(E, N, H)
    uw = synth.normal_bf16(seed, rng_stream + 1, E * N * H, 0.02).reshape(E, N, H)
    dw = synth.normal_bf16(seed, rng_stream + 2, E * H * N, 0.02).reshape(E, H, N)
    g = 128
    gp, gs = zip(*[oracle.rtn_pack(gw[e], g)[:2] for e in range(E)])
    up, us = zip(*[oracle.rtn_pack(uw[e], g)[:2] for e in range(E)])
    dp, ds = zip(*[oracle.rtn_pack(dw[e], g)[:2] for e in range(E)])
    sh = {}
    shd = {}
    if n_shared:
        for i, key in enumerate(("sh_gate", "sh_up", "sh_down")):
            shape = (n_shared, shared_N, H) if i < 2 else (n_shared, H, shared_N)
            a = synth.normal_bf16(seed, rng_stream + 3 + i, int(np.prod(shape)), 0.02).reshape(shape)
            sh[key] = a
            shd[key] = to_dev_bf16(a)
    hl = oracle.Layer(E, H, N, np.stack(gp), np.stack(up), np.stack(dp), np.stack(gs),
                      np.stack(us), np.stack(ds), **sh)
    dl = moe.make_layer(to_dev_bf16(gw), to_dev_bf16(uw), to_dev_bf16(dw), **shd)
    torch.cuda.synchronize()
    assert np.array_equal(dl.gate_packed.cpu().numpy(), hl.gate_packed)
    assert np.array_equal(bits(dl.down_scales), hl.down_scales)
    return hl, dl


def _report(**kv):
    """One JSON line per parity check (the test, worst output error as a fraction of rule 3's
    tolerance, FP8 code differences) appended to $MOE_PARITY_REPORT when it is set."""
    path = os.environ.get("MOE_PARITY_REPORT")
    if path:
        kv["test"] = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
        with open(path, "a") as f:
            f.write(json.dumps(kv) + "\n")


def _check_output_rules(hl, x, logits, k, got_out, ref, gpu_hq_pairs, gpu_sh_pairs, allow=None):
    """Rule 3 against the oracle alone.  `allow` = (format and seeded case, cap): only a test
    that names the case needing it gets rule 2's allowance for outputs of tokens whose
    requantized codes differ (tests/parity.py), and for at most `cap` outputs.  Returns the
    number of outputs that needed the allowance."""
    ratio = output_errors(got_out, ref["out"])
    worst = float(ratio.max(initial=0.0))
    n_bad = int((ratio > 1.0).sum())
    _report(worst_out_err_over_tol=round(worst, 4), outputs=int(ratio.size), out_of_tol=n_bad,
            allowance=None if allow is None else allow[0])
    if n_bad == 0:
        return 0
    assert allow is not None, f"{n_bad} outputs out of tolerance; worst {worst:.3f}x tol"
    T = x.shape[0]
    ref_pairs = ref["hq"][ref["row_of_pair"]]
    flipped = (gpu_hq_pairs != ref_pairs).reshape(T, -1).any(axis=1)
    alt, _ = oracle.moe_forward_given_h(hl, x, logits, k, gpu_hq_pairs, gpu_sh_pairs)
    return check_output_explained(got_out, ref["out"], alt, flipped, max_explained=allow[1])


def _run_and_compare(hl, dl, x, logits, k, allow=None):
    T = x.shape[0]
    ref = oracle.moe_forward(hl, x, logits, k)
    xd, ld = to_dev_bf16(x), torch.from_numpy(logits).cuda()
    ws = moe.alloc_workspace(dl, T, k)
    out = moe.forward(dl, xd, ld, k, ws=ws)
    torch.cuda.synchronize()
    assert moe.moe_last_device_status() == 0
    v = ws_views(dl, ws, T, k)
    for key in ("ids", "offsets", "sorted_pairs", "row_of_pair"):
        assert np.array_equal(v[key], ref[key]), key
    np.testing.assert_allclose(v["gates"], ref["gates"], rtol=1e-6)
    # first-stage FP8: codes and scales of every token are exact
    assert np.array_equal(v["xq"], ref["xq"])
    assert np.array_equal(v["s_x"], ref["s_x"])
    n_diff, frac = check_fp8_codes(v["hq"], ref["hq"])
    _report(hq_codes=int(v["hq"].size), hq_diff=n_diff)
    np.testing.assert_allclose(v["s_h"], ref["s_h"], rtol=2e-5)
    n_explained = _check_output_rules(hl, x, logits, k, bits(out), ref, v["hq"][v["row_of_pair"]],
                                      v["s_h"][v["row_of_pair"]], allow)
    return dict(hq_diff=n_diff, hq_frac=frac, explained=n_explained, out=bits(out))


def test_forward_tiny_workload():
    wl = synth.WORKLOADS["tiny"]
    hl = oracle.pack_workload_layer(wl)
    dl = device_layer(wl)
    assert np.array_equal(dl.up_packed.cpu().numpy(), hl.up_packed)
    r1 = _run_and_compare(hl, dl, synth.tokens(wl), synth.logits(wl), wl.k)
    r2 = _run_and_compare(hl, dl, synth.tokens(wl), synth.logits(wl), wl.k)
    assert np.array_equal(r1["out"], r2["out"])        # deterministic


@pytest.mark.parametrize("E,H,N,k,T", [(5, 384, 256, 3, 37), (1, 256, 128, 1, 9), (8, 256, 128, 2, 1),
                                       (16, 512, 384, 8, 130), (3, 1024, 128, 2, 700),
                                       (64, 1024, 1024, 6, 16), (4, 512, 256, 2, 500)])
def test_forward_ragged_shapes(E, H, N, k, T):
    hl, dl = _host_layer_and_dev(E, H, N, seed=E * 7 + T)
    x = synth.normal_bf16(3, 777 + T, T * H).reshape(T, H)
    logits = synth.normal_f32(3, 778 + T, T * E).reshape(T, E)
    _run_and_compare(hl, dl, x, logits, k)


@pytest.mark.parametrize("E,H,N,k,T,skew", [(16, 4096, 2048, 2, 400, 3.0), (32, 4096, 2048, 4, 600, 2.0),
                                              (8, 4096, 2048, 2, 600, 0.0), (16, 256, 128, 2, 260, 0.0),
                                              (8, 1024, 1024, 2, 600, 0.0)])
def test_forward_split_short_segments(E, H, N, k, T, skew):
    """Layers on 128-row tiles at the model's depths (H, N >= 2048) run their segments of at most
    32 rows on 32-row tiles (unsigned widening, sorted rows in its K order) and the others on
    128-row tiles: skewed routing gives both kinds in one layer (the third case, uniform, leaves the
    narrow launch empty).  The last two layers are too shallow for the split and stay on 128-row
    tiles: the 256 x 128 one put an output at 2.8 x the tolerance when it split (0.78 x unsplit).
    The 1024 x 1024 one has, split or not, one requantized code one step from the oracle's (rule 2),
    which moves two outputs of its token to 1.2 x the tolerance: the only W4A8 case that needs the
    named allowance (a step of one of N = 1024 activations weighs 2 x what it does at 2048)."""
    hl, dl = _host_layer_and_dev(E, H, N, seed=31 + E, n_shared=1, shared_N=128)
    x = synth.normal_bf16(33, 73_000, T * H, 1.0).reshape(T, H)
    logits = synth.normal_f32(33, 73_001, T * E, 1.0).reshape(T, E)
    logits += (skew * np.linspace(1.0, 0.0, E)).astype(np.float32)   # early experts preferred
    lay = moe.moe_w4a8_workspace_layout(dl, T, k)
    assert lay["act_order"] == (2 if H >= 2048 and N >= 2048 else 0)
    allow = ("w4a8 1024 x 1024 uniform, layer seed 39, inputs seed 33", 4) if (H, N) == (1024, 1024) else None
    r = _run_and_compare(hl, dl, x, logits, k, allow=allow)
    seg = np.diff(oracle.moe_forward(hl, x, logits, k)["offsets"])
    if skew > 0 or H < 1024:
        assert (seg[seg > 0] <= 32).any() and (seg > 32).any()   # both kinds of segment
    _report(short_segments=int(((seg > 0) & (seg <= 32)).sum()), long_segments=int((seg > 32).sum()))
    assert r["hq_frac"] <= 1e-3


def _random_nibble_layer(E, H, N, seed):
    """Packed words of uniformly random nibbles (so code -8, nibble 0, is as common as any other
    code: pack-quantized storage allows it although RTN never writes it) and random bf16 group
    scales, built directly as words and given unchanged to the oracle and the GPU.  A few rows
    are set to all -8, all +7 and alternating -8 / +7 codes."""
    rng = np.random.default_rng(seed)
    def words(rows, K):
        w = rng.integers(0, 2 ** 32, size=(E, rows, K // 8), dtype=np.uint64).astype(np.uint32)
        w[:, 0, :] = 0x00000000                        # every code -8
        w[:, 1, : K // 16] = 0xFFFFFFFF                # +7 in the first half of the row
        w[:, 2, :] = 0xF0F0F0F0                        # -8, +7, -8, +7, ...
        return w.view(np.int32)
    def scales(rows, K):
        return _f32_to_bf16_bits(rng.uniform(0.003, 0.012, size=(E, rows, K // 128)))
    gp, up, dp = words(N, H), words(N, H), words(H, N)
    gs, us, ds = scales(N, H), scales(N, H), scales(H, N)
    hl = oracle.Layer(E, H, N, gp, up, dp, gs, us, ds)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    dl = moe.Layer(E, H, N, dev(gp), dev(up), dev(dp), dev(gs.view(np.int16)).view(torch.bfloat16),
                   dev(us.view(np.int16)).view(torch.bfloat16), dev(ds.view(np.int16)).view(torch.bfloat16))
    return hl, dl


# token tiles of 16 and 32 rows (decode: unsigned widening of gate/up, gathered rows) and of 128
# and 192 rows (prefill: signed widening), each on packed words in which nibble 0 (code -8) is
# as frequent as every other nibble
@pytest.mark.parametrize("E,H,N,k,T", [(64, 512, 256, 6, 8), (64, 512, 256, 6, 64), (16, 512, 256, 6, 40),
                                       (4, 512, 256, 2, 100), (2, 512, 256, 1, 400)])
def test_forward_code_minus8(E, H, N, k, T):
    hl, dl = _random_nibble_layer(E, H, N, seed=E + T)
    assert (oracle.unpack(hl.gate_packed[0], H) == -8).mean() > 0.05
    x = synth.normal_bf16(12, 700 + T, T * H).reshape(T, H)
    logits = synth.normal_f32(12, 701 + T, T * E).reshape(T, E)
    logits[:, :3] += 4.0                               # the all -8 / +7 rows' experts are routed
    _run_and_compare(hl, dl, x, logits, k)


# the largest supported dimensions: H = 16384 (128 K-groups), N = 8192, E = 1024 with top-8
@pytest.mark.parametrize("w8", [False, True])
@pytest.mark.parametrize("E,H,N,k,T", [(2, 16384, 256, 1, 5), (2, 256, 8192, 2, 3), (1024, 256, 128, 8, 40)])
def test_forward_max_shapes(w8, E, H, N, k, T):
    hl, dl = (_host_layer_and_dev_w8a8 if w8 else _host_layer_and_dev)(E, H, N, seed=E + H + N)
    x = synth.normal_bf16(9, 860 + T, T * H).reshape(T, H)
    logits = synth.normal_f32(9, 861 + T, T * E).reshape(T, E)
    _run_and_compare(hl, dl, x, logits, k)


def test_forward_nan_logits_route_to_valid_experts():
    """NaN logits are outside the input domain; the GPU ranks them as -inf, so every selected
    id is a valid expert, and a NaN expert is never chosen while a finite one is left."""
    hl, dl = _host_layer_and_dev(8, 256, 128, seed=77)
    T, k = 6, 2
    x = synth.normal_bf16(10, 850, T * 256).reshape(T, 256)
    logits = synth.normal_f32(10, 851, T * 8).reshape(T, 8)
    logits[0, :] = np.nan                               # all NaN: still k valid ids
    logits[1, 3] = np.nan
    logits[2, :7] = np.nan                              # one finite expert: it is chosen first
    xd, ld = to_dev_bf16(x), torch.from_numpy(logits).cuda()
    ws = moe.alloc_workspace(dl, T, k)
    out = moe.forward(dl, xd, ld, k, ws=ws)
    torch.cuda.synchronize()
    assert moe.moe_last_device_status() == 0
    ids = ws_views(dl, ws, T, k)["ids"]
    assert ((ids >= 0) & (ids < 8)).all()
    assert all(len(set(r)) == k for r in ids.tolist())
    assert 3 not in ids[1].tolist()
    assert ids[2, 0] == 7
    finite = ~np.isnan(logits).any(axis=1)
    ref_ids, _ = oracle.route_topk(np.where(np.isnan(logits), -np.inf, logits).astype(np.float32), k)
    assert np.array_equal(ids[finite], ref_ids[finite])
    assert np.isfinite(bf16_to_f32(bits(out))[finite]).all()


def test_forward_shared_experts_small():
    hl, dl = _host_layer_and_dev(4, 256, 128, seed=5, n_shared=2, shared_N=256)
    T = 21
    x = synth.normal_bf16(4, 901, T * 256).reshape(T, 256)
    logits = synth.normal_f32(4, 902, T * 4).reshape(T, 4)
    _run_and_compare(hl, dl, x, logits, 2)


def test_forward_zero_tokens_and_zero_rows():
    hl, dl = _host_layer_and_dev(4, 256, 128, seed=9)
    x = synth.normal_bf16(5, 903, 6 * 256).reshape(6, 256)
    x[2, :] = 0                                        # zero row: s_x = 0, codes 0, output 0
    logits = synth.normal_f32(5, 904, 6 * 4).reshape(6, 4)
    r = _run_and_compare(hl, dl, x, logits, 2)
    assert not bf16_to_f32(r["out"][2]).any()
    xd = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    ld = torch.empty(0, 4, dtype=torch.float32, device="cuda")
    out = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    moe.moe_w4a8_forward(dl, xd, ld, 2, out, torch.empty(256, dtype=torch.uint8, device="cuda"))


# ---- router logits (the step upstream of top-k) ---------------------------------------------------

@pytest.mark.parametrize("T,E,H", [(1, 256, 4096), (8, 256, 4096), (37, 20, 1000), (300, 256, 1024),
                                   (2048, 256, 4096)])
def test_router_logits_vs_oracle(T, E, H):
    """CUDA-core path for small T, tensor-core path for T >= 256: logits within the fp32
    summation bound of the oracle's, top-k selection equal wherever the oracle's margin at the
    k-th place exceeds that bound."""
    x = synth.normal_bf16(6, 990 + T, T * H).reshape(T, H)
    wr = synth.normal_bf16(6, 991 + E, E * H, 1.0 / np.sqrt(H)).reshape(E, H)
    ref = oracle.router_logits(x, wr).astype(np.float64)
    got = torch.empty(T, E, dtype=torch.float32, device="cuda")
    moe.moe_router_logits(to_dev_bf16(x), to_dev_bf16(wr), got)
    torch.cuda.synchronize()
    g = got.cpu().numpy().astype(np.float64)
    xa = np.abs(bf16_to_f32(x).astype(np.float64))
    wa = np.abs(bf16_to_f32(wr).astype(np.float64))
    bound = 2 * H * 2.0 ** -24 * (xa @ wa.T) + 1e-30     # both sums within H*2^-24*sum|xw| of exact
    assert np.all(np.abs(g - ref) <= bound)
    # the selection is unique wherever the oracle's gap at the k-th place exceeds twice the
    # largest logit difference seen; there the ids must agree
    k = min(6, E)
    ids_ref, _ = oracle.route_topk(ref.astype(np.float32), k)
    ids_got, _ = oracle.route_topk(g.astype(np.float32), k)
    srt = -np.sort(-ref, axis=1)
    margin = srt[:, k - 1] - (srt[:, k] if k < E else -np.inf)
    clear = margin > 2 * np.abs(g - ref).max() + 1e-12
    assert clear.sum() >= 0.8 * T
    assert np.array_equal(ids_got[clear], ids_ref[clear])


@pytest.mark.parametrize("T,E,H,k", [(1, 256, 4096, 6), (8, 256, 4096, 6), (16, 64, 512, 8),
                                     (37, 20, 1000, 3), (300, 256, 1024, 6), (2048, 256, 4096, 6),
                                     (70, 1000, 256, 2)])
def test_router_topk_fused(T, E, H, k):
    """Router + top-k in one call: the logits equal moe_router_logits' bit for bit (same kernels,
    same summation order), and the ids / gates are the oracle's top-k of those logits (ids exact;
    gates to the last bits of expf)."""
    x = synth.normal_bf16(7, 880 + T, T * H).reshape(T, H)
    wr = synth.normal_bf16(7, 881 + E, E * H, 1.0 / np.sqrt(H)).reshape(E, H)
    xd, wd = to_dev_bf16(x), to_dev_bf16(wr)
    lg = torch.empty(T, E, dtype=torch.float32, device="cuda")
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    gw = torch.empty(T, k, dtype=torch.float32, device="cuda")
    ws = torch.full((moe.moe_router_topk_workspace_bytes(T, E, k),), 0xAB, dtype=torch.uint8, device="cuda")
    for _ in range(2):                                 # the counters are reused by the second call
        moe.moe_router_topk(xd, wd, k, lg, ids, gw, ws)
    lg2 = torch.empty(T, E, dtype=torch.float32, device="cuda")
    moe.moe_router_logits(xd, wd, lg2)
    torch.cuda.synchronize()
    assert moe.moe_last_device_status() == 0
    g = lg.cpu().numpy()
    assert np.array_equal(g.view(np.uint32), lg2.cpu().numpy().view(np.uint32))
    ids_ref, gates_ref = oracle.route_topk(g, k)
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    np.testing.assert_allclose(gw.cpu().numpy(), gates_ref, rtol=1e-6)
    ref = oracle.router_logits(x, wr).astype(np.float64)
    bound = 2 * H * 2.0 ** -24 * (np.abs(bf16_to_f32(x).astype(np.float64)) @
                                  np.abs(bf16_to_f32(wr).astype(np.float64)).T) + 1e-30
    assert np.all(np.abs(g.astype(np.float64) - ref) <= bound)


@pytest.mark.parametrize("w8", [False, True, "nvfp4"])
@pytest.mark.parametrize("E,H,N,k,T", [(16, 256, 128, 2, 8), (16, 256, 128, 2, 40),
                                       (16, 256, 128, 2, 300), (128, 256, 128, 2, 300)])
def test_forward_router_matches_logits_path(w8, E, H, N, k, T):
    """The layer fed by the router weight equals, bit for bit, the layer fed by the logits that
    moe_router_logits computes (decode front: router + quantization + top-k in one kernel;
    16 < T: fused router + top-k, then quantization; E = 128, T = 300: tensor-core router)."""
    make = (_host_layer_and_dev_nvfp4 if w8 == "nvfp4" else _host_layer_and_dev_w8a8 if w8
            else _host_layer_and_dev)
    hl, dl = make(E, H, N, seed=30 + E + T)
    x = synth.normal_bf16(8, 870 + T, T * H).reshape(T, H)
    wr = synth.normal_bf16(8, 871 + E, E * H, 1.0 / np.sqrt(H)).reshape(E, H)
    xd, wd = to_dev_bf16(x), to_dev_bf16(wr)
    lg = torch.empty(T, E, dtype=torch.float32, device="cuda")
    moe.moe_router_logits(xd, wd, lg)
    ws_a, ws_b = moe.alloc_workspace(dl, T, k), moe.alloc_workspace(dl, T, k)
    out_a = moe.forward(dl, xd, lg, k, ws=ws_a)
    out_b = torch.empty_like(out_a)
    (moe.moe_nvfp4_forward_router if w8 == "nvfp4" else moe.moe_w8a8_forward_router if w8
     else moe.moe_w4a8_forward_router)(dl, xd, wd, k, out_b, ws_b)
    torch.cuda.synchronize()
    assert moe.moe_last_device_status() == 0
    assert np.array_equal(bits(out_a), bits(out_b))
    va, vb = ws_views(dl, ws_a, T, k), ws_views(dl, ws_b, T, k)
    for key in ("ids", "offsets", "sorted_pairs", "xq", "s_x", "hq", "s_h"):
        assert np.array_equal(va[key], vb[key]), key
    # and the routing is the oracle's top-k of those logits
    ids_ref, _ = oracle.route_topk(lg.cpu().numpy(), k)
    assert np.array_equal(vb["ids"], ids_ref)


def test_router_logits_zero_tokens():
    wr = torch.zeros(8, 64, dtype=torch.bfloat16, device="cuda")
    moe.moe_router_logits(torch.empty(0, 64, dtype=torch.bfloat16, device="cuda"), wr,
                          torch.empty(0, 8, dtype=torch.float32, device="cuda"))


# ---- the layer at full size: every token at decode, hundreds at prefill ----------------------------

FULL = ["decode_t8", "decode_t64", "prefill_t2048_zipf", "prefill_t16384_shared"]
FULL_WL = "prefill_t16384_shared"          # the full-size configs share its routed-expert weights


def _boundary_tokens(v, T, k, n_min, tile_rows, rng):
    """Tokens of a batch whose routed rows sit where token tiles start and end: the first and
    last rows of the six longest expert segments and the rows on both sides of each tile
    boundary inside them, the first and last rows of the last (partly filled) tile of 48 other
    segments, every token routed to a one-row segment; then random tokens up to n_min."""
    off, sp = v["offsets"], v["sorted_pairs"]
    lens = np.diff(off)
    rows = set()
    for e in np.argsort(-lens, kind="stable")[:6]:
        r0, r1 = int(off[e]), int(off[e + 1])
        if r1 > r0:
            rows |= {r0, r1 - 1}
            for bn in tile_rows:
                for b in range(r0 + bn, r1, bn):
                    rows |= {b - 1, b}
    live = np.flatnonzero(lens > 0)
    for e in rng.permutation(live)[:48]:
        r0, r1 = int(off[e]), int(off[e + 1])
        rows.add(r1 - 1)
        for bn in tile_rows:
            rows.add(r0 + (r1 - r0 - 1) // bn * bn)
    for e in np.flatnonzero(lens == 1):
        rows.add(int(off[e]))
    toks = {int(sp[r]) // k for r in rows}
    while len(toks) < min(n_min, T):
        toks.add(int(rng.integers(0, T)))
    return sorted(toks)


class _HostLayers:
    """The oracle's copies of the full-size weights, packed expert by expert as tests need them
    (one per format; the routed weights of every full-size config are the same draws)."""

    def __init__(self):
        self.layers, self.done = {}, {}

    def get(self, fmt, experts, wl):
        build = {"w4a8": oracle.pack_workload_layer, "w8a8": oracle.quant_workload_layer_w8a8,
                 "nvfp4": oracle.quant_workload_layer_nvfp4}[fmt]
        full = synth.WORKLOADS[FULL_WL]
        if fmt not in self.layers:
            self.layers[fmt] = build(full, experts=[])
            self.done[fmt] = set()
        todo = sorted(set(experts) - self.done[fmt])
        if todo:
            build(full, experts=todo, into=self.layers[fmt])
            self.done[fmt] |= set(todo)
        L = self.layers[fmt]
        if not wl.n_shared:                            # the same routed weights, no shared experts
            import copy
            L = copy.copy(L)
            L.sh_gate = L.sh_up = L.sh_down = None
            L.n_shared = L.shared_N = 0
        return L


@pytest.fixture(scope="module")
def host_layers():
    return _HostLayers()


def _full_size_check(name, dl, fmt, host_layers, n_batches=1, n_prefill_tokens=256, tile_rows=(128, 192),
                     allow=None):
    """The layer at full size on the GPU; every token of `n_batches` batches at decode (T <= 64),
    at prefill at least `n_prefill_tokens` tokens chosen at token-tile boundaries, compared with
    the oracle on those tokens (tokens are independent, so the oracle's sub-batch gives the same
    rows) under the three rules; routing properties on the whole batch."""
    wl = synth.WORKLOADS[name]
    rng = np.random.default_rng(wl.T)
    picks = []                                         # (first token of the batch, tokens, views, out)
    for b in range(n_batches):
        t0 = b * wl.T
        x, lg = device_inputs(wl, t0=t0, T=wl.T)
        ws = moe.alloc_workspace(dl, wl.T, wl.k)
        out = moe.forward(dl, x, lg, wl.k, ws=ws)
        torch.cuda.synchronize()
        assert moe.moe_last_device_status() == 0
        v = ws_views(dl, ws, wl.T, wl.k)
        P = wl.P
        off = v["offsets"]
        assert off[0] == 0 and off[-1] == P and np.all(np.diff(off) >= 0)
        assert np.array_equal(np.sort(v["sorted_pairs"]), np.arange(P))
        assert np.array_equal(v["row_of_pair"][v["sorted_pairs"]], np.arange(P))
        seg = np.repeat(np.arange(wl.E), np.diff(off))
        assert np.array_equal(v["ids"].reshape(-1)[v["sorted_pairs"]], seg)
        for e in range(wl.E):
            s_ = v["sorted_pairs"][off[e]:off[e + 1]]
            assert np.all(np.diff(s_) > 0)
        outb = bits(out)
        assert np.isfinite(bf16_to_f32(outb)).all()
        toks = (list(range(wl.T)) if wl.T <= 64 else
                _boundary_tokens(v, wl.T, wl.k, n_prefill_tokens, tile_rows, rng))
        picks.append((t0, toks, v, outb))
        del ws, out
    xs = np.concatenate([synth.tokens(wl, t0 + t, 1) for t0, toks, _, _ in picks for t in toks])
    ls = np.concatenate([synth.logits(wl, t0 + t, 1) for t0, toks, _, _ in picks for t in toks])
    ids = np.concatenate([v["ids"][toks] for _, toks, v, _ in picks])
    hl = host_layers.get(fmt, sorted(set(ids.reshape(-1).tolist())), wl)
    ref = oracle.moe_forward(hl, xs, ls, wl.k)
    assert np.array_equal(ids, ref["ids"])
    np.testing.assert_allclose(np.concatenate([v["gates"][toks] for _, toks, v, _ in picks]), ref["gates"],
                               rtol=1e-6)
    assert np.array_equal(np.concatenate([v["xq"][toks] for _, toks, v, _ in picks]), ref["xq"])
    assert np.array_equal(np.concatenate([v["s_x"][toks] for _, toks, v, _ in picks]), ref["s_x"])
    rows = [v["row_of_pair"].reshape(wl.T, wl.k)[toks].reshape(-1) for _, toks, v, _ in picks]
    hq = np.concatenate([v["hq"][r] for (_, _, v, _), r in zip(picks, rows)])
    s_h = np.concatenate([v["s_h"][r] for (_, _, v, _), r in zip(picks, rows)])
    n_diff, _ = check_fp8_codes(hq, ref["hq"][ref["row_of_pair"]])
    _report(hq_codes=int(hq.size), hq_diff=n_diff, tokens=int(xs.shape[0]))
    np.testing.assert_allclose(s_h, ref["s_h"][ref["row_of_pair"]], rtol=2e-5)
    outb = np.concatenate([o[toks] for _, toks, _, o in picks])
    _check_output_rules(hl, xs, ls, wl.k, outb, ref, hq, s_h, allow)
    return int(hq.size)


@pytest.fixture(scope="module")
def full_layer():
    return device_layer(synth.WORKLOADS[FULL_WL])     # same weights for all full-size configs


def _no_shared(dl):
    cls = type(dl)
    if cls is moe.Layer:
        return moe.Layer(dl.E, dl.H, dl.N, dl.gate_packed, dl.up_packed, dl.down_packed,
                         dl.gate_scales, dl.up_scales, dl.down_scales)
    if cls is moe.Layer8:
        return moe.Layer8(dl.E, dl.H, dl.N, dl.gate_w8, dl.up_w8, dl.down_w8, dl.gate_rs, dl.up_rs,
                          dl.down_rs)
    return moe.Layer4(dl.E, dl.H, dl.N, dl.gate_f4, dl.up_f4, dl.down_f4, dl.gate_bs, dl.up_bs, dl.down_bs,
                      dl.gate_s2, dl.up_s2, dl.down_s2)


@pytest.mark.parametrize("name", FULL)
def test_forward_full_size(name, full_layer, host_layers):
    """W4A8 at full size: decode_t8 over all eight benchmark batches (64 tokens), decode_t64 all
    64 tokens, the prefill configs at >= 256 tokens at tile boundaries; >= 0.5 M requantized codes
    each under rule 2."""
    wl = synth.WORKLOADS[name]
    dl = full_layer if wl.n_shared else _no_shared(full_layer)
    n = _full_size_check(name, dl, "w4a8", host_layers, n_batches=8 if name == "decode_t8" else 1)
    assert n >= 500_000


# ---- failure detection: a bounded device wait that runs out -------------------------------------

def test_bounded_wait_reports_timeout_and_context_survives():
    assert moe.moe_last_device_status() == 0
    moe.moe_selftest_bounded_wait(50_000_000)          # 50 ms on a barrier nothing completes
    assert moe.moe_last_device_status() == -6          # MOE_ERR_TIMEOUT
    assert moe.moe_last_device_status() == 0          # read-and-clear
    wl = synth.WORKLOADS["tiny"]                        # the context is still usable
    hl = oracle.pack_workload_layer(wl)
    dl = device_layer(wl)
    _run_and_compare(hl, dl, synth.tokens(wl), synth.logits(wl), wl.k)


# ---- row-scaled FP8 (W8A8) experts ---------------------------------------------------------------

def test_w8a8_quant_weights_bitexact():
    rng = np.random.default_rng(21)
    w = (rng.standard_normal((300, 512)) * 0.02 * 2.0 ** rng.uniform(-6, 6, (300, 1))).astype(np.float32)
    w[5] = 0.0                                         # zero row: scale 0, codes 0
    w[6, 7] = 1e30                                     # huge outlier: every other code flushes to 0
    w[7, :] = -3.0e-38                                 # subnormal-scale row
    wb = _f32_to_bf16_bits(w)
    q_ref, s_ref = oracle.quant_rows(wb)
    q = torch.empty(300, 512, dtype=torch.uint8, device="cuda")
    sc = torch.empty(300, dtype=torch.float32, device="cuda")
    moe.w8a8_quant_weights(to_dev_bf16(wb), q, sc)
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


def _host_layer_and_dev_w8a8(E, H, N, seed, n_shared=0, shared_N=0):
    """Seeded random layer, rows scaled over 2^-3..2^3: row-quantized on the host by the oracle
    and on the GPU by the library."""
    rng_stream = 60_000 + seed * 10
    def w(stream, rows, K):
        a = synth.normal_f32(seed, stream, E * rows * K, 0.02).reshape(E, rows, K)
        scale = 2.0 ** np.round(synth.normal_f32(seed, stream + 5, E * rows).reshape(E, rows, 1) * 1.5)
        return _f32_to_bf16_bits((a * scale).astype(np.float32))
    gw, uw, dw = w(rng_stream, N, H), w(rng_stream + 1, N, H), w(rng_stream + 2, H, N)
    def rq(W):
        qs = [oracle.quant_rows(W[e]) for e in range(E)]
        return np.stack([a for a, _ in qs]), np.stack([b for _, b in qs])
    (gq, gs), (uq, us), (dq, ds) = rq(gw), rq(uw), rq(dw)
    sh, shd = {}, {}
    if n_shared:
        for i, key in enumerate(("sh_gate", "sh_up", "sh_down")):
            shape = (n_shared, shared_N, H) if i < 2 else (n_shared, H, shared_N)
            a = synth.normal_bf16(seed, rng_stream + 3 + i, int(np.prod(shape)), 0.02).reshape(shape)
            sh[key] = a
            shd[key] = to_dev_bf16(a)
    hl = oracle.Layer.w8a8(E, H, N, gq, uq, dq, gs, us, ds, **sh)
    dl = moe.make_layer_w8a8(to_dev_bf16(gw), to_dev_bf16(uw), to_dev_bf16(dw), **shd)
    torch.cuda.synchronize()
    assert np.array_equal(dl.gate_w8.cpu().numpy(), gq)
    assert np.array_equal(dl.down_w8.cpu().numpy(), dq)
    assert np.array_equal(dl.up_rs.cpu().numpy(), us)
    return hl, dl


def test_w8a8_forward_tiny_workload():
    wl = synth.WORKLOADS["tiny"]
    hl = oracle.quant_workload_layer_w8a8(wl)
    dl = device_layer_w8a8(wl)
    assert np.array_equal(dl.up_w8.cpu().numpy(), hl.up_w8)
    assert np.array_equal(dl.down_rs.cpu().numpy(), hl.down_rs)
    r1 = _run_and_compare(hl, dl, synth.tokens(wl), synth.logits(wl), wl.k)
    r2 = _run_and_compare(hl, dl, synth.tokens(wl), synth.logits(wl), wl.k)
    assert np.array_equal(r1["out"], r2["out"])        # deterministic


# token tiles of 16 (decode, gathered rows), 32 (gathered) and 256 rows (with the MMA's N
# following the live rows: segments of every length from 1 to several hundred rows)
@pytest.mark.parametrize("E,H,N,k,T", [(5, 384, 256, 3, 37), (1, 256, 128, 1, 9), (8, 256, 128, 2, 1),
                                       (8, 256, 256, 2, 200), (16, 512, 384, 8, 130),
                                       (8, 256, 256, 2, 600), (3, 1024, 128, 2, 700),
                                       (2, 512, 256, 1, 1000), (64, 1024, 1024, 6, 16)])
def test_w8a8_forward_ragged_shapes(E, H, N, k, T):
    hl, dl = _host_layer_and_dev_w8a8(E, H, N, seed=E * 7 + T)
    x = synth.normal_bf16(3, 777 + T, T * H).reshape(T, H)
    logits = synth.normal_f32(3, 778 + T, T * E).reshape(T, E)
    _run_and_compare(hl, dl, x, logits, k)


def test_w8a8_forward_shared_experts_and_zero_rows():
    hl, dl = _host_layer_and_dev_w8a8(4, 256, 128, seed=5, n_shared=2, shared_N=256)
    T = 21
    x = synth.normal_bf16(4, 901, T * 256).reshape(T, 256)
    x[3, :] = 0
    logits = synth.normal_f32(4, 902, T * 4).reshape(T, 4)
    r = _run_and_compare(hl, dl, x, logits, 2)
    ref = oracle.moe_forward(hl, x, logits, 2)
    assert np.array_equal(r["out"][3], ref["out"][3])  # shared experts of a zero row: exactly 0
    xd = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    ld = torch.empty(0, 4, dtype=torch.float32, device="cuda")
    out = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    moe.moe_w8a8_forward(dl, xd, ld, 2, out, torch.empty(256, dtype=torch.uint8, device="cuda"))


@pytest.fixture(scope="module")
def full_layer_w8a8():
    return device_layer_w8a8(synth.WORKLOADS[FULL_WL])


@pytest.mark.parametrize("name", FULL)
def test_w8a8_forward_full_size(name, full_layer_w8a8, host_layers):
    """Row-scaled FP8 experts at full size: every token of one batch at decode, >= 64 tokens at
    tile boundaries (128/192/256 rows) at prefill."""
    wl = synth.WORKLOADS[name]
    dl = full_layer_w8a8 if wl.n_shared else _no_shared(full_layer_w8a8)
    _full_size_check(name, dl, "w8a8", host_layers, n_prefill_tokens=64, tile_rows=(128, 256))


# ---- NVFP4 experts -------------------------------------------------------------------------------

def test_nvfp4_quant_weights_bitexact():
    rng = np.random.default_rng(41)
    E, rows, K = 3, 100, 512
    w = (rng.standard_normal((E, rows, K)) * 0.02 * 2.0 ** rng.uniform(-5, 5, (E, rows, 1))).astype(np.float32)
    w[0, 4, 32:48] = 0.0                               # a zero block
    w[1, 7, :16] = [6, 3, 1.25, -0.75, 0.25, -6, 0, 2.5, 5, -1.75, 0.5, 4, -3.5, 1, 0, 0]  # ties
    w[2] = 0.0                                         # a zero expert: scale2 0, everything 0
    wb = _f32_to_bf16_bits(w)
    codes = torch.empty(E, rows, K // 2, dtype=torch.uint8, device="cuda")
    scales = torch.empty(E, rows, K // 16, dtype=torch.uint8, device="cuda")
    s2 = torch.empty(E, dtype=torch.float32, device="cuda")
    moe.nvfp4_quant_weights(to_dev_bf16(wb), codes, scales, s2)
    torch.cuda.synchronize()
    for e in range(E):
        c_ref, s_ref, s2_ref = oracle.nvfp4_quant(wb[e])
        assert np.array_equal(codes[e].cpu().numpy(), c_ref), e
        assert np.array_equal(scales[e].cpu().numpy(), s_ref), e
        assert s2[e].item() == s2_ref, e


def _host_layer_and_dev_nvfp4(E, H, N, seed, n_shared=0, shared_N=0):
    """Seeded random layer, rows scaled over 2^-4..2^4: NVFP4-quantized on the host by the oracle
    and on the GPU by the library."""
    rng_stream = 70_000 + seed * 10
    def w(stream, rows, K):
        a = synth.normal_f32(seed, stream, E * rows * K, 0.02).reshape(E, rows, K)
        scale = 2.0 ** np.round(synth.normal_f32(seed, stream + 5, E * rows).reshape(E, rows, 1) * 1.5)
        return _f32_to_bf16_bits((a * scale).astype(np.float32))
    gw, uw, dw = w(rng_stream, N, H), w(rng_stream + 1, N, H), w(rng_stream + 2, H, N)
    def qp(W):
        r = [oracle.nvfp4_quant(W[e]) for e in range(E)]
        return (np.stack([a for a, _, _ in r]), np.stack([b for _, b, _ in r]),
                np.array([c for _, _, c in r], np.float32))
    g, u, d = qp(gw), qp(uw), qp(dw)
    sh, shd = {}, {}
    if n_shared:
        for i, key in enumerate(("sh_gate", "sh_up", "sh_down")):
            shape = (n_shared, shared_N, H) if i < 2 else (n_shared, H, shared_N)
            a = synth.normal_bf16(seed, rng_stream + 3 + i, int(np.prod(shape)), 0.02).reshape(shape)
            sh[key] = a
            shd[key] = to_dev_bf16(a)
    hl = oracle.Layer.nvfp4(E, H, N, g[0], u[0], d[0], g[1], u[1], d[1], g[2], u[2], d[2], **sh)
    dl = moe.make_layer_nvfp4(to_dev_bf16(gw), to_dev_bf16(uw), to_dev_bf16(dw), **shd)
    torch.cuda.synchronize()
    assert np.array_equal(dl.gate_f4.cpu().numpy(), g[0])
    assert np.array_equal(dl.down_bs.cpu().numpy(), d[1])
    assert np.array_equal(dl.up_s2.cpu().numpy(), u[2])
    return hl, dl


def test_nvfp4_forward_tiny_workload():
    wl = synth.WORKLOADS["tiny"]
    hl = oracle.quant_workload_layer_nvfp4(wl)
    dl = device_layer_nvfp4(wl)
    assert np.array_equal(dl.up_f4.cpu().numpy(), hl.up_f4)
    assert np.array_equal(dl.down_s2.cpu().numpy(), hl.down_s2)
    r1 = _run_and_compare(hl, dl, synth.tokens(wl), synth.logits(wl), wl.k)
    r2 = _run_and_compare(hl, dl, synth.tokens(wl), synth.logits(wl), wl.k)
    assert np.array_equal(r1["out"], r2["out"])


@pytest.mark.parametrize("E,H,N,k,T", [(5, 384, 256, 3, 37), (1, 256, 128, 1, 9), (8, 256, 128, 2, 1),
                                       (8, 256, 256, 2, 200), (16, 512, 384, 8, 130),
                                       (3, 1024, 128, 2, 700), (64, 1024, 1024, 6, 16)])
def test_nvfp4_forward_ragged_shapes(E, H, N, k, T):
    hl, dl = _host_layer_and_dev_nvfp4(E, H, N, seed=E * 7 + T)
    x = synth.normal_bf16(3, 777 + T, T * H).reshape(T, H)
    logits = synth.normal_f32(3, 778 + T, T * E).reshape(T, E)
    # NVFP4, E=3 H=1024 N=128 top-2 T=700 (seed 721): a permitted requantized-code flip moves one
    # output of its token 1.26x past rule 3 through the short (N = 128) down projection
    allow = ("nvfp4 E3 H1024 N128 k2 T700 seed 721", 4) if (E, H, N, k, T) == (3, 1024, 128, 2, 700) else None
    _run_and_compare(hl, dl, x, logits, k, allow=allow)


def test_nvfp4_forward_shared_experts():
    hl, dl = _host_layer_and_dev_nvfp4(4, 256, 128, seed=5, n_shared=2, shared_N=256)
    T = 21
    x = synth.normal_bf16(4, 901, T * 256).reshape(T, 256)
    logits = synth.normal_f32(4, 902, T * 4).reshape(T, 4)
    _run_and_compare(hl, dl, x, logits, 2)


@pytest.fixture(scope="module")
def full_layer_nvfp4():
    return device_layer_nvfp4(synth.WORKLOADS[FULL_WL])


@pytest.mark.parametrize("name", FULL)
def test_nvfp4_forward_full_size(name, full_layer_nvfp4, host_layers):
    """NVFP4 experts at full size: every token of one batch at decode, >= 64 tokens at tile
    boundaries at prefill."""
    wl = synth.WORKLOADS[name]
    dl = full_layer_nvfp4 if wl.n_shared else _no_shared(full_layer_nvfp4)
    # the NVFP4 GEMM sums all of K in TMEM (f16 tensor cores), so ~7e-5 of the requantized codes
    # of prefill_t2048_zipf (seed 0) sit one step from the oracle's (rule 2), and 13 outputs of
    # those tokens pass only under rule 2's allowance (cap 64, under 1e-4 of the outputs checked)
    allow = ("nvfp4 prefill_t2048_zipf seed 0", 64) if name == "prefill_t2048_zipf" else None
    _full_size_check(name, dl, "nvfp4", host_layers, n_prefill_tokens=64, tile_rows=(128, 256), allow=allow)


# ---- hybrid layers: NVFP4 hot experts, W4A8 cold experts -------------------------------------------

def _host_hybrid(w4: "oracle.Layer", f4: "oracle.Layer", hot_ids):
    hot_ids = np.array(hot_ids, np.int32)
    cold_ids = np.array([e for e in range(w4.E) if e not in set(hot_ids.tolist())], np.int32)
    cold = oracle.Layer(len(cold_ids), w4.H, w4.N, w4.gate_packed[cold_ids], w4.up_packed[cold_ids],
                        w4.down_packed[cold_ids], w4.gate_scales[cold_ids], w4.up_scales[cold_ids],
                        w4.down_scales[cold_ids], sh_gate=w4.sh_gate, sh_up=w4.sh_up, sh_down=w4.sh_down)
    hot = oracle.Layer.nvfp4(len(hot_ids), w4.H, w4.N, f4.gate_f4[hot_ids], f4.up_f4[hot_ids],
                             f4.down_f4[hot_ids], f4.gate_bs[hot_ids], f4.up_bs[hot_ids], f4.down_bs[hot_ids],
                             f4.gate_s2[hot_ids], f4.up_s2[hot_ids], f4.down_s2[hot_ids])
    return oracle.Layer.hybrid(cold, hot, hot_ids, cold_ids)


def _host_layer_and_dev_hybrid(E, H, N, seed, hot_ids):
    """One set of seeded weights, W4A8-packed and NVFP4-quantized on both sides; the hybrid takes
    the NVFP4 slabs of the hot experts and the W4A8 slabs of the rest."""
    rng_stream = 80_000 + seed * 10
    gw = synth.normal_bf16(seed, rng_stream + 0, E * N * H, 0.02).reshape(E, N, H)
    uw = synth.normal_bf16(seed, rng_stream + 1, E * N * H, 0.02).reshape(E, N, H)
    dw = synth.normal_bf16(seed, rng_stream + 2, E * H * N, 0.02).reshape(E, H, N)
    gp, gs = zip(*[oracle.rtn_pack(gw[e])[:2] for e in range(E)])
    up, us = zip(*[oracle.rtn_pack(uw[e])[:2] for e in range(E)])
    dp, ds = zip(*[oracle.rtn_pack(dw[e])[:2] for e in range(E)])
    w4 = oracle.Layer(E, H, N, np.stack(gp), np.stack(up), np.stack(dp), np.stack(gs), np.stack(us), np.stack(ds))
    def qp(W):
        r = [oracle.nvfp4_quant(W[e]) for e in range(E)]
        return (np.stack([a for a, _, _ in r]), np.stack([b for _, b, _ in r]),
                np.array([c for _, _, c in r], np.float32))
    g, u, d = qp(gw), qp(uw), qp(dw)
    f4 = oracle.Layer.nvfp4(E, H, N, g[0], u[0], d[0], g[1], u[1], d[1], g[2], u[2], d[2])
    hl = _host_hybrid(w4, f4, hot_ids)
    dgw, duw, ddw = to_dev_bf16(gw), to_dev_bf16(uw), to_dev_bf16(dw)
    dl = moe.hybrid_from(moe.make_layer(dgw, duw, ddw), moe.make_layer_nvfp4(dgw, duw, ddw), hot_ids)
    torch.cuda.synchronize()
    return hl, dl


@pytest.mark.parametrize("E,H,N,k,T,hot", [(16, 256, 128, 2, 8, [0, 5, 9]), (16, 256, 128, 2, 40, [3]),
                                           (8, 256, 256, 2, 600, [2, 7]), (4, 256, 128, 2, 21, [0, 1, 2, 3]),
                                           (4, 256, 128, 2, 21, []), (64, 1024, 1024, 6, 16, list(range(0, 64, 7)))])
def test_hybrid_forward(E, H, N, k, T, hot):
    """Hot experts on the NVFP4 GEMM, cold ones on the W4A8 GEMM, in one layer (decode: both
    GEMMs write their rows of h and Y before the shared requantization and combine; prefill;
    all hot; all cold)."""
    hl, dl = _host_layer_and_dev_hybrid(E, H, N, seed=E + T + len(hot), hot_ids=hot)
    x = synth.normal_bf16(11, 840 + T, T * H).reshape(T, H)
    logits = synth.normal_f32(11, 841 + T, T * E).reshape(T, E)
    _run_and_compare(hl, dl, x, logits, k)


def test_hybrid_full_size_decode_sampled():
    """decode_t8 with 15 % of the experts hot (the page's 512k tier keeps 14.8 % in NVFP4)."""
    wl = synth.WORKLOADS["decode_t8"]
    hot = [int(e) for e in np.random.default_rng(5).choice(wl.E, 38, replace=False)]
    dl = moe.hybrid_from(device_layer(wl), device_layer_nvfp4(wl), hot)
    x, lg = device_inputs(wl)
    ws = moe.alloc_workspace(dl, wl.T, wl.k)
    out = moe.forward(dl, x, lg, wl.k, ws=ws)
    torch.cuda.synchronize()
    assert moe.moe_last_device_status() == 0
    v = ws_views(dl, ws, wl.T, wl.k)
    ids_ref, _ = oracle.route_topk(synth.logits(wl), wl.k)
    experts = sorted(set(ids_ref.reshape(-1).tolist()))
    assert any(e in hot for e in experts) and any(e not in hot for e in experts)
    hl = _host_hybrid(oracle.pack_workload_layer(wl, experts=experts),
                      oracle.quant_workload_layer_nvfp4(wl, experts=experts), hot)
    xs, ls = synth.tokens(wl), synth.logits(wl)
    ref = oracle.moe_forward(hl, xs, ls, wl.k)
    assert np.array_equal(v["ids"], ref["ids"])
    check_fp8_codes(v["hq"][v["row_of_pair"]], ref["hq"][ref["row_of_pair"]])
    _check_output_rules(hl, xs, ls, wl.k, bits(out), ref, v["hq"][v["row_of_pair"]], v["s_h"][v["row_of_pair"]])
