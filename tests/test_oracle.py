"""Pins of the CPU oracle against facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself: hand-worked
values under tests/golden/ (derived from the pages' rules), exhaustive
brute-force searches, independent library routines (numpy sorts, fp64
softmax, an fp64 dense MLP) and invariants.
"""
import math

import numpy as np
import pytest

import oracle
import synth
from conftest import golden_lines


# ------------------------------------------------------------------------------------------------
# E4M3
# ------------------------------------------------------------------------------------------------

def _all_finite_codes():
    return [c for c in range(256) if (c & 0x7F) != 0x7F]


def test_e4m3_decode_table_shape():
    vals = oracle.e4m3_decode_table()
    nan_codes = [c for c in range(256) if np.isnan(vals[c])]
    assert nan_codes == [0x7F, 0xFF]
    finite = vals[~np.isnan(vals)]
    assert len(finite) == 254
    assert len(set(finite.tolist())) == 253          # +0 and -0 compare equal
    assert finite.max() == 448.0 and finite.min() == -448.0
    pos = np.sort(np.unique(np.abs(finite)))
    assert pos[1] == 2.0 ** -9                        # smallest subnormal
    # subnormals + first binade are the equally spaced ladder 0..15 * 2^-9
    assert np.array_equal(pos[:16], np.arange(16) * 2.0 ** -9)


@pytest.mark.parametrize("line", list(golden_lines("e4m3_worked.txt")))
def test_e4m3_worked_values(line):
    x, code = line.split()
    assert oracle.e4m3_encode(float(x)) == int(code, 16)


def test_e4m3_roundtrip_all_codes():
    for c in _all_finite_codes():
        v = oracle.e4m3_decode(c)
        assert oracle.e4m3_encode(v) == c, hex(c)


def test_int4_codes_exact_in_e4m3():
    for i in range(-8, 8):
        c = oracle.e4m3_encode(float(i))
        assert oracle.e4m3_decode(c) == float(i)


def _brute_nearest(xs):
    """Nearest finite E4M3 code by exhaustive search; ties to the even code; saturate."""
    codes = np.array([c for c in range(128) if c != 0x7F], np.int64)   # non-negative magnitudes
    mags = np.array([oracle.e4m3_decode(int(c)) for c in codes], np.float64)
    out = []
    for x in xs:
        a = min(abs(float(x)), 448.0)
        d = np.abs(mags - a)
        best = np.flatnonzero(d == d.min())
        if len(best) > 1:
            best = [b for b in best if codes[b] % 2 == 0]
        c = int(codes[best[0]])
        if np.signbit(np.float32(x)):
            c |= 0x80
        out.append(c)
    return out


def test_e4m3_encode_vs_brute_force():
    rng = np.random.default_rng(1)
    mags = np.array(sorted(set(abs(oracle.e4m3_decode(c)) for c in _all_finite_codes())),
                    np.float64)
    mids = (mags[1:] + mags[:-1]) / 2
    probes = []
    for m in np.concatenate([mids, mags]):
        f = np.float32(m)
        probes += [f, np.nextafter(f, np.float32(np.inf)), np.nextafter(f, np.float32(0))]
    probes += list(rng.standard_normal(4000).astype(np.float32) * 30)
    probes += list((rng.standard_normal(2000) * 0.01).astype(np.float32))
    probes += list(np.float32(2.0) ** rng.uniform(-14, 10, 2000).astype(np.float32))
    probes = np.array(probes, np.float32)
    probes = np.concatenate([probes, -probes])
    got = [oracle.e4m3_encode(float(x)) for x in probes]
    want = _brute_nearest(probes)
    bad = [(float(p), g, w) for p, g, w in zip(probes, got, want) if g != w]
    assert not bad, bad[:10]


# ------------------------------------------------------------------------------------------------
# INT4 RTN + pack-quantized storage
# ------------------------------------------------------------------------------------------------

def _f32_to_bf16_bits(x):
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


@pytest.mark.parametrize("line", list(golden_lines("pack_words.txt")))
def test_pack_words_golden(line):
    f = line.split()
    codes = np.array([int(v) for v in f[:8]], np.int8)
    word = np.array([int(f[8], 16)], np.uint32).view(np.int32)
    # the inverse (unpack) holds for every word, -8 included
    assert np.array_equal(oracle.unpack(np.array([[word[0]]], np.int32), 8)[0], codes)
    if codes.min() < -7:
        return      # RTN with scale amax/7 never yields -8; packing it is covered via unpack
    # build one 128-element group whose RTN codes are exactly `codes` in its first word:
    # scale 2^-4 forced by a +-7*2^-4 element elsewhere in the group.
    w = np.zeros((1, 128), np.float32)
    w[0, :8] = codes.astype(np.float32) * 0.0625
    w[0, 100] = 7 * 0.0625
    packed, scales, got_codes = oracle.rtn_pack(_f32_to_bf16_bits(w))
    assert oracle.bf16_to_f32(scales)[0, 0] == 0.0625
    assert np.array_equal(got_codes[0, :8], codes)
    assert packed[0, 0] == word[0]


def test_unpack_every_nibble_every_position():
    for pos in range(8):
        for nib in range(16):
            word = np.array([0x88888888 & ~(0xF << (4 * pos)) | (nib << (4 * pos))],
                            np.uint32).view(np.int32)
            codes = oracle.unpack(word.reshape(1, 1), 8)[0]
            want = np.zeros(8, np.int8)
            want[pos] = nib - 8
            assert np.array_equal(codes, want), (pos, nib)


def test_pack_roundtrip_random():
    rng = np.random.default_rng(2)
    w = _f32_to_bf16_bits(rng.standard_normal((64, 512)).astype(np.float32) * 0.02)
    packed, scales, codes = oracle.rtn_pack(w)
    assert codes.min() >= -8 and codes.max() <= 7
    assert np.array_equal(oracle.unpack(packed, 512), codes)


def test_rtn_worked_case():
    groups = {}
    scales_want = {}
    for line in golden_lines("rtn_worked_case.txt"):
        f = line.split()
        if f[1] == "scale":
            scales_want[f[0]] = float(f[2])
        else:
            groups.setdefault(f[0], []).append((int(f[1]), float(f[2]), int(f[3])))
    names = sorted(groups)
    w = np.zeros((len(names), 128), np.float32)
    for gi, name in enumerate(names):
        for idx, val, _ in groups[name]:
            w[gi, idx] = val
    wb = _f32_to_bf16_bits(w)
    assert np.array_equal(oracle.bf16_to_f32(wb), w)      # listed values are exact bf16
    packed, scales, codes = oracle.rtn_pack(wb)
    for gi, name in enumerate(names):
        assert oracle.bf16_to_f32(scales)[gi, 0] == scales_want[name]
        for idx, _, code in groups[name]:
            assert codes[gi, idx] == code, (name, idx)


def test_rtn_error_bound_and_zero_group():
    rng = np.random.default_rng(3)
    w = rng.standard_normal((32, 1024)).astype(np.float32) * 0.02
    w[5, 128:256] = 0.0                                  # an all-zero group
    wb = _f32_to_bf16_bits(w)
    packed, scales, codes = oracle.rtn_pack(wb)
    wf = oracle.bf16_to_f32(wb).astype(np.float64)
    s = np.repeat(oracle.bf16_to_f32(scales).astype(np.float64), 128, axis=1)
    assert scales[5, 1] == 0 and not codes[5, 128:256].any()
    nz = s > 0
    # amax/s <= 7*(1+2^-8) so no code is clamped, and rounding error is at most half a step
    assert np.all(np.abs(wf - codes * s)[nz] <= 0.5 * s[nz] * (1 + 2 ** -20))
    assert codes.min() >= -7                              # RTN with scale amax/7 never gives -8


# ------------------------------------------------------------------------------------------------
# per-token FP8
# ------------------------------------------------------------------------------------------------

def test_token_quant_closed_form():
    x = np.zeros((3, 256), np.float32)
    x[0, 0] = 1.0                 # amax 1 -> s = fp32(1/448)
    x[0, 1] = 0.5                 # 0.5*448 = 224 exactly representable -> 0x76
    x[0, 2] = 0.30078125          # bf16(0.3): 134.75 -> 128 (spacing 16) -> 0x70
    x[0, 3] = -1.0
    x[2, :] = 0.875               # s = 2^-9 exactly, all codes 0x7e
    q, s = oracle.quant_tokens(_f32_to_bf16_bits(x))
    assert s[0] == np.float32(1.0) / np.float32(448.0)
    assert list(q[0, :4]) == [0x7E, 0x76, 0x70, 0xFE]
    assert s[1] == 0.0 and not q[1].any()                # zero row
    assert s[2] == 2.0 ** -9 and np.all(q[2] == 0x7E)


def test_token_quant_properties():
    wl = synth.WORKLOADS["decode_t8"]
    x = synth.tokens(wl)
    q, s = oracle.quant_tokens(x)
    xf = oracle.bf16_to_f32(x)
    amax = np.abs(xf).max(axis=1)
    assert np.array_equal(s, (amax / np.float32(448)).astype(np.float32))
    dec = oracle.e4m3_decode_table()
    for t in range(x.shape[0]):
        i = np.argmax(np.abs(xf[t]))
        assert q[t, i] in (0x7E, 0xFE)
        # dequantized value within half an E4M3 step (relative 2^-4 for normals) of x
        d = dec[q[t]].astype(np.float64) * s[t]
        err = np.abs(d - xf[t])
        bound = np.maximum(np.abs(xf[t]) * 2.0 ** -4, 2.0 ** -10 * s[t]) * (1 + 1e-6)
        assert np.all(err <= bound)


# ------------------------------------------------------------------------------------------------
# routing + permutation
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("line", list(golden_lines("routing_worked.txt")))
def test_routing_worked(line):
    k, l, ids, gates = [p.split() for p in line.split("|")]
    k = int(k[0])
    got_ids, got_g = oracle.route_topk(np.array([[float(v) for v in l]], np.float32), k)
    assert got_ids[0].tolist() == [int(v) for v in ids]
    assert np.array_equal(got_g[0], np.array([float(v) for v in gates], np.float32))


def test_routing_vs_sort_and_softmax():
    rng = np.random.default_rng(4)
    logits = rng.standard_normal((300, 64)).astype(np.float32)
    logits[:10, 5] = logits[:10, 9]                      # planted ties
    for k in (1, 2, 6, 64):
        ids, gates = oracle.route_topk(logits, k)
        for t in range(logits.shape[0]):
            order = np.lexsort((np.arange(64), -logits[t].astype(np.float64)))
            assert ids[t].tolist() == order[:k].tolist()
            sel = logits[t, order[:k]].astype(np.float64)
            ref = np.exp(sel - sel.max())
            ref /= ref.sum()
            assert np.allclose(gates[t], ref, rtol=2e-6, atol=1e-7)
            assert abs(float(gates[t].astype(np.float64).sum()) - 1.0) < 1e-6 * k
        if k == 64:   # k = E: the gate is the full softmax
            full = np.exp(logits - logits.max(1, keepdims=True))
            full /= full.sum(1, keepdims=True)
            back = np.zeros_like(full)
            np.put_along_axis(back, ids, gates, 1)
            assert np.allclose(back, full, rtol=2e-6, atol=1e-7)


# ------------------------------------------------------------------------------------------------
# Router logits (the step upstream of top-k)
# ------------------------------------------------------------------------------------------------

def _bf16(a):
    """fp32 array -> bf16 bits, round to nearest even (numpy, independent of the oracle)."""
    u = np.asarray(a, np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def _f32(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def test_router_one_hot_rows_select_weight_columns():
    """x = e_j picks column j of the router weight: catches a transposed or shifted operand."""
    rng = np.random.default_rng(11)
    E, H = 12, 256
    wr = _bf16(rng.standard_normal((E, H)) / 16)
    cols = [0, 1, 77, 128, 255]
    x = np.zeros((len(cols), H), np.uint16)
    for t, j in enumerate(cols):
        x[t, j] = 0x3F80                                    # bf16 1.0
    got = oracle.router_logits(x, wr)
    assert np.array_equal(got, _f32(wr[:, cols]).T)


def test_router_two_terms_round_once():
    """Two non-zero inputs: each bf16 product is exact in fp32, the sum rounds once."""
    rng = np.random.default_rng(12)
    E, H = 9, 384
    wr = _bf16(rng.standard_normal((E, H)))
    x = np.zeros((20, H), np.uint16)
    want = np.zeros((20, E), np.float32)
    for t in range(20):
        j1, j2 = sorted(rng.choice(H, 2, replace=False))
        a, b = _bf16(rng.standard_normal(2) * 3)
        x[t, j1], x[t, j2] = a, b
        exact = (_f32(a).astype(np.float64) * _f32(wr[:, j1]).astype(np.float64)
                 + _f32(b).astype(np.float64) * _f32(wr[:, j2]).astype(np.float64))
        want[t] = exact.astype(np.float32)
    assert np.array_equal(oracle.router_logits(x, wr), want)


def test_router_within_sequential_fp32_bound():
    """|fp32 sequential sum - exact| <= (H-1) * 2^-24 * sum |x_k w_k| (standard summation bound)."""
    rng = np.random.default_rng(13)
    T, E, H = 7, 40, 512
    x = _bf16(rng.standard_normal((T, H)))
    wr = _bf16(rng.standard_normal((E, H)) / math.sqrt(H))
    got = oracle.router_logits(x, wr).astype(np.float64)
    xf, wf = _f32(x).astype(np.float64), _f32(wr).astype(np.float64)
    exact = xf @ wf.T
    bound = (H - 1) * 2.0 ** -24 * (np.abs(xf) @ np.abs(wf).T)
    assert np.all(np.abs(got - exact) <= bound)
    assert np.abs(got - exact).max() > 0                   # it is a real fp32 sum, not fp64


def test_permutation_vs_stable_sort():
    rng = np.random.default_rng(5)
    for T, k, E in ((50, 6, 256), (16, 2, 8), (1, 1, 1), (0, 2, 8), (333, 3, 17)):
        ids = rng.integers(0, E, (T, k)).astype(np.int32) if T else np.zeros((0, k), np.int32)
        offsets, sorted_pairs, rop = oracle.permute(ids, E)
        flat = ids.reshape(-1)
        ref = np.argsort(flat, kind="stable")
        assert np.array_equal(sorted_pairs, ref)
        assert np.array_equal(offsets, np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))]))
        assert offsets[-1] == T * k and np.all(np.diff(offsets) >= 0)
        assert np.array_equal(rop[sorted_pairs], np.arange(T * k))


# ------------------------------------------------------------------------------------------------
# the layer
# ------------------------------------------------------------------------------------------------

def _tiny_layer(wl):
    return oracle.pack_workload_layer(wl)


def test_layer_dense_brute_force_matches_permuted():
    wl = synth.WORKLOADS["tiny"]
    layer = _tiny_layer(wl)
    x, lg = synth.tokens(wl), synth.logits(wl)
    r = oracle.moe_forward(layer, x, lg, wl.k)
    d = oracle.moe_forward_dense(layer, x, lg, wl.k)
    assert np.array_equal(r["out"], d["out"])
    assert np.array_equal(r["out_f32"], d["out_f32"])
    for p in range(wl.P):
        t, j = divmod(p, wl.k)
        e = r["ids"][t, j]
        row = r["row_of_pair"][p]
        assert np.array_equal(r["hq"][row], d["hq"][t, e])
        assert r["s_h"][row] == d["s_h"][t, e]
        assert np.array_equal(r["y"][row], d["y"][t, e])


def test_expert_rows_match_dense_brute_force():
    """The expert-parallel receive step (S4-S6 on given FP8 rows) against the dense brute force,
    which runs every (token, expert) pair without any permutation: any (token, expert), routed
    or not, in any row order, and through a slice of the experts."""
    wl = synth.WORKLOADS["tiny"]
    layer = _tiny_layer(wl)
    x, lg = synth.tokens(wl), synth.logits(wl)
    d = oracle.moe_forward_dense(layer, x, lg, wl.k)
    xq, sx = oracle.quant_tokens(x)
    rng = np.random.default_rng(5)
    t = rng.integers(0, wl.T, 40)
    e = rng.integers(0, wl.E, 40)
    y = oracle.expert_rows(layer, xq[t], sx[t], e)
    for i in range(40):
        assert np.array_equal(y[i], d["y"][t[i], e[i]]), i
    e0, e1 = 2, 6
    sel = (e >= e0) & (e < e1)
    ys = oracle.expert_rows(oracle.expert_slice(layer, e0, e1), xq[t[sel]], sx[t[sel]], e[sel] - e0)
    assert np.array_equal(ys, y[sel])
    with pytest.raises(ValueError):
        oracle.expert_rows(layer, xq[:1], sx[:1], np.array([wl.E]))


def test_combine_closed_form_and_forward_decomposition():
    """S7 alone: constant rows give bf16(sum_j g_j c_j); and the layer's own routed rows, gates
    and shared experts put back together give the layer's output bit for bit."""
    T, H, N, E, k = 3, 128, 128, 4, 2
    z = np.zeros((E, N, H // 8), np.int32)
    layer = oracle.Layer(E, H, N, z, z, np.zeros((E, H, N // 8), np.int32),
                         np.zeros((E, N, 1), np.uint16), np.zeros((E, N, 1), np.uint16),
                         np.zeros((E, H, 1), np.uint16))
    gates = np.array([[0.25, 0.75], [0.5, 0.5], [1.0, 0.0]], np.float32)
    c = np.array([[3.0, -1.5], [1.0, 2.0], [-7.0, 100.0]], np.float32)
    y = np.repeat(c.reshape(T * k, 1), H, axis=1).astype(np.float32)
    out = oracle.bf16_to_f32(oracle.combine(layer, np.zeros((T, H), np.uint16), gates, y, k))
    for t, want in enumerate((-0.375, 1.5, -7.0)):
        assert np.all(out[t] == want), (t, out[t, :2])
    wl = synth.WORKLOADS["tiny"]
    full = oracle.pack_workload_layer(wl)
    x, lg = synth.tokens(wl), synth.logits(wl)
    r = oracle.moe_forward(full, x, lg, wl.k)
    assert np.array_equal(oracle.combine(full, x, r["gates"], r["y"][r["row_of_pair"]], wl.k), r["out"])


def test_layer_constant_closed_form():
    want = {}
    for line in golden_lines("constant_layer.txt"):
        t, o, hq = line.split()
        want[int(t)] = (float(o), int(hq, 16))
    T, H, N, E, k = 4, 128, 128, 2, 1
    w0 = 0.02734375
    def packed(sign, rows, K):
        wb = _f32_to_bf16_bits(np.full((rows, K), sign * w0, np.float32))
        return oracle.rtn_pack(wb)
    gp = np.stack([packed(+1, N, H)[0], packed(-1, N, H)[0]])
    gs = np.stack([packed(+1, N, H)[1], packed(-1, N, H)[1]])
    dp = np.stack([packed(+1, H, N)[0], packed(-1, H, N)[0]])
    ds = np.stack([packed(+1, H, N)[1], packed(-1, H, N)[1]])
    layer = oracle.Layer(E, H, N, gp, gp, dp, gs, gs, ds)
    x = _f32_to_bf16_bits(np.full((T, H), 0.875, np.float32))
    lg = np.array([[1, 0], [0, 1], [1, 0], [0, 1]], np.float32)
    r = oracle.moe_forward(layer, x, lg, k)
    out = oracle.bf16_to_f32(r["out"])
    for t in range(T):
        assert np.all(out[t] == want[t][0]), (t, out[t, :4])
        assert np.all(r["hq"][r["row_of_pair"][t]] == want[t][1])
    assert np.all(r["s_x"] == 2.0 ** -9)
    # closed form of the float result before the final rounding: y = +-3.5 * 9.37890625 * sigmoid(+-3.0625)
    sig = lambda v: 1.0 / (1.0 + math.exp(-v))
    for t in range(T):
        s = 1.0 if t % 2 == 0 else -1.0
        ref = s * 3.5 * 9.37890625 * sig(s * 3.0625)
        assert np.allclose(r["out_f32"][t], ref, rtol=1e-6)


def test_layer_single_expert_vs_fp64_mlp():
    """E = 1, k = 1: the layer is one quantized SwiGLU MLP.  Compare with a textbook fp64
    MLP on the dequantized weights and the unquantized input: the difference is the FP8
    activation quantization error only (relative step 2^-4 per element, averaged)."""
    rng = np.random.default_rng(6)
    T, H, N = 24, 512, 256
    def wts(rows, K):
        return _f32_to_bf16_bits(rng.standard_normal((rows, K)).astype(np.float32) * 0.02)
    Wg, Wu, Wd = wts(N, H), wts(N, H), wts(H, N)
    pg, sg, cg = oracle.rtn_pack(Wg)
    pu, su, cu = oracle.rtn_pack(Wu)
    pd, sd, cd = oracle.rtn_pack(Wd)
    layer = oracle.Layer(1, H, N, pg[None], pu[None], pd[None], sg[None], su[None], sd[None])
    x = _f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    lg = np.zeros((T, 1), np.float32)
    r = oracle.moe_forward(layer, x, lg, 1)
    deq = lambda c, s: c.astype(np.float64) * np.repeat(oracle.bf16_to_f32(s).astype(np.float64), 128, 1)
    Dg, Du, Dd = deq(cg, sg), deq(cu, su), deq(cd, sd)
    xf = oracle.bf16_to_f32(x).astype(np.float64)
    g = xf @ Dg.T
    u = xf @ Du.T
    h = g / (1 + np.exp(-g)) * u
    ref = h @ Dd.T
    got = r["out_f32"].astype(np.float64)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel < 0.05, rel
    assert np.corrcoef(got.ravel(), ref.ravel())[0, 1] > 0.998
    # a wrong sign of the SwiGLU or a transposed weight would be far outside this band
    assert r["gates"].min() == 1.0


def _shared_layer(H, Ns, sh_gate, sh_up, sh_down, E=2):
    """A layer whose routed experts are all zero (scale 0, codes 0: routed output exactly 0), so
    that out_f32 is the shared experts' sum alone."""
    z = lambda rows, K: np.zeros((E, rows, K), np.int32)
    zs = lambda rows, K: np.zeros((E, rows, K // 128), np.uint16)
    return oracle.Layer(E, H, 128, z(128, H // 8), z(128, H // 8), z(H, 128 // 8), zs(128, H),
                        zs(128, H), zs(H, 128), sh_gate=sh_gate, sh_up=sh_up, sh_down=sh_down)


def test_shared_experts_constant_closed_form():
    """Two shared experts with constant weights (tests/golden/shared_constant.txt): the output is
    2 * 1.75 * silu(0.875) - 0.875 * silu(1.75), rounded once to bf16."""
    (want_f32, want_bf16), = [tuple(map(float, l.split())) for l in golden_lines("shared_constant.txt")]
    H, Ns, T = 128, 256, 2
    c = lambda v, shape: np.full(shape, _f32_to_bf16_bits(np.float32(v)), np.uint16)
    sg = np.stack([c(2.0 ** -7, (Ns, H)), c(2.0 ** -6, (Ns, H))])
    su = np.stack([c(2.0 ** -6, (Ns, H)), c(-(2.0 ** -7), (Ns, H))])
    sd = np.stack([c(2.0 ** -7, (H, Ns)), c(2.0 ** -8, (H, Ns))])
    layer = _shared_layer(H, Ns, sg, su, sd)
    x = _f32_to_bf16_bits(np.full((T, H), 0.875, np.float32))
    r = oracle.moe_forward(layer, x, np.array([[1, 0], [0, 1]], np.float32), 1)
    silu = lambda v: v / (1.0 + math.exp(-v))
    closed = 2 * 1.75 * silu(0.875) - 0.875 * silu(1.75)
    assert abs(closed - want_f32) < 1e-6
    # fp32 sums of exact terms, two expf calls and a handful of roundings: a few ulp of 2.2
    np.testing.assert_allclose(r["out_f32"], closed, rtol=0, atol=4e-6)
    assert np.all(oracle.bf16_to_f32(r["out"]) == want_bf16)


def test_shared_experts_vs_fp64_swiglu():
    """Two random bf16 shared experts (H != Ns, so a transposed down weight reads other values)
    against a textbook fp64 SwiGLU MLP per shared expert, summed.  The oracle's fp32 result lies
    within the sequential-fp32 error bound of the fp64 value; swapped gate/up, a missing silu or a
    transposed down projection fall far outside it."""
    rng = np.random.default_rng(19)
    H, Ns, S, T = 256, 384, 2, 7
    def w(shape):
        return _f32_to_bf16_bits((rng.standard_normal(shape) * 0.05).astype(np.float32))
    sg, su, sd = w((S, Ns, H)), w((S, Ns, H)), w((S, H, Ns))
    x = _f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    layer = _shared_layer(H, Ns, sg, su, sd)
    r = oracle.moe_forward(layer, x, rng.standard_normal((T, 2)).astype(np.float32), 1)
    got = r["out_f32"].astype(np.float64)
    xf = oracle.bf16_to_f32(x).astype(np.float64)
    Wg, Wu, Wd = (oracle.bf16_to_f32(a).astype(np.float64) for a in (sg, su, sd))
    eps = 2.0 ** -24

    def seq_dot(a, b):
        """fp64 value of sum_i a[..., i] * b[..., i] and the error bound of evaluating it in fp32
        in increasing i: every product and every partial sum s_i rounds once, so the error is at
        most eps * (sum |p_i| + sum_{i>=2} |s_i|) (partial sums taken in fp64, 1 % margin)."""
        prod = a[..., None, :] * b[None, ...]
        part = np.cumsum(prod, axis=-1)
        bnd = eps * (np.abs(prod).sum(-1) + np.abs(part[..., 1:]).sum(-1)) * 1.01
        return part[..., -1], bnd

    def mlp(gate_first=True, with_silu=True, down_T=False):
        y = np.zeros((T, H))
        bound = np.zeros((T, H))
        for s in range(S):
            (g, dg), (u, du) = seq_dot(xf, Wg[s]), seq_dot(xf, Wu[s])
            if not gate_first:
                g, u, dg, du = u, g, du, dg
            sig = 1.0 / (1.0 + np.exp(-g))
            a = (g * sig if with_silu else g) * u
            # g and u errors carried through silu(g) * u (|d silu / dg| < 1.1), plus expf's ulps
            # and the four roundings of g / (1 + e) * u on a itself
            da = 1.1 * dg * np.abs(u) + np.abs(g * sig) * du + 8 * eps * np.abs(a)
            D = Wd[s].reshape(Ns, H).T if down_T else Wd[s]
            ys, dy = seq_dot(a, D)
            y += ys
            bound += da @ np.abs(D).T + dy
        return y, bound + 4 * eps * np.abs(y)          # the two shared outputs summed, then added

    ref, bound = mlp()
    assert np.all(np.abs(got - ref) <= bound)
    rms = np.sqrt((ref ** 2).mean())
    assert bound.max() < 1e-3 * rms                     # the bound is tight enough to mean something
    for wrong in (dict(gate_first=False), dict(with_silu=False), dict(down_T=True)):
        alt, _ = mlp(**wrong)
        assert np.abs(alt - ref).max() > 100 * bound.max(), wrong
    # and the bf16 output is the single rounding of that fp32 sum
    assert np.array_equal(r["out"], _f32_to_bf16_bits(r["out_f32"]))


def test_layer_empty_batch():
    wl = synth.WORKLOADS["tiny"]
    layer = _tiny_layer(wl)
    r = oracle.moe_forward(layer, np.zeros((0, wl.H), np.uint16), np.zeros((0, wl.E), np.float32),
                           wl.k)
    assert r["out"].shape == (0, wl.H)
    assert np.all(r["offsets"] == 0)


# ------------------------------------------------------------------------------------------------
# row-scaled FP8 (W8A8) experts
# ------------------------------------------------------------------------------------------------

def test_row_quant_closed_form():
    w = np.zeros((4, 128), np.float32)
    w[0, :] = 0.02734375          # 7 * 2^-8: scale = 2^-14 exactly, every code E4M3(448) = 0x7e
    w[1, 0] = -1.0                # scale = fp32(1/448); -448 -> 0xfe
    w[1, 1] = 0.25                # 112 = 1.75 * 2^6 -> 0x6e
    w[3, 5] = 0.875               # scale 2^-9; the other entries 0 -> code 0
    q, s = oracle.quant_rows(_f32_to_bf16_bits(w))
    assert s[0] == 2.0 ** -14 and np.all(q[0] == 0x7E)
    assert s[1] == np.float32(1.0) / np.float32(448.0)
    assert list(q[1, :3]) == [0xFE, 0x6E, 0x00]
    assert s[2] == 0.0 and not q[2].any()
    assert s[3] == 2.0 ** -9 and q[3, 5] == 0x7E and int(q[3].astype(np.int64).sum()) == 0x7E


def _w8_layer_from_f32(Wg, Wu, Wd):
    """Row-quantize fp32 expert weights [E,N,H],[E,N,H],[E,H,N] (rounded to bf16 first)."""
    E, N, H = Wg.shape
    def rq(W):
        qs = [oracle.quant_rows(_f32_to_bf16_bits(W[e])) for e in range(E)]
        return np.stack([a for a, _ in qs]), np.stack([b for _, b in qs])
    (gq, gs), (uq, us), (dq, ds) = rq(Wg), rq(Wu), rq(Wd)
    return oracle.Layer.w8a8(E, H, N, gq, uq, dq, gs, us, ds), (gq, gs, uq, us, dq, ds)


def test_w8a8_constant_closed_form():
    want = {}
    for line in golden_lines("constant_layer.txt"):
        t, o, hq = line.split()
        want[int(t)] = (float(o), int(hq, 16))
    T, H, N, E, k = 4, 128, 128, 2, 1
    w0 = 0.02734375
    sgn = np.array([1.0, -1.0], np.float32)[:, None, None]
    Wg = np.broadcast_to(sgn * w0, (E, N, H)).astype(np.float32)
    Wd = np.broadcast_to(sgn * w0, (E, H, N)).astype(np.float32)
    layer, (gq, gs, _, _, dq, ds) = _w8_layer_from_f32(Wg, Wg, Wd)
    assert np.all(gs == 2.0 ** -14) and np.all(ds == 2.0 ** -14)
    assert np.all(gq[0] == 0x7E) and np.all(gq[1] == 0xFE)
    x = _f32_to_bf16_bits(np.full((T, H), 0.875, np.float32))
    lg = np.array([[1, 0], [0, 1], [1, 0], [0, 1]], np.float32)
    r = oracle.moe_forward(layer, x, lg, k)
    out = oracle.bf16_to_f32(r["out"])
    sig = lambda v: 1.0 / (1.0 + math.exp(-v))
    for t in range(T):
        assert np.all(out[t] == want[t][0]), (t, out[t, :4])
        assert np.all(r["hq"][r["row_of_pair"][t]] == want[t][1])
        s = 1.0 if t % 2 == 0 else -1.0
        assert np.allclose(r["out_f32"][t], s * 3.5 * 9.37890625 * sig(s * 3.0625), rtol=1e-6)


def test_w8a8_down_projection_within_fp32_bound():
    """y[r, m] = (sum_n dec(hq[r,n]) dec(wd[e,m,n])) * s_wd[e,m] * s_h[r], checked row by row
    against an fp64 sum of the same codes within the sequential-fp32 error bound.  Rows of the
    weights are scaled over 2^-3..2^3 so that a scale applied per column, or a transposed
    weight, is far outside the bound."""
    rng = np.random.default_rng(11)
    T, H, N, E, k = 12, 256, 128, 4, 2
    rs_g = 2.0 ** rng.uniform(-3, 3, (E, N, 1))
    rs_d = 2.0 ** rng.uniform(-3, 3, (E, H, 1))
    Wg = (rng.standard_normal((E, N, H)) * 0.02 * rs_g).astype(np.float32)
    Wu = (rng.standard_normal((E, N, H)) * 0.02 * rs_g[:, ::-1]).astype(np.float32)
    Wd = (rng.standard_normal((E, H, N)) * 0.02 * rs_d).astype(np.float32)
    layer, (_, _, _, _, dq, ds) = _w8_layer_from_f32(Wg, Wu, Wd)
    x = _f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    lg = rng.standard_normal((T, E)).astype(np.float32)
    r = oracle.moe_forward(layer, x, lg, k)
    dec = oracle.e4m3_decode_table().astype(np.float64)
    for e in range(E):
        for row in range(r["offsets"][e], r["offsets"][e + 1]):
            terms = dec[r["hq"][row]][None, :] * dec[dq[e]]          # [H, N]
            exact = terms.sum(axis=1)
            bound = N * 2.0 ** -24 * np.abs(terms).sum(axis=1)
            acc = r["y"][row].astype(np.float64) / (ds[e].astype(np.float64) * r["s_h"][row])
            # the two final fp32 multiplies add at most 2 ulp of the result each
            slack = 4 * 2.0 ** -24 * np.abs(exact)
            assert np.all(np.abs(acc - exact) <= bound + slack + 1e-30), (e, row)


def test_w8a8_single_expert_vs_fp64_mlp():
    """E = 1, k = 1: a row-scaled FP8 SwiGLU MLP against a textbook fp64 MLP on the dequantized
    FP8 weights and the unquantized input: the gap is the FP8 activation rounding only."""
    rng = np.random.default_rng(12)
    T, H, N = 24, 512, 256
    Wg = (rng.standard_normal((1, N, H)) * 0.02 * 2.0 ** rng.uniform(-3, 3, (1, N, 1))).astype(np.float32)
    Wu = (rng.standard_normal((1, N, H)) * 0.02 * 2.0 ** rng.uniform(-3, 3, (1, N, 1))).astype(np.float32)
    Wd = (rng.standard_normal((1, H, N)) * 0.02 * 2.0 ** rng.uniform(-3, 3, (1, H, 1))).astype(np.float32)
    layer, (gq, gs, uq, us, dq, ds) = _w8_layer_from_f32(Wg, Wu, Wd)
    x = _f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    r = oracle.moe_forward(layer, x, np.zeros((T, 1), np.float32), 1)
    dec = oracle.e4m3_decode_table().astype(np.float64)
    Dg = dec[gq[0]] * gs[0][:, None]
    Du = dec[uq[0]] * us[0][:, None]
    Dd = dec[dq[0]] * ds[0][:, None]
    xf = oracle.bf16_to_f32(x).astype(np.float64)
    g, u = xf @ Dg.T, xf @ Du.T
    ref = (g / (1 + np.exp(-g)) * u) @ Dd.T
    got = r["out_f32"].astype(np.float64)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel < 0.05, rel
    assert np.corrcoef(got.ravel(), ref.ravel())[0, 1] > 0.998


def test_w8a8_dense_brute_force_matches_permuted():
    wl = synth.WORKLOADS["tiny"]
    layer = oracle.quant_workload_layer_w8a8(wl)
    assert layer.fmt == oracle.FMT_W8A8
    x, lg = synth.tokens(wl), synth.logits(wl)
    r = oracle.moe_forward(layer, x, lg, wl.k)
    d = oracle.moe_forward_dense(layer, x, lg, wl.k)
    assert np.array_equal(r["out"], d["out"])
    for p in range(wl.P):
        t, j = divmod(p, wl.k)
        e = r["ids"][t, j]
        row = r["row_of_pair"][p]
        assert np.array_equal(r["hq"][row], d["hq"][t, e])
        assert np.array_equal(r["y"][row], d["y"][t, e])
    # the two formats agree to the INT4 weight-rounding gap (a step of amax/7 per weight,
    # through three projections), not bit for bit
    w4 = oracle.moe_forward(_tiny_layer(wl), x, lg, wl.k)
    a, b = r["out_f32"].astype(np.float64), w4["out_f32"].astype(np.float64)
    assert np.linalg.norm(a - b) / np.linalg.norm(a) < 0.35
    assert not np.array_equal(r["out"], w4["out"])


# ------------------------------------------------------------------------------------------------
# NVFP4 experts
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("line", list(golden_lines("e2m1_lut.txt")))
def test_e2m1_lut_golden(line):
    c, v = line.split()
    got = oracle.e2m1_decode(int(c))
    assert got == float(v) and math.copysign(1.0, got) == math.copysign(1.0, float(v))


def _e2m1_nearest_numpy(x):
    """Nearest of the 16 E2M1 values by sorting distances (ties: the even code), sign kept."""
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float64)
    out = []
    for v in np.asarray(x, np.float64):
        d = np.abs(abs(v) - grid)
        cand = np.flatnonzero(d == d.min())
        i = int(cand[0]) if len(cand) == 1 else int(cand[cand % 2 == 0][0])
        out.append(i | (8 if math.copysign(1.0, v) < 0 else 0))
    return np.array(out)


def test_e2m1_encode_vs_brute_force():
    rng = np.random.default_rng(31)
    mids = np.array([.25, .75, 1.25, 1.75, 2.5, 3.5, 5.0])
    xs = np.concatenate([rng.uniform(-8, 8, 3000), mids, -mids, np.nextafter(mids, 0), np.nextafter(mids, 9),
                         [0.0, -0.0, 6.0, 7.9, 100.0, -100.0]]).astype(np.float32)
    got = np.array([oracle.e2m1_encode(float(v)) for v in xs])
    assert np.array_equal(got, _e2m1_nearest_numpy(xs))


def test_nvfp4_worked_row():
    want = {}
    for line in golden_lines("nvfp4_worked.txt"):
        kind, i, v = line.split()
        want[(kind, int(i))] = int(v, 16)
    b0 = np.array([6, 3, 1.25, -0.75, 0.25, -6, 0, 2.5, 5, -1.75, 0.5, 4, -3.5, 1, 0, 0], np.float32) * 2.0 ** -4
    b1 = np.zeros(16, np.float32)
    b1[0] = 1.5 * 2.0 ** -6
    codes, scales, s2 = oracle.nvfp4_quant(_f32_to_bf16_bits(np.concatenate([b0, b1])[None, :]))
    assert s2 == np.float32(0.375) / np.float32(2688)
    for (kind, i), v in want.items():
        assert (scales[0, i] if kind == "scale" else codes[0, i]) == v, (kind, i)


def _nvfp4_dequant(codes, scales, s2):
    """The page's dequant math in fp64: LUT[code] * scale[block] * scale2, low nibble first."""
    lut = np.array([oracle.e2m1_decode(c) for c in range(16)])
    e4 = oracle.e4m3_decode_table().astype(np.float64)
    rows, half = codes.shape
    c = np.empty((rows, 2 * half), np.int64)
    c[:, 0::2] = codes & 15
    c[:, 1::2] = codes >> 4
    return lut[c] * np.repeat(e4[scales], 16, axis=1) * float(s2)


def test_nvfp4_roundtrip_error_bound():
    """Every weight is within half an E2M1 step (relative 1/4 of the block's spacing; the
    grid's widest gap is 2 at the top) of its dequantized value, block by block, and the
    row maximum maps to +-6 * scale * scale2 of its block."""
    rng = np.random.default_rng(32)
    w = (rng.standard_normal((64, 256)) * 0.02 * 2.0 ** rng.uniform(-4, 4, (64, 1))).astype(np.float32)
    w[3, 16:32] = 0.0                                  # an all-zero block: scale 0, codes 0
    wb = _f32_to_bf16_bits(w)
    codes, scales, s2 = oracle.nvfp4_quant(wb)
    wf = oracle.bf16_to_f32(wb).astype(np.float64)
    deq = _nvfp4_dequant(codes, scales, s2)
    assert scales[3, 1] == 0 and not codes[3, 8:16].any()
    e4 = oracle.e4m3_decode_table().astype(np.float64)
    d = np.repeat(e4[scales], 16, axis=1) * float(s2)           # the block's unit
    assert np.all(np.abs(deq - wf) <= d * 1.0 + 1e-30)         # half of the widest gap (2) of the grid
    # relative error of the grid: at most half a step of 2^-1 relative spacing above 1
    big = np.abs(wf) >= d
    assert np.all(np.abs(deq - wf)[big] <= 0.25 * np.abs(wf)[big] + 1e-12)
    # the largest weight of the tensor saturates the top code exactly
    r, c = np.unravel_index(np.argmax(np.abs(wf)), wf.shape)
    assert (codes[r, c // 2] >> (4 * (c % 2))) & 7 == 7


def _f4_layer_from_f32(Wg, Wu, Wd):
    E = Wg.shape[0]
    def qp(W):
        r = [oracle.nvfp4_quant(_f32_to_bf16_bits(W[e])) for e in range(E)]
        return (np.stack([a for a, _, _ in r]), np.stack([b for _, b, _ in r]),
                np.array([c for _, _, c in r], np.float32))
    g, u, d = qp(Wg), qp(Wu), qp(Wd)
    N, H = Wg.shape[1], Wg.shape[2]
    return oracle.Layer.nvfp4(E, H, N, g[0], u[0], d[0], g[1], u[1], d[1], g[2], u[2], d[2]), (g, u, d)


def test_nvfp4_constant_closed_form():
    """The constant layer of tests/golden/constant_layer.txt in NVFP4: every weight is 6 x
    block scale 448 x scale2 (= w0 / 2688) = w0 up to scale2's rounding, so the outputs match
    the same golden values."""
    want = {}
    for line in golden_lines("constant_layer.txt"):
        t, o, hq = line.split()
        want[int(t)] = (float(o), int(hq, 16))
    T, H, N, E, k = 4, 128, 128, 2, 1
    w0 = 0.02734375
    sgn = np.array([1.0, -1.0], np.float32)[:, None, None]
    Wg = np.broadcast_to(sgn * w0, (E, N, H)).astype(np.float32)
    Wd = np.broadcast_to(sgn * w0, (E, H, N)).astype(np.float32)
    layer, (g, _, _) = _f4_layer_from_f32(Wg, Wg, Wd)
    assert np.all(g[0][0] == 0x77) and np.all(g[0][1] == 0xFF) and np.all(g[1] == 0x7E)
    x = _f32_to_bf16_bits(np.full((T, H), 0.875, np.float32))
    lg = np.array([[1, 0], [0, 1], [1, 0], [0, 1]], np.float32)
    r = oracle.moe_forward(layer, x, lg, k)
    out = oracle.bf16_to_f32(r["out"])
    for t in range(T):
        assert np.all(out[t] == want[t][0]), (t, out[t, :4])
        assert np.all(r["hq"][r["row_of_pair"][t]] == want[t][1])


def test_nvfp4_single_expert_vs_fp64_mlp():
    """E = 1, k = 1: the NVFP4 layer against a textbook fp64 SwiGLU MLP on the weights
    dequantized by the page's formula and the unquantized input."""
    rng = np.random.default_rng(33)
    T, H, N = 24, 512, 256
    def w(rows, K):
        return (rng.standard_normal((1, rows, K)) * 0.02 * 2.0 ** rng.uniform(-3, 3, (1, rows, 1))).astype(np.float32)
    layer, (g, u, d) = _f4_layer_from_f32(w(N, H), w(N, H), w(H, N))
    x = _f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    r = oracle.moe_forward(layer, x, np.zeros((T, 1), np.float32), 1)
    Dg, Du, Dd = (_nvfp4_dequant(p[0][0], p[1][0], p[2][0]) for p in (g, u, d))
    xf = oracle.bf16_to_f32(x).astype(np.float64)
    gg, uu = xf @ Dg.T, xf @ Du.T
    ref = (gg / (1 + np.exp(-gg)) * uu) @ Dd.T
    got = r["out_f32"].astype(np.float64)
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 0.05
    assert np.corrcoef(got.ravel(), ref.ravel())[0, 1] > 0.998


def test_nvfp4_dense_brute_force_matches_permuted():
    wl = synth.WORKLOADS["tiny"]
    layer = oracle.quant_workload_layer_nvfp4(wl)
    assert layer.fmt == oracle.FMT_NVFP4
    x, lg = synth.tokens(wl), synth.logits(wl)
    r = oracle.moe_forward(layer, x, lg, wl.k)
    d = oracle.moe_forward_dense(layer, x, lg, wl.k)
    assert np.array_equal(r["out"], d["out"])
    for p in range(wl.P):
        t, j = divmod(p, wl.k)
        e = r["ids"][t, j]
        row = r["row_of_pair"][p]
        assert np.array_equal(r["hq"][row], d["hq"][t, e])
        assert np.array_equal(r["y"][row], d["y"][t, e])


def _hybrid_from(wl, hot_ids):
    """A hybrid layer of workload `wl`: the NVFP4 slabs of the hot experts, the W4A8 slabs of the
    others, both taken from the single-format layers of the same seeded weights."""
    w4 = oracle.pack_workload_layer(wl)
    f4 = oracle.quant_workload_layer_nvfp4(wl)
    hot_ids = np.array(hot_ids, np.int32)
    cold_ids = np.array([e for e in range(wl.E) if e not in set(hot_ids.tolist())], np.int32)
    cold = oracle.Layer(wl.E - len(hot_ids), wl.H, wl.N, w4.gate_packed[cold_ids], w4.up_packed[cold_ids],
                        w4.down_packed[cold_ids], w4.gate_scales[cold_ids], w4.up_scales[cold_ids],
                        w4.down_scales[cold_ids])
    hot = oracle.Layer.nvfp4(len(hot_ids), wl.H, wl.N, f4.gate_f4[hot_ids], f4.up_f4[hot_ids],
                             f4.down_f4[hot_ids], f4.gate_bs[hot_ids], f4.up_bs[hot_ids], f4.down_bs[hot_ids],
                             f4.gate_s2[hot_ids], f4.up_s2[hot_ids], f4.down_s2[hot_ids])
    return oracle.Layer.hybrid(cold, hot, hot_ids, cold_ids), w4, f4


def test_hybrid_dispatches_each_expert_to_its_format():
    """Every routed pair of the hybrid layer computes exactly what the single-format layer of
    its expert's format computes for it (hot experts: NVFP4, the rest: W4A8)."""
    wl = synth.WORKLOADS["tiny"]
    hot_ids = [6, 1, 3]                                 # slab order differs from expert order
    hy, w4, f4 = _hybrid_from(wl, hot_ids)
    x, lg = synth.tokens(wl), synth.logits(wl)
    rh = oracle.moe_forward(hy, x, lg, wl.k)
    r4 = oracle.moe_forward(w4, x, lg, wl.k)
    rf = oracle.moe_forward(f4, x, lg, wl.k)
    assert np.array_equal(rh["ids"], r4["ids"])
    for p in range(wl.P):
        t, j = divmod(p, wl.k)
        ref = rf if rh["ids"][t, j] in hot_ids else r4
        assert np.array_equal(rh["hq"][rh["row_of_pair"][p]], ref["hq"][ref["row_of_pair"][p]])
        assert np.array_equal(rh["y"][rh["row_of_pair"][p]], ref["y"][ref["row_of_pair"][p]])
    d = oracle.moe_forward_dense(hy, x, lg, wl.k)
    assert np.array_equal(d["out"], rh["out"])


def test_hybrid_rejects_lists_that_do_not_cover_every_expert():
    wl = synth.WORKLOADS["tiny"]
    hy, _, _ = _hybrid_from(wl, [6, 1, 3])
    hy.cold_ids = hy.cold_ids[:-1].copy()               # an expert in neither list
    with pytest.raises(ValueError):
        oracle.moe_forward(hy, synth.tokens(wl), synth.logits(wl), wl.k)


# ------------------------------------------------------------------------------------------------
# rule 3 with rule 2's allowance (tests/parity.py)
# ------------------------------------------------------------------------------------------------

def test_given_h_reproduces_the_forward():
    wl = synth.WORKLOADS["tiny"]
    for layer in (oracle.pack_workload_layer(wl), oracle.quant_workload_layer_nvfp4(wl)):
        x, lg = synth.tokens(wl), synth.logits(wl)
        r = oracle.moe_forward(layer, x, lg, wl.k)
        out, out_f32 = oracle.moe_forward_given_h(layer, x, lg, wl.k, r["hq"][r["row_of_pair"]],
                                                  r["s_h"][r["row_of_pair"]])
        assert np.array_equal(out, r["out"]) and np.array_equal(out_f32, r["out_f32"])


def test_planted_code_flip_is_local_and_only_explained_for_its_token():
    from parity import check_output, check_output_explained
    wl = synth.WORKLOADS["tiny"]
    layer = oracle.pack_workload_layer(wl)
    x, lg = synth.tokens(wl), synth.logits(wl)
    r = oracle.moe_forward(layer, x, lg, wl.k)
    hq = r["hq"][r["row_of_pair"]].copy()
    sh = r["s_h"][r["row_of_pair"]].copy()
    t = 5
    p = t * wl.k
    n = int(np.argmax(oracle.e4m3_decode_table()[hq[p]]))   # the largest code of the row
    hq[p, n] += 1 if hq[p, n] & 0x7F < 0x7E else -1         # one E4M3 step
    alt, _ = oracle.moe_forward_given_h(layer, x, lg, wl.k, hq, sh)
    changed = (alt != r["out"]).any(axis=1)
    assert changed[t] and changed.sum() == 1                  # only the token of the flipped row
    flipped = np.zeros(wl.T, bool)
    flipped[t] = True
    check_output_explained(alt, r["out"], alt, flipped)       # explained by its own flip
    # the same outputs with the allowance withheld: fail unless already within tolerance
    within = True
    try:
        check_output(alt, r["out"])
    except AssertionError:
        within = False
    if not within:
        with pytest.raises(AssertionError):
            check_output_explained(alt, r["out"], alt, np.zeros(wl.T, bool))


# ------------------------------------------------------------------------------------------------
# the generator (input recipe)
# ------------------------------------------------------------------------------------------------

def test_generator_moments_and_determinism():
    a = synth.normal_f32(0, 77, 2_000_000)
    b = synth.normal_f32(0, 77, 1000, start=500)
    assert np.array_equal(a[500:1500], b)
    assert abs(a.mean()) < 3e-3 and abs(a.std() - 1) < 3e-3
    assert abs((a.astype(np.float64) ** 4).mean() - 3) < 0.03
    assert not np.array_equal(a[:100], synth.normal_f32(1, 77, 100))


def test_workload_recipe():
    wl = synth.WORKLOADS["decode_t8"]
    m = synth.outlier_mask(wl)
    assert int(m.sum()) == 41
    x = oracle.bf16_to_f32(synth.tokens(wl))
    assert x.shape == (8, 4096)
    assert np.abs(x[:, m == 1]).mean() > 10 * np.abs(x[:, m == 0]).mean()
    z = synth.WORKLOADS["prefill_t2048_zipf"]
    ranks = synth.expert_ranks(z)
    assert sorted(ranks.tolist()) == list(range(1, 257))
    b = synth.logit_bias(z)
    assert np.allclose(b, -1.1 * np.log(ranks), rtol=0, atol=1e-12)
