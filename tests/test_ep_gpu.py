"""Expert-parallel entry points on the GPU, called through the C ABI.

* moe_ep_dispatch's records and counts against the oracle, byte for byte (rule 1: FP8 codes,
  scales, routing);
* one rank (EpLayer with no process group) against moe_w4a8_forward, bit for bit;
* 2 and 4 ranks emulated on one GPU (each rank's calls in turn, the exchanges done by copying
  row ranges between the ranks' buffers; no kernel waits on another) against the oracle's layer
  on all tokens under rule 3;
* a record naming an expert outside the receiver's range: a zero row and the device-status
  word, no fault; empty batches."""
import numpy as np
import pytest

import oracle
import synth
from conftest import cuda_ok
from parity import output_errors

pytestmark = pytest.mark.gpu

if cuda_ok():
    import torch
    import bit_quantized_moe_token_b200 as moe
    from bit_quantized_moe_token_b200.ep import EpLayer, local_experts
    from test_parity_gpu import _host_layer_and_dev, _report, bits, to_dev_bf16


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not cuda_ok():
        pytest.skip("no CUDA device")


def _inputs(seed, T, E, H):
    x = synth.normal_bf16(seed, 72_000, T * H, 1.0).reshape(T, H)
    logits = synth.normal_f32(seed, 72_001, T * E, 1.0).reshape(T, E)
    return x, logits


def _expected_records(x, logits, E, k, n_ranks):
    """The records and counts the C ABI declares, built from the oracle's S1-S3."""
    T, H = x.shape
    xq, sx = oracle.quant_tokens(x)
    ids, _ = oracle.route_topk(logits, k)
    offsets, _, rop = oracle.permute(ids, E)
    El = E // n_ranks
    rec = np.zeros((T * k, H + 16), np.uint8)
    for p in range(T * k):
        rec[rop[p], :H] = xq[p // k]
        rec[rop[p], H:H + 4] = np.frombuffer(np.float32(sx[p // k]).tobytes(), np.uint8)
        rec[rop[p], H + 4:H + 8] = np.frombuffer(np.int32(ids.flat[p] % El).tobytes(), np.uint8)
    counts = np.array([offsets[(r + 1) * El] - offsets[r * El] for r in range(n_ranks)], np.int32)
    return rec, counts


# (E, H, N, k, T): narrow 16- and 32-row token tiles, 192-row tiles, 128-row tiles with the short
# segments (9 of 16 here) on 32-row tiles
CASES = [(8, 256, 128, 2, 5), (8, 256, 128, 2, 37), (16, 256, 128, 4, 64), (8, 512, 256, 2, 700),
         (16, 4096, 2048, 2, 260)]


@pytest.mark.parametrize("E,H,N,k,T", CASES)
@pytest.mark.parametrize("n_ranks", [1, 2, 4])
def test_ep_dispatch_records_bitexact(E, H, N, k, T, n_ranks):
    x, logits = _inputs(11, T, E, H)
    s = moe.layer_struct(E, H, N)
    counts = torch.empty(n_ranks, dtype=torch.int32, device="cuda")
    rec = torch.empty((T * k, moe.ep_record_bytes(H)), dtype=torch.uint8, device="cuda")
    ws = torch.empty(moe.moe_ep_dispatch_workspace_bytes(s, T, k), dtype=torch.uint8, device="cuda")
    moe.moe_ep_dispatch(s, to_dev_bf16(x), torch.from_numpy(logits).cuda(), k, n_ranks, counts, rec, ws)
    torch.cuda.synchronize()
    assert moe.moe_last_device_status() == 0
    want_rec, want_counts = _expected_records(x, logits, E, k, n_ranks)
    assert np.array_equal(counts.cpu().numpy(), want_counts)
    assert np.array_equal(rec.cpu().numpy(), want_rec)


@pytest.mark.parametrize("E,H,N,k,T", CASES)
@pytest.mark.parametrize("n_shared", [0, 1])
def test_ep_one_rank_equals_forward(E, H, N, k, T, n_shared):
    _, dl = _host_layer_and_dev(E, H, N, seed=21, n_shared=n_shared, shared_N=128 if n_shared else 0)
    x, logits = _inputs(12, T, E, H)
    xd, ld = to_dev_bf16(x), torch.from_numpy(logits).cuda()
    want = moe.forward(dl, xd, ld, k)
    ep = EpLayer(dl, local_experts(dl, 0, 1))
    got = ep.forward(xd, ld, k)
    torch.cuda.synchronize()
    assert moe.moe_last_device_status() == 0
    assert ep.stats.sent == ep.stats.received == [T * k]
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))


def _emulated_ranks(dl, x, logits, k, T_of_rank, n_ranks):
    """Every rank's three calls on one GPU, the exchanges as copies of row ranges."""
    E, H = dl.E, dl.H
    rb = moe.ep_record_bytes(H)
    locs = [local_experts(dl, r, n_ranks) for r in range(n_ranks)]
    t0 = np.concatenate([[0], np.cumsum(T_of_rank)])
    xs, ws, sends, counts = [], [], [], []
    for r in range(n_ranks):
        T = T_of_rank[r]
        xr = to_dev_bf16(np.ascontiguousarray(x[t0[r]:t0[r + 1]]))
        lr = torch.from_numpy(np.ascontiguousarray(logits[t0[r]:t0[r + 1]])).cuda()
        w = torch.empty(max(moe.moe_ep_dispatch_workspace_bytes(dl, T, k), 256), dtype=torch.uint8, device="cuda")
        c = torch.empty(n_ranks, dtype=torch.int32, device="cuda")
        s = torch.empty((T * k, rb), dtype=torch.uint8, device="cuda")
        moe.moe_ep_dispatch(dl, xr, lr, k, n_ranks, c, s, w)
        xs.append(xr), ws.append(w), sends.append(s), counts.append(c)
    cnt = torch.stack(counts).cpu().numpy()              # cnt[sender, owner]
    soff = np.concatenate([np.zeros((n_ranks, 1), np.int64), np.cumsum(cnt, axis=1)], axis=1)
    ys = []
    for o in range(n_ranks):                              # owner o: records from senders 0, 1, ...
        recv = torch.cat([sends[s][soff[s, o]:soff[s, o + 1]] for s in range(n_ranks)])
        y = torch.empty((recv.shape[0], H), dtype=torch.float32, device="cuda")
        we = torch.empty(max(moe.moe_ep_experts_workspace_bytes(locs[o], recv.shape[0]), 256),
                         dtype=torch.uint8, device="cuda")
        moe.moe_ep_experts_forward(locs[o], recv, y, we)
        ys.append(y)
    roff = np.concatenate([np.zeros((1, n_ranks), np.int64), np.cumsum(cnt, axis=0)], axis=0)  # per owner
    outs = []
    for s in range(n_ranks):                              # sender s: rows back from owners 0, 1, ...
        y_back = torch.cat([ys[o][roff[s, o]:roff[s + 1, o]] for o in range(n_ranks)])
        out = torch.empty((T_of_rank[s], H), dtype=torch.bfloat16, device="cuda")
        moe.moe_ep_combine(dl, xs[s], y_back, k, out, ws[s])
        outs.append(out)
    torch.cuda.synchronize()
    assert moe.moe_last_device_status() == 0
    return np.concatenate([bits(o) for o in outs]), cnt


@pytest.mark.parametrize("E,H,N,k,T", CASES)
@pytest.mark.parametrize("n_ranks", [2, 4])
def test_ep_emulated_ranks_vs_oracle(E, H, N, k, T, n_ranks):
    hl, dl = _host_layer_and_dev(E, H, N, seed=22, n_shared=1, shared_N=128)
    x, logits = _inputs(13, T, E, H)
    # ragged token counts per rank, one rank possibly without tokens
    cuts = np.sort(np.random.default_rng(T + n_ranks).integers(0, T + 1, n_ranks - 1))
    T_of_rank = list(np.diff(np.concatenate([[0], cuts, [T]])).astype(int))
    got, cnt = _emulated_ranks(dl, x, logits, k, T_of_rank, n_ranks)
    ref = oracle.moe_forward(hl, x, logits, k)
    assert cnt.sum() == T * k
    ratio = output_errors(got, ref["out"])
    worst = float(ratio.max(initial=0.0))
    _report(worst_out_err_over_tol=round(worst, 4), outputs=int(ratio.size), out_of_tol=int((ratio > 1).sum()))
    assert worst <= 1.0, f"{int((ratio > 1).sum())} outputs out of tolerance; worst {worst:.3f}x tol"


def test_ep_bad_expert_index_gives_zero_row_and_status():
    E, H, N, k, T = 8, 256, 128, 2, 9
    _, dl = _host_layer_and_dev(E, H, N, seed=23)
    x, logits = _inputs(14, T, E, H)
    s = moe.layer_struct(E, H, N)
    counts = torch.empty(1, dtype=torch.int32, device="cuda")
    rec = torch.empty((T * k, moe.ep_record_bytes(H)), dtype=torch.uint8, device="cuda")
    ws = torch.empty(moe.moe_ep_dispatch_workspace_bytes(s, T, k), dtype=torch.uint8, device="cuda")
    moe.moe_ep_dispatch(s, to_dev_bf16(x), torch.from_numpy(logits).cuda(), k, 1, counts, rec, ws)
    torch.cuda.synchronize()
    bad = rec.clone()
    bad[3, H + 4:H + 8] = torch.tensor(np.frombuffer(np.int32(E).tobytes(), np.uint8).copy())
    bad[7, H + 4:H + 8] = torch.tensor(np.frombuffer(np.int32(-1).tobytes(), np.uint8).copy())
    for gather_tiles in (True, False):
        recs = bad if gather_tiles else bad.repeat(40, 1)      # 720 records: wide tiles
        R = recs.shape[0]
        y = torch.full((R, H), float("nan"), dtype=torch.float32, device="cuda")
        we = torch.empty(moe.moe_ep_experts_workspace_bytes(dl, R), dtype=torch.uint8, device="cuda")
        moe.moe_ep_experts_forward(dl, recs, y, we)
        torch.cuda.synchronize()
        assert moe.moe_last_device_status() == -1                            # MOE_ERR_INVALID_ARG
        assert moe.moe_last_device_status() == 0                             # read and cleared
        yh = y.cpu().numpy()
        assert np.all(yh[3] == 0) and np.all(yh[7] == 0)
        assert np.all(np.isfinite(yh))


def test_ep_empty_batches():
    E, H, N, k = 8, 256, 128, 2
    _, dl = _host_layer_and_dev(E, H, N, seed=24)
    counts = torch.full((2,), 7, dtype=torch.int32, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    x = torch.empty((0, H), dtype=torch.bfloat16, device="cuda")
    lg = torch.empty((0, E), dtype=torch.float32, device="cuda")
    rec = torch.empty((0, moe.ep_record_bytes(H)), dtype=torch.uint8, device="cuda")
    moe.moe_ep_dispatch(dl, x, lg, k, 2, counts, rec, ws)
    moe.moe_ep_experts_forward(local_experts(dl, 0, 2), rec, torch.empty((0, H), device="cuda"), ws)
    out = torch.empty((0, H), dtype=torch.bfloat16, device="cuda")
    moe.moe_ep_combine(dl, x, torch.empty((0, H), device="cuda"), k, out, ws)
    torch.cuda.synchronize()
    assert counts.cpu().tolist() == [0, 0]
    assert moe.moe_last_device_status() == 0


_NCCL_ONE_RANK = r'''
import os, sys, numpy as np, torch, torch.distributed as dist
from datetime import timedelta
sys.path.insert(0, os.environ["MOE_ROOT"]); sys.path.insert(0, os.path.join(os.environ["MOE_ROOT"], "tests"))
torch.cuda.set_device(0)
dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=60), device_id=torch.device("cuda", 0))
try:
    import bit_quantized_moe_token_b200 as moe
    from bit_quantized_moe_token_b200.ep import EpLayer, local_experts
    from test_parity_gpu import _host_layer_and_dev, to_dev_bf16
    from test_ep_gpu import _inputs
    for (E, H, N, k, T) in ((8, 256, 128, 2, 37), (8, 512, 256, 2, 700)):
        _, dl = _host_layer_and_dev(E, H, N, seed=25, n_shared=1, shared_N=128)
        x, logits = _inputs(15, T, E, H)
        xd, ld = to_dev_bf16(x), torch.from_numpy(logits).cuda()
        want = moe.forward(dl, xd, ld, k)
        ep = EpLayer(dl, local_experts(dl, 0, 1))
        assert ep.grouped and ep.n_ranks == 1
        got = ep.forward(xd, ld, k)
        torch.cuda.synchronize()
        assert moe.moe_last_device_status() == 0
        assert torch.equal(got.view(torch.int16), want.view(torch.int16)), (E, H, N, k, T)
    print("nccl one rank ok")
finally:
    dist.destroy_process_group()
'''


def test_ep_nccl_exchanges_one_rank():
    """The NCCL all-to-all exchanges of EpLayer on one GPU (a process group of one rank: the
    exchanges run, no rank waits on another): bit-exact against moe_w4a8_forward."""
    import os
    import socket
    import subprocess
    import sys
    from conftest import ROOT
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    env = dict(os.environ, MOE_ROOT=ROOT, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
               NCCL_NVLS_ENABLE="0")
    r = subprocess.run([sys.executable, "-c", _NCCL_ONE_RANK], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "nccl one rank ok" in r.stdout
