"""Expert-parallel forward over 2 and 4 gloo ranks on the CPU.

What runs is EpLayer's host logic (bit_quantized_moe_token_b200/ep.py): the per-owner counts,
the two all-to-all exchanges of records and output rows, and the bookkeeping that brings each
row back to its pair.  The three library calls are replaced by OracleEpOps, the oracle's
restatement of each of them on CPU tensors with the record layout the C ABI declares
(MOE_EP_RECORD_BYTES).  The ranks' outputs, put together, must equal the oracle's one-process
layer on all tokens bit for bit: every expert row and every combine is the same oracle
arithmetic, so any difference is a record sent to the wrong owner, a row returned to the wrong
slot, or a wrong expert index.  (On the GPU the same calls run in the library's kernels; see
tests/test_ep_gpu.py.)"""
import os
import socket
import sys
from datetime import timedelta

import numpy as np
import pytest

from conftest import ROOT

H, N, E, K = 256, 128, 8, 2
META = 16   # record bytes after the codes: scale, local expert, padding


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer(seed, n_shared):
    import oracle
    import synth
    base = 70_000 + seed * 10
    gw = synth.normal_bf16(seed, base + 0, E * N * H, 0.02).reshape(E, N, H)
    uw = synth.normal_bf16(seed, base + 1, E * N * H, 0.02).reshape(E, N, H)
    dw = synth.normal_bf16(seed, base + 2, E * H * N, 0.02).reshape(E, H, N)
    gp, gs = zip(*[oracle.rtn_pack(gw[e], 128)[:2] for e in range(E)])
    up, us = zip(*[oracle.rtn_pack(uw[e], 128)[:2] for e in range(E)])
    dp, ds = zip(*[oracle.rtn_pack(dw[e], 128)[:2] for e in range(E)])
    sh = {}
    if n_shared:
        Ns = 128
        sh = dict(sh_gate=synth.normal_bf16(seed, base + 3, n_shared * Ns * H, 0.02).reshape(n_shared, Ns, H),
                  sh_up=synth.normal_bf16(seed, base + 4, n_shared * Ns * H, 0.02).reshape(n_shared, Ns, H),
                  sh_down=synth.normal_bf16(seed, base + 5, n_shared * H * Ns, 0.02).reshape(n_shared, H, Ns))
    return oracle.Layer(E, H, N, np.stack(gp), np.stack(up), np.stack(dp), np.stack(gs), np.stack(us),
                        np.stack(ds), **sh)


def _inputs(seed, T, skew):
    import synth
    x = synth.normal_bf16(seed, 71_000, T * H, 1.0).reshape(T, H)
    logits = synth.normal_f32(seed, 71_001, T * E, 1.0).reshape(T, E)
    if skew:   # every token prefers the first owner's experts: the other owners receive nothing
        logits[:, : E // 4] += 50.0
    return x, logits


class OracleEpOps:
    """The three library calls of an expert-parallel forward restated with the oracle, on CPU
    tensors.  State that the library keeps in the dispatch workspace (gates, record slot of each
    pair) is kept here."""

    def __init__(self):
        self.kept = {}

    @staticmethod
    def dispatch_workspace_bytes(layer, T, k):
        return 256

    @staticmethod
    def experts_workspace_bytes(local, R):
        return 256

    def dispatch(self, layer, x, logits, k, n_ranks, send_counts, send, ws):
        import oracle
        x16 = x.view(__import__("torch").int16).numpy().view(np.uint16)
        xq, sx = oracle.quant_tokens(x16)
        ids, gates = oracle.route_topk(logits.numpy(), k)
        offsets, _, rop = oracle.permute(ids, layer.E)
        El = layer.E // n_ranks
        rec = send.numpy()
        rec[:] = 0
        for p in range(ids.size):
            slot, t = rop[p], p // k
            rec[slot, :layer.H] = xq[t]
            rec[slot, layer.H:layer.H + 4] = np.frombuffer(np.float32(sx[t]).tobytes(), np.uint8)
            rec[slot, layer.H + 4:layer.H + 8] = np.frombuffer(np.int32(ids.flat[p] % El).tobytes(), np.uint8)
        send_counts.numpy()[:] = [offsets[(r + 1) * El] - offsets[r * El] for r in range(n_ranks)]
        self.kept[ws.data_ptr()] = (gates, rop)

    def experts_forward(self, local, recv, y_rows, ws):
        import oracle
        r = recv.numpy()
        if r.shape[0] == 0:
            return
        h = local.H
        q = np.ascontiguousarray(r[:, :h])
        s = np.ascontiguousarray(r[:, h:h + 4]).view(np.float32).ravel()
        e = np.ascontiguousarray(r[:, h + 4:h + 8]).view(np.int32).ravel()
        y_rows.numpy()[:] = oracle.expert_rows(local, q, s, e)

    def combine(self, layer, x, y_back, k, out, ws):
        import oracle
        import torch
        gates, rop = self.kept[ws.data_ptr()]
        y_pairs = y_back.numpy()[rop]            # pair p's row came back to its record slot rop[p]
        x16 = x.view(torch.int16).numpy().view(np.uint16)
        out.view(torch.int16).numpy().view(np.uint16)[:] = oracle.combine(layer, x16, gates, y_pairs, k)


def _worker(rank, world, port, q, T_of_rank, seed, n_shared, skew):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch
    import torch.distributed as dist
    import oracle
    from bit_quantized_moe_token_b200.ep import EpLayer

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        full = _layer(seed, n_shared)
        El = E // world
        local = oracle.expert_slice(full, rank * El, (rank + 1) * El)
        x, logits = _inputs(seed, sum(T_of_rank), skew)
        t0 = sum(T_of_rank[:rank])
        mine = slice(t0, t0 + T_of_rank[rank])
        xt = torch.from_numpy(np.ascontiguousarray(x[mine]).view(np.int16)).view(torch.bfloat16)
        lt = torch.from_numpy(np.ascontiguousarray(logits[mine]))
        ep = EpLayer(full, local, ops=OracleEpOps())
        out = ep.forward(xt, lt, K)
        q.put((rank, out.view(torch.int16).numpy().view(np.uint16).copy(), ep.stats.sent, ep.stats.received))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _run(world, T_of_rank, seed=1, n_shared=0, skew=False):
    import torch.multiprocessing as mp
    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, T_of_rank, seed, n_shared, skew))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    full = _layer(seed, n_shared)
    x, logits = _inputs(seed, sum(T_of_rank), skew)
    ref = oracle.moe_forward(full, x, logits, K)
    got = np.concatenate([r[1] for r in res])
    assert np.array_equal(got, ref["out"])
    # what each rank sent is what its owners received, and every pair went to its expert's owner
    sent = np.array([r[2] for r in res])
    recv = np.array([r[3] for r in res])
    assert np.array_equal(sent.T, recv)
    El = E // world
    for r, n_t in enumerate(T_of_rank):
        t0 = sum(T_of_rank[:r])
        owners = ref["ids"][t0:t0 + n_t].ravel() // El
        assert list(sent[r]) == [int((owners == o).sum()) for o in range(world)]
    return sent


def test_ep_two_ranks_matches_one_process_layer():
    _run(2, [5, 3])


def test_ep_four_ranks_ragged_and_shared_experts():
    _run(4, [7, 1, 4, 2], seed=2, n_shared=1)


def test_ep_owner_receiving_nothing_and_rank_without_tokens():
    sent = _run(4, [6, 0, 3, 5], seed=3, skew=True)
    assert sent[:, 1:].sum() == 0          # the skew sends every record to the first owner
