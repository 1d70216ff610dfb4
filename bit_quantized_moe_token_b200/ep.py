"""Expert-parallel W4A8 MoE layer: one process per GPU, the routed experts split over the ranks.

Rank r of n holds experts [r E/n, (r+1) E/n) as its own W4A8 layer and the shared experts in
full.  A forward on each rank's own tokens runs the three library calls of
``include/moe_w4a8.h`` (``moe_ep_dispatch``, ``moe_ep_experts_forward``, ``moe_ep_combine``) with
two exchanges through ``torch.distributed`` between them: the FP8 records to the experts'
owners, the fp32 output rows back.  The exchanges are the only work done here; every step of
the layer runs in the library's kernels.

The pages serve the layer tensor-parallel (TP4 on the Inkling-512k-NVFP4-AQLM-hybrid card,
"Serving"; TP8 in the Inkling 2 Small FP8 for AMD MI300X card's launch command); splitting the
independent experts instead is the plainest multi-GPU form of the same computation.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

from . import _binding as B


def local_experts(layer: B.Layer, rank: int, n_ranks: int) -> B.Layer:
    """Rank `rank`'s experts of `layer` as a layer of their own (views, no copy; no shared
    experts)."""
    if layer.E % n_ranks:
        raise ValueError(f"E = {layer.E} does not split over {n_ranks} ranks")
    El = layer.E // n_ranks
    sl = slice(rank * El, (rank + 1) * El)
    return B.Layer(El, layer.H, layer.N, layer.gate_packed[sl], layer.up_packed[sl],
                   layer.down_packed[sl], layer.gate_scales[sl], layer.up_scales[sl],
                   layer.down_scales[sl], group=layer.group)


class CudaEpOps:
    """The library calls of one expert-parallel forward (the default; see EpLayer)."""

    dispatch = staticmethod(B.moe_ep_dispatch)
    experts_forward = staticmethod(B.moe_ep_experts_forward)
    combine = staticmethod(B.moe_ep_combine)
    dispatch_workspace_bytes = staticmethod(B.moe_ep_dispatch_workspace_bytes)
    experts_workspace_bytes = staticmethod(B.moe_ep_experts_workspace_bytes)


@dataclass
class EpStats:
    """What the last forward moved: records sent / received (one per routed pair)."""
    sent: list
    received: list


class EpLayer:
    """This rank's part of an expert-parallel layer.

    layer   the full layer's shapes and shared experts (a B.Layer whose routed-expert tensors may
            be None on this rank: only E, H, N, group and the shared experts are read)
    local   this rank's experts (local_experts(full, rank, n_ranks) when the full layer is here)
    group   the process group of the n_ranks ranks (None: the default group; with no process
            group initialised the layer runs alone, n_ranks = 1)
    ops     the calls that do the work (CudaEpOps: the library's kernels)
    """

    def __init__(self, layer, local: B.Layer, group=None, ops=CudaEpOps):
        self.layer = layer
        self.local = local
        self.group = group
        self.ops = ops
        # with a process group the exchanges go through it (at one rank too); without one the
        # layer runs alone and the rows stay where they are
        self.grouped = dist.is_available() and dist.is_initialized()
        if self.grouped:
            self.rank = dist.get_rank(group)
            self.n_ranks = dist.get_world_size(group)
        else:
            self.rank, self.n_ranks = 0, 1
        if layer.E != local.E * self.n_ranks:
            raise ValueError(f"{self.n_ranks} ranks of {local.E} experts do not make E = {layer.E}")
        self._ws = {}
        self.stats = None

    def _workspace(self, key, nbytes: int, device):
        ws = self._ws.get(key)
        if ws is None or ws.numel() < nbytes:
            ws = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
            self._ws[key] = ws
        return ws

    def _exchange(self, inp, rows: int, out_splits=None, in_splits=None):
        """All-to-all of inp's rows (in_splits[r] of them to rank r); returns the `rows` rows
        received (out_splits[r] from rank r).  Alone, the rows stay where they are."""
        if not self.grouped:
            return inp
        out = torch.empty((rows,) + tuple(inp.shape[1:]), dtype=inp.dtype, device=inp.device)
        dist.all_to_all_single(out, inp, out_splits, in_splits, group=self.group)
        return out

    def forward(self, x, logits, k: int, out=None):
        """x bf16 [T, H] and router logits fp32 [T, E] of this rank's tokens -> bf16 [T, H]."""
        T, H = x.shape
        dev = x.device
        n = self.n_ranks
        rb = B.ep_record_bytes(H)
        if out is None:
            out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        ws_d = self._workspace("dispatch", self.ops.dispatch_workspace_bytes(self.layer, T, k), dev)
        send_counts = torch.empty(n, dtype=torch.int32, device=dev)
        send = torch.empty((T * k, rb), dtype=torch.uint8, device=dev)
        self.ops.dispatch(self.layer, x, logits, k, n, send_counts, send, ws_d)
        if self.grouped:
            # how many records go each way: one int per rank pair, then to the host for the splits
            recv_counts = self._exchange(send_counts, n)
            counts = torch.cat([send_counts, recv_counts]).cpu().tolist()
            sc, rc = counts[:n], counts[n:]
        else:
            sc = rc = [T * k]   # alone: every record stays here, and nothing needs the host
        R = sum(rc)
        recv = self._exchange(send, R, rc, sc)
        y_rows = torch.empty((R, H), dtype=torch.float32, device=dev)
        ws_e = self._workspace("experts", self.ops.experts_workspace_bytes(self.local, R), dev)
        self.ops.experts_forward(self.local, recv, y_rows, ws_e)
        y_back = self._exchange(y_rows, T * k, sc, rc)
        self.ops.combine(self.layer, x, y_back, k, out, ws_d)
        self.stats = EpStats(sc, rc)
        return out
