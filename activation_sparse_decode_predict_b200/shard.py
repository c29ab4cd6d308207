"""Neuron-sharded FFN layers across ranks (one process per GPU).

Every rank holds a slice of each layer's neurons -- a contiguous part of the
hot rows and a contiguous part of the cold rows, stored hot-first like a whole
layer -- plus a replica of the predictor's first matrix P1 and the P2 rows of
its cold neurons.  A rank's predictor picks active neurons among its own cold
rows only, its sparse FFN produces a partial y over its own neurons, and the
partial outputs are summed across ranks (one all-reduce of B x d fp32 per
layer) before the residual + RMSNorm glue.  Because each rank's slice is an
ordinary hot-first layer, the library's calls serve it unchanged.

This is the multi-GPU reading of the pages' neuron placement (unite.ai,
"Nöron Yerleştirme ve Yönetimi": neurons are placed across processing units
by the offline stage, a neuron table maps them back): here the units are GPUs
instead of a CPU and a GPU.

Only host-side bookkeeping and the per-layer call sequence live here; every
FFN step runs in libpi's kernels and the sum across ranks in
torch.distributed (NCCL on GPUs).
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import torch

from . import _binding as _b
from . import make_desc, layer_weights, layer as _layer, residual_rmsnorm, workspace
from ._binding import FfnDesc


def neuron_shards(n_hot: int, n_cold: int, world: int) -> List[Tuple[int, int, int, int]]:
    """(h0, h1, c0, c1) per rank: hot rows [h0, h1) and cold rows [c0, c1) of
    the cold block, contiguous and balanced; together they cover every neuron
    exactly once."""
    if world < 1:
        raise ValueError("world must be >= 1")
    return [(n_hot * r // world, n_hot * (r + 1) // world, n_cold * r // world, n_cold * (r + 1) // world)
            for r in range(world)]


def shard_rows(n_hot: int, shard: Tuple[int, int, int, int]) -> torch.Tensor:
    """Storage rows of the whole layer held by a shard, in the shard's own
    (hot-first) order: the shard's neuron table."""
    h0, h1, c0, c1 = shard
    return torch.cat([torch.arange(h0, h1), n_hot + torch.arange(c0, c1)]).to(torch.int64)


def _rows(t, rows: torch.Tensor):
    if t is None:
        return None
    if isinstance(t, tuple):          # Q4_0 weight planes
        return tuple(x.index_select(0, rows.to(x.device)).contiguous() for x in t)
    return t.index_select(0, rows.to(t.device)).contiguous()


def _pred_rows(P, rows: torch.Tensor):
    """Rows of a predictor matrix; a Q4_0 one stays one buffer (codes, then scales)."""
    if P is None:
        return None
    if isinstance(P, tuple):
        qs, sc = (x.index_select(0, rows.to(x.device)) for x in P)
        n = qs.numel()
        buf = torch.empty(n + 2 * sc.numel(), dtype=torch.uint8, device=qs.device)
        buf[:n] = qs.reshape(-1)
        buf[n:] = sc.reshape(-1).view(torch.uint8)
        return buf[:n].view(qs.shape), buf[n:].view(torch.float16).view(sc.shape)
    return P.index_select(0, rows.to(P.device)).contiguous()


def shard_layer(L: dict, n_hot: int, n_cold: int, world: int, rank: int) -> dict:
    """The slice of one layer (the dict of pi_workload.make_layer / layer_weights)
    that `rank` holds.  Keys as for a whole layer, plus n_hot / ffn of the
    shard and its neuron table `rows`; b2 is kept on rank 0 only, so that the
    sum over ranks adds it once."""
    sh = neuron_shards(n_hot, n_cold, world)[rank]
    h0, h1, c0, c1 = sh
    rows = shard_rows(n_hot, sh)
    cold = torch.arange(c0, c1, dtype=torch.int64)
    out = {k: v for k, v in L.items() if k in ("thr", "rank")}
    out["P1"] = L["P1"]
    out["P2"] = _pred_rows(L.get("P2"), cold) if c1 > c0 else None
    out["bp"] = L["bp"].index_select(0, cold.to(L["bp"].device)).contiguous() if L.get("bp") is not None else None
    for k in ("Wg", "Wu", "WdT"):
        out[k] = _rows(L.get(k), rows)
    out["b1"] = L["b1"].index_select(0, rows.to(L["b1"].device)).contiguous() if L.get("b1") is not None else None
    out["b2"] = L.get("b2") if rank == 0 else None
    out["n_hot"], out["ffn"], out["rows"] = h1 - h0, (h1 - h0) + (c1 - c0), rows
    return out


def shard_desc(desc: FfnDesc, shard: dict) -> FfnDesc:
    """The descriptor of a shard: the layer's, with the shard's neuron counts."""
    names = {v: k for k, v in _b.DTYPES.items()}
    acts = {v: k for k, v in _b.ACTS.items()}
    return make_desc(desc.d, shard["ffn"], shard["n_hot"], desc.rank, names[desc.wtype], names[desc.ptype],
                     acts[desc.act])


class ShardedStack:
    """One decode step through sharded FFN layers on this rank: per layer the
    rank's predictor + sparse FFN (pi_layer) on its shard, the sum of the
    partial outputs over the ranks of `group` (no group: this rank alone),
    then the residual + RMSNorm glue."""

    def __init__(self, desc: FfnDesc, shards: Sequence[dict], batch: int, group=None, device=None):
        dev = device or "cuda"
        self.desc = desc
        self.shards = list(shards)
        self.group = group
        self.descs = [shard_desc(desc, s) for s in self.shards]
        self.weights = [layer_weights(s) for s in self.shards]
        self.ws = [workspace(d, batch, device=dev) for d in self.descs]
        self.y = torch.empty(batch, desc.d, dtype=torch.float32, device=dev)
        self.idx = [torch.empty(max(s["ffn"] - s["n_hot"], 1), dtype=torch.int32, device=dev) for s in self.shards]
        self.count = [torch.zeros(1, dtype=torch.int32, device=dev) for _ in self.shards]

    def step(self, h_in: torch.Tensor, h_out: torch.Tensor, eps: float) -> None:
        import torch.distributed as dist
        n = len(self.shards)
        bufs = (torch.empty_like(h_in), torch.empty_like(h_in))
        cur = h_in
        for l in range(n):
            _layer(self.descs[l], cur, self.weights[l], self.idx[l], self.count[l], self.y, self.ws[l])
            if self.group is not None and dist.get_world_size(self.group) > 1:
                dist.all_reduce(self.y, op=dist.ReduceOp.SUM, group=self.group)
            nxt = h_out if l == n - 1 else bufs[l & 1]
            residual_rmsnorm(cur, self.y, eps, nxt)
            cur = nxt

    def active_rows(self, l: int) -> torch.Tensor:
        """Layer l's active cold neurons picked by this rank, as storage rows of the whole layer."""
        n = int(self.count[l].item())
        local = self.idx[l][:n].long().cpu()
        return self.shards[l]["rows"].index_select(0, local)
