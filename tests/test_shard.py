"""Neuron-sharded layers: the bookkeeping on the host, and the sharded FFN
(each rank's predictor and masked FFN on its own slice, partial outputs
summed across ranks) against the whole layer -- with the CPU oracle on
world-size-2 gloo ranks.  No GPU: the library runs on shards in
tests/test_gpu_shard.py."""
import os
import socket

import numpy as np
import pytest
import torch

import pi_workload as W
from activation_sparse_decode_predict_b200 import shard


@pytest.mark.parametrize("n_hot,n_cold,world", [(103, 1945, 2), (0, 900, 4), (11, 0, 3), (5, 7, 8)])
def test_shards_cover_every_neuron_once(n_hot, n_cold, world):
    shards = shard.neuron_shards(n_hot, n_cold, world)
    rows = torch.cat([shard.shard_rows(n_hot, s) for s in shards])
    assert torch.equal(torch.sort(rows).values, torch.arange(n_hot + n_cold))
    for (h0, h1, c0, c1) in shards:
        assert 0 <= h1 - h0 <= n_hot // world + 1 and 0 <= c1 - c0 <= n_cold // world + 1


def _wl():
    return W.Workload("shard", 61, 256, 1200, 1, "reglu", "f16", "f16", 0.88, 1.2, 0.1, 32, (2,), 1)


def _rank_result(rank, world, wl):
    """This rank's predictor list (as storage rows of the whole layer) and partial y, by the oracle."""
    import oracle
    L = W.make_layer(wl, 0)
    S = shard.shard_layer(L, wl.n_hot, wl.n_cold, world, rank)
    h = W.make_tokens(wl, 2, 3).numpy()
    np_ = lambda v: None if v is None else (tuple(x.numpy() for x in v) if isinstance(v, tuple) else v.numpy())
    r = oracle.predict(h, np_(S["P1"]), np_(S["P2"]), np_(S["bp"]), S["thr"], S["n_hot"], S["ffn"])
    y = oracle.masked_ffn(h, r["idx"], np_(S["Wg"]), np_(S["Wu"]), np_(S["WdT"]), np_(S["b1"]), np_(S["b2"]),
                          wl.act, S["n_hot"], S["ffn"])
    rows = S["rows"].numpy()[r["idx"]] if len(r["idx"]) else np.zeros(0, np.int64)
    return rows, y, L, h


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rows, y, _, _ = _rank_result(rank, world, _wl())
        yt = torch.from_numpy(y)
        dist.all_reduce(yt, op=dist.ReduceOp.SUM)
        gathered = [None] * world
        dist.all_gather_object(gathered, rows.tolist())
        if rank == 0:
            q.put((yt.numpy(), sorted(sum(gathered, []))))
    finally:
        dist.destroy_process_group()


def test_sharded_layer_sums_to_the_whole_layer_on_two_gloo_ranks():
    import multiprocessing as mp
    import oracle
    wl = _wl()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    with socket.socket() as s_:
        s_.bind(("127.0.0.1", 0))
        port = s_.getsockname()[1]
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    y_sum, rows = q.get(timeout=240)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # the whole layer, unsharded
    L = W.make_layer(wl, 0)
    h = W.make_tokens(wl, 2, 3).numpy()
    r = oracle.predict(h, L["P1"].numpy(), L["P2"].numpy(), L["bp"].numpy(), L["thr"], wl.n_hot, wl.ffn)
    assert rows == r["idx"].tolist()          # the ranks' lists together are the whole layer's list
    y = oracle.masked_ffn(h, r["idx"], L["Wg"].numpy(), L["Wu"].numpy(), L["WdT"].numpy(), L["b1"].numpy(), None,
                          wl.act, wl.n_hot, wl.ffn)
    assert np.abs(y_sum - y).max() <= 1e-12 * np.abs(y).max()
