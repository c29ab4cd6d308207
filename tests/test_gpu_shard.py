"""Neuron-sharded layers on the GPU (one device: the ranks' shards run in
turn): the library on each shard, the partial outputs summed, against the
oracle of the whole layer; and the per-rank decode step of shard.ShardedStack."""
import numpy as np
import pytest
import torch

import activation_sparse_decode_predict_b200 as pi
import pi_workload as W
from activation_sparse_decode_predict_b200 import shard
from gpu_util import TOL, check_index_list, gpu_ffn, gpu_predict, oracle_layer, oracle_predict, rel_err, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world,wt,B", [(2, "f16", 2), (4, "f16", 1), (3, "q4_0", 3)])
def test_shards_sum_to_the_whole_layer(world, wt, B):
    wl = W.Workload("gshard", 62, 1024, 3000, 1, "reglu", wt, "f16", 0.88, 1.2, 0.1, 64, (B,), 1)
    L = W.make_layer(wl, 0, device="cuda")
    h = W.make_tokens(wl, B, 4, device="cuda")
    desc = pi.desc_for(wl)
    y_sum = np.zeros((B, wl.d))
    rows = []
    for r in range(world):
        S = shard.shard_layer(L, wl.n_hot, wl.n_cold, world, r)
        sd = shard.shard_desc(desc, S)
        ws = pi.workspace(sd, B)
        gidx, idx_t, cnt_t = gpu_predict(sd, h, S, ws)
        y_sum += gpu_ffn(sd, h, S, idx_t, cnt_t, ws)
        rows += S["rows"].numpy()[gidx].tolist()
        assert pi.device_status(ws) == 0
    rows = np.sort(np.array(rows, dtype=np.int64))
    h_np = to_np(h)
    check_index_list(rows, oracle_predict(L, h_np, wl), wl.thr, wl.n_hot, wl.ffn)
    assert rel_err(y_sum, oracle_layer(L, h_np, wl, rows)) <= TOL[wt]


def test_sharded_stack_on_one_rank_equals_the_decode_stack():
    wl = W.Workload("gshard2", 63, 512, 1500, 3, "relu", "f16", "f16", 0.88, 1.2, 0.08, 32, (1,), 1, has_b2=True)
    layers = [W.make_layer(wl, l, device="cuda") for l in range(3)]
    desc = pi.desc_for(wl)
    st = shard.ShardedStack(desc, [shard.shard_layer(L, wl.n_hot, wl.n_cold, 1, 0) for L in layers], 1)
    h0 = W.make_tokens(wl, 1, 8, device="cuda")
    h_a = torch.empty_like(h0)
    st.step(h0, h_a, W.RMS_EPS)
    h_b = torch.empty_like(h0)
    ws = pi.workspace(desc, 1)
    idx = torch.empty(3, wl.n_cold, dtype=torch.int32, device="cuda")
    counts = torch.zeros(3, dtype=torch.int32, device="cuda")
    pi.decode_stack(desc, pi.layer_array([pi.layer_weights(L) for L in layers]), h0, h_b, idx, counts, None,
                    W.RMS_EPS, ws)
    torch.cuda.synchronize()
    assert (h_a.float() - h_b.float()).abs().max().item() <= 2 ** -8 * h_b.float().abs().max().item()
    # the two paths run different predictor kernels (CUDA-core and tensor-core
    # dots), so near-threshold neurons may differ; nothing else may
    for l in range(3):
        a = set(st.active_rows(l).tolist())
        b = set(idx[l, :int(counts[l])].long().cpu().tolist())
        assert len(a ^ b) <= 2 + 0.01 * len(b), l
