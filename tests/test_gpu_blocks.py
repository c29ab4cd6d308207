"""A whole decode step through attention + FFN blocks (pi_decode_blocks)
against the CPU oracle, teacher-forced per sub-step on the GPU's own inputs
(the trace): the head list, the attention output through the glue, the FFN
list and output through the glue."""
import numpy as np
import pytest
import torch

import activation_sparse_decode_predict_b200 as pi
import oracle
import pi_workload as W
from gpu_util import check_index_list, oracle_layer, oracle_predict, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("wt,B", [("f16", 1), ("f16", 3), ("q4_0", 3)])
def test_decode_blocks_match_oracle(wt, B):
    n_layers, L, s_max = 2, 40, 64
    wl = W.Workload("blocks-" + wt, 88, 512, 1500, n_layers, "reglu", wt, "f16", 0.88, 1.2, 0.1, 64, (B,), 1)
    H, n_hot_h, head_rank = 8, 1, 32
    fdesc = pi.desc_for(wl)
    adesc = pi.attn_desc(wl.d, H, n_hot_h, s_max)
    layers = [W.make_layer(wl, l, device="cuda") for l in range(n_layers)]
    attn = [W.make_attention(wl.d, H, n_hot_h, head_rank, B, s_max, seed=300 + l, device="cuda")
            for l in range(n_layers)]
    caches0 = [(a["K"].clone(), a["V"].clone()) for a in attn]
    blocks = (pi.BlockWeights * n_layers)(*[pi.block_weights(Lw, A, head_rank) for Lw, A in zip(layers, attn)])
    h0 = W.make_tokens(wl, B, 11, device="cuda")
    h_out = torch.zeros_like(h0)
    hidx = torch.full((n_layers, H), -1, dtype=torch.int32, device="cuda")
    hcnt = torch.zeros(n_layers, dtype=torch.int32, device="cuda")
    idx = torch.full((n_layers, wl.n_cold), -1, dtype=torch.int32, device="cuda")
    counts = torch.zeros(n_layers, dtype=torch.int32, device="cuda")
    trace = torch.zeros(n_layers, 2, B, wl.d, dtype=torch.float16, device="cuda")
    ws = pi.blocks_workspace(fdesc, adesc, B)
    pi.decode_blocks(fdesc, adesc, blocks, h0, h_out, L, hidx, hcnt, idx, counts, W.RMS_EPS, ws, trace=trace)
    torch.cuda.synchronize()
    assert pi.device_status(ws) == 0
    assert torch.equal(trace[0, 0], h0)
    for l in range(n_layers):
        A = attn[l]
        h_l, g_l = to_np(trace[l, 0]), to_np(trace[l, 1])
        # head list: the head predictor on h_l
        nh = int(hcnt[l].item())
        heads = hidx[l, :nh].cpu().numpy()
        orc = oracle.predict(h_l, to_np(A["P1"]), to_np(A["P2"]), to_np(A["bp"]), A["thr"], n_hot_h, H)
        check_index_list(heads, orc, A["thr"], n_hot_h, H)
        # attention over those heads, then the glue -> g_l
        K0, V0 = (to_np(c) for c in caches0[l])
        a = oracle.attention(h_l, heads, *(to_np(A[k]) for k in ("Wq", "Wk", "Wv", "WoT")), K0, V0, L, H, n_hot_h)
        g_ref = oracle.residual_rmsnorm(h_l, a["y"], W.RMS_EPS)
        assert np.abs(g_l.astype(np.float64) - g_ref).max() <= 4e-3 * np.abs(g_ref).max(), "layer %d attention" % l
        # the FFN on g_l: its list and, through the glue, the next input
        n = int(counts[l].item())
        gidx = idx[l, :n].cpu().numpy()
        check_index_list(gidx, oracle_predict(layers[l], g_l, wl), wl.thr, wl.n_hot, wl.ffn)
        y = oracle_layer(layers[l], g_l, wl, gidx)
        nxt_ref = oracle.residual_rmsnorm(g_l, y, W.RMS_EPS)
        nxt = to_np(trace[l + 1, 0]) if l + 1 < n_layers else to_np(h_out)
        assert np.abs(nxt.astype(np.float64) - nxt_ref).max() <= 4e-3 * np.abs(nxt_ref).max(), "layer %d ffn" % l
