"""GPU parity of predictors sized per layer (unite.ai "Adaptif Sparsite
Predictor’ları": each layer's predictor has its own size): a rank per layer
and Q4_0 predictor matrices, through the per-kernel calls, the persistent
decode-step kernel and the token-block path, against the CPU oracle."""
import numpy as np
import pytest
import torch

import activation_sparse_decode_predict_b200 as pi
import pi_workload as W
from gpu_util import TOL, check_index_list, gpu_ffn, gpu_predict, oracle_layer, oracle_predict, rel_err, to_dev, to_np
from test_gpu_parity import _stack_check

pytestmark = pytest.mark.gpu


def _wl(name, d, ffn, hot, rank, act, wt, pt, B, layers=1, steps=(), sparsity=0.88):
    return W.Workload(name, 70 + len(name), d, ffn, layers, act, wt, pt, sparsity, 1.2, hot, rank, (B,), 1,
                      has_b2=(act != "reglu"), rank_steps=steps)


def _layer(wl, layer=0):
    # made on the device: a Q4_0 predictor's scales must stay right after its
    # codes in one buffer, which a per-tensor copy would not keep
    return W.make_layer(wl, layer, device="cuda")


# (name, d, ffn, hot, rank, act, wtype, ptype, batch)
Q4_PRED = [
    ("q4pred-f16w-b1", 512, 2000, 0.1, 128, "reglu", "f16", "q4_0", 1),
    ("q4pred-q4w-b2", 512, 1500, 0.08, 64, "relu", "q4_0", "q4_0", 2),
    ("q4pred-f16w-b5", 1024, 2600, 0.1, 96, "reglu", "f16", "q4_0", 5),
    ("q4pred-f32w-b3", 256, 900, 0.05, 32, "relu2", "f32", "q4_0", 3),
]


@pytest.mark.parametrize("case", Q4_PRED, ids=[c[0] for c in Q4_PRED])
def test_q4_0_predictor_single_layer_matches_oracle(case):
    """pi_predict and pi_sparse_ffn with a Q4_0 predictor (fp16 tokens)."""
    name, d, ffn, hot, rank, act, wt, pt, B = case
    wl = _wl(name, d, ffn, hot, rank, act, wt, pt, B)
    L = _layer(wl)
    assert isinstance(L["P1"], tuple) and L["P1"][0].dtype == torch.uint8
    h = to_dev(W.make_tokens(wl, B, 2))
    assert h.dtype == torch.float16
    desc = pi.desc_for(wl)
    ws = pi.workspace(desc, B)
    gidx, idx_t, cnt_t = gpu_predict(desc, h, L, ws)
    orc = oracle_predict(L, to_np(h), wl)
    check_index_list(gidx, orc, wl.thr, wl.n_hot, wl.ffn)
    assert 0 < len(gidx) < wl.n_cold
    y = gpu_ffn(desc, h, L, idx_t, cnt_t, ws)
    assert rel_err(y, oracle_layer(L, to_np(h), wl, gidx)) <= TOL[wl.wtype]
    assert pi.device_status(ws) == 0


# (name, d, ffn, hot, rank, act, wtype, ptype, batch, layers, rank_steps)
STACKS = [
    # persistent kernel: Q4_0 weights with a Q4_0 predictor, ranks 256..768 per layer
    ("stack-q4-q4pred-b1", 512, 1500, 0.1, 768, "reglu", "q4_0", "q4_0", 1, 3, (768, 256, 512)),
    ("stack-q4-q4pred-b2", 1024, 2500, 0.1, 512, "relu2", "q4_0", "q4_0", 2, 3, (256, 512)),
    # persistent kernel: fp16 predictors whose rank changes per layer
    ("stack-f16-ranks-b1", 1024, 3000, 0.1, 128, "reglu", "f16", "f16", 1, 3, (128, 48, 96)),
    ("stack-f16-ranks-b2", 512, 2000, 0.08, 64, "relu", "f16", "f16", 2, 3, (32, 64)),
    # per-layer kernels (token blocks of 3+): Q4_0 predictor, ranks per layer
    ("stack-f16-q4pred-b4", 512, 1800, 0.1, 256, "reglu", "f16", "q4_0", 4, 3, (256, 96, 160)),
    ("stack-q4-q4pred-b3", 512, 1200, 0.1, 128, "relu", "q4_0", "q4_0", 3, 2, (64, 128)),
]


@pytest.mark.parametrize("case", STACKS, ids=[c[0] for c in STACKS])
def test_stack_with_per_layer_predictors_matches_oracle(case):
    name, d, ffn, hot, rank, act, wt, pt, B, L, steps = case
    wl = _wl(name, d, ffn, hot, rank, act, wt, pt, B, layers=L, steps=steps)
    fused = B <= 2
    assert (pi.stack_launches(pi.desc_for(wl), B, L) == 1) == fused
    _stack_check(wl, B, L, seed_step=4)


def test_full_size_13b_q4_0_with_q4_0_predictor():
    """The 13B-shaped Q4_0 stack with its predictor in Q4_0 too (0.5625 bytes
    per element instead of 2): two layers through the persistent kernel,
    every list entry checked, y on 48 sampled columns."""
    wl = W.WORKLOADS["13b-reglu-q4_0"].with_(ptype="q4_0")
    assert pi.stack_launches(pi.desc_for(wl), 1, 2) == 1
    cols = np.sort(np.random.default_rng(13).choice(wl.d, size=48, replace=False)).astype(np.int32)
    _stack_check(wl, 1, 2, cols=cols, seed_step=1)
    # the predictor bytes per layer drop from 2 to 18/32 bytes per element
    fp16 = W.layer_bytes(W.WORKLOADS["13b-reglu-q4_0"], 1, 560.0)
    q4 = W.layer_bytes(wl, 1, 560.0)
    assert q4 < 0.55 * fp16
