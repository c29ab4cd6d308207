"""GPU parity: libpi (through its C ABI) against the CPU oracle on the same
seeded inputs, at sizes the oracle finishes in seconds that still span
several tiles and ragged tails, plus edge cases and integer-exact layers."""
import numpy as np
import pytest
import torch

import activation_sparse_decode_predict_b200 as pi
import oracle
import pi_workload as W
from gpu_util import (BAND, TOL, check_index_list, gpu_ffn, gpu_predict, oracle_layer, oracle_predict, rel_err,
                      to_dev, to_np, token_ffn)

pytestmark = pytest.mark.gpu

# (name, d, ffn, hot_frac, rank, act, wtype, ptype, batch)
SHAPES = [
    ("tiny-relu-fp32", 512, 2048, 0.05, 64, "relu", "f32", "f32", 1),
    ("ragged-reglu-f16-b3", 264, 777, 0.017, 24, "reglu", "f16", "f16", 3),
    ("relu2-f16-nohot", 128, 513, 0.0, 16, "relu2", "f16", "f16", 1),
    ("reglu-q4-b2", 160, 300, 0.10, 32, "reglu", "q4_0", "f16", 2),
    ("relu-q4-b5", 256, 1100, 0.08, 32, "relu", "q4_0", "f16", 5),
    ("relu-f32w-f16tok", 64, 100, 0.10, 8, "relu", "f32", "f16", 1),
    ("reglu-f16-b16", 256, 1000, 0.10, 32, "reglu", "f16", "f16", 16),
    ("reglu-f16-b8", 1024, 2600, 0.10, 128, "reglu", "f16", "f16", 8),
    ("relu2-f32-b4", 96, 700, 0.05, 16, "relu2", "f32", "f32", 4),
    # tensor-core token-block path: 256-column chunks, d split in parts, no hot rows
    ("relu2-f16-b12", 1280, 1500, 0.05, 32, "relu2", "f16", "f16", 12),
    ("reglu-f16-b16-split", 4096, 1200, 0.10, 64, "reglu", "f16", "f16", 16),
    ("relu-f16-b3-nohot", 512, 900, 0.0, 32, "relu", "f16", "f16", 3),
    # tensor-core predictor of a token block (rank % 128 == 0), P2 split in parts
    ("relu-f16-b16-bigrank", 2048, 1500, 0.10, 2048, "relu", "f16", "f16", 16),
    ("reglu-f16-b4-pred", 512, 1200, 0.10, 128, "reglu", "f16", "f16", 4),
    # Q4_0 token blocks: gate/up rows decoded onto the tensor cores, d in parts, ragged lists
    ("reglu-q4-b8", 512, 1300, 0.10, 64, "reglu", "q4_0", "f16", 8),
    ("relu2-q4-b16-parts", 4096, 900, 0.05, 32, "relu2", "q4_0", "f16", 16),
    ("reglu-q4-b3-ragged", 768, 999, 0.02, 48, "reglu", "q4_0", "f16", 3),
]


def _workload(name, d, ffn, hot, rank, act, wt, pt, B, sparsity=0.88):
    return W.Workload(name, 40 + len(name), d, ffn, 1, act, wt, pt, sparsity, 1.2, hot, rank, (B,), 1,
                      has_b2=(act != "reglu"))


def _layer(wl, layer=0):
    L = W.make_layer(wl, layer, device="cpu")
    return {k: to_dev(v) if k not in ("perm", "p", "thr") else v for k, v in L.items()}


# the shapes whose FFN the tcgen05 token-block kernels take (fp16, d % 256 == 0, B = 3..16)
TC_SHAPES = [s for s in SHAPES if s[6] == "f16" and s[7] == "f16" and s[1] % 256 == 0 and 3 <= s[-1] <= 16]


@pytest.mark.parametrize("shape", SHAPES, ids=[s[0] for s in SHAPES])
def test_predict_and_sparse_ffn_match_oracle(shape):
    _shape_check(shape)


@pytest.mark.parametrize("shape", TC_SHAPES, ids=[s[0] for s in TC_SHAPES])
def test_token_blocks_on_tcgen05_match_oracle(shape):
    """The same checks with the token-block FFN on the tcgen05 kernels."""
    with token_ffn("tcgen05"):
        _shape_check(shape)


def _shape_check(shape):
    wl = _workload(*shape)
    B = shape[-1]
    L = _layer(wl)
    h = to_dev(W.make_tokens(wl, B, 0))
    desc = pi.desc_for(wl)
    ws = pi.workspace(desc, B)
    gidx, idx_t, cnt_t = gpu_predict(desc, h, L, ws)
    h_np = to_np(h)
    orc = oracle_predict(L, h_np, wl)
    check_index_list(gidx, orc, wl.thr, wl.n_hot, wl.ffn)
    assert 0 < len(gidx) < wl.n_cold
    y = gpu_ffn(desc, h, L, idx_t, cnt_t, ws)
    ref = oracle_layer(L, h_np, wl, gidx)
    assert rel_err(y, ref) <= TOL[wl.wtype]
    assert pi.device_status(ws) == 0
    # the fused layer call gives the same list and output
    y2 = torch.zeros(B, wl.d, device="cuda")
    idx2 = torch.zeros_like(idx_t)
    cnt2 = torch.zeros_like(cnt_t)
    pi.layer(desc, h, pi.layer_weights(L), idx2, cnt2, y2, ws)
    torch.cuda.synchronize()
    assert int(cnt2.item()) == len(gidx)
    assert np.array_equal(idx2[: len(gidx)].cpu().numpy(), gidx)
    assert rel_err(y2.cpu().numpy(), ref) <= TOL[wl.wtype]


INT_CASES = [
    (256, 600, 40, 32, "reglu", "f16", "f16", 1),
    (256, 600, 0, 32, "relu", "f16", "f16", 4),
    (96, 333, 33, 16, "relu2", "f32", "f32", 3),
    (128, 520, 20, 16, "reglu", "q4_0", "f16", 2),
    (160, 300, 300, 16, "relu", "q4_0", "f16", 1),
    (256, 700, 70, 32, "reglu", "f16", "f16", 16),
    (256, 700, 70, 32, "relu", "f16", "f16", 8),
    # Q4_0 token blocks: codes decoded into tensor-core fragments, down on the CUDA cores
    (256, 600, 30, 32, "reglu", "q4_0", "f16", 4),
    (512, 700, 50, 32, "relu", "q4_0", "f16", 16),
]


@pytest.mark.parametrize("path", ["warp_mma", "tcgen05"])
@pytest.mark.parametrize("case", INT_CASES)
def test_integer_exact_layers_are_bit_identical(case, path):
    """Every product and partial sum is an exact small integer (or dyadic), so
    the GPU must equal the oracle bit for bit in any summation order (token
    blocks through either FFN kernel family)."""
    with token_ffn(path):
        _int_check(case)


def _int_check(case):
    d, ffn, n_hot, rank, act, wt, pt, B = case
    L = W.make_int_layer(d, ffn, n_hot, rank, act, wt, pt, B, seed=d + ffn + B)
    L = {k: to_dev(v) if k not in ("perm", "thr") else v for k, v in L.items()}
    desc = pi.make_desc(d, ffn, n_hot, rank, wt, pt, act)
    ws = pi.workspace(desc, B)
    h = L["h"]
    gidx, idx_t, cnt_t = gpu_predict(desc, h, L, ws)
    h_np = to_np(h)
    orc = oracle.predict(h_np, to_np(L["P1"]), to_np(L["P2"]), to_np(L["bp"]), 0.5, n_hot, ffn)
    assert np.array_equal(gidx, orc["idx"])
    y = gpu_ffn(desc, h, L, idx_t, cnt_t, ws)
    ref = oracle.masked_ffn(h_np, gidx, to_np(L["Wg"]), to_np(L["Wu"]), to_np(L["WdT"]), to_np(L["b1"]),
                            to_np(L["b2"]), act, n_hot, ffn)
    assert np.array_equal(y, ref)


def test_threshold_extremes_and_no_cold_neurons():
    wl = _workload("edge", 128, 600, 0.1, 16, "reglu", "f16", "f16", 2)
    L = _layer(wl)
    h = to_dev(W.make_tokens(wl, 2, 3))
    desc = pi.desc_for(wl)
    ws = pi.workspace(desc, 2)
    h_np = to_np(h)
    # everything active: equals the dense FFN
    L_all = dict(L, thr=-1e30)
    gidx, idx_t, cnt_t = gpu_predict(desc, h, L_all, ws)
    assert np.array_equal(gidx, np.arange(wl.n_hot, wl.ffn))
    y = gpu_ffn(desc, h, L_all, idx_t, cnt_t, ws)
    Ln = {k: to_np(L[k]) for k in ("Wg", "Wu", "WdT", "b1")}
    dense = oracle.dense_ffn(h_np, Ln["Wg"], Ln["Wu"], Ln["WdT"], Ln["b1"], None, "reglu", wl.n_hot, wl.ffn)
    assert rel_err(y, dense) <= TOL["f16"]
    # nothing active: hot part only
    L_none = dict(L, thr=1e30)
    gidx, idx_t, cnt_t = gpu_predict(desc, h, L_none, ws)
    assert len(gidx) == 0
    y = gpu_ffn(desc, h, L_none, idx_t, cnt_t, ws)
    hot = oracle.masked_ffn(h_np, [], Ln["Wg"], Ln["Wu"], Ln["WdT"], Ln["b1"], None, "reglu", wl.n_hot, wl.ffn)
    assert rel_err(y, hot) <= TOL["f16"]
    # all neurons hot: no predictor matrix at all
    desc_h = pi.make_desc(128, 600, 600, 16, "f16", "f16", "reglu")
    ws_h = pi.workspace(desc_h, 2)
    idx = torch.zeros(1, dtype=torch.int32, device="cuda")
    cnt = torch.full((1,), 5, dtype=torch.int32, device="cuda")
    pi.predict(desc_h, h, L["P1"], None, None, 0.5, idx, cnt, ws_h)
    torch.cuda.synchronize()
    assert int(cnt.item()) == 0
    y = torch.zeros(2, 128, device="cuda")
    pi.sparse_ffn(desc_h, h, idx, cnt, L["Wg"], L["Wu"], L["WdT"], L["b1"], None, y, ws_h)
    torch.cuda.synchronize()
    full = oracle.masked_ffn(h_np, [], Ln["Wg"], Ln["Wu"], Ln["WdT"], Ln["b1"], None, "reglu", 600, 600)
    assert rel_err(y.cpu().numpy(), full) <= TOL["f16"]


@pytest.mark.parametrize("path", ["warp_mma", "tcgen05"])
def test_token_block_extremes(path):
    """Token blocks (fp16, d % 256 == 0, B = 3..16) through either FFN kernel
    family: an empty list (no hot rows and nothing predicted: y = b2), every
    neuron active (the dense FFN), and one workspace reused by calls whose
    lists differ in length (on tcgen05 the per-tile and per-chunk writer
    counters are back at zero after every call)."""
    with token_ffn(path):
        _token_block_extremes()


def test_q4_token_block_extremes():
    """The Q4_0 token-block path (gate/up codes on the tensor cores, down on the
    CUDA cores) with an empty list, every neuron active, and one workspace
    reused by lists of different lengths."""
    _token_block_extremes("q4_0")


def _token_block_extremes(wt="f16"):
    for act, B in (("relu", 4), ("reglu", 16)):
        wl = _workload("tc-edge-" + act + "-" + wt, 512, 1000, 0.0, 32, act, wt, "f16", B)
        L = _layer(wl)
        h = to_dev(W.make_tokens(wl, B, 5))
        h_np = to_np(h)
        desc = pi.desc_for(wl)
        ws = pi.workspace(desc, B)
        for thr in (1e30, -1e30, wl.thr, 1e30, wl.thr, -1e30):
            Lt = dict(L, thr=thr)
            gidx, idx_t, cnt_t = gpu_predict(desc, h, Lt, ws)
            if thr == 1e30:
                assert len(gidx) == 0
            if thr == -1e30:
                assert len(gidx) == wl.n_cold
            y = gpu_ffn(desc, h, Lt, idx_t, cnt_t, ws)
            assert rel_err(y, oracle_layer(Lt, h_np, wl, gidx)) <= TOL[wt], (act, thr)
            assert pi.device_status(ws) == 0


BAD_LIST = [("per-kernel", 128, "relu", "f16", 1, "warp_mma"),
            ("token-block", 256, "reglu", "f16", 4, "warp_mma"),
            ("token-block-tcgen05", 256, "reglu", "f16", 4, "tcgen05"),
            ("token-block-q4", 256, "relu", "q4_0", 4, "warp_mma")]


@pytest.mark.parametrize("name,d,act,wt,B,path", BAD_LIST, ids=[c[0] for c in BAD_LIST])
def test_bad_device_list_is_flagged_and_skipped(name, d, act, wt, B, path):
    """An entry of the list outside [n_hot, ffn) sets PI_ERR_INDEX and adds
    nothing; a count above the capacity sets PI_ERR_CAPACITY and is clamped
    -- on every FFN path."""
    wl = _workload("badidx-" + name, d, 500, 0.1, 16, act, wt, "f16", B)
    L = _layer(wl)
    h = to_dev(W.make_tokens(wl, B, 0))
    desc = pi.desc_for(wl)
    ws = pi.workspace(desc, B)
    good = [wl.n_hot + 3, wl.n_hot + 40, wl.ffn - 1]
    idx = torch.tensor(good[:2] + [wl.ffn + 5] + good[2:], dtype=torch.int32, device="cuda")
    cnt = torch.tensor([4], dtype=torch.int32, device="cuda")
    with token_ffn(path):
        y = gpu_ffn(desc, h, L, idx, cnt, ws)
    assert pi.device_status(ws, clear=True) == pi._binding.PI_ERR_INDEX
    ref = oracle_layer(L, to_np(h), wl, good)
    assert rel_err(y, ref) <= TOL[wt]
    assert pi.device_status(ws) == 0
    # a count above the list's capacity is flagged and clamped
    full = torch.arange(wl.n_hot, wl.ffn, dtype=torch.int32, device="cuda")
    cnt = torch.tensor([wl.n_cold + 1000], dtype=torch.int32, device="cuda")
    with token_ffn(path):
        y = gpu_ffn(desc, h, L, full, cnt, ws)
    assert pi.device_status(ws, clear=True) == pi._binding.PI_ERR_CAPACITY
    ref = oracle_layer(L, to_np(h), wl, full.cpu().numpy())
    assert rel_err(y, ref) <= TOL[wt]


@pytest.mark.parametrize("htype", ["f32", "f16"])
def test_residual_rmsnorm_matches_oracle(htype):
    g = torch.Generator().manual_seed(5)
    B, d = 3, 520
    h = (torch.randn(B, d, generator=g)).to(torch.float32 if htype == "f32" else torch.float16)
    y = torch.randn(B, d, generator=g) * 0.3
    out = torch.empty_like(h, device="cuda")
    pi.residual_rmsnorm(h.cuda(), y.cuda(), 1e-6, out)
    torch.cuda.synchronize()
    ref = oracle.residual_rmsnorm(h.numpy(), y.numpy().astype(np.float64), 1e-6)
    got = out.float().cpu().numpy()
    tol = 2e-6 if htype == "f32" else 2 ** -10
    assert np.abs(got - ref).max() <= tol * np.abs(ref).max()


def _stack_check(wl, B, n_layers, cols=None, seed_step=0, thr=None, dense=False):
    """pi_decode_stack (the benchmark's launch) against the oracle, teacher-forced
    per layer on the GPU's own layer inputs (h_trace).  `thr` overrides every
    layer's threshold; `dense` also compares each layer with the oracle's dense
    FFN (every neuron listed).  Returns the number of (layer, cold row) pairs
    whose score fell in the 1e-3 band, which is bounded so that the list check
    never becomes vacuous."""
    desc = pi.desc_for(wl)
    layers = [W.make_layer(wl, l, device="cuda") for l in range(n_layers)]
    if thr is not None:
        for L in layers:
            L["thr"] = thr
    arr = pi.layer_array([pi.layer_weights(L) for L in layers])
    h0 = W.make_tokens(wl, B, seed_step, device="cuda")
    ws = pi.workspace(desc, B)
    C = wl.n_cold
    idx = torch.full((n_layers, max(C, 1)), -1, dtype=torch.int32, device="cuda")
    counts = torch.zeros(n_layers, dtype=torch.int32, device="cuda")
    y = torch.zeros(n_layers, B, wl.d, device="cuda")
    trace = torch.zeros(n_layers, B, wl.d, dtype=h0.dtype, device="cuda")
    h_out = torch.zeros_like(h0)
    pi.decode_stack(desc, arr, h0, h_out, idx, counts, y, W.RMS_EPS, ws, h_trace=trace)
    torch.cuda.synchronize()
    assert pi.device_status(ws) == 0
    assert torch.equal(trace[0], h0)
    n_amb = 0
    for l, L in enumerate(layers):
        h_l = to_np(trace[l])
        n = int(counts[l].item())
        gidx = idx[l, :n].cpu().numpy()
        if C == 0:
            assert n == 0
        orc = oracle_predict(L, h_l, wl)
        n_amb += check_index_list(gidx, orc, L["thr"], wl.n_hot, wl.ffn)
        ref = oracle_layer(L, h_l, wl, gidx, cols=cols)
        got = to_np(y[l]).astype(np.float64)
        if cols is not None:
            got = got[:, cols]
        assert rel_err(got, ref) <= TOL[wl.wtype], "layer %d" % l
        if dense:
            Ln = {k: to_np(L[k]) for k in ("Wg", "Wu", "WdT", "b1", "b2")}
            ref_d = oracle.dense_ffn(h_l, Ln["Wg"], Ln["Wu"], Ln["WdT"], Ln["b1"], Ln["b2"], wl.act, wl.n_hot,
                                     wl.ffn)
            assert rel_err(to_np(y[l]).astype(np.float64), ref_d) <= TOL[wl.wtype], "layer %d (dense)" % l
        # glue: the next layer's input (or h_out) is RMSNorm(h_l + y_l)
        nxt = to_np(trace[l + 1]) if l + 1 < n_layers else to_np(h_out)
        glue = oracle.residual_rmsnorm(h_l, to_np(y[l]).astype(np.float64), W.RMS_EPS)
        assert np.abs(nxt.astype(np.float64) - glue).max() <= 2 ** -9 * np.abs(glue).max()
    # about 2e-3 of N(0, 1)-like scores fall within 1e-3 of the threshold; a
    # much larger count would mean the band hides real disagreements
    amb_max = 0.01 * max(C, 1) * n_layers + 8
    print("%s B=%d: %d of %d (layer, cold row) pairs in the 1e-3 band" % (wl.name, B, n_amb, C * n_layers))
    assert n_amb <= amb_max, "%d (layer, cold row) pairs in the band, bound %d" % (n_amb, amb_max)
    return n_amb, counts.cpu().numpy()


def test_decode_stack_small_matches_oracle():
    wl = _workload("stack", 256, 900, 0.1, 32, "reglu", "f16", "f16", 2).with_(layers=3)
    _stack_check(wl, 2, 3)


FULL = [("7b-reglu-fp16", 1), ("13b-reglu-q4_0", 1), ("13b-reglu-q4_0", 4), ("13b-reglu-q4_0", 16),
        ("40b-relu-fp16", 1), ("40b-relu-fp16", 2), ("40b-relu-fp16", 8), ("70b-reglu-fp16", 1),
        ("70b-reglu-fp16", 4), ("70b-reglu-fp16", 16)]


@pytest.mark.parametrize("name,B", FULL, ids=["%s-b%d" % f for f in FULL])
def test_full_size_workloads_two_layers_sampled(name, B):
    """Full workload shapes through pi_decode_stack; every active-list entry is
    checked, y on 48 sampled columns (the oracle computes them one by one)."""
    _full_check(name, B)


FULL_TB = [f for f in FULL if f[1] >= 3 and "q4" not in f[0]]  # the switch is for fp16 weights


@pytest.mark.parametrize("name,B", FULL_TB, ids=["%s-b%d" % f for f in FULL_TB])
def test_full_size_token_blocks_on_tcgen05(name, B):
    """The full-size token blocks with their FFN on the tcgen05 kernels."""
    with token_ffn("tcgen05"):
        _full_check(name, B)


def test_down_projection_ranges_longer_than_one_staging_pass():
    """The CUDA-core down kernel stages at most 1024 list positions of its
    range at a time: wide rows (d = 8192: 16 column chunks, 27 ranges) and a
    list of every neuron (30000) give ranges of ~1111 positions, so every
    range takes two passes.  Q4_0 token block of 3 through the decode stack,
    every neuron active (the dense FFN), sampled columns."""
    wl = _workload("q4-long-ranges", 8192, 30000, 0.05, 128, "reglu", "q4_0", "f16", 3)
    rng = np.random.default_rng(11)
    cols = np.sort(rng.choice(wl.d, size=48, replace=False)).astype(np.int32)
    _, counts = _stack_check(wl, 3, 1, cols=cols, thr=-1e30)
    assert int(counts[0]) == wl.n_cold


FULL_DEPTH = [("7b-reglu-fp16", 1), ("13b-reglu-q4_0", 1)]


@pytest.mark.parametrize("name,B", FULL_DEPTH, ids=["%s-b%d" % f for f in FULL_DEPTH])
def test_full_depth_stack_every_column(name, B):
    """Every layer of a full-depth stack in the benchmark's one launch (32 and
    40 layers), every output column, each layer against the oracle fed that
    layer's GPU input; the glue between layers is checked too."""
    wl = W.WORKLOADS[name]
    _stack_check(wl, B, wl.layers, seed_step=7)


def _full_check(name, B):
    wl = W.WORKLOADS[name]
    rng = np.random.default_rng(B)
    cols = np.sort(rng.choice(wl.d, size=48, replace=False)).astype(np.int32)
    _stack_check(wl, B, 2, cols=cols, seed_step=B)


# Shapes the persistent decode-step kernel takes (d % 512 == 0, token blocks of 1 or 2).
FUSED = [
    ("fused-f32-relu", 512, 2048, 0.05, 64, "relu", "f32", "f32", 1, 2),
    ("fused-f16-reglu-b2", 1024, 3000, 0.10, 64, "reglu", "f16", "f16", 2, 3),
    ("fused-q4-relu2", 512, 1500, 0.08, 32, "relu2", "q4_0", "f16", 1, 2),
    ("fused-f16-relu", 1536, 5000, 0.08, 128, "relu", "f16", "f16", 1, 2),
    ("fused-q4-reglu-b2", 1024, 2500, 0.10, 64, "reglu", "q4_0", "f16", 2, 2),
    ("fused-f16-reglu-allhot", 512, 700, 1.0, 32, "reglu", "f16", "f16", 1, 2),
    ("fused-f16-relu-nohot", 512, 900, 0.0, 32, "relu", "f16", "f16", 2, 2),
]


@pytest.mark.parametrize("case", FUSED, ids=[f[0] for f in FUSED])
def test_fused_stack_matches_oracle(case):
    name, d, ffn, hot, rank, act, wt, pt, B, L = case
    wl = _workload(name, d, ffn, hot, rank, act, wt, pt, B).with_(layers=L)
    assert pi.stack_launches(pi.desc_for(wl), B, L) == 1
    _stack_check(wl, B, L, seed_step=3)


# (name, d, ffn, hot_frac, rank, act, wtype, ptype, batch, layers)
EXTREMES = [
    ("ext-f16-reglu", 1024, 3000, 0.10, 64, "reglu", "f16", "f16", 1, 3),
    ("ext-f16-relu-b2", 1536, 5000, 0.08, 128, "relu", "f16", "f16", 2, 3),
    ("ext-q4-reglu-b2", 1024, 2500, 0.10, 64, "reglu", "q4_0", "f16", 2, 3),
    ("ext-f32-relu2", 512, 2048, 0.05, 64, "relu2", "f32", "f32", 1, 3),
]


@pytest.mark.parametrize("case", EXTREMES, ids=[e[0] for e in EXTREMES])
def test_fused_stack_every_cold_neuron_active_equals_dense(case):
    """Threshold -1e30 on every layer: the persistent kernel's lists are every
    cold row, so each layer must equal the dense FFN (skipping no neuron leaves
    the output unchanged: unite.ai, "Nöron Bilinçli Operatör").  Every CTA's
    local list is its whole P2 share: the longest lists the kernel can see."""
    name, d, ffn, hot, rank, act, wt, pt, B, L = case
    wl = _workload(name, d, ffn, hot, rank, act, wt, pt, B).with_(layers=L)
    assert pi.stack_launches(pi.desc_for(wl), B, L) == 1
    n_amb, counts = _stack_check(wl, B, L, seed_step=5, thr=-1e30, dense=True)
    assert n_amb == 0
    assert np.all(counts == wl.n_cold)


@pytest.mark.parametrize("case", EXTREMES, ids=[e[0] for e in EXTREMES])
def test_fused_stack_no_cold_neuron_active_is_hot_slice(case):
    """Threshold +1e30 on every layer: empty lists, and each layer's output is
    the hot slice alone."""
    name, d, ffn, hot, rank, act, wt, pt, B, L = case
    wl = _workload(name, d, ffn, hot, rank, act, wt, pt, B).with_(layers=L)
    assert pi.stack_launches(pi.desc_for(wl), B, L) == 1
    n_amb, counts = _stack_check(wl, B, L, seed_step=6, thr=1e30)
    assert n_amb == 0
    assert np.all(counts == 0)


def test_full_size_70b_sparsity_80_token_block_of_2():
    """The densest full-size setting of the persistent kernel: 70B-shaped
    layers at 80 % sparsity with a token block of 2 (the longest per-CTA lists
    and hand-overs); every list entry checked, y on 48 sampled columns."""
    wl = W.WORKLOADS["70b-reglu-fp16"].with_(sparsity=0.80)
    assert pi.stack_launches(pi.desc_for(wl), 2, 2) == 1
    rng = np.random.default_rng(80)
    cols = np.sort(rng.choice(wl.d, size=48, replace=False)).astype(np.int32)
    _, counts = _stack_check(wl, 2, 2, cols=cols, seed_step=2)
    assert np.all(counts > 0.1 * wl.n_cold)


@pytest.mark.parametrize("case", [(512, 900, 60, 32, "reglu", "f16", "f16", 1),
                                  (1024, 1200, 0, 32, "relu", "f16", "f16", 2),
                                  (512, 640, 40, 16, "relu2", "q4_0", "f16", 1),
                                  (512, 500, 50, 16, "relu", "f32", "f32", 2)])
def test_fused_stack_integer_exact(case):
    """One integer-exact layer through the persistent kernel: list and output
    are bit-identical to the oracle (fp32 sums of small integers are exact in
    any order, atomics included)."""
    d, ffn, n_hot, rank, act, wt, pt, B = case
    L = W.make_int_layer(d, ffn, n_hot, rank, act, wt, pt, B, seed=3 * d + ffn)
    L = {k: to_dev(v) if k not in ("perm", "thr") else v for k, v in L.items()}
    desc = pi.make_desc(d, ffn, n_hot, rank, wt, pt, act)
    assert pi.stack_launches(desc, B, 1) == 1
    ws = pi.workspace(desc, B)
    arr = pi.layer_array([pi.layer_weights(L)])
    C = ffn - n_hot
    idx = torch.full((1, max(C, 1)), -1, dtype=torch.int32, device="cuda")
    counts = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = torch.zeros(1, B, d, device="cuda")
    h_out = torch.zeros_like(L["h"])
    pi.decode_stack(desc, arr, L["h"], h_out, idx, counts, y, 1e-6, ws)
    torch.cuda.synchronize()
    assert pi.device_status(ws) == 0
    h_np = to_np(L["h"])
    orc = oracle.predict(h_np, to_np(L["P1"]), to_np(L["P2"]), to_np(L["bp"]), 0.5, n_hot, ffn)
    n = int(counts[0].item())
    assert np.array_equal(idx[0, :n].cpu().numpy(), orc["idx"])
    ref = oracle.masked_ffn(h_np, orc["idx"], to_np(L["Wg"]), to_np(L["Wu"]), to_np(L["WdT"]), to_np(L["b1"]),
                            to_np(L["b2"]), act, n_hot, ffn)
    assert np.array_equal(y[0].cpu().numpy().astype(np.float64), ref)


def test_fused_stack_repeated_calls_and_graph_replay():
    """The persistent kernel leaves its barrier state clean, and what varies
    between identical calls is bounded.  Its split-K adds each CTA's fp32
    partial with atomics, and which CTA takes a claimed hot chunk or a
    handed-over row depends on timing, so y may differ in its last fp32 bits.
    Everything else is fixed: the first layer's list (its input is the same
    token block) is identical on every call, later layers' lists agree with
    the oracle outside the 1e-3 band, y agrees to 1e-5 and h_out to one fp16
    ulp."""
    wl = _workload("replay", 1024, 3000, 0.1, 64, "reglu", "f16", "f16", 1).with_(layers=4)
    desc = pi.desc_for(wl)
    layers = [W.make_layer(wl, l, device="cuda") for l in range(4)]
    arr = pi.layer_array([pi.layer_weights(L) for L in layers])
    h0 = W.make_tokens(wl, 1, 9, device="cuda")
    ws = pi.workspace(desc, 1)
    outs = []
    s = torch.cuda.Stream()
    idx = torch.zeros(4, wl.n_cold, dtype=torch.int32, device="cuda")
    counts = torch.zeros(4, dtype=torch.int32, device="cuda")
    y = torch.zeros(4, 1, wl.d, device="cuda")
    trace = torch.zeros(4, 1, wl.d, dtype=h0.dtype, device="cuda")
    h_out = torch.zeros_like(h0)

    def keep():
        outs.append({"counts": counts.clone(), "idx": idx.clone(), "h": h_out.clone(), "y": y.clone(),
                     "trace": trace.clone()})

    with torch.cuda.stream(s):
        for _ in range(3):
            pi.decode_stack(desc, arr, h0, h_out, idx, counts, y, W.RMS_EPS, ws, h_trace=trace, stream=s)
            s.synchronize()
            keep()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            pi.decode_stack(desc, arr, h0, h_out, idx, counts, y, W.RMS_EPS, ws, h_trace=trace, stream=s)
        for _ in range(3):
            g.replay()
            s.synchronize()
            keep()
    assert pi.device_status(ws) == 0
    ref = outs[0]
    orcs = [oracle_predict(L, to_np(ref["trace"][l]), wl) for l, L in enumerate(layers)]
    n0 = int(ref["counts"][0].item())
    for o in outs[1:]:
        assert int(o["counts"][0].item()) == n0
        assert torch.equal(o["idx"][0, :n0], ref["idx"][0, :n0])
        for l in range(4):
            n = int(o["counts"][l].item())
            check_index_list(o["idx"][l, :n].cpu().numpy(), orcs[l], wl.thr, wl.n_hot, wl.ffn)
            same_in = torch.equal(o["trace"][l], ref["trace"][l])
            same_list = n == int(ref["counts"][l].item()) and torch.equal(o["idx"][l, :n], ref["idx"][l, :n])
            if same_in and same_list:   # same work, summed in another order
                dy = (o["y"][l] - ref["y"][l]).abs().max().item()
                assert dy <= 1e-5 * ref["y"][l].abs().max().item(), "layer %d" % l
        if all(torch.equal(o["trace"][l], ref["trace"][l]) for l in range(4)):
            assert (o["h"].float() - ref["h"].float()).abs().max().item() <= 2 ** -9
