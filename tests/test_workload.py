"""The seeded synthetic workloads have the statistics they claim."""
import math

import numpy as np
import pytest
import torch

import oracle
import pi_workload as W


def test_zipf_probabilities():
    for n, a, mean in ((2048, 1.1, 0.10), (11008, 1.2, 0.12), (28672, 1.2, 0.05)):
        p = W.zipf_probs(n, a, mean)
        assert abs(p.mean() - mean) < 1e-9
        assert np.all(np.diff(p) <= 0) and p.max() <= 0.99 and p.min() > 0


def test_hot_first_layout_is_a_permutation_with_hot_rows_first():
    w = W.WORKLOADS["7b-reglu-fp16"]
    p, perm = W.neuron_layout(w, 3)
    assert np.array_equal(np.sort(perm), np.arange(w.ffn))
    ps = p[perm]
    assert ps[: w.n_hot].min() >= ps[w.n_hot:].max()
    assert np.all(np.diff(perm[: w.n_hot]) > 0) and np.all(np.diff(perm[w.n_hot:]) > 0)
    assert w.n_hot == 1101


def test_hot_counts_match_workload_statements():
    assert [W.WORKLOADS[k].n_hot for k in W.WORKLOADS] == [103, 1101, 1383, 2622, 2868]


SMALL = W.Workload("small", 9, 256, 1500, 2, "reglu", "f32", "f32", 0.88, 1.2, 0.10, 64, (1,), 4)


def test_generated_layer_statistics():
    w = SMALL
    L = W.make_layer(w, 0)
    assert L["Wg"].shape == (w.ffn, w.d) and L["P1"].shape == (w.rank, w.d) and L["P2"].shape == (w.n_cold, w.rank)
    assert torch.allclose(L["b1"].double(), torch.special.ndtri(torch.as_tensor(L["p"])), atol=1e-6)
    hs = np.concatenate([W.make_tokens(w, 1, t).numpy() for t in range(48)])
    assert np.allclose((hs.astype(np.float64) ** 2).sum(1), w.d, rtol=1e-5)
    sup = oracle.true_support(hs, L["Wg"].numpy(), L["Wu"].numpy(), L["b1"].numpy(), "reglu", w.ffn)
    # per-token firing fraction ~ 1 - sparsity
    assert abs(sup.mean() - (1 - w.sparsity)) < 0.02
    # hot neurons fire far more often than cold ones
    assert sup[:, : w.n_hot].mean() > 4 * sup[:, w.n_hot:].mean()
    # the predictor recovers most of the true cold support
    rec, prec = [], []
    for t in range(16):
        r = oracle.predict(hs[t:t + 1], L["P1"].numpy(), L["P2"].numpy(), L["bp"].numpy(), w.thr, w.n_hot, w.ffn)
        pred = np.zeros(w.n_cold, bool)
        pred[r["idx"] - w.n_hot] = True
        true = sup[t, w.n_hot:].astype(bool)
        rec.append((pred & true).sum() / max(true.sum(), 1))
        prec.append((pred & true).sum() / max(pred.sum(), 1))
    assert np.mean(rec) > 0.6 and np.mean(prec) > 0.6


def test_predictor_construction_is_the_low_rank_part_of_the_gate():
    w = SMALL
    L = W.make_layer(w, 1)
    h = W.make_tokens(w, 2, 0).numpy()
    r = oracle.predict(h, L["P1"].numpy(), L["P2"].numpy(), L["bp"].numpy(), w.thr, w.n_hot, w.ffn)
    # s - thr correlates strongly with the true gate pre-activation (rho = 0.9)
    g = h.astype(np.float64) @ L["Wg"].numpy().astype(np.float64).T + L["b1"].numpy()
    c = np.corrcoef((r["s"] - w.thr).ravel(), g[:, w.n_hot:].ravel())[0, 1]
    assert c > 0.9


def test_q4_0_quantizer_roundtrip():
    g = torch.Generator().manual_seed(0)
    x = torch.randn(6, 128, generator=g) / math.sqrt(128)
    qs, sc = W.quantize_q4_0(x)
    assert qs.dtype == torch.uint8 and qs.shape == (6, 64) and sc.shape == (6, 4)
    dec = oracle.decode_matrix((qs.numpy(), sc.numpy()), 128)
    s = np.repeat(np.abs(sc.numpy().astype(np.float64)), 32, axis=1)
    err = np.abs(dec - x.numpy())
    # rounding error <= s/2, except where q = 16 is clamped to 15 (x = -m): error <= s
    assert np.all(err <= 1.001 * s + 1e-7)
    assert np.mean(err <= 0.5 * s * 1.001 + 1e-7) > 0.95
    blk = x.numpy().reshape(6, 4, 32)
    m = np.take_along_axis(blk, np.abs(blk).argmax(-1)[..., None], -1)[..., 0]
    assert np.allclose(dec.reshape(6, 4, 32)[np.arange(6)[:, None], np.arange(4)[None], np.abs(blk).argmax(-1)], m,
                       rtol=2e-3)


def test_integer_layer_is_exact_in_fp16():
    L = W.make_int_layer(256, 300, 30, 32, "reglu", "f16", "f16", 2, seed=1)
    for k in ("Wg", "Wu", "WdT", "P1", "P2", "h"):
        v = L[k].float()
        assert torch.equal(v, torch.round(v))
    Lq = W.make_int_layer(256, 300, 30, 32, "relu", "q4_0", "f16", 1, seed=2)
    qs, sc = Lq["Wu"]
    assert qs.shape == (300, 128) and sc.shape == (300, 8)


def test_algorithmic_bytes_per_layer():
    w = W.WORKLOADS["7b-reglu-fp16"]
    A = W.expected_active(w, 1)
    assert 500 < A < 650
    mb = W.layer_bytes(w, 1, A) / 1e6
    assert 68 < mb < 72
    w5 = W.WORKLOADS["70b-reglu-fp16"]
    assert 330 < W.layer_bytes(w5, 1, W.expected_active(w5, 1)) / 1e6 < 345


def test_relu_stack_keeps_the_tokens_of_a_block_apart():
    """b2 removes the common part of the ReLU FFN output, so the stack glue does
    not pull the tokens of a block together (their active sets stay distinct)."""
    import torch
    for act in ("relu", "relu2", "reglu"):
        wl = W.Workload("apart", 93, 512, 2048, 6, act, "f32", "f32", 0.92, 1.3, 0.08, 64, (8,), 1)
        h = W.make_tokens(wl, 8, 1).double()
        for l in range(6):
            L = W.make_layer(wl, l)
            z = h @ L["Wu"].double().T
            if act == "reglu":
                a = torch.relu(h @ L["Wg"].double().T + L["b1"].double()) * z
            else:
                a = torch.relu(z + L["b1"].double())
                if act == "relu2":
                    a = a * a
            y = a @ L["WdT"].double()
            if L["b2"] is not None:
                y = y + L["b2"].double()
            x = h + y
            h = x / torch.sqrt((x * x).mean(1, keepdim=True) + 1e-6)
        hn = h / h.norm(dim=1, keepdim=True)
        cos = (hn @ hn.T)[~torch.eye(8, dtype=torch.bool)]
        assert cos.abs().mean().item() < 0.3, (act, cos.abs().mean().item())  # uncentred ReLU: > 0.8


@pytest.mark.parametrize("act,wtype,ptype,batch", [("reglu", "f16", "f16", 1), ("relu", "f32", "f32", 2),
                                                   ("relu2", "f16", "f16", 3), ("reglu", "q4_0", "f16", 1)])
def test_layer_bytes_counts_the_bytes_of_the_tensors_read(act, wtype, ptype, batch):
    """The roofline's algorithmic bytes equal the bytes of the tensors an ideal
    pass reads and writes, counted from a generated layer: both predictor
    matrices and bp, the listed rows of every weight matrix with their b1
    entries, the index list, the token block in, the fp32 output out and b2."""
    w = W.WORKLOADS["tiny-relu-fp32"].with_(d=256, ffn=1024, rank=32, act=act, wtype=wtype, ptype=ptype)
    L = W.make_layer(w, 0)
    n_active = 37

    def row_bytes(m):
        if isinstance(m, tuple):  # Q4_0 planes
            return m[0][0].numel() * m[0].element_size() + m[1][0].numel() * m[1].element_size()
        return m[0].numel() * m.element_size()

    mats = [L["Wg"], L["Wu"], L["WdT"]] if w.gated else [L["Wu"], L["WdT"]]
    n_list = w.n_hot + n_active
    tok = torch.empty(0, dtype=L["P1"].dtype).element_size()
    expect = (L["P1"].numel() * L["P1"].element_size() + L["P2"].numel() * L["P2"].element_size()
              + L["bp"].numel() * 4
              + sum(row_bytes(m) for m in mats) * n_list + 4 * n_list
              + 4 * n_active
              + batch * w.d * tok + batch * w.d * 4
              + (L["b2"].numel() * 4 if L["b2"] is not None else 0))
    assert W.layer_bytes(w, batch, n_active) == pytest.approx(expect, rel=0, abs=1e-6)
