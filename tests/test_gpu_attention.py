"""GPU parity of the head-sparse decode attention (unite.ai "Adaptif Sparsite
Predictor’ları": a second per-layer predictor picks the self-attention heads
to compute) against the CPU oracle: given head lists, the head predictor
feeding it, the cache append, and the edge cases."""
import numpy as np
import pytest
import torch

import activation_sparse_decode_predict_b200 as pi
import oracle
import pi_workload as W
from gpu_util import TOL, check_index_list, rel_err, to_np

pytestmark = pytest.mark.gpu


def _inputs(d, H, n_hot, rank, B, s_max, seed, wt="f16", xt="f16", ct="f16"):
    A = W.make_attention(d, H, n_hot, rank, B, s_max, seed, wtype=wt, ctype=ct, device="cuda")
    g = torch.Generator(device="cpu").manual_seed(seed + 1)
    x = torch.randn(B, d, generator=g, dtype=torch.float64)
    x = (x * (d ** 0.5) / x.norm(dim=1, keepdim=True)).to(torch.float16 if xt == "f16" else torch.float32).cuda()
    return A, x


def _run(desc, x, hidx, hcnt, A, length, ws):
    y = torch.full((x.shape[0], desc.d), float("nan"), dtype=torch.float32, device="cuda")
    pi.sparse_attention(desc, x, hidx, hcnt, A["Wq"], A["Wk"], A["Wv"], A["WoT"], A["K"], A["V"], length, y, ws)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


# (name, d, n_heads, n_hot, B, len, s_max, wtype, xtype, ctype)
CASES = [
    ("7b-heads-b1", 4096, 32, 4, 1, 300, 512, "f16", "f16", "f16"),
    ("dh64-b3", 512, 8, 1, 3, 37, 64, "f16", "f16", "f16"),
    ("dh32-b2-fp32", 256, 8, 0, 2, 5, 16, "f32", "f32", "f32"),
    ("dh256-b16", 2048, 8, 2, 16, 150, 160, "f16", "f16", "f16"),
    ("empty-cache-b2", 512, 4, 0, 2, 0, 8, "f16", "f16", "f16"),
    ("f32w-f16x-f32cache", 512, 4, 1, 1, 64, 80, "f32", "f16", "f32"),
    ("long-cache-b1", 1024, 8, 0, 1, 3000, 3072, "f16", "f16", "f16"),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_sparse_attention_matches_oracle(case):
    name, d, H, n_hot, B, L, s_max, wt, xt, ct = case
    A, x = _inputs(d, H, n_hot, 32, B, s_max, seed=d + H + B + L, wt=wt, xt=xt, ct=ct)
    rng = np.random.default_rng(L + 7)
    cold = np.arange(n_hot, H)
    listed = np.sort(rng.choice(cold, size=max(1, len(cold) // 2), replace=False)).astype(np.int32) if len(cold) \
        else np.zeros(0, np.int32)
    hidx = torch.tensor(listed if len(listed) else [0], dtype=torch.int32, device="cuda")
    hcnt = torch.tensor([len(listed)], dtype=torch.int32, device="cuda")
    desc = pi.attn_desc(d, H, n_hot, s_max, wt, xt, ct)
    ws = pi.attn_workspace(desc, B)
    K0, V0 = A["K"].clone(), A["V"].clone()
    ref = oracle.attention(to_np(x), listed, *(to_np(A[k]) for k in ("Wq", "Wk", "Wv", "WoT")), to_np(K0), to_np(V0),
                           L, H, n_hot)
    y = _run(desc, x, hidx, hcnt, A, L, ws)
    assert pi.device_status(ws) == 0
    assert rel_err(y, ref["y"]) <= TOL["f16"], name
    # the listed heads' k and v are appended at position len; nothing else in the caches moves
    heads = list(range(n_hot)) + listed.tolist()
    tol = 2 ** -10 if ct == "f16" else 1e-5
    for p, h in enumerate(heads):
        for cache, new in ((A["K"], ref["k"]), (A["V"], ref["v"])):
            got = cache[:, h, L].double().cpu().numpy()
            assert np.abs(got - new[:, p]).max() <= tol * max(1.0, np.abs(new[:, p]).max()), (name, h)
    touched = torch.zeros(H, dtype=torch.bool)
    touched[heads] = True
    for cache, orig in ((A["K"], K0), (A["V"], V0)):
        same = cache.clone()
        same[:, touched.cuda(), L] = orig[:, touched.cuda(), L]
        assert torch.equal(same, orig), name


def test_head_predictor_feeds_sparse_attention():
    """pi_predict with the heads as its neurons picks the heads; the attention
    over exactly those heads matches the oracle's predictor and attention."""
    d, H, n_hot, rank, B, L, s_max = 2048, 16, 2, 64, 2, 200, 256
    A, x = _inputs(d, H, n_hot, rank, B, s_max, seed=5)
    fdesc = pi.make_desc(d, H, n_hot, rank, "f16", "f16", "relu")
    fws = pi.workspace(fdesc, B)
    hidx = torch.full((H - n_hot,), -1, dtype=torch.int32, device="cuda")
    hcnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    pi.predict(fdesc, x, A["P1"], A["P2"], A["bp"], A["thr"], hidx, hcnt, fws)
    torch.cuda.synchronize()
    n = int(hcnt.item())
    listed = hidx[:n].cpu().numpy()
    orc = oracle.predict(to_np(x), to_np(A["P1"]), to_np(A["P2"]), to_np(A["bp"]), A["thr"], n_hot, H)
    check_index_list(listed, orc, A["thr"], n_hot, H)
    assert 0 < n < H - n_hot
    desc = pi.attn_desc(d, H, n_hot, s_max)
    ws = pi.attn_workspace(desc, B)
    ref = oracle.attention(to_np(x), listed, *(to_np(A[k]) for k in ("Wq", "Wk", "Wv", "WoT", "K", "V")), L, H, n_hot)
    y = _run(desc, x, hidx, hcnt, A, L, ws)
    assert pi.device_status(ws) == 0
    assert rel_err(y, ref["y"]) <= TOL["f16"]


def test_all_heads_listed_is_dense_attention_and_bad_heads_are_flagged():
    d, H, B, L, s_max = 1024, 8, 2, 50, 64
    A, x = _inputs(d, H, 0, 32, B, s_max, seed=9)
    desc = pi.attn_desc(d, H, 0, s_max)
    ws = pi.attn_workspace(desc, B)
    K0, V0 = to_np(A["K"]), to_np(A["V"])
    every = np.arange(H, dtype=np.int32)
    ref = oracle.attention(to_np(x), every, *(to_np(A[k]) for k in ("Wq", "Wk", "Wv", "WoT")), K0, V0, L, H, 0)
    y = _run(desc, x, torch.tensor(every, device="cuda"), torch.tensor([H], dtype=torch.int32, device="cuda"), A, L, ws)
    assert rel_err(y, ref["y"]) <= TOL["f16"]
    # an index outside [n_hot, n_heads) is reported and skipped
    bad = torch.tensor([1, 99, 4], dtype=torch.int32, device="cuda")
    y = _run(desc, x, bad, torch.tensor([3], dtype=torch.int32, device="cuda"), A, L, ws)
    assert pi.device_status(ws, clear=True) == pi._binding.PI_ERR_INDEX
    ref = oracle.attention(to_np(x), [1, 4], *(to_np(A[k]) for k in ("Wq", "Wk", "Wv", "WoT")), K0, V0, L, H, 0)
    assert rel_err(y, ref["y"]) <= TOL["f16"]
    # no head listed: y = 0
    y = _run(desc, x, bad, torch.tensor([0], dtype=torch.int32, device="cuda"), A, L, ws)
    assert np.all(y == 0) and pi.device_status(ws) == 0
