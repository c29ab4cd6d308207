"""Helpers shared by the GPU parity tests: run libpi through its C ABI and
compare with the CPU oracle on the same seeded inputs."""
import contextlib

import numpy as np
import torch

import activation_sparse_decode_predict_b200 as pi
import oracle

# Acceptance bars: active-index lists are exact outside a 1e-3 band around
# the threshold; FFN outputs meet max|gpu - oracle| / max|oracle| <= 2e-3
# (fp32/fp16 weights) or 5e-3 (Q4_0), with the oracle fed the GPU's list.
BAND = 1e-3
TOL = {"f32": 2e-3, "f16": 2e-3, "q4_0": 5e-3}


def to_np(x):
    if x is None:
        return None
    if isinstance(x, tuple):
        return tuple(to_np(t) for t in x)
    return np.ascontiguousarray(x.detach().cpu().numpy())


def to_dev(x, dev="cuda"):
    if x is None:
        return None
    if isinstance(x, tuple):
        return tuple(to_dev(t, dev) for t in x)
    if isinstance(x, torch.Tensor):
        return x.to(dev).contiguous()
    return x


def gpu_predict(desc, h, L, ws):
    C = desc.ffn - desc.n_hot
    idx = torch.full((max(C, 1),), -7, dtype=torch.int32, device="cuda")
    count = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    pi.predict(desc, h, L["P1"], L["P2"], L["bp"], L["thr"], idx, count, ws)
    torch.cuda.synchronize()
    n = int(count.item())
    return idx[:n].cpu().numpy(), idx, count


def gpu_ffn(desc, h, L, idx, count, ws):
    y = torch.full((h.shape[0], desc.d), float("nan"), dtype=torch.float32, device="cuda")
    pi.sparse_ffn(desc, h, idx, count, L.get("Wg"), L["Wu"], L["WdT"], L.get("b1"), L.get("b2"), y, ws)
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


def check_index_list(gpu_idx, orc, thr, n_hot, ffn):
    """The GPU list is ascending, unique, inside [n_hot, ffn), and equals the
    oracle's list on every neuron whose scores are all outside the band."""
    C = ffn - n_hot
    gpu_idx = np.asarray(gpu_idx)
    assert np.all(np.diff(gpu_idx) > 0), "list not strictly ascending"
    if len(gpu_idx):
        assert gpu_idx[0] >= n_hot and gpu_idx[-1] < ffn
    g = np.zeros(C, bool)
    g[gpu_idx - n_hot] = True
    o = orc["mask"].astype(bool)
    amb = (np.abs(orc["s"] - thr) <= BAND).any(axis=0) if C else np.zeros(0, bool)
    bad = np.nonzero((g != o) & ~amb)[0]
    assert len(bad) == 0, "index lists differ outside the band at cold rows %s" % bad[:10]
    return int(amb.sum())


def rel_err(y, ref):
    den = np.abs(ref).max()
    return float(np.abs(y - ref).max() / (den if den > 0 else 1.0))


def oracle_layer(L, h_np, wl, idx, cols=None):
    """The oracle's y for list [0, n_hot) ++ idx."""
    Ln = {k: to_np(L[k]) if k in L else None for k in ("Wg", "Wu", "WdT", "b1", "b2")}
    return oracle.masked_ffn(h_np, idx, Ln["Wg"], Ln["Wu"], Ln["WdT"], Ln["b1"], Ln["b2"], wl.act, wl.n_hot, wl.ffn,
                             cols=cols)


def oracle_predict(L, h_np, wl):
    return oracle.predict(h_np, to_np(L["P1"]), to_np(L["P2"]), to_np(L["bp"]), L["thr"], wl.n_hot, wl.ffn)


@contextlib.contextmanager
def token_ffn(path):
    """Run the body with the token-block FFN kernels `path` ("warp_mma" or
    "tcgen05"), then restore the previous choice."""
    old = pi.token_block_ffn()
    pi.set_token_block_ffn(path)
    try:
        yield
    finally:
        pi.set_token_block_ffn(old)
