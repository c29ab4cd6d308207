"""Seeded synthetic workloads for the activation-sparse decode FFN.

This module only *makes inputs*: weights, predictor matrices, biases and token
blocks with the shapes and statistics of the five benchmark workloads.  It
holds none of the method's arithmetic (no predictor evaluation, no FFN, no
decoding of Q4_0); both the CUDA path and the CPU oracle consume what it
makes, and neither is imported here.

Statistics (the pages give none of these numerically; each choice is the
plainest one that reproduces the property the pages describe):

* Power-law neuron activity ([AB] "Hot-Cold-Neuron-Mechanismus"; [UA]
  "Offline Aşama"): neuron of Zipf rank k fires with probability
  p_k = min(0.99, c * k^-alpha), c bisected so that mean_k p_k = 1 - sparsity.
  The rank -> neuron-id map is a seeded random permutation.
* The firing rate is set through the bias b1 = Phi^-1(p) on the gate (ReGLU)
  or the up projection (ReLU, squared ReLU): with ||h||^2 = d and rows of
  variance 1/d, w.h ~ N(0, 1), so P(w.h + b1 > 0) = p.
* Predictor: W_gate (or W_up) = U V + sqrt(1 - rho) E with U ~ N(0, rho/r'),
  V ~ N(0, 1/d), E ~ N(0, 1/d), r' = rank / 2, rho = 0.9.  P1 = [V; -V] and
  P2 = [U, -U] (cold rows only), bp = b1 + thr, so that
  P2 ReLU(P1 h) + bp - thr = U V h + b1, the low-rank part of the true
  pre-activation.
* Hot set: the top ceil(hot_frac * ffn) neurons by firing probability.  The
  offline layout stores them first ([UA] "Nöron Yerleştirme ve Yönetimi":
  a neuron table maps each placed neuron back to its original row); ``perm``
  is that table (storage row -> original row).
* Q4_0 ([GN] "Kuantisasi dan kompatibilitas"): 32-element blocks along d,
  scale s = m / -8 where m is the block element of largest magnitude (sign
  kept), rounded to fp16; q = clamp(round_half_away(x / s) + 8, 0, 15); byte k
  of a block holds q[k] (low nibble) and q[k + 16] (high nibble).  Split
  planes: qs [rows, d/2] uint8 and sc [rows, d/32] fp16.
* Tokens: h ~ N(0, 1)^d, scaled so that ||h||^2 = d.

Pages: [GN] GeekNews "Serving model bahasa besar berkecepatan tinggi pada PC
dengan GPU konsumen"; [AB] aibars.net "PowerInfer - Hochgeschwindigkeits-
Inferenz-Engine für große Sprachmodelle"; [UA] unite.ai "PowerInfer: Tüketici
Düzeyinde bir GPU ile Hızlı Büyük Dil Modeli Sunucusu".
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np
import torch

RHO = 0.9
THRESHOLD = 0.5
RMS_EPS = 1e-6


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    cfg_id: int
    d: int
    ffn: int
    layers: int
    act: str          # "relu" | "reglu" | "relu2"
    wtype: str        # "f32" | "f16" | "q4_0"
    ptype: str        # "f32" | "f16" | "q4_0" (predictor dtype; tokens are fp32 with fp32 predictors, else fp16)
    sparsity: float
    alpha: float
    hot_frac: float
    rank: int
    batches: tuple
    steps: int
    has_b2: bool = False
    thr: float = THRESHOLD
    # per-layer predictor ranks (layer l takes rank_steps[l % len]); empty: every layer has `rank`
    rank_steps: tuple = ()

    @property
    def n_hot(self) -> int:
        return int(math.ceil(self.hot_frac * self.ffn - 1e-9))

    @property
    def n_cold(self) -> int:
        return self.ffn - self.n_hot

    @property
    def gated(self) -> bool:
        return self.act == "reglu"

    @property
    def htype(self) -> str:
        """Token-block dtype: fp32 with fp32 predictors, fp16 otherwise."""
        return "f32" if self.ptype == "f32" else "f16"

    def layer_rank(self, layer: int) -> int:
        """Predictor rank of a layer ([UA] "Adaptif Sparsite Predictor’ları":
        the predictor's size is chosen per layer); never above `rank`."""
        if not self.rank_steps:
            return self.rank
        r = int(self.rank_steps[layer % len(self.rank_steps)])
        assert 0 < r <= self.rank
        return r

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five synthetic workloads (shapes of OPT-tiny, ReluLLaMA-7B, Llama2-13B,
# Falcon-40B and Llama2-70B FFNs).  Steps for the last three are not fixed by
# their statement; 512 / 128 / 128 bound the run time.
WORKLOADS: Dict[str, Workload] = {
    "tiny-relu-fp32": Workload("tiny-relu-fp32", 1, 512, 2048, 2, "relu", "f32", "f32", 0.90, 1.1, 0.05, 64,
                               (1,), 256, has_b2=True),
    "7b-reglu-fp16": Workload("7b-reglu-fp16", 2, 4096, 11008, 32, "reglu", "f16", "f16", 0.88, 1.2, 0.10, 1024,
                              (1,), 512),
    "13b-reglu-q4_0": Workload("13b-reglu-q4_0", 3, 5120, 13824, 40, "reglu", "q4_0", "f16", 0.90, 1.2, 0.10, 1024,
                               (1,), 512),
    "40b-relu-fp16": Workload("40b-relu-fp16", 4, 8192, 32768, 60, "relu", "f16", "f16", 0.92, 1.3, 0.08, 1536,
                              (1, 8), 128),
    "70b-reglu-fp16": Workload("70b-reglu-fp16", 5, 8192, 28672, 80, "reglu", "f16", "f16", 0.90, 1.2, 0.10, 2048,
                               (1, 4, 16), 128),
}
SPARSITY_SWEEP_70B = (0.80, 0.90, 0.95)

_TORCH_DT = {"f32": torch.float32, "f16": torch.float16}


def _seed(w: Workload, layer: int, tensor: int) -> int:
    key = (w.cfg_id * 1_000_003 + int(round(w.sparsity * 1000))) * 10_007 + layer
    return (key * 131 + tensor) & 0x7FFF_FFFF_FFFF


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def zipf_probs(n: int, alpha: float, mean: float, pmax: float = 0.99) -> np.ndarray:
    """p[k-1] = min(pmax, c k^-alpha) for Zipf rank k = 1..n with mean(p) = mean (bisection on c)."""
    base = np.arange(1, n + 1, dtype=np.float64) ** (-alpha)
    lo, hi = 0.0, 1.0 / base[-1]
    for _ in range(200):
        c = 0.5 * (lo + hi)
        if np.minimum(pmax, c * base).mean() < mean:
            lo = c
        else:
            hi = c
    return np.minimum(pmax, 0.5 * (lo + hi) * base)


def neuron_layout(w: Workload, layer: int):
    """Firing probabilities and the hot-first neuron table for one layer.

    Returns (p_orig [ffn] float64 by original neuron id, perm [ffn] int64 with
    perm[storage row] = original id: hot ids ascending, then cold ids ascending).
    """
    p_rank = zipf_probs(w.ffn, w.alpha, 1.0 - w.sparsity)
    rng = np.random.default_rng(_seed(w, layer, 1))
    rank_to_id = rng.permutation(w.ffn)
    p_orig = np.empty(w.ffn, np.float64)
    p_orig[rank_to_id] = p_rank
    hot_ids = np.sort(rank_to_id[: w.n_hot])
    is_hot = np.zeros(w.ffn, bool)
    is_hot[hot_ids] = True
    perm = np.concatenate([hot_ids, np.nonzero(~is_hot)[0]]).astype(np.int64)
    return p_orig, perm


def quantize_q4_0(x: torch.Tensor):
    """Q4_0 split planes of a [rows, d] tensor (d % 32 == 0): (qs uint8 [rows, d/2], sc fp16 [rows, d/32])."""
    rows, d = x.shape
    assert d % 32 == 0
    blk = x.float().reshape(rows, d // 32, 32)
    amax_i = blk.abs().argmax(dim=-1, keepdim=True)
    m = torch.gather(blk, -1, amax_i)
    s16 = (m / -8.0).to(torch.float16)
    s = s16.float()
    safe = torch.where(s == 0, torch.ones_like(s), s)
    v = blk / safe
    q = torch.sign(v) * torch.floor(v.abs() + 0.5) + 8.0
    q = torch.where(s == 0, torch.full_like(q, 8.0), q).clamp_(0, 15).to(torch.uint8)
    qs = (q[..., :16] | (q[..., 16:] << 4)).reshape(rows, d // 2).contiguous()
    sc = s16.reshape(rows, d // 32).contiguous()
    return qs, sc


def pack_q4_0(x: torch.Tensor):
    """Q4_0 planes of a [rows, cols] matrix in ONE buffer, scales after the
    codes (the C ABI's layout of a Q4_0 predictor matrix); returns the pair
    (qs, sc) of views into that buffer."""
    qs, sc = quantize_q4_0(x.to(torch.float16))
    n = qs.numel()
    buf = torch.empty(n + 2 * sc.numel(), dtype=torch.uint8, device=x.device)
    buf[:n] = qs.reshape(-1)
    buf[n:] = sc.reshape(-1).view(torch.uint8)
    rows, cols = x.shape
    return buf[:n].view(rows, cols // 2), buf[n:].view(torch.float16).view(rows, cols // 32)


def _as_ptype(x: torch.Tensor, ptype: str):
    if ptype == "q4_0":
        return pack_q4_0(x)
    return x.to(_TORCH_DT[ptype]).contiguous()


def _as_wtype(x: torch.Tensor, wtype: str):
    if wtype == "q4_0":
        return quantize_q4_0(x.to(torch.float16))
    return x.to(_TORCH_DT[wtype]).contiguous()


def make_layer(w: Workload, layer: int, device="cpu") -> dict:
    """All tensors of one layer in storage (hot-first) order, on `device`.

    Keys: Wg (ReGLU only), Wu, WdT (each a tensor [ffn, d] or a Q4_0 pair),
    b1 fp32 [ffn], b2 fp32 [d] or None, P1 [rank, d], P2 [n_cold, rank], bp fp32
    [n_cold], perm int64 [ffn], p fp64 [ffn] (storage order), thr.
    """
    d, F, r = w.d, w.ffn, w.layer_rank(layer)
    assert r % 2 == 0
    rh = r // 2
    p_orig, perm = neuron_layout(w, layer)
    perm_t = torch.as_tensor(perm, device=device)
    inv_sd = 1.0 / math.sqrt(d)

    U = torch.randn(F, rh, generator=_gen(device, _seed(w, layer, 2)), device=device) * math.sqrt(RHO / rh)
    V = torch.randn(rh, d, generator=_gen(device, _seed(w, layer, 3)), device=device) * inv_sd
    E = torch.randn(F, d, generator=_gen(device, _seed(w, layer, 4)), device=device) * inv_sd
    W_pred = U @ V
    W_pred.add_(E, alpha=math.sqrt(1.0 - RHO))
    del E
    W_other = torch.randn(F, d, generator=_gen(device, _seed(w, layer, 5)), device=device) * inv_sd
    WdT = torch.randn(F, d, generator=_gen(device, _seed(w, layer, 6)), device=device) * inv_sd

    b1_orig = torch.special.ndtri(torch.as_tensor(p_orig, dtype=torch.float64)).to(torch.float32)
    b1 = b1_orig.to(device)[perm_t].contiguous()
    b2 = None
    if w.has_b2:
        b2 = (torch.randn(d, generator=_gen(device, _seed(w, layer, 7)), device=device) * 0.05).float()
    if not w.gated:
        # ReLU / squared ReLU: every token's output has a common part, the
        # expected activations (positive for the often-firing neurons) times
        # their down rows.  Added layer after layer it would pull the tokens of
        # a block onto one direction, and the union of their active sets would
        # shrink to a single token's.  b2 removes it: b2 -= sum_j E[a_j] WdT[j],
        # with z_j = w_j . h + b1_j ~ N(b1_j, |w_j|^2) for ||h||^2 = d, taken on
        # the rows before they are rounded to their storage type.  (ReGLU
        # needs nothing: its up dot has mean zero.)
        z_sd = W_pred.norm(dim=1).double()[perm_t]
        bz = b1.double()
        t = bz / z_sd
        pdf = torch.exp(-0.5 * t * t) / math.sqrt(2.0 * math.pi)
        cdf = 0.5 * torch.erfc(-t / math.sqrt(2.0))
        if w.act == "relu2":
            ea = (bz * bz + z_sd * z_sd) * cdf + bz * z_sd * pdf
        else:
            ea = bz * cdf + z_sd * pdf
        ea_orig = torch.zeros(F, dtype=torch.float32, device=device)
        ea_orig[perm_t] = ea.float()
        common = (ea_orig.unsqueeze(0) @ WdT).squeeze(0)
        b2 = (-common if b2 is None else b2 - common).float().contiguous()
    out = {"perm": perm, "p": p_orig[perm], "thr": w.thr}
    if w.gated:
        out["Wg"] = _as_wtype(W_pred[perm_t], w.wtype)
        out["Wu"] = _as_wtype(W_other[perm_t], w.wtype)
    else:
        out["Wg"] = None
        out["Wu"] = _as_wtype(W_pred[perm_t], w.wtype)
    del W_pred, W_other
    out["WdT"] = _as_wtype(WdT[perm_t], w.wtype)
    del WdT
    out["b1"] = b1
    out["b2"] = b2
    out["P1"] = _as_ptype(torch.cat([V, -V], dim=0), w.ptype)
    U_cold = U[perm_t[w.n_hot:]]
    out["P2"] = _as_ptype(torch.cat([U_cold, -U_cold], dim=1), w.ptype) if w.n_cold > 0 else None
    out["rank"] = r
    out["bp"] = (b1[w.n_hot:] + w.thr).float().contiguous()
    return out


def make_tokens(w: Workload, batch: int, step: int, device="cpu") -> torch.Tensor:
    """Token block h [batch, d] for decode step `step`: N(0,1) rows scaled to ||h||^2 = d."""
    g = _gen(device, _seed(w, 0xF0, step))
    h = torch.randn(batch, w.d, generator=g, device=device, dtype=torch.float64)
    h = h * (math.sqrt(w.d) / h.norm(dim=1, keepdim=True))
    return h.to(_TORCH_DT[w.htype]).contiguous()


def make_int_layer(d: int, ffn: int, n_hot: int, rank: int, act: str, wtype: str, ptype: str, batch: int,
                   seed: int, density: float = 0.05, device="cpu") -> dict:
    """A layer whose every product and partial sum is exact in fp16/fp32/double.

    Weights, predictor entries and tokens are small integers (Q4_0: s * (q - 8)
    with s a power of two), most of them zero, so that dot products are small
    integers and fp32 accumulation is exact in any order.  bp is an integer
    and thr = 0.5, so no score ever ties the threshold.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)

    def sparse_int(shape, lo, hi, dens):
        v = torch.randint(lo, hi + 1, shape, generator=g).float()
        keep = torch.rand(shape, generator=g) < dens
        return v * keep

    h = sparse_int((batch, d), -2, 2, 0.5)
    out = {"h": h.to(_TORCH_DT[ptype]).to(device), "thr": 0.5, "perm": np.arange(ffn)}
    if wtype == "q4_0":
        def qmat():
            q = torch.randint(0, 16, (ffn, d), generator=g)
            keep = torch.rand((ffn, d), generator=g) < density
            q = torch.where(keep, q, torch.full_like(q, 8)).to(torch.uint8).reshape(ffn, d // 32, 32)
            qs = (q[..., :16] | (q[..., 16:] << 4)).reshape(ffn, d // 2).contiguous()
            e = torch.randint(-2, 1, (ffn, d // 32), generator=g).float()
            sc = torch.pow(2.0, e).to(torch.float16).contiguous()
            return qs.to(device), sc.to(device)
        Wg, Wu, WdT = (qmat() if act == "reglu" else None), qmat(), qmat()
    else:
        dt = _TORCH_DT[wtype]
        Wg = sparse_int((ffn, d), -2, 2, density).to(dt).to(device) if act == "reglu" else None
        Wu = sparse_int((ffn, d), -2, 2, density).to(dt).to(device)
        WdT = sparse_int((ffn, d), -2, 2, density).to(dt).to(device)
    out.update(Wg=Wg, Wu=Wu, WdT=WdT)
    out["b1"] = torch.randint(-1, 2, (ffn,), generator=g).float().to(device)
    out["b2"] = torch.randint(-2, 3, (d,), generator=g).float().to(device)
    pt = _TORCH_DT[ptype]
    out["P1"] = sparse_int((rank, d), -1, 1, min(1.0, 8.0 / d + density)).to(pt).to(device)
    out["P2"] = sparse_int((ffn - n_hot, rank), -1, 1, min(1.0, 4.0 / rank + density)).to(pt).to(device)
    out["bp"] = torch.randint(-2, 2, (ffn - n_hot,), generator=g).float().to(device)
    return out


def layer_bytes(w: Workload, batch: int, n_active: float, rank: Optional[int] = None) -> float:
    """Algorithmic bytes one layer must move for one token block with n_active
    predicted-active cold neurons: both predictor matrices (of the layer's
    rank), the listed weight rows (hot + active), their biases, the index
    list, and the token block in and the fp32 output out."""
    e = {"f32": 4.0, "f16": 2.0, "q4_0": 18.0 / 32.0}
    e_p = e[w.ptype]
    e_h = 4 if w.htype == "f32" else 2
    e_w = e[w.wtype]
    r = w.rank if rank is None else rank
    mats = 3 if w.gated else 2
    n_list = w.n_hot + n_active
    pred = (r * w.d + w.n_cold * r) * e_p + 4 * w.n_cold                   # P1, P2, bp
    ffn = mats * n_list * w.d * e_w + 4 * n_list                           # rows + b1
    idx = 4 * n_active
    io = batch * w.d * e_h + batch * w.d * 4 + (4 * w.d if (w.has_b2 or not w.gated) else 0)
    return pred + ffn + idx + io


def expected_active(w: Workload, batch: int) -> float:
    """E[|union of cold actives|] under the Zipf model, for planning only."""
    p_rank = zipf_probs(w.ffn, w.alpha, 1.0 - w.sparsity)
    cold = p_rank[w.n_hot:]
    return float(np.sum(1.0 - (1.0 - cold) ** batch))


def make_attention(d: int, n_heads: int, n_hot: int, rank: int, batch: int, s_max: int, seed: int,
                   wtype: str = "f16", ctype: str = "f16", device="cpu") -> dict:
    """Inputs of one head-sparse attention step: Wq, Wk, Wv, WoT [d, d] with
    rows of variance 1/d (head h = rows h*dh .. h*dh+dh-1), caches K, V
    [batch, n_heads, s_max, dh] ~ N(0, 1), and a head predictor built like
    the FFN's (P1 = [V; -V], P2 = [U, -U] for the cold heads, bp = thr), so
    each cold head's score sits around the threshold and about half of them
    are active for a token."""
    g = _gen(device, seed)
    dh = d // n_heads
    wdt = _TORCH_DT[wtype]
    out = {}
    for k in ("Wq", "Wk", "Wv", "WoT"):
        out[k] = (torch.randn(d, d, generator=g, device=device) / math.sqrt(d)).to(wdt).contiguous()
    for k in ("K", "V"):
        out[k] = torch.randn(batch, n_heads, s_max, dh, generator=g, device=device).to(_TORCH_DT[ctype]).contiguous()
    rh = rank // 2
    U = torch.randn(n_heads - n_hot, rh, generator=g, device=device) * math.sqrt(RHO / rh)
    V = torch.randn(rh, d, generator=g, device=device) / math.sqrt(d)
    out["P1"] = torch.cat([V, -V], dim=0).to(torch.float16).contiguous()
    out["P2"] = torch.cat([U, -U], dim=1).to(torch.float16).contiguous() if n_heads > n_hot else None
    out["bp"] = torch.full((n_heads - n_hot,), THRESHOLD, dtype=torch.float32, device=device)
    out["thr"] = THRESHOLD
    return out
