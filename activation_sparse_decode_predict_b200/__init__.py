"""Activation-sparse decode FFN for NVIDIA B200 (sm_100a).

Python face of libpi (include/pi.h).  The functions here only marshal torch
CUDA tensors into the C ABI: every step of the hot path runs in the library's
CUDA kernels.  There is no CPU path and no fallback: without the built
library, or without a CUDA device, the calls raise.

Pages: unite.ai "PowerInfer: Tüketici Düzeyinde bir GPU ile Hızlı Büyük Dil
Modeli Sunucusu" ("Adaptif Sparsite Predictor’ları", "Nöron Bilinçli
Operatör", "Nöron Yerleştirme ve Yönetimi"); GeekNews "Serving model bahasa
besar berkecepatan tinggi pada PC dengan GPU konsumen" ("Keterbatasan dan
FAQ", "Kuantisasi dan kompatibilitas").
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence, Tuple, Union

import torch

from . import _binding as _b
from ._binding import (ACTS, DTYPES, EXPORTS, MAX_BATCH, AttnDesc, BlockWeights, FfnDesc, LayerWeights, PiError,
                       Weight)

_lib = None

WeightT = Union[torch.Tensor, Tuple[torch.Tensor, torch.Tensor]]


def lib():
    """The loaded libpi (raises ImportError if it was not built)."""
    global _lib
    if _lib is None:
        _lib = _b.load()
    return _lib


def _check(status: int) -> None:
    if status != 0:
        raise PiError(status, lib().pi_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch tensor, got %r" % type(t))
    if not t.is_cuda:
        raise ValueError("libpi takes CUDA tensors only (got a %s tensor)" % t.device)
    if not t.is_contiguous():
        raise ValueError("libpi takes contiguous tensors only")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def make_desc(d: int, ffn: int, n_hot: int, rank: int, wtype: str, ptype: str, act: str) -> FfnDesc:
    return FfnDesc(d, ffn, n_hot, rank, DTYPES[wtype], DTYPES[ptype], ACTS[act])


def desc_for(w) -> FfnDesc:
    """Descriptor of a pi_workload.Workload."""
    return make_desc(w.d, w.ffn, w.n_hot, w.rank, w.wtype, w.ptype, w.act)


def workspace_bytes(desc: FfnDesc, batch: int) -> int:
    n = lib().pi_workspace_bytes(ctypes.byref(desc), int(batch))
    if n == 0:
        raise PiError(_b.PI_ERR_INVALID_ARG, lib().pi_last_error().decode())
    return int(n)


def workspace(desc: FfnDesc, batch: int, device=None, stream=None) -> torch.Tensor:
    """A zero-initialised workspace tensor (allocated by torch, not by libpi)."""
    n = workspace_bytes(desc, batch)
    ws = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
    _check(lib().pi_workspace_init(_ptr(ws), n, _stream(stream)))
    return ws


def weight(w: Optional[WeightT]) -> Weight:
    if w is None:
        return Weight(None, None)
    if isinstance(w, tuple):
        return Weight(_ptr(w[0]), _ptr(w[1]))
    return Weight(_ptr(w), None)


def _pred_ptr(P):
    """Device pointer of a predictor matrix: a tensor, or a Q4_0 pair (codes,
    scales) whose scales follow its codes in one buffer (the C ABI's layout)."""
    if isinstance(P, tuple):
        qs, sc = P
        if sc.data_ptr() != qs.data_ptr() + qs.numel():
            raise ValueError("Q4_0 predictor scales must follow its codes in the same buffer")
        return _ptr(qs)
    return _ptr(P)


def layer_weights(L: dict) -> LayerWeights:
    """pi_layer_weights from a dict with keys P1, P2, bp, Wg, Wu, WdT, b1, b2,
    thr and optionally rank (this layer's predictor rank; 0 = the descriptor's)."""
    return LayerWeights(_pred_ptr(L["P1"]), _pred_ptr(L["P2"]), _ptr(L.get("bp")), weight(L.get("Wg")),
                        weight(L["Wu"]), weight(L["WdT"]), _ptr(L.get("b1")), _ptr(L.get("b2")), float(L["thr"]),
                        int(L.get("rank", 0)))


def predict(desc: FfnDesc, h: torch.Tensor, P1, P2, bp, threshold: float, idx: torch.Tensor, count: torch.Tensor,
            ws: torch.Tensor, stream=None) -> None:
    _check(lib().pi_predict(ctypes.byref(desc), h.shape[0], _ptr(h), _pred_ptr(P1), _pred_ptr(P2), _ptr(bp),
                            float(threshold),
                            _ptr(idx), _ptr(count), _ptr(ws), ws.numel(), _stream(stream)))


def sparse_ffn(desc: FfnDesc, h: torch.Tensor, idx: torch.Tensor, count: torch.Tensor, Wg: Optional[WeightT],
               Wu: WeightT, WdT: WeightT, b1, b2, y: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    _check(lib().pi_sparse_ffn(ctypes.byref(desc), h.shape[0], _ptr(h), _ptr(idx), _ptr(count), weight(Wg),
                               weight(Wu), weight(WdT), _ptr(b1), _ptr(b2), _ptr(y), _ptr(ws), ws.numel(),
                               _stream(stream)))


def layer(desc: FfnDesc, h: torch.Tensor, lw: LayerWeights, idx: torch.Tensor, count: torch.Tensor,
          y: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    _check(lib().pi_layer(ctypes.byref(desc), h.shape[0], _ptr(h), ctypes.byref(lw), _ptr(idx), _ptr(count), _ptr(y),
                          _ptr(ws), ws.numel(), _stream(stream)))


def residual_rmsnorm(h: torch.Tensor, y: torch.Tensor, eps: float, h_out: torch.Tensor, stream=None) -> None:
    ht = {torch.float32: 0, torch.float16: 1}[h.dtype]
    _check(lib().pi_residual_rmsnorm(h.shape[0], h.shape[1], ht, _ptr(h), _ptr(y), float(eps), _ptr(h_out),
                                     _stream(stream)))


def layer_array(layers: Sequence[LayerWeights]):
    arr = (LayerWeights * len(layers))(*layers)
    return arr


def decode_stack(desc: FfnDesc, layers, h_in: torch.Tensor, h_out: torch.Tensor, idx: torch.Tensor,
                 counts: torch.Tensor, y: Optional[torch.Tensor], eps: float, ws: torch.Tensor,
                 h_trace: Optional[torch.Tensor] = None, stream=None) -> None:
    """One decode step through len(layers) layers (layers: a ctypes array from layer_array, host memory)."""
    _check(lib().pi_decode_stack(ctypes.byref(desc), h_in.shape[0], len(layers), layers, _ptr(h_in), _ptr(h_out),
                                 _ptr(idx), _ptr(counts), _ptr(y), _ptr(h_trace), float(eps), _ptr(ws), ws.numel(),
                                 _stream(stream)))


def set_token_block_ffn(path: str) -> None:
    """Kernels for the sparse FFN of token blocks of 3-16 (fp16 weights):
    "warp_mma" (row dots on warp-level mma.sync, the default) or "tcgen05"
    (gathered tiles on the fifth-generation tensor cores).  Process-wide."""
    if path not in _b.TOKEN_FFN:
        raise ValueError("path must be one of %s" % sorted(_b.TOKEN_FFN))
    _check(lib().pi_set_token_block_ffn(_b.TOKEN_FFN[path]))


def token_block_ffn() -> str:
    """The current token-block FFN kernels ("warp_mma" or "tcgen05")."""
    v = lib().pi_get_token_block_ffn()
    return {i: k for k, i in _b.TOKEN_FFN.items()}[v]


def stack_launches(desc: FfnDesc, batch: int, n_layers: int) -> int:
    n = lib().pi_stack_launches(ctypes.byref(desc), int(batch), int(n_layers))
    if n < 0:
        raise PiError(_b.PI_ERR_INVALID_ARG, "invalid stack arguments")
    return int(n)


def device_status(ws: torch.Tensor, clear: bool = False, stream=None) -> int:
    v = ctypes.c_int32(0)
    _check(lib().pi_get_device_status(_ptr(ws), ctypes.byref(v), int(bool(clear)), _stream(stream)))
    return int(v.value)


def selftest_bounded_wait(ws: torch.Tensor, kind: int, stream=None) -> None:
    """Launch a wait that can only time out (kind 0: mbarrier, 1: grid barrier)."""
    _check(lib().pi_selftest_bounded_wait(_ptr(ws), int(kind), _stream(stream)))


def attn_desc(d: int, n_heads: int, n_hot: int, s_max: int, wtype: str = "f16", xtype: str = "f16",
              ctype: str = "f16") -> AttnDesc:
    return AttnDesc(d, n_heads, n_hot, s_max, DTYPES[wtype], DTYPES[xtype], DTYPES[ctype])


def attn_workspace(desc: AttnDesc, batch: int, device=None, stream=None) -> torch.Tensor:
    """A zero-initialised workspace for pi_sparse_attention (allocated by torch)."""
    n = lib().pi_attn_workspace_bytes(ctypes.byref(desc), int(batch))
    if n == 0:
        raise PiError(_b.PI_ERR_INVALID_ARG, lib().pi_last_error().decode())
    ws = torch.empty(int(n), dtype=torch.uint8, device=device or "cuda")
    _check(lib().pi_workspace_init(_ptr(ws), int(n), _stream(stream)))
    return ws


def sparse_attention(desc: AttnDesc, x: torch.Tensor, head_idx, head_count: torch.Tensor, Wq, Wk, Wv, WoT,
                     K: torch.Tensor, V: torch.Tensor, length: int, y: torch.Tensor, ws: torch.Tensor,
                     stream=None) -> None:
    """One decode step of the self-attention block over the listed heads (pi_sparse_attention)."""
    _check(lib().pi_sparse_attention(ctypes.byref(desc), x.shape[0], _ptr(x), _ptr(head_idx), _ptr(head_count),
                                     _ptr(Wq), _ptr(Wk), _ptr(Wv), _ptr(WoT), _ptr(K), _ptr(V), int(length), _ptr(y),
                                     _ptr(ws), ws.numel(), _stream(stream)))


def block_weights(L: dict, A: dict, head_rank: int) -> BlockWeights:
    """pi_block_weights from an FFN layer dict (layer_weights) and an attention
    dict with keys P1, P2, bp, thr (head predictor), Wq, Wk, Wv, WoT, K, V."""
    return BlockWeights(layer_weights(L), _pred_ptr(A["P1"]), _pred_ptr(A.get("P2")), _ptr(A.get("bp")), _ptr(A["Wq"]),
                        _ptr(A["Wk"]), _ptr(A["Wv"]), _ptr(A["WoT"]), _ptr(A["K"]), _ptr(A["V"]), float(A["thr"]),
                        int(head_rank))


def blocks_workspace(fdesc: FfnDesc, adesc: AttnDesc, batch: int, device=None, stream=None) -> torch.Tensor:
    n = lib().pi_blocks_workspace_bytes(ctypes.byref(fdesc), ctypes.byref(adesc), int(batch))
    if n == 0:
        raise PiError(_b.PI_ERR_INVALID_ARG, lib().pi_last_error().decode())
    ws = torch.empty(int(n), dtype=torch.uint8, device=device or "cuda")
    _check(lib().pi_workspace_init(_ptr(ws), int(n), _stream(stream)))
    return ws


def decode_blocks(fdesc: FfnDesc, adesc: AttnDesc, blocks, h_in: torch.Tensor, h_out: torch.Tensor, length: int,
                  head_idx: torch.Tensor, head_counts: torch.Tensor, idx: torch.Tensor, counts: torch.Tensor,
                  eps: float, ws: torch.Tensor, trace: Optional[torch.Tensor] = None, stream=None) -> None:
    """One decode step through len(blocks) attention + FFN blocks (blocks: a ctypes array of BlockWeights)."""
    _check(lib().pi_decode_blocks(ctypes.byref(fdesc), ctypes.byref(adesc), h_in.shape[0], len(blocks), blocks,
                                  _ptr(h_in), _ptr(h_out), int(length), _ptr(head_idx), _ptr(head_counts), _ptr(idx),
                                  _ptr(counts), _ptr(trace), float(eps), _ptr(ws), ws.numel(), _stream(stream)))


def version() -> str:
    return lib().pi_version().decode()
