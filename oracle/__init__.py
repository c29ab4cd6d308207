"""CPU oracle for the activation-sparse decode FFN (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports it.

The arithmetic lives in ``pi_oracle.c`` (plain C, IEEE double, ascending
summation order); this module compiles it with gcc on first use and marshals
numpy arrays into it.  See the header of ``pi_oracle.c`` for the definitions
and the pages each function follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pi_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

WTYPES = {"f32": 0, "f16": 1, "q4_0": 2}
ACTS = {"relu": 0, "reglu": 1, "relu2": 2}


def build(force: bool = False) -> str:
    """Compile pi_oracle.c into liboracle.so (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _bind(path: str):
    """Load a compiled oracle library and declare its C signatures."""
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
    lib.orc_half_to_double.argtypes = [ctypes.c_uint16]
    lib.orc_half_to_double.restype = f64
    lib.orc_elem.argtypes = [i32, P, P, i64, i64, i64]
    lib.orc_elem.restype = f64
    lib.orc_predict.argtypes = [i32, i32, i32, i32, i32, i32, i32, P, P, P, P, P, P, f64, P, P, P, P]
    lib.orc_predict.restype = i64
    lib.orc_masked_ffn.argtypes = [i32, i32, i32, i32, i32, i32, i32, P, P, i64, P, P, P, P, P, P, P, P,
                                   P, i32, P, P]
    lib.orc_masked_ffn.restype = None
    lib.orc_true_support.argtypes = [i32, i32, i32, i32, i32, i32, P, P, P, P, P, P, P]
    lib.orc_true_support.restype = None
    lib.orc_attention.argtypes = [i32, i32, i32, i32, i32, i32, i32, P, P, i64, P, P, P, P, P, P, i32, i32, P, P,
                                  P]
    lib.orc_attention.restype = None
    lib.orc_residual_rmsnorm.argtypes = [i32, i32, i32, P, P, f64, P]
    lib.orc_residual_rmsnorm.restype = None
    lib.orc_set_threads.argtypes = [i32]
    lib.orc_get_threads.restype = i32
    return lib


_override = None


def _load():
    global _lib
    if _override is not None:
        return _override
    with _lock:
        if _lib is None:
            _lib = _bind(build())
    return _lib


class use_library:
    """Context manager: route this module's functions to another compiled
    oracle (the tests use it to check that the pins reject planted mistakes)."""

    def __init__(self, path: str):
        self.lib = _bind(path)

    def __enter__(self):
        global _override
        self._prev = _override
        _override = self.lib
        return self

    def __exit__(self, *exc):
        global _override
        _override = self._prev
        return False


def _ptr(a):
    if a is None:
        return None
    assert isinstance(a, np.ndarray) and a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous numpy arrays"
    return a.ctypes.data


def _htype(h: np.ndarray) -> int:
    if h.dtype == np.float32:
        return WTYPES["f32"]
    if h.dtype == np.float16:
        return WTYPES["f16"]
    raise TypeError("token block must be float32 or float16, got %s" % h.dtype)


def _wtype_of(w) -> int:
    if isinstance(w, tuple):
        return WTYPES["q4_0"]
    return _htype(w)


def _wparts(w):
    """A weight is an fp32/fp16 array [rows, d] or a Q4_0 pair (qs uint8 [rows, d/2], sc float16 [rows, d/32])."""
    if w is None:
        return None, None
    if isinstance(w, tuple):
        qs, sc = w
        assert qs.dtype == np.uint8 and sc.dtype == np.float16
        return qs, sc
    return w, None


def set_threads(n: int) -> None:
    _load().orc_set_threads(int(n))


def get_threads() -> int:
    return int(_load().orc_get_threads())


def half_to_double(bits: int) -> float:
    return float(_load().orc_half_to_double(int(bits) & 0xFFFF))


def decode_matrix(w, d: int) -> np.ndarray:
    """Decode a whole weight matrix to float64 through the oracle's element decoder."""
    lib = _load()
    data, sc = _wparts(w)
    rows = data.shape[0]
    t = _wtype_of(w)
    out = np.empty((rows, d), dtype=np.float64)
    for r in range(rows):
        for c in range(d):
            out[r, c] = lib.orc_elem(t, _ptr(data), _ptr(sc), r, c, d)
    return out


def predict(h, P1, P2, bp, thr, n_hot: int, ffn: int):
    """Returns dict(u [B,r], s [B,C], mask [C] uint8, idx int32 ascending).

    P1 [r, d] and P2 [C, r] are fp32/fp16 arrays, or Q4_0 pairs (qs uint8
    [rows, cols/2], sc float16 [rows, cols/32]) with blocks along d (P1) and
    along the rank (P2)."""
    lib = _load()
    h = np.ascontiguousarray(h)
    B, d = h.shape
    p1, p1_sc = _wparts(P1)
    p2, p2_sc = _wparts(P2)
    q4 = isinstance(P1, tuple)
    r = p1.shape[0]
    C = ffn - n_hot
    assert p1.shape == ((r, d // 2) if q4 else (r, d))
    assert P2 is None and C == 0 or p2.shape == ((C, r // 2) if q4 else (C, r))
    assert (P2 is None) or isinstance(P2, tuple) == q4
    u = np.empty((B, r), np.float64)
    s = np.empty((B, C), np.float64)
    mask = np.empty((C,), np.uint8)
    idx = np.empty((max(C, 1),), np.int32)
    bp_ = None if bp is None else np.ascontiguousarray(bp, dtype=np.float32)
    n = lib.orc_predict(d, ffn, n_hot, r, _htype(h), _wtype_of(P1), B, _ptr(h), _ptr(p1), _ptr(p1_sc), _ptr(p2),
                        _ptr(p2_sc), _ptr(bp_), float(thr), _ptr(u), _ptr(s), _ptr(mask), _ptr(idx))
    return {"u": u, "s": s, "mask": mask, "idx": idx[:n].copy()}


def masked_ffn(h, idx, Wg, Wu, WdT, b1, b2, act: str, n_hot: int, ffn: int, cols=None, want_a: bool = False):
    """y [B, d] (or [B, len(cols)]) of the FFN over the list [0, n_hot) ++ idx, in float64."""
    lib = _load()
    h = np.ascontiguousarray(h)
    B, d = h.shape
    idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
    wg, wg_sc = _wparts(Wg)
    wu, wu_sc = _wparts(Wu)
    wd, wd_sc = _wparts(WdT)
    wt = _wtype_of(Wu)
    if act == "reglu":
        assert Wg is not None and _wtype_of(Wg) == wt
    assert _wtype_of(WdT) == wt
    cols_ = None if cols is None else np.ascontiguousarray(np.asarray(cols, dtype=np.int32))
    n_out = d if cols_ is None else len(cols_)
    y = np.empty((B, n_out), np.float64)
    n_list = n_hot + len(idx)
    a = np.empty((B, max(n_list, 1)), np.float64) if want_a else None
    b1_ = None if b1 is None else np.ascontiguousarray(b1, dtype=np.float32)
    b2_ = None if b2 is None else np.ascontiguousarray(b2, dtype=np.float32)
    lib.orc_masked_ffn(d, ffn, n_hot, wt, ACTS[act], _htype(h), B, _ptr(h), _ptr(idx), len(idx), _ptr(wg),
                       _ptr(wg_sc), _ptr(wu), _ptr(wu_sc), _ptr(wd), _ptr(wd_sc), _ptr(b1_), _ptr(b2_), _ptr(cols_),
                       n_out, _ptr(y), _ptr(a))
    if want_a:
        return y, a[:, :n_list]
    return y


def dense_ffn(h, Wg, Wu, WdT, b1, b2, act: str, n_hot: int, ffn: int, cols=None):
    """The dense FFN: the masked FFN with every cold neuron listed (same routine, same order)."""
    return masked_ffn(h, np.arange(n_hot, ffn, dtype=np.int32), Wg, Wu, WdT, b1, b2, act, n_hot, ffn, cols)


def true_support(h, Wg, Wu, b1, act: str, ffn: int) -> np.ndarray:
    """support [B, ffn] uint8: the (gate for ReGLU, else up) pre-activation incl. b1 is > 0."""
    lib = _load()
    h = np.ascontiguousarray(h)
    B, d = h.shape
    wg, wg_sc = _wparts(Wg)
    wu, wu_sc = _wparts(Wu)
    out = np.empty((B, ffn), np.uint8)
    b1_ = None if b1 is None else np.ascontiguousarray(b1, dtype=np.float32)
    lib.orc_true_support(d, ffn, _wtype_of(Wu), ACTS[act], _htype(h), B, _ptr(h), _ptr(wg), _ptr(wg_sc), _ptr(wu),
                         _ptr(wu_sc), _ptr(b1_), _ptr(out))
    return out


def attention(x, idx, Wq, Wk, Wv, WoT, K, V, length: int, n_heads: int, n_hot: int):
    """Head-sparse decode attention over the heads [0, n_hot) ++ idx: dict(y [B, d],
    k [B, n_list, dh], v [B, n_list, dh]) in float64.  K, V: caches [B, n_heads, s_max, dh]."""
    lib = _load()
    x = np.ascontiguousarray(x)
    B, d = x.shape
    idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
    K = np.ascontiguousarray(K)
    V = np.ascontiguousarray(V)
    assert K.shape == V.shape and K.shape[0] == B and K.shape[1] == n_heads and K.shape[3] == d // n_heads
    assert 0 <= length <= K.shape[2]
    wt = _htype(Wq)
    for w in (Wk, Wv, WoT):
        assert _htype(w) == wt and w.shape == (d, d)
    n_list = n_hot + len(idx)
    dh = d // n_heads
    y = np.empty((B, d), np.float64)
    k = np.empty((B, max(n_list, 1), dh), np.float64)
    v = np.empty((B, max(n_list, 1), dh), np.float64)
    lib.orc_attention(d, n_heads, n_hot, wt, _htype(x), _htype(K), B, _ptr(x), _ptr(idx), len(idx), _ptr(Wq),
                      _ptr(Wk), _ptr(Wv), _ptr(WoT), _ptr(K), _ptr(V), K.shape[2], int(length), _ptr(y), _ptr(k),
                      _ptr(v))
    return {"y": y, "k": k[:, :n_list], "v": v[:, :n_list]}


def residual_rmsnorm(h, y, eps: float) -> np.ndarray:
    """x = h + y; x / sqrt(mean(x^2) + eps), per token, float64."""
    lib = _load()
    h = np.ascontiguousarray(h)
    B, d = h.shape
    y = np.ascontiguousarray(y, dtype=np.float64)
    out = np.empty((B, d), np.float64)
    lib.orc_residual_rmsnorm(B, d, _htype(h), _ptr(h), _ptr(y), float(eps), _ptr(out))
    return out
