"""ctypes binding of libpi (include/pi.h): argument marshalling only.

Every function takes torch tensors that already live on the CUDA device and
passes their data pointers, sizes and the current CUDA stream to the C ABI.
No arithmetic of the hot path runs here.  If libpi.so is missing the import
fails loudly; there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpi.so")

PI_OK, PI_ERR_INVALID_ARG, PI_ERR_UNSUPPORTED, PI_ERR_CUDA, PI_ERR_CAPACITY, PI_ERR_TIMEOUT, PI_ERR_INDEX = \
    0, -1, -2, -3, -4, -5, -6
STATUS_NAMES = {0: "PI_OK", -1: "PI_ERR_INVALID_ARG", -2: "PI_ERR_UNSUPPORTED", -3: "PI_ERR_CUDA",
                -4: "PI_ERR_CAPACITY", -5: "PI_ERR_TIMEOUT", -6: "PI_ERR_INDEX"}
DTYPES = {"f32": 0, "f16": 1, "q4_0": 2}
ACTS = {"relu": 0, "reglu": 1, "relu2": 2}
MAX_BATCH = 16
TOKEN_FFN = {"warp_mma": 0, "tcgen05": 1}

# Every symbol include/pi.h declares.
EXPORTS = ("pi_workspace_bytes", "pi_workspace_init", "pi_predict", "pi_sparse_ffn", "pi_layer",
           "pi_residual_rmsnorm", "pi_decode_stack", "pi_stack_launches", "pi_set_token_block_ffn",
           "pi_get_token_block_ffn", "pi_get_device_status",
           "pi_attn_workspace_bytes", "pi_sparse_attention", "pi_blocks_workspace_bytes", "pi_decode_blocks",
           "pi_predict_static", "pi_selftest_bounded_wait",
           "pi_last_error", "pi_version")


class FfnDesc(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("ffn", ctypes.c_int32), ("n_hot", ctypes.c_int32),
                ("rank", ctypes.c_int32), ("wtype", ctypes.c_int), ("ptype", ctypes.c_int), ("act", ctypes.c_int)]


class Weight(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


class LayerWeights(ctypes.Structure):
    _fields_ = [("P1", ctypes.c_void_p), ("P2", ctypes.c_void_p), ("bp", ctypes.c_void_p),
                ("W_gate", Weight), ("W_up", Weight), ("W_downT", Weight),
                ("b1", ctypes.c_void_p), ("b2", ctypes.c_void_p), ("threshold", ctypes.c_float),
                ("rank", ctypes.c_int32)]


class AttnDesc(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("n_heads", ctypes.c_int32), ("n_hot", ctypes.c_int32),
                ("s_max", ctypes.c_int32), ("wtype", ctypes.c_int), ("xtype", ctypes.c_int), ("ctype", ctypes.c_int)]


class BlockWeights(ctypes.Structure):
    _fields_ = [("ffn", LayerWeights), ("P1h", ctypes.c_void_p), ("P2h", ctypes.c_void_p), ("bph", ctypes.c_void_p),
                ("Wq", ctypes.c_void_p), ("Wk", ctypes.c_void_p), ("Wv", ctypes.c_void_p), ("WoT", ctypes.c_void_p),
                ("K", ctypes.c_void_p), ("V", ctypes.c_void_p), ("thr_h", ctypes.c_float), ("head_rank", ctypes.c_int32)]


class PiError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__("%s: %s" % (STATUS_NAMES.get(status, status), msg))
        self.status = status


def load(path: str = LIB_PATH):
    if not os.path.exists(path):
        raise ImportError("libpi.so not built (%s); run activation_sparse_decode_predict_b200/build.py" % path)
    lib = ctypes.CDLL(path)
    P, S, i32, f32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_float
    st = ctypes.c_int
    D = ctypes.POINTER(FfnDesc)
    lib.pi_workspace_bytes.argtypes = [D, i32]
    lib.pi_workspace_bytes.restype = S
    lib.pi_workspace_init.argtypes = [P, S, P]
    lib.pi_workspace_init.restype = st
    lib.pi_predict.argtypes = [D, i32, P, P, P, P, f32, P, P, P, S, P]
    lib.pi_predict.restype = st
    lib.pi_sparse_ffn.argtypes = [D, i32, P, P, P, Weight, Weight, Weight, P, P, P, P, S, P]
    lib.pi_sparse_ffn.restype = st
    lib.pi_layer.argtypes = [D, i32, P, ctypes.POINTER(LayerWeights), P, P, P, P, S, P]
    lib.pi_layer.restype = st
    lib.pi_residual_rmsnorm.argtypes = [i32, i32, ctypes.c_int, P, P, f32, P, P]
    lib.pi_residual_rmsnorm.restype = st
    lib.pi_decode_stack.argtypes = [D, i32, i32, ctypes.POINTER(LayerWeights), P, P, P, P, P, P, f32, P, S, P]
    lib.pi_decode_stack.restype = st
    lib.pi_stack_launches.argtypes = [D, i32, i32]
    lib.pi_stack_launches.restype = i32
    lib.pi_set_token_block_ffn.argtypes = [i32]
    lib.pi_set_token_block_ffn.restype = ctypes.c_int
    lib.pi_get_token_block_ffn.argtypes = []
    lib.pi_get_token_block_ffn.restype = i32
    lib.pi_get_device_status.argtypes = [P, ctypes.POINTER(ctypes.c_int32), i32, P]
    lib.pi_get_device_status.restype = st
    A = ctypes.POINTER(AttnDesc)
    lib.pi_attn_workspace_bytes.argtypes = [A, i32]
    lib.pi_attn_workspace_bytes.restype = S
    lib.pi_sparse_attention.argtypes = [A, i32, P, P, P, P, P, P, P, P, P, i32, P, P, S, P]
    lib.pi_sparse_attention.restype = st
    lib.pi_blocks_workspace_bytes.argtypes = [D, A, i32]
    lib.pi_blocks_workspace_bytes.restype = S
    lib.pi_decode_blocks.argtypes = [D, A, i32, i32, ctypes.POINTER(BlockWeights), P, P, i32, P, P, P, P, P, f32, P,
                                     S, P]
    lib.pi_decode_blocks.restype = st
    lib.pi_predict_static.argtypes = [D, i32, P, P, P, P, f32, P, P, P]
    lib.pi_predict_static.restype = st
    lib.pi_selftest_bounded_wait.argtypes = [P, i32, P]
    lib.pi_selftest_bounded_wait.restype = st
    lib.pi_last_error.restype = ctypes.c_char_p
    lib.pi_version.restype = ctypes.c_char_p
    return lib
