"""libpi loads on a machine without a GPU, exports every symbol include/pi.h
declares, and rejects bad arguments on the host before launching anything."""
import ctypes
import os
import re

import pytest

import activation_sparse_decode_predict_b200 as pi
from activation_sparse_decode_predict_b200 import _binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "pi.h"), encoding="utf-8").read()
    return sorted(set(re.findall(r"PI_API\s+[\w\s\*]+?\b(pi_\w+)\s*\(", src)))


def test_header_declares_the_binding_exports():
    assert _declared() == sorted(B.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = pi.lib()
    for name in _declared():
        assert hasattr(lib, name), name
    assert pi.version().count(".") == 2


def _desc(**kw):
    base = dict(d=4096, ffn=11008, n_hot=1101, rank=1024, wtype="f16", ptype="f16", act="reglu")
    base.update(kw)
    return pi.make_desc(**base)


def test_workspace_bytes_is_host_only_and_grows_with_batch():
    n1 = pi.workspace_bytes(_desc(), 1)
    n16 = pi.workspace_bytes(_desc(), 16)
    assert 0 < n1 < n16
    assert n1 % 256 == 0


@pytest.mark.parametrize("kw,batch", [
    (dict(d=4100), 1),            # d % 8
    (dict(ffn=0), 1),
    (dict(n_hot=-1), 1),
    (dict(n_hot=20000), 1),       # n_hot > ffn
    (dict(rank=1020), 1),         # rank % 8
    (dict(wtype="q4_0", d=4104), 1),  # Q4_0 needs d % 32
    ({}, 0),
    ({}, 17),
])
def test_invalid_descriptors_are_rejected(kw, batch):
    lib = pi.lib()
    assert lib.pi_workspace_bytes(ctypes.byref(_desc(**kw)), batch) == 0
    assert lib.pi_last_error()


def test_bad_pointers_fail_before_any_launch():
    lib = pi.lib()
    d = _desc()
    fake = ctypes.c_void_p(1 << 20)        # aligned, never dereferenced: every call below fails first
    mis = ctypes.c_void_p((1 << 20) + 4)   # misaligned for 16-byte tensors
    P = ctypes.c_void_p
    # NULL h
    st = lib.pi_predict(ctypes.byref(d), 1, None, fake, fake, None, 0.5, fake, fake, fake, 1 << 40, None)
    assert st == B.PI_ERR_INVALID_ARG and b"h" in lib.pi_last_error()
    # misaligned P1
    st = lib.pi_predict(ctypes.byref(d), 1, fake, mis, fake, None, 0.5, fake, fake, fake, 1 << 40, None)
    assert st == B.PI_ERR_INVALID_ARG
    # workspace too small
    st = lib.pi_predict(ctypes.byref(d), 1, fake, fake, fake, None, 0.5, fake, fake, fake, 1024, None)
    assert st == B.PI_ERR_CAPACITY
    # NULL desc
    st = lib.pi_predict(None, 1, fake, fake, fake, None, 0.5, fake, fake, fake, 1 << 40, None)
    assert st == B.PI_ERR_INVALID_ARG
    # sparse FFN: Q4_0 without scales
    dq = _desc(wtype="q4_0", d=4096)
    w = B.Weight(fake, None)
    st = lib.pi_sparse_ffn(ctypes.byref(dq), 1, fake, fake, fake, w, w, w, None, None, fake, fake, 1 << 40, None)
    assert st == B.PI_ERR_INVALID_ARG and b"scales" in lib.pi_last_error()
    # ReGLU needs W_gate
    w0 = B.Weight(None, None)
    wf = B.Weight(fake, None)
    st = lib.pi_sparse_ffn(ctypes.byref(d), 1, fake, fake, fake, w0, wf, wf, None, None, fake, fake, 1 << 40, None)
    assert st == B.PI_ERR_INVALID_ARG and b"W_gate" in lib.pi_last_error()
    # rmsnorm: bad batch / eps
    assert lib.pi_residual_rmsnorm(0, 64, 1, fake, fake, 1e-6, fake, None) == B.PI_ERR_INVALID_ARG
    assert lib.pi_residual_rmsnorm(1, 64, 1, fake, fake, -1.0, fake, None) == B.PI_ERR_INVALID_ARG
    # decode stack: aliasing output and too many layers
    arr = (B.LayerWeights * 1)()
    st = lib.pi_decode_stack(ctypes.byref(d), 1, 1, arr, fake, fake, fake, fake, None, None, 1e-6, fake, 1 << 40,
                             None)
    assert st == B.PI_ERR_INVALID_ARG and b"alias" in lib.pi_last_error()
    st = lib.pi_decode_stack(ctypes.byref(d), 1, 129, arr, fake, P(2 << 20), fake, fake, None, None, 1e-6, fake,
                             1 << 40, None)
    assert st == B.PI_ERR_INVALID_ARG
    # status read needs an output pointer
    assert lib.pi_get_device_status(fake, None, 0, None) == B.PI_ERR_INVALID_ARG


def test_python_layer_refuses_cpu_tensors():
    import torch
    d = _desc(d=64, ffn=100, n_hot=10, rank=8)
    with pytest.raises(ValueError, match="CUDA"):
        pi.residual_rmsnorm(torch.zeros(1, 64), torch.zeros(1, 64), 1e-6, torch.zeros(1, 64))


def test_launch_plan_is_host_only():
    """pi_stack_launches plans a decode step without a GPU: one persistent
    launch for token blocks of 1-2 on every workload shape; for token blocks of
    3-16 an fp16 predictor runs on the tensor cores (P1 and P2 row dots,
    threshold, compaction), the FFN on the warp-level kernels (gate/up row
    dots, down, reduce) or, when chosen, fp16 weights (d % 256 == 0) on the
    tcgen05 kernels (up with the activation, down with the reduction), then
    the glue: 8 per layer (7 on tcgen05; 8 with Q4_0 weights); a shape the
    persistent kernel does not take runs the CUDA-core kernels (u, scores,
    compaction; gate/up, down, reduce; glue: 7 per layer, 5 with no cold
    neurons); -1 for invalid arguments."""
    import pi_workload as W
    lib = pi.lib()
    for w in W.WORKLOADS.values():
        desc = pi.desc_for(w)
        for batch in (1, 2):
            assert lib.pi_stack_launches(ctypes.byref(desc), batch, w.layers) == 1, (w.name, batch)
        pred = 4 if w.ptype == "f16" else 3
        for path in ("warp_mma", "tcgen05"):
            pi.set_token_block_ffn(path)
            ffn = 2 if (path == "tcgen05" and w.wtype == "f16" and w.ptype == "f16") else 3
            for batch in (3, 8, 16):
                want = (pred + ffn + 1) * w.layers
                assert lib.pi_stack_launches(ctypes.byref(desc), batch, w.layers) == want, (w.name, batch, path)
        pi.set_token_block_ffn("warp_mma")
    odd = _desc(d=520, ffn=2048, n_hot=103, rank=64, act="relu")  # d not a multiple of 256
    assert lib.pi_stack_launches(ctypes.byref(odd), 1, 4) == 28
    all_hot = _desc(d=512, ffn=2048, n_hot=2048, rank=64, act="relu", wtype="f32", ptype="f32")
    assert lib.pi_stack_launches(ctypes.byref(all_hot), 3, 4) == 20
    assert lib.pi_stack_launches(ctypes.byref(_desc()), 1, 0) == -1
    assert lib.pi_stack_launches(ctypes.byref(_desc()), 0, 4) == -1
    assert lib.pi_stack_launches(ctypes.byref(_desc(d=100)), 1, 4) == -1


def test_static_predict_checks_like_predict_before_any_launch():
    """pi_predict_static applies pi_predict's descriptor and pointer checks
    (same alignments: h, P1, P2 16 bytes; bp, idx, count 4 bytes) and returns
    before touching the device.  The addresses are never dereferenced: every
    call here fails on the host."""
    lib = pi.lib()
    d = _desc(d=512, ffn=2048, n_hot=100, rank=64)
    fake = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 2)   # not 4-byte aligned
    mis16 = ctypes.c_void_p((1 << 20) + 4)  # 4- but not 16-byte aligned

    def call(desc=d, batch=1, h=fake, P1=fake, P2=fake, bp=None, idx=fake, count=fake):
        return lib.pi_predict_static(ctypes.byref(desc) if desc is not None else None, batch, h, P1, P2, bp, 0.5,
                                     idx, count, None)

    assert call(bp=odd) == B.PI_ERR_INVALID_ARG and b"bp" in lib.pi_last_error()
    assert call(count=odd) == B.PI_ERR_INVALID_ARG and b"count" in lib.pi_last_error()
    assert call(idx=odd) == B.PI_ERR_INVALID_ARG and b"idx" in lib.pi_last_error()
    assert call(h=mis16) == B.PI_ERR_INVALID_ARG and b"h" in lib.pi_last_error()
    assert call(P2=mis16) == B.PI_ERR_INVALID_ARG and b"P2" in lib.pi_last_error()
    assert call(desc=None) == B.PI_ERR_INVALID_ARG
    assert call(batch=17) == B.PI_ERR_INVALID_ARG
    # the limits pi_predict enforces through its descriptor check
    assert call(desc=_desc(d=16392, ffn=2048, n_hot=100, rank=64)) == B.PI_ERR_UNSUPPORTED
    assert call(desc=_desc(d=512, ffn=2048, n_hot=100, rank=65544)) == B.PI_ERR_UNSUPPORTED
    bad_act = _desc(d=512, ffn=2048, n_hot=100, rank=64)
    bad_act.act = 7
    assert call(desc=bad_act) == B.PI_ERR_INVALID_ARG


def test_sparse_attention_checks_before_any_launch():
    """pi_sparse_attention's descriptor, length and pointer checks run on the
    host; the fake addresses below are never dereferenced."""
    lib = pi.lib()
    fake = ctypes.c_void_p(1 << 20)
    good = pi.attn_desc(4096, 32, 4, 512)
    assert lib.pi_attn_workspace_bytes(ctypes.byref(good), 1) > 0
    assert lib.pi_attn_workspace_bytes(ctypes.byref(good), 17) == 0

    def call(desc, length=10, x=fake, hidx=fake, y=fake, ws_bytes=1 << 40):
        return lib.pi_sparse_attention(ctypes.byref(desc), 1, x, hidx, fake, fake, fake, fake, fake, fake, fake,
                                       length, y, fake, ws_bytes, None)

    assert call(pi.attn_desc(96, 2, 0, 16)) == B.PI_ERR_UNSUPPORTED          # head dimension 48
    assert call(pi.attn_desc(4096, 3, 0, 16)) == B.PI_ERR_INVALID_ARG        # 3 does not divide 4096
    assert call(pi.attn_desc(512, 4, 0, 16, "f16", "f32")) == B.PI_ERR_UNSUPPORTED  # fp32 tokens, fp16 weights
    assert call(good, length=512) == B.PI_ERR_INVALID_ARG                    # len must be < s_max
    assert call(good, length=-1) == B.PI_ERR_INVALID_ARG
    assert call(good, x=ctypes.c_void_p((1 << 20) + 8)) == B.PI_ERR_INVALID_ARG and b"x" in lib.pi_last_error()
    assert call(good, hidx=None) == B.PI_ERR_INVALID_ARG and b"head_idx" in lib.pi_last_error()
    assert call(good, ws_bytes=4096) == B.PI_ERR_CAPACITY


def test_token_block_ffn_switch():
    """The token-block FFN kernels are chosen process-wide; warp_mma is the
    default, any other value than the two paths is refused."""
    lib = pi.lib()
    assert pi.token_block_ffn() == "warp_mma"
    pi.set_token_block_ffn("tcgen05")
    assert lib.pi_get_token_block_ffn() == 1
    assert lib.pi_set_token_block_ffn(7) == B.PI_ERR_INVALID_ARG
    assert pi.token_block_ffn() == "tcgen05"
    pi.set_token_block_ffn("warp_mma")
    assert lib.pi_get_token_block_ffn() == 0
    with pytest.raises(ValueError):
        pi.set_token_block_ffn("cuda_cores")
