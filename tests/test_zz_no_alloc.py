"""pi_predict_static: the predictor for callers that cannot allocate device
memory (hosts that give the library only its inputs and outputs).  Its
scratch is a fixed 1 MiB array inside libpi; it must give the same active
lists as pi_predict with a caller workspace, call after call."""
import ctypes

import numpy as np
import pytest
import torch

import activation_sparse_decode_predict_b200 as pi
import pi_workload as W
from activation_sparse_decode_predict_b200 import _binding as B

pytestmark = pytest.mark.gpu


def _static_predict(lib, desc, h, L, idx, count):
    st = lib.pi_predict_static(ctypes.byref(desc), h.shape[0], h.data_ptr(), L["P1"].data_ptr(),
                               L["P2"].data_ptr(), L["bp"].data_ptr(), float(L["thr"]), idx.data_ptr(),
                               count.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == B.PI_OK, lib.pi_last_error()


def test_static_scratch_predict_matches_workspace_predict_twice():
    lib = pi.lib()
    wl = W.Workload("noalloc", 91, 1024, 3000, 1, "reglu", "f16", "f16", 0.88, 1.2, 0.1, 128, (2,), 2)
    L = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in W.make_layer(wl, 0).items()}
    desc = pi.desc_for(wl)
    ws = pi.workspace(desc, 2)
    C = wl.n_cold
    for step in range(2):                      # two calls in a row, different token blocks
        h = W.make_tokens(wl, 2, 50 + step, device="cuda")
        idx_ref = torch.full((C,), -1, dtype=torch.int32, device="cuda")
        cnt_ref = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        pi.predict(desc, h, L["P1"], L["P2"], L["bp"], L["thr"], idx_ref, cnt_ref, ws)
        idx = torch.full((C,), -2, dtype=torch.int32, device="cuda")
        cnt = torch.full((1,), -2, dtype=torch.int32, device="cuda")
        _static_predict(lib, desc, h, L, idx, cnt)
        torch.cuda.synchronize()
        n = int(cnt_ref.item())
        assert 0 < n < C
        assert int(cnt.item()) == n
        assert torch.equal(idx[:n], idx_ref[:n])
        assert np.all(np.diff(idx[:n].cpu().numpy()) > 0)


def test_static_scratch_rejects_sizes_beyond_its_limit():
    """A request whose scratch does not fit is refused before anything runs.
    Real tensors of the requested shape: 16 tokens x rank 16384 x 4 bytes of u
    fill the 1 MiB alone, the tile masks push it over; count keeps its
    sentinel, so nothing was launched."""
    lib = pi.lib()
    d, ffn, rank, batch = 64, 256, 16384, 16
    desc = pi.make_desc(d, ffn, 0, rank, "f16", "f16", "relu")
    h = torch.zeros(batch, d, dtype=torch.float16, device="cuda")
    P1 = torch.zeros(rank, d, dtype=torch.float16, device="cuda")
    P2 = torch.zeros(ffn, rank, dtype=torch.float16, device="cuda")
    idx = torch.full((ffn,), -3, dtype=torch.int32, device="cuda")
    cnt = torch.full((1,), -3, dtype=torch.int32, device="cuda")
    st = lib.pi_predict_static(ctypes.byref(desc), batch, h.data_ptr(), P1.data_ptr(), P2.data_ptr(), None, 0.5,
                               idx.data_ptr(), cnt.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == B.PI_ERR_CAPACITY
    assert b"1 MiB" in lib.pi_last_error()
    torch.cuda.synchronize()
    assert int(cnt.item()) == -3
    assert bool((idx == -3).all())


def test_static_scratch_token_block_of_8_matches_oracle():
    """fp16 predictor, 8 tokens: pi_predict takes its tensor-core predictor
    there and this call the CUDA-core one, so both lists are compared with
    the oracle, exact outside the 1e-3 band around the threshold."""
    from gpu_util import check_index_list, oracle_predict, to_np
    lib = pi.lib()
    wl = W.Workload("noalloc8", 93, 512, 1800, 1, "reglu", "f16", "f16", 0.88, 1.2, 0.1, 128, (8,), 2)
    L = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in W.make_layer(wl, 0).items()}
    desc = pi.desc_for(wl)
    C = wl.n_cold
    for step in range(2):
        h = W.make_tokens(wl, 8, 70 + step, device="cuda")
        idx = torch.full((C,), -2, dtype=torch.int32, device="cuda")
        cnt = torch.full((1,), -2, dtype=torch.int32, device="cuda")
        _static_predict(lib, desc, h, L, idx, cnt)
        torch.cuda.synchronize()
        n = int(cnt.item())
        assert 0 < n < C
        orc = oracle_predict(L, to_np(h), wl)
        check_index_list(idx[:n].cpu().numpy(), orc, wl.thr, wl.n_hot, wl.ffn)
