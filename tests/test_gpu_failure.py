"""Failure detection on the GPU without a fault: the persistent kernel's
bounded waits give up, record PI_ERR_TIMEOUT and leave the context usable."""
import time

import numpy as np
import pytest
import torch

import activation_sparse_decode_predict_b200 as pi
import oracle
import pi_workload as W
from activation_sparse_decode_predict_b200 import _binding as B

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind", [0, 1], ids=["mbarrier", "grid-barrier"])
def test_bounded_wait_times_out_and_context_survives(kind):
    wl = W.Workload("fail", 61, 512, 1500, 1, "relu", "f16", "f16", 0.88, 1.2, 0.1, 32, (1,), 1)
    desc = pi.desc_for(wl)
    ws = pi.workspace(desc, 1)
    t0 = time.time()
    pi.selftest_bounded_wait(ws, kind)
    torch.cuda.synchronize()
    dt = time.time() - t0
    assert pi.device_status(ws) == B.PI_ERR_TIMEOUT
    assert 1.5 < dt < 30.0
    # after re-initialising the workspace the decode step runs and is correct
    pi.lib().pi_workspace_init(ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)
    L = W.make_layer(wl, 0, device="cuda")
    arr = pi.layer_array([pi.layer_weights(L)])
    h0 = W.make_tokens(wl, 1, 0, device="cuda")
    idx = torch.zeros(1, wl.n_cold, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = torch.zeros(1, 1, wl.d, device="cuda")
    h_out = torch.zeros_like(h0)
    pi.decode_stack(desc, arr, h0, h_out, idx, cnt, y, W.RMS_EPS, ws)
    torch.cuda.synchronize()
    assert pi.device_status(ws) == 0
    n = int(cnt.item())
    ref = oracle.masked_ffn(h0.cpu().numpy(), idx[0, :n].cpu().numpy(), None, L["Wu"].cpu().numpy(),
                            L["WdT"].cpu().numpy(), L["b1"].cpu().numpy(),
                            None if L["b2"] is None else L["b2"].cpu().numpy(), "relu", wl.n_hot, wl.ffn)
    err = np.abs(y[0].cpu().numpy() - ref).max() / np.abs(ref).max()
    assert err <= 2e-3
