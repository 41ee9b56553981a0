"""Failure detection without a fault: a kernel whose bounded wait runs out (on a flag that nothing
sets) records TTT_ERR_TIMEOUT in the workspace error word; ttt_workspace_status reports it once and
clears it, and the context stays usable for the next call."""
import pytest
import torch

import oracle
from tests.parity import TOL, rel_max_err
from vision_test_token_b200 import capi, forward_linear, workspace_status
from vision_test_token_b200.inputs import random_unit

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_recovers(cuda_dev):
    ws = torch.zeros(256, dtype=torch.uint8, device=cuda_dev)
    assert workspace_status(ws) == capi.TTT_OK
    st = capi.ttt_selftest_wait_timeout(ws.data_ptr(), ws.numel(), 2_000_000, torch.cuda.current_stream().cuda_stream)
    assert st == capi.TTT_OK
    assert workspace_status(ws) == capi.TTT_ERR_TIMEOUT
    assert workspace_status(ws) == capi.TTT_OK                     # reported once, then cleared
    assert capi.ttt_last_error() == capi.TTT_OK                   # no CUDA error: the kernel returned
    _, x = random_unit(2, 2, 9, 9, dtype="bf16", seed=21)          # the next call works as before
    Z = forward_linear(x["Q"].to(cuda_dev), x["K"].to(cuda_dev), x["V"].to(cuda_dev), x["W0_lin"].to(cuda_dev),
                       0.5, 9, 9)
    torch.cuda.synchronize()
    Zr, _ = oracle.linear(x["Q"], x["K"], x["V"], x["W0_lin"], 0.5)
    assert rel_max_err(Z, Zr) <= TOL["bf16"]
