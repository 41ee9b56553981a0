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


def test_conv_kernel_wait_runs_out_and_recovers(cuda_dev):
    """A real kernel's give-up path.  The depthwise-conv head's readout waits for its unit's W1, which
    the unit's last gradient partial publishes (a ready flag raised once the unit's partial counter
    reaches its task count).  A counter pre-set in the zero-filled workspace -- a count the tasks can
    never complete -- leaves that flag down.  With every device-side wait bounded at 2 ms the call
    records TTT_ERR_TIMEOUT in the workspace (no CUDA error: the kernel returns), the status is
    reported once, and after ttt_workspace_init the same workspace gives a correct next call."""
    from vision_test_token_b200 import forward_dwconv
    from vision_test_token_b200.layer import _shape_of
    w, x = random_unit(2, 1, 12, 12, dtype="bf16", seed=31, kind="mixed", conv_heads=1)
    Q, K, V = (x[k].to(cuda_dev) for k in ("Q", "K", "V"))
    W0 = x["W0_conv"].to(cuda_dev)
    nbytes = capi.ttt_workspace_bytes(capi.TTT_HEAD_DWCONV, _shape_of(Q, 12, 12))
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=cuda_dev)
    words = ws.view(torch.int32)
    words[64 + 1] = 1 << 30            # header (256 B), then done, unit_count[0], ...: unit 0 never completes
    assert capi.ttt_set_wait_limit(2_000_000) == capi.TTT_OK
    try:
        forward_dwconv(Q, K, V, W0, 0.5, 12, 12, ws=ws)
        torch.cuda.synchronize()
        assert capi.ttt_last_error() == capi.TTT_OK
        assert workspace_status(ws) == capi.TTT_ERR_TIMEOUT
        assert workspace_status(ws) == capi.TTT_OK
    finally:
        assert capi.ttt_set_wait_limit(1_000_000_000) == capi.TTT_OK
    st = capi.ttt_workspace_init(ws.data_ptr(), nbytes, torch.cuda.current_stream().cuda_stream)
    assert st == capi.TTT_OK
    Z = forward_dwconv(Q, K, V, W0, 0.5, 12, 12, ws=ws)
    torch.cuda.synchronize()
    assert workspace_status(ws) == capi.TTT_OK
    Zr, _ = oracle.dwconv(x["Q"], x["K"], x["V"], x["W0_conv"], 0.5, 12, 12)
    assert rel_max_err(Z, Zr) <= TOL["bf16"]

