"""GPU test of ttt_forward_linear_noalloc, the linear-head entry point for callers that cannot
allocate device memory (a plugin handed only its input/output buffers, code with a fixed memory
budget).  It must give the same result as ttt_forward_linear -- within the parity tolerance of the
other tests -- on two calls in a row, since the second call finds the first call's leftovers in the
shared scratch array.  The file is named so that pytest collects it last."""
import pytest
import torch

from tests.parity import TOL, rel_max_err
from vision_test_token_b200 import capi, forward_linear
from vision_test_token_b200.inputs import random_unit

pytestmark = pytest.mark.gpu


def _noalloc(x, eta, H, W, dev):
    Q, K, V = (x[k].to(dev) for k in ("Q", "K", "V"))
    W0 = x["W0_lin"].to(dev).contiguous()
    B, h, N, d = Q.shape
    Z = torch.full_like(Q, float("nan"))
    W1 = torch.full((B, h, d, d), float("nan"), device=dev)
    dtype = capi.TTT_BF16 if Q.dtype == torch.bfloat16 else capi.TTT_FP32
    shape = capi.make_shape(B, h, H, W, d, Q.stride(0), Q.stride(1), dtype)
    st = capi.ttt_forward_linear_noalloc(Q.data_ptr(), K.data_ptr(), V.data_ptr(), W0.data_ptr(), Z.data_ptr(),
                                         float(eta), shape, W1.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == capi.TTT_OK, capi.status_string(st)
    torch.cuda.synchronize()
    return Z, W1


@pytest.mark.parametrize("dtype,B,h,H,W", [("bf16", 4, 5, 78, 78), ("bf16", 3, 2, 20, 25), ("fp32", 1, 1, 14, 14)])
def test_noalloc_matches_workspace_entry_point_twice(cuda_dev, dtype, B, h, H, W):
    _, x = random_unit(B, h, H, W, dtype=dtype, seed=B + h + H)
    eta = 0.5
    Q, K, V = (x[k].to(cuda_dev) for k in ("Q", "K", "V"))
    W1_ref = torch.empty((B, h, 64, 64), device=cuda_dev)
    Z_ref = forward_linear(Q, K, V, x["W0_lin"].to(cuda_dev), eta, H, W, W1_out=W1_ref)
    torch.cuda.synchronize()
    for _ in range(2):
        Z, W1 = _noalloc(x, eta, H, W, cuda_dev)
        assert rel_max_err(Z, Z_ref.double().cpu().numpy()) <= TOL[dtype]
        assert rel_max_err(W1, W1_ref.double().cpu().numpy()) <= TOL[dtype]


def test_noalloc_allocates_nothing(cuda_dev):
    """Around a pair of calls (the first one on this shape included) neither PyTorch's allocator nor
    the device's free memory changes: the entry point draws only on its library-owned array.  (One
    call on another shape first, so that the kernel's code is already loaded on the device.)"""
    _noalloc(random_unit(1, 1, 9, 9, dtype="bf16", seed=4)[1], 0.5, 9, 9, cuda_dev)
    _, x = random_unit(2, 3, 16, 16, dtype="bf16", seed=5)
    Q, K, V = (x[k].to(cuda_dev) for k in ("Q", "K", "V"))
    W0 = x["W0_lin"].to(cuda_dev).contiguous()
    Z = torch.empty_like(Q)
    W1 = torch.empty((2, 3, 64, 64), device=cuda_dev)
    shape = capi.make_shape(2, 3, 16, 16, 64, Q.stride(0), Q.stride(1), capi.TTT_BF16)
    stream = torch.cuda.current_stream().cuda_stream
    torch.cuda.synchronize()
    n0 = torch.cuda.memory_stats(cuda_dev).get("allocation.all.allocated", 0)
    f0, _ = torch.cuda.mem_get_info(cuda_dev)
    for _ in range(2):
        st = capi.ttt_forward_linear_noalloc(Q.data_ptr(), K.data_ptr(), V.data_ptr(), W0.data_ptr(), Z.data_ptr(),
                                             0.5, shape, W1.data_ptr(), stream)
        assert st == capi.TTT_OK
    torch.cuda.synchronize()
    assert torch.cuda.memory_stats(cuda_dev).get("allocation.all.allocated", 0) == n0
    assert torch.cuda.mem_get_info(cuda_dev)[0] == f0
    assert capi.ttt_noalloc_status(stream) == capi.TTT_OK


def test_noalloc_fp32_counters_left_by_a_larger_call(cuda_dev):
    """fp32 keeps counters and partial slots in the scratch: a call over 6 units, then one over 1 unit
    (which finds the first call's leftovers), both correct."""
    for (B, h) in [(2, 3), (1, 1)]:
        _, x = random_unit(B, h, 14, 14, dtype="fp32", seed=40 + B)
        Q, K, V = (x[k].to(cuda_dev) for k in ("Q", "K", "V"))
        W1_ref = torch.empty((B, h, 64, 64), device=cuda_dev)
        Z_ref = forward_linear(Q, K, V, x["W0_lin"].to(cuda_dev), 0.5, 14, 14, W1_out=W1_ref)
        torch.cuda.synchronize()
        Z, W1 = _noalloc(x, 0.5, 14, 14, cuda_dev)
        assert rel_max_err(Z, Z_ref.double().cpu().numpy()) <= TOL["fp32"]
        assert rel_max_err(W1, W1_ref.double().cpu().numpy()) <= TOL["fp32"]


def test_noalloc_rejects_shapes_beyond_its_scratch(cuda_dev):
    big = torch.zeros(1, device=cuda_dev)
    p = big.data_ptr()
    shape = capi.make_shape(64, 12, 80, 80, 64, 12 * 6400 * 64, 6400 * 64, capi.TTT_FP32)
    assert capi.ttt_workspace_bytes(capi.TTT_HEAD_LINEAR, shape) > (8 << 20)
    st = capi.ttt_forward_linear_noalloc(p, p, p, p, p, 0.5, shape, None, torch.cuda.current_stream().cuda_stream)
    assert st == capi.TTT_ERR_WORKSPACE


def test_noalloc_status_reports_a_timeout_once(cuda_dev):
    """A bounded wait that runs out on the library-owned array (the self-test kernel pointed at it) is
    reported by ttt_noalloc_status once, and the next no-alloc call is still correct."""
    stream = torch.cuda.current_stream().cuda_stream
    _, x = random_unit(2, 2, 12, 12, dtype="bf16", seed=17)
    _noalloc(x, 0.5, 12, 12, cuda_dev)
    assert capi.ttt_noalloc_status(stream) == capi.TTT_OK
    assert capi.ttt_selftest_wait_timeout(None, 0, 2_000_000, stream) == capi.TTT_OK
    assert capi.ttt_noalloc_status(stream) == capi.TTT_ERR_TIMEOUT
    assert capi.ttt_noalloc_status(stream) == capi.TTT_OK
    Q, K, V = (x[k].to(cuda_dev) for k in ("Q", "K", "V"))
    W1_ref = torch.empty((2, 2, 64, 64), device=cuda_dev)
    Z_ref = forward_linear(Q, K, V, x["W0_lin"].to(cuda_dev), 0.5, 12, 12, W1_out=W1_ref)
    Z, W1 = _noalloc(x, 0.5, 12, 12, cuda_dev)
    assert rel_max_err(Z, Z_ref.double().cpu().numpy()) <= TOL["bf16"]
    assert rel_max_err(W1, W1_ref.double().cpu().numpy()) <= TOL["bf16"]
    assert capi.ttt_noalloc_status(stream) == capi.TTT_OK
