"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every symbol that
include/ttt.h declares, sizes workspaces and rejects invalid requests before touching the GPU."""
import ctypes
import os
import re

import pytest

from vision_test_token_b200 import build, capi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return capi.lib()


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "ttt.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ttt_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    declared = _declared_functions()
    assert declared, "no declarations parsed"
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(capi.EXPORTED) == declared


def test_status_strings_and_version(lib):
    assert capi.status_string(capi.TTT_OK) == "TTT_OK"
    assert capi.status_string(capi.TTT_ERR_TIMEOUT) == "TTT_ERR_TIMEOUT"
    assert capi.ttt_version() >= 103


def _shape(**kw):
    base = dict(batch=8, heads=5, H=78, W=78, d=64, batch_stride=6 * 6084 * 64, head_stride=6084 * 64,
                dtype=capi.TTT_BF16, hidden=0)
    base.update(kw)
    return capi.make_shape(**base)


def test_workspace_sizes(lib):
    s = _shape()
    n = capi.ttt_workspace_bytes(capi.TTT_HEAD_LINEAR, s)
    # bf16 linear: the cluster kernel keeps its intermediates on chip, only the error word remains
    assert n == 256
    nf = capi.ttt_workspace_bytes(capi.TTT_HEAD_LINEAR, _shape(dtype=capi.TTT_FP32, batch_stride=6 * 6084 * 64))
    assert 40 * 64 * 64 * 4 < nf < 16 << 20           # fp32: counters, W1 and partial slots
    nc = capi.ttt_workspace_bytes(capi.TTT_HEAD_DWCONV, s)
    # conv: header, control words (done, 40 unit counters, 40 ready flags) padded to 256 B,
    # then per unit room for one task per row pair (39) of 576-float partials, then W1 per unit
    assert nc == 256 + 512 + 40 * 39 * 576 * 4 + 40 * 576 * 4
    assert capi.ttt_workspace_bytes(capi.TTT_HEAD_LINEAR, _shape(d=32)) == 0
    assert capi.ttt_workspace_bytes(capi.TTT_HEAD_LINEAR, _shape(batch=0)) == 0
    assert capi.ttt_workspace_bytes(7, s) == 0


def test_layer_workspace_sizes(lib):
    s = _shape(heads=6)
    # the linear range's workspace (bf16: the error word), then the conv range's (8 units)
    assert capi.ttt_layer_workspace_bytes(s, 1) == 256 + (256 + 256 + 8 * 39 * 576 * 4 + 8 * 576 * 4)
    assert capi.ttt_layer_workspace_bytes(s, 0) == 256
    assert capi.ttt_layer_workspace_bytes(s, 6) == capi.ttt_workspace_bytes(capi.TTT_HEAD_DWCONV, s)
    assert capi.ttt_layer_workspace_bytes(s, 7) == 0
    assert capi.ttt_layer_workspace_bytes(s, -1) == 0


def test_layer_rejects_bad_head_split(lib):
    s = _shape(heads=6)
    fake = ctypes.c_void_p(1 << 20)
    for ch in (-1, 7):
        st = capi.ttt_forward_layer(fake, fake, fake, fake, fake, ctypes.c_void_p(1 << 40), 0.5, s, ch, fake,
                                    1 << 30, None, None, None)
        assert st == capi.TTT_ERR_INVALID_ARG


@pytest.mark.parametrize("kw,expected", [
    (dict(d=32), capi.TTT_ERR_UNSUPPORTED),
    (dict(batch=0), capi.TTT_ERR_INVALID_ARG),
    (dict(H=0), capi.TTT_ERR_INVALID_ARG),
    (dict(dtype=5), capi.TTT_ERR_INVALID_ARG),
    (dict(max_sms=-1), capi.TTT_ERR_INVALID_ARG),
    (dict(loss=2), capi.TTT_ERR_INVALID_ARG),
    (dict(loss=-1), capi.TTT_ERR_INVALID_ARG),
    (dict(head_stride=100), capi.TTT_ERR_INVALID_ARG),          # heads would overlap
    (dict(head_stride=6084 * 64 + 4), capi.TTT_ERR_ALIGNMENT),  # not a 16-byte multiple for bf16
])
def test_invalid_shapes_are_rejected_before_any_launch(lib, kw, expected):
    s = _shape(**kw)
    st = capi.ttt_forward_linear(None, None, None, None, None, 0.5, s, None, 0, None, None)
    assert st == expected


def test_null_pointers_and_workspace(lib):
    s = _shape()
    assert capi.ttt_forward_linear(None, None, None, None, None, 0.5, s, None, 0, None, None) == capi.TTT_ERR_INVALID_ARG
    fake = ctypes.c_void_p(1 << 20)
    st = capi.ttt_forward_linear(fake, fake, fake, fake, ctypes.c_void_p(1 << 40), 0.5, s, None, 0, None, None)
    assert st == capi.TTT_ERR_WORKSPACE
    st = capi.ttt_forward_linear(fake, fake, fake, fake, ctypes.c_void_p(1 << 40), float("nan"), s, fake, 1 << 30,
                                 None, None)
    assert st == capi.TTT_ERR_INVALID_ARG


def test_mlp_rejects_unsupported_requests(lib):
    s = _shape(hidden=256, dtype=capi.TTT_FP32)
    assert capi.ttt_forward_mlp(None, None, None, None, None, None, 0.5, s, None, 0, None, None, None) == \
        capi.TTT_ERR_UNSUPPORTED
    s = _shape(hidden=100)
    assert capi.ttt_forward_mlp(None, None, None, None, None, None, 0.5, s, None, 0, None, None, None) == \
        capi.TTT_ERR_INVALID_ARG
    s = _shape(hidden=256, loss=capi.TTT_LOSS_DOT)       # the MLP head implements the L2 loss only
    assert capi.ttt_forward_mlp(None, None, None, None, None, None, 0.5, s, None, 0, None, None, None) == \
        capi.TTT_ERR_UNSUPPORTED
    assert capi.ttt_workspace_bytes(capi.TTT_HEAD_MLP, s) == 0


def test_dot_loss_shapes_size_like_l2(lib):
    """The dot-product loss uses the same workspaces as the L2 loss."""
    for kind in (capi.TTT_HEAD_LINEAR, capi.TTT_HEAD_DWCONV):
        for dt in (capi.TTT_BF16, capi.TTT_FP32):
            a = capi.ttt_workspace_bytes(kind, _shape(dtype=dt))
            b = capi.ttt_workspace_bytes(kind, _shape(dtype=dt, loss=capi.TTT_LOSS_DOT))
            assert a == b and a > 0
    s = _shape(heads=6, loss=capi.TTT_LOSS_DOT)
    assert capi.ttt_layer_workspace_bytes(s, 1) == capi.ttt_layer_workspace_bytes(_shape(heads=6), 1)


def test_selftest_rejects_bad_arguments(lib):
    fake = ctypes.c_void_p(1 << 20)
    assert capi.ttt_selftest_wait_timeout(None, 256, 0, None) == capi.TTT_ERR_INVALID_ARG   # checked first
    assert capi.ttt_selftest_wait_timeout(fake, 100, 1000, None) == capi.TTT_ERR_WORKSPACE
    assert capi.ttt_selftest_wait_timeout(ctypes.c_void_p((1 << 20) + 16), 256, 1000, None) == capi.TTT_ERR_ALIGNMENT
    assert capi.ttt_selftest_wait_timeout(fake, 256, 0, None) == capi.TTT_ERR_INVALID_ARG
    assert capi.ttt_selftest_wait_timeout(fake, 256, 2_000_000_000, None) == capi.TTT_ERR_INVALID_ARG


def test_minibatch_rejects_bad_arguments(lib):
    s = _shape()
    fake = ctypes.c_void_p(1 << 20)
    call = lambda shape, b, mode: capi.ttt_forward_linear_minibatch(fake, fake, fake, fake, ctypes.c_void_p(1 << 40),
                                                                   0.5, shape, b, mode, fake, 256, None, None)
    assert call(s, 0, capi.TTT_MB_PREFIX) == capi.TTT_ERR_INVALID_ARG          # empty mini-batches
    assert call(s, 16, 2) == capi.TTT_ERR_INVALID_ARG                          # unknown mode
    assert call(_shape(loss=capi.TTT_LOSS_DOT), 16, capi.TTT_MB_PREFIX) == capi.TTT_ERR_UNSUPPORTED
    assert call(_shape(d=32), 16, capi.TTT_MB_EPOCH) == capi.TTT_ERR_UNSUPPORTED
    assert capi.ttt_forward_linear_minibatch(None, None, None, None, None, 0.5, s, 16, capi.TTT_MB_PREFIX, fake, 256,
                                             None, None) == capi.TTT_ERR_INVALID_ARG
    assert capi.ttt_forward_linear_minibatch(fake, fake, fake, fake, ctypes.c_void_p(1 << 40), 0.5, s, 16,
                                             capi.TTT_MB_PREFIX, None, 0, None, None) == capi.TTT_ERR_WORKSPACE


def test_backward_workspace_and_validation(lib):
    s = _shape()
    n = capi.ttt_workspace_bytes(capi.TTT_HEAD_LINEAR_BACKWARD, s)
    units = 8 * 5
    # counters, then partial slots for up to 320 CTAs + one per unit ([G ; C ; dW1] = 192 x 64 fp32),
    # the unit matrices (4 x 64 x 64), each unit's dW0 and deta, and the bf16 operand images of the
    # per-token maps (8 x 64 x 64 bf16 per unit)
    assert n > (320 + units) * 192 * 64 * 4 + units * 5 * 64 * 64 * 4 + units * 8 * 64 * 64 * 2
    assert capi.ttt_workspace_bytes(capi.TTT_HEAD_LINEAR_BACKWARD, _shape(batch=0)) == 0
    fake = ctypes.c_void_p(1 << 20)
    far = ctypes.c_void_p(1 << 40)
    call = lambda shape, dZ=fake, ws=fake, nbytes=1 << 30: capi.ttt_backward_linear(
        fake, fake, fake, fake, dZ, 0.5, shape, ws, nbytes, far, far, far, None, None, None)
    assert call(_shape(loss=capi.TTT_LOSS_DOT)) == capi.TTT_ERR_UNSUPPORTED     # L2 only
    assert call(s, dZ=None) == capi.TTT_ERR_INVALID_ARG
    assert call(s, ws=None, nbytes=0) == capi.TTT_ERR_WORKSPACE
    assert call(s, nbytes=n - 1) == capi.TTT_ERR_WORKSPACE
    assert call(_shape(d=32)) == capi.TTT_ERR_UNSUPPORTED


def test_header_is_plain_c(tmp_path):
    """include/ttt.h is a C header: a C99 translation unit that includes it and takes the address of
    every declared function compiles with gcc in pedantic mode."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    names = _declared_functions()
    src = tmp_path / "use_header.c"
    src.write_text('#include "ttt.h"\n' + "".join(f"void (*p_{n})(void) = (void (*)(void)){n};\n" for n in names) +
                   "int main(void) { ttt_shape s = {0}; (void)s; return 0; }\n")
    r = subprocess.run([gcc, "-std=c99", "-pedantic", "-Wall", "-Werror", "-fsyntax-only",
                        "-I", os.path.join(ROOT, "include"), str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_wait_limit_bounds(lib):
    """The bound of every device-side wait is settable from the host (1 ns .. 1 s); other values are
    rejected and leave it unchanged."""
    assert capi.ttt_set_wait_limit(0) == capi.TTT_ERR_INVALID_ARG
    assert capi.ttt_set_wait_limit(10 ** 10) == capi.TTT_ERR_INVALID_ARG
    assert capi.ttt_set_wait_limit(1_000_000_000) == capi.TTT_OK
