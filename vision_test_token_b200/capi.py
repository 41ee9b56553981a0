"""ctypes binding of libttt.so: the C ABI declared in include/ttt.h, one Python name per C entry
point, argument marshalling only.  Importing this module loads the in-tree library and fails
loudly if it is missing or does not export every declared symbol."""
import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libttt.so")

TTT_OK, TTT_ERR_INVALID_ARG, TTT_ERR_UNSUPPORTED, TTT_ERR_ALIGNMENT = 0, 1, 2, 3
TTT_ERR_WORKSPACE, TTT_ERR_CUDA, TTT_ERR_TIMEOUT = 4, 5, 6
TTT_FP32, TTT_BF16 = 0, 1
TTT_HEAD_LINEAR, TTT_HEAD_DWCONV, TTT_HEAD_MLP, TTT_HEAD_LINEAR_BACKWARD, TTT_HEAD_CONV3X3 = 0, 1, 2, 3, 4
TTT_HEAD_DWCONV_BACKWARD, TTT_HEAD_MLP_BACKWARD = 5, 6
TTT_LOSS_L2, TTT_LOSS_DOT = 0, 1
TTT_MB_PREFIX, TTT_MB_EPOCH = 0, 1

# Every symbol that include/ttt.h declares.
EXPORTED = (
    "ttt_workspace_bytes", "ttt_workspace_init", "ttt_workspace_status",
    "ttt_forward_linear", "ttt_forward_dwconv", "ttt_forward_conv3x3", "ttt_forward_mlp", "ttt_forward_linear_noalloc", "ttt_noalloc_status",
    "ttt_forward_linear_minibatch", "ttt_backward_linear", "ttt_backward_dwconv", "ttt_backward_mlp",
    "ttt_layer_workspace_bytes", "ttt_forward_layer", "ttt_selftest_wait_timeout", "ttt_set_wait_limit",
    "ttt_status_string", "ttt_last_error", "ttt_version",
)


class TttShape(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int), ("heads", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
        ("d", ctypes.c_int), ("hidden", ctypes.c_int),
        ("batch_stride", ctypes.c_longlong), ("head_stride", ctypes.c_longlong),
        ("dtype", ctypes.c_int), ("max_sms", ctypes.c_int), ("loss", ctypes.c_int),
    ]


class TttError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


_lib = None


def lib():
    """Load libttt.so (once).  Raises if the library was not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libttt.so not found at {LIB_PATH}: run `python -m vision_test_token_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i, f = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
        shp = ctypes.POINTER(TttShape)
        L.ttt_workspace_bytes.argtypes = [i, shp]
        L.ttt_workspace_bytes.restype = sz
        L.ttt_workspace_init.argtypes = [vp, sz, vp]
        L.ttt_workspace_init.restype = i
        L.ttt_workspace_status.argtypes = [vp, vp]
        L.ttt_workspace_status.restype = i
        L.ttt_forward_linear.argtypes = [vp, vp, vp, vp, vp, f, shp, vp, sz, vp, vp]
        L.ttt_forward_linear.restype = i
        L.ttt_forward_linear_noalloc.argtypes = [vp, vp, vp, vp, vp, f, shp, vp, vp]
        L.ttt_noalloc_status.argtypes = [vp]
        L.ttt_noalloc_status.restype = i
        L.ttt_forward_linear_noalloc.restype = i
        L.ttt_forward_linear_minibatch.argtypes = [vp, vp, vp, vp, vp, f, shp, i, i, vp, sz, vp, vp]
        L.ttt_forward_linear_minibatch.restype = i
        L.ttt_backward_linear.argtypes = [vp, vp, vp, vp, vp, f, shp, vp, sz, vp, vp, vp, vp, vp, vp]
        L.ttt_backward_dwconv.argtypes = [vp, vp, vp, vp, vp, f, shp, vp, sz, vp, vp, vp, vp, vp, vp]
        L.ttt_backward_dwconv.restype = i
        L.ttt_backward_mlp.argtypes = [vp, vp, vp, vp, vp, vp, f, shp, vp, sz, vp, vp, vp, vp, vp, vp, vp]
        L.ttt_backward_mlp.restype = i
        L.ttt_backward_linear.restype = i
        L.ttt_forward_dwconv.argtypes = [vp, vp, vp, vp, vp, f, shp, vp, sz, vp, vp]
        L.ttt_forward_conv3x3.argtypes = [vp, vp, vp, vp, vp, f, shp, vp, sz, vp, vp]
        L.ttt_forward_conv3x3.restype = i
        L.ttt_forward_dwconv.restype = i
        L.ttt_forward_mlp.argtypes = [vp, vp, vp, vp, vp, vp, f, shp, vp, sz, vp, vp, vp]
        L.ttt_forward_mlp.restype = i
        L.ttt_layer_workspace_bytes.argtypes = [shp, i]
        L.ttt_layer_workspace_bytes.restype = sz
        L.ttt_forward_layer.argtypes = [vp, vp, vp, vp, vp, vp, f, shp, i, vp, sz, vp, vp, vp]
        L.ttt_forward_layer.restype = i
        L.ttt_selftest_wait_timeout.argtypes = [vp, sz, ctypes.c_ulonglong, vp]
        L.ttt_selftest_wait_timeout.restype = i
        L.ttt_set_wait_limit.argtypes = [ctypes.c_ulonglong]
        L.ttt_set_wait_limit.restype = i
        L.ttt_status_string.argtypes = [i]
        L.ttt_status_string.restype = ctypes.c_char_p
        L.ttt_last_error.argtypes = []
        L.ttt_last_error.restype = i
        L.ttt_version.argtypes = []
        L.ttt_version.restype = i
        for name in EXPORTED:
            getattr(L, name)
        _lib = L
    return _lib


def status_string(st):
    return lib().ttt_status_string(int(st)).decode()


def make_shape(batch, heads, H, W, d, batch_stride, head_stride, dtype, hidden=0, max_sms=0, loss=TTT_LOSS_L2):
    return TttShape(batch, heads, H, W, d, hidden, batch_stride, head_stride, dtype, max_sms, loss)


def ttt_workspace_bytes(kind, shape):
    return lib().ttt_workspace_bytes(kind, ctypes.byref(shape))


def ttt_workspace_init(ws, nbytes, stream):
    return lib().ttt_workspace_init(ws, nbytes, stream)


def ttt_workspace_status(ws, stream):
    return lib().ttt_workspace_status(ws, stream)


def ttt_forward_linear(Q, K, V, W0, Z, eta, shape, ws, ws_bytes, W1_out, stream):
    return lib().ttt_forward_linear(Q, K, V, W0, Z, eta, ctypes.byref(shape), ws, ws_bytes, W1_out, stream)


def ttt_forward_linear_noalloc(Q, K, V, W0, Z, eta, shape, W1_out, stream):
    return lib().ttt_forward_linear_noalloc(Q, K, V, W0, Z, eta, ctypes.byref(shape), W1_out, stream)


def ttt_noalloc_status(stream):
    return lib().ttt_noalloc_status(stream)


def ttt_forward_linear_minibatch(Q, K, V, W0, Z, eta, shape, batch_tokens, mode, ws, ws_bytes, W1_out, stream):
    return lib().ttt_forward_linear_minibatch(Q, K, V, W0, Z, eta, ctypes.byref(shape), batch_tokens, mode, ws,
                                              ws_bytes, W1_out, stream)


def ttt_backward_linear(Q, K, V, W0, dZ, eta, shape, ws, ws_bytes, dQ, dK, dV, dW0_out, deta_out, stream):
    return lib().ttt_backward_linear(Q, K, V, W0, dZ, eta, ctypes.byref(shape), ws, ws_bytes, dQ, dK, dV, dW0_out,
                                     deta_out, stream)


def ttt_backward_dwconv(Q, K, V, W0, dZ, eta, shape, ws, ws_bytes, dQ, dK, dV, dW0_out, deta_out, stream):
    return lib().ttt_backward_dwconv(Q, K, V, W0, dZ, eta, ctypes.byref(shape), ws, ws_bytes, dQ, dK, dV, dW0_out,
                                     deta_out, stream)


def ttt_backward_mlp(Q, K, V, Wa, Wb, dZ, eta, shape, ws, ws_bytes, dQ, dK, dV, dWa_out, dWb_out, deta_out, stream):
    return lib().ttt_backward_mlp(Q, K, V, Wa, Wb, dZ, eta, ctypes.byref(shape), ws, ws_bytes, dQ, dK, dV, dWa_out,
                                  dWb_out, deta_out, stream)


def ttt_forward_dwconv(Q, K, V, W0, Z, eta, shape, ws, ws_bytes, W1_out, stream):
    return lib().ttt_forward_dwconv(Q, K, V, W0, Z, eta, ctypes.byref(shape), ws, ws_bytes, W1_out, stream)


def ttt_forward_conv3x3(Q, K, V, W0, Z, eta, shape, ws, ws_bytes, W1_out, stream):
    return lib().ttt_forward_conv3x3(Q, K, V, W0, Z, eta, ctypes.byref(shape), ws, ws_bytes, W1_out, stream)


def ttt_forward_mlp(Q, K, V, Wa, Wb, Z, eta, shape, ws, ws_bytes, Wa_out, Wb_out, stream):
    return lib().ttt_forward_mlp(Q, K, V, Wa, Wb, Z, eta, ctypes.byref(shape), ws, ws_bytes, Wa_out, Wb_out,
                                 stream)


def ttt_layer_workspace_bytes(shape, conv_heads):
    return lib().ttt_layer_workspace_bytes(ctypes.byref(shape), conv_heads)


def ttt_forward_layer(Q, K, V, W0_lin, W0_conv, Z, eta, shape, conv_heads, ws, ws_bytes, W1_lin_out, W1_conv_out,
                      stream):
    return lib().ttt_forward_layer(Q, K, V, W0_lin, W0_conv, Z, eta, ctypes.byref(shape), conv_heads, ws, ws_bytes,
                                   W1_lin_out, W1_conv_out, stream)


def ttt_selftest_wait_timeout(ws, ws_bytes, limit_ns, stream):
    return lib().ttt_selftest_wait_timeout(ws, ws_bytes, limit_ns, stream)


def ttt_set_wait_limit(limit_ns):
    return lib().ttt_set_wait_limit(limit_ns)


def ttt_last_error():
    return lib().ttt_last_error()


def ttt_version():
    return lib().ttt_version()
