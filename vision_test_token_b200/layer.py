"""Torch-facing wrappers over the C ABI: they take CUDA tensors, check layouts, hand raw device
pointers and the current stream to libttt.so and raise on any non-OK status.  PyTorch only
allocates memory and supplies the stream; every step of the layer runs in the library's kernels.

Tensor layout: Q, K, V (and Z) are [B][heads][N][d] views whose last two dimensions are contiguous
(row stride d, element stride 1); the batch and head strides may be anything the library accepts,
so a slice of heads of a larger buffer (e.g. ``X[:, :5]``) is passed without a copy.
"""
import torch

from . import capi

_DTYPES = {torch.bfloat16: capi.TTT_BF16, torch.float32: capi.TTT_FP32}
# inner loss of the one-step training: "l2" = (1/N) sum ||f(k) - v||^2, "dot" = -(1/N) sum <f(k), v>
_LOSSES = {"l2": capi.TTT_LOSS_L2, "dot": capi.TTT_LOSS_DOT}
_ws_cache = {}


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream_handle(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _shape_of(Q, H, W, hidden=0, max_sms=0, loss="l2"):
    if Q.dim() != 4:
        raise ValueError("Q/K/V must be [B][heads][N][d]")
    B, heads, N, d = Q.shape
    if H * W != N:
        raise ValueError(f"grid {H}x{W} does not match N={N}")
    if Q.stride(3) != 1 or Q.stride(2) != d:
        raise ValueError("token rows of Q/K/V/Z must be contiguous")
    if Q.dtype not in _DTYPES:
        raise ValueError(f"unsupported dtype {Q.dtype}")
    if loss not in _LOSSES:
        raise ValueError(f"loss must be one of {sorted(_LOSSES)}")
    return capi.make_shape(B, heads, H, W, d, Q.stride(0), Q.stride(1), _DTYPES[Q.dtype], hidden, max_sms,
                           _LOSSES[loss])


def _same_layout(ref, *others):
    for t in others:
        if t.shape != ref.shape or t.stride() != ref.stride() or t.dtype != ref.dtype or t.device != ref.device:
            raise ValueError("Q, K, V and Z must share shape, strides, dtype and device")


def workspace(kind, shape, device):
    """A zero-initialised workspace for (kind, shape) on `device`, cached and reused.  None when the
    library sizes none (an invalid or unsupported shape: the call itself then reports why)."""
    nbytes = capi.ttt_workspace_bytes(kind, shape)
    if nbytes == 0:
        return None
    key = (kind, str(device), nbytes)
    ws = _ws_cache.get(key)
    if ws is None:
        ws = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


def _ws_args(ws):
    return (None, 0) if ws is None else (_ptr(ws), ws.numel())


def _check(st, where):
    if st != capi.TTT_OK:
        raise capi.TttError(st, where)


def _out_like(Q, Z):
    if Z is None:
        Z = torch.empty_like(Q, memory_format=torch.contiguous_format)
        if Z.stride() != Q.stride():
            raise ValueError("pass Z explicitly when Q is a strided view")
    return Z


def forward_linear(Q, K, V, W0, eta, H, W, Z=None, W1_out=None, ws=None, stream=None, max_sms=0, loss="l2"):
    """Linear inner model.  W0: [heads][d][d] fp32 CUDA tensor.  Returns Z.  `max_sms` (0 = all)
    bounds the SMs the call spreads over; `loss` is "l2" or "dot" (the inner loss)."""
    shape = _shape_of(Q, H, W, max_sms=max_sms, loss=loss)
    Z = _out_like(Q, Z)
    _same_layout(Q, K, V, Z)
    W0 = W0.contiguous()
    if ws is None:
        ws = workspace(capi.TTT_HEAD_LINEAR, shape, Q.device)
    st = capi.ttt_forward_linear(_ptr(Q), _ptr(K), _ptr(V), _ptr(W0), _ptr(Z), float(eta), shape, *_ws_args(ws),
                                 _ptr(W1_out), _stream_handle(stream))
    _check(st, "ttt_forward_linear")
    return Z


_MB_MODES = {"prefix": capi.TTT_MB_PREFIX, "epoch": capi.TTT_MB_EPOCH}


def _error_word_workspace(device):
    """The 256-byte zero-filled workspace (an error word) of the calls that need no other scratch."""
    key = ("error_word", str(device))
    ws = _ws_cache.get(key)
    if ws is None:
        ws = torch.zeros(256, dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


def forward_linear_minibatch(Q, K, V, W0, eta, H, W, batch_tokens, mode="prefix", Z=None, W1_out=None, ws=None,
                             stream=None, max_sms=0):
    """Linear inner model trained by mini-batch gradient descent over consecutive batches of
    `batch_tokens` tokens.  mode "prefix": causal prefix sums inside a mini-batch, z_t = W_t q_t;
    mode "epoch": one mean-gradient step per mini-batch, every query read out with the final
    weights.  W1_out (optional, [B][heads][d][d] fp32) receives the weights after the last batch."""
    if mode not in _MB_MODES:
        raise ValueError(f"mode must be one of {sorted(_MB_MODES)}")
    shape = _shape_of(Q, H, W, max_sms=max_sms)
    Z = _out_like(Q, Z)
    _same_layout(Q, K, V, Z)
    W0 = W0.contiguous()
    if ws is None:
        ws = _error_word_workspace(Q.device)
    st = capi.ttt_forward_linear_minibatch(_ptr(Q), _ptr(K), _ptr(V), _ptr(W0), _ptr(Z), float(eta), shape,
                                           int(batch_tokens), _MB_MODES[mode], *_ws_args(ws), _ptr(W1_out),
                                           _stream_handle(stream))
    _check(st, "ttt_forward_linear_minibatch")
    return Z


def backward_linear(Q, K, V, W0, eta, H, W, dZ, out=None, ws=None, stream=None, max_sms=0):
    """Backward pass of the full-batch linear head (L2 loss) for the upstream gradient dZ of Z.
    Returns (dQ, dK, dV, dW0 [heads][d][d] fp32 summed over images, deta: a 1-element fp32 tensor
    summed over every unit), all on Q's device; `out` may supply those five tensors."""
    shape = _shape_of(Q, H, W, max_sms=max_sms)
    _same_layout(Q, K, V, dZ)
    heads = Q.shape[1]
    if out is None:
        dQ, dK, dV = (_out_like(Q, None) for _ in range(3))
        dW0 = torch.empty((heads, Q.shape[3], Q.shape[3]), dtype=torch.float32, device=Q.device)
        deta = torch.empty(1, dtype=torch.float32, device=Q.device)
    else:
        dQ, dK, dV, dW0, deta = out
    _same_layout(Q, dQ, dK, dV)
    W0 = W0.contiguous()
    if ws is None:
        ws = workspace(capi.TTT_HEAD_LINEAR_BACKWARD, shape, Q.device)
    st = capi.ttt_backward_linear(_ptr(Q), _ptr(K), _ptr(V), _ptr(W0), _ptr(dZ), float(eta), shape, *_ws_args(ws),
                                  _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dW0), _ptr(deta), _stream_handle(stream))
    _check(st, "ttt_backward_linear")
    return dQ, dK, dV, dW0, deta


def backward_dwconv(Q, K, V, W0, eta, H, W, dZ, out=None, ws=None, stream=None):
    """Backward pass of the depthwise-conv head (L2 loss) for the upstream gradient dZ of Z.
    Returns (dQ, dK, dV, dW0 [heads][d][3][3] fp32 summed over images, deta: a 1-element fp32 tensor
    summed over every unit); `out` may supply those five tensors."""
    shape = _shape_of(Q, H, W)
    _same_layout(Q, K, V, dZ)
    heads = Q.shape[1]
    if out is None:
        dQ, dK, dV = (_out_like(Q, None) for _ in range(3))
        dW0 = torch.empty((heads, Q.shape[3], 3, 3), dtype=torch.float32, device=Q.device)
        deta = torch.empty(1, dtype=torch.float32, device=Q.device)
    else:
        dQ, dK, dV, dW0, deta = out
    _same_layout(Q, dQ, dK, dV)
    W0 = W0.contiguous()
    if ws is None:
        ws = workspace(capi.TTT_HEAD_DWCONV_BACKWARD, shape, Q.device)
    st = capi.ttt_backward_dwconv(_ptr(Q), _ptr(K), _ptr(V), _ptr(W0), _ptr(dZ), float(eta), shape, *_ws_args(ws),
                                  _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dW0), _ptr(deta), _stream_handle(stream))
    _check(st, "ttt_backward_dwconv")
    return dQ, dK, dV, dW0, deta


def backward_mlp(Q, K, V, Wa, Wb, eta, H, W, dZ, out=None, ws=None, stream=None):
    """Backward pass of the MLP head (L2 loss) for the upstream gradient dZ of Z.  Returns (dQ, dK, dV,
    dWa [heads][hidden][d], dWb [heads][d][hidden] fp32 summed over images, deta: a 1-element fp32 tensor
    summed over every unit); `out` may supply those six tensors."""
    shape = _shape_of(Q, H, W, hidden=Wa.shape[1])
    _same_layout(Q, K, V, dZ)
    if out is None:
        dQ, dK, dV = (_out_like(Q, None) for _ in range(3))
        dWa = torch.empty(Wa.shape, dtype=torch.float32, device=Q.device)
        dWb = torch.empty(Wb.shape, dtype=torch.float32, device=Q.device)
        deta = torch.empty(1, dtype=torch.float32, device=Q.device)
    else:
        dQ, dK, dV, dWa, dWb, deta = out
    _same_layout(Q, dQ, dK, dV)
    Wa, Wb = Wa.contiguous(), Wb.contiguous()
    if ws is None:
        ws = workspace(capi.TTT_HEAD_MLP_BACKWARD, shape, Q.device)
    st = capi.ttt_backward_mlp(_ptr(Q), _ptr(K), _ptr(V), _ptr(Wa), _ptr(Wb), _ptr(dZ), float(eta), shape,
                               *_ws_args(ws), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dWa), _ptr(dWb), _ptr(deta),
                               _stream_handle(stream))
    _check(st, "ttt_backward_mlp")
    return dQ, dK, dV, dWa, dWb, deta


def forward_dwconv(Q, K, V, W0, eta, H, W, Z=None, W1_out=None, ws=None, stream=None, max_sms=0, loss="l2"):
    """3x3 depthwise-conv inner model.  W0: [heads][d][3][3] fp32 CUDA tensor.  Returns Z."""
    shape = _shape_of(Q, H, W, max_sms=max_sms, loss=loss)
    Z = _out_like(Q, Z)
    _same_layout(Q, K, V, Z)
    W0 = W0.contiguous()
    if ws is None:
        ws = workspace(capi.TTT_HEAD_DWCONV, shape, Q.device)
    st = capi.ttt_forward_dwconv(_ptr(Q), _ptr(K), _ptr(V), _ptr(W0), _ptr(Z), float(eta), shape, *_ws_args(ws),
                                 _ptr(W1_out), _stream_handle(stream))
    _check(st, "ttt_forward_dwconv")
    return Z


def forward_conv3x3(Q, K, V, W0, eta, H, W, Z=None, W1_out=None, ws=None, stream=None, max_sms=0):
    """Full 3x3 conv inner model (every output channel reads every input channel).  W0:
    [heads][d][d][3][3] fp32 CUDA tensor; bf16 Q, K, V.  Returns Z."""
    shape = _shape_of(Q, H, W, max_sms=max_sms)
    Z = _out_like(Q, Z)
    _same_layout(Q, K, V, Z)
    W0 = W0.contiguous()
    if ws is None:
        ws = workspace(capi.TTT_HEAD_CONV3X3, shape, Q.device)
    st = capi.ttt_forward_conv3x3(_ptr(Q), _ptr(K), _ptr(V), _ptr(W0), _ptr(Z), float(eta), shape, *_ws_args(ws),
                                  _ptr(W1_out), _stream_handle(stream))
    _check(st, "ttt_forward_conv3x3")
    return Z


def forward_mlp(Q, K, V, Wa, Wb, eta, H, W, Z=None, Wa_out=None, Wb_out=None, ws=None, stream=None, max_sms=0,
                loss="l2"):
    """One-hidden-layer GELU MLP inner model.  Wa: [heads][hidden][d], Wb: [heads][d][hidden].
    Only the "l2" loss is implemented (the library rejects "dot" with TTT_ERR_UNSUPPORTED)."""
    shape = _shape_of(Q, H, W, hidden=Wa.shape[1], max_sms=max_sms, loss=loss)
    Z = _out_like(Q, Z)
    _same_layout(Q, K, V, Z)
    Wa, Wb = Wa.contiguous(), Wb.contiguous()
    if ws is None:
        ws = workspace(capi.TTT_HEAD_MLP, shape, Q.device)
    st = capi.ttt_forward_mlp(_ptr(Q), _ptr(K), _ptr(V), _ptr(Wa), _ptr(Wb), _ptr(Z), float(eta), shape,
                              *_ws_args(ws), _ptr(Wa_out), _ptr(Wb_out), _stream_handle(stream))
    _check(st, "ttt_forward_mlp")
    return Z


def layer_workspace(shape, conv_heads, device):
    """A zero-initialised workspace for ttt_forward_layer(shape, conv_heads), cached and reused (None
    when the library sizes none)."""
    nbytes = capi.ttt_layer_workspace_bytes(shape, conv_heads)
    if nbytes == 0:
        return None
    key = ("layer", str(device), nbytes)
    ws = _ws_cache.get(key)
    if ws is None:
        ws = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


def forward_layer(Q, K, V, weights, eta, H, W, conv_heads=0, Z=None, W1_lin_out=None, W1_conv_out=None, ws=None,
                  stream=None, concurrent=True, max_sms=0, loss="l2"):
    """A layer whose first heads are linear and whose last `conv_heads` heads are depthwise-conv
    heads, over head ranges of the same buffers.  weights: {"W0_lin": [heads-conv_heads][d][d],
    "W0_conv": [conv_heads][d][3][3]}.  With `concurrent` (the default) one ttt_forward_layer call
    runs both kernels at the same time; otherwise ttt_forward_linear and ttt_forward_dwconv run one
    after the other on the stream."""
    Z = _out_like(Q, Z)
    _same_layout(Q, K, V, Z)
    heads = Q.shape[1]
    nl = heads - conv_heads
    W0l = weights["W0_lin"].contiguous() if nl else None
    W0c = weights["W0_conv"].contiguous() if conv_heads else None
    if concurrent:
        shape = _shape_of(Q, H, W, max_sms=max_sms, loss=loss)
        if ws is None:
            ws = layer_workspace(shape, conv_heads, Q.device)
        st = capi.ttt_forward_layer(_ptr(Q), _ptr(K), _ptr(V), _ptr(W0l), _ptr(W0c), _ptr(Z), float(eta), shape,
                                    conv_heads, *_ws_args(ws), _ptr(W1_lin_out), _ptr(W1_conv_out),
                                    _stream_handle(stream))
        _check(st, "ttt_forward_layer")
        return Z
    if nl:
        forward_linear(Q[:, :nl], K[:, :nl], V[:, :nl], W0l, eta, H, W, Z=Z[:, :nl], W1_out=W1_lin_out,
                       stream=stream, max_sms=max_sms, loss=loss)
    if conv_heads:
        forward_dwconv(Q[:, nl:], K[:, nl:], V[:, nl:], W0c, eta, H, W, Z=Z[:, nl:], W1_out=W1_conv_out,
                       stream=stream, max_sms=max_sms, loss=loss)
    return Z


def workspace_status(ws, stream=None):
    """Synchronises and returns the library status recorded in `ws` (TTT_OK or TTT_ERR_TIMEOUT)."""
    return capi.ttt_workspace_status(_ptr(ws), _stream_handle(stream))
