"""fp64 CPU oracle for the ViT^3 test-time-training layer -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline / reference leg of
``bench.py`` may import this package.  The CUDA product path never does, and it shares no code
with it.  Every function takes numpy arrays in the layout documented in ``ttt_oracle.c``
([B][heads][N][d] for Q, K, V, Z), widens them exactly to float64 and returns float64 results.

Functions and the definitions they follow (page titles and sections; see ``ttt_oracle.c``):
  linear(...)       L2 loss, one full-batch gradient step on W (d x d), z = W1 q  -- per-pair form
  linear_gram(...)  the same step written as W0 - eta (2/N) (W0 K K^T - V K^T)
  dwconv(...)       the same loss with a 3x3 depthwise cross-correlation inner model
  conv3x3(...)      the same loss with a full 3x3 cross-correlation (d -> d channels) inner model
  mlp(...)          the same loss with f(x) = Wb gelu_tanh(Wa x)
  linear_dot(...), dwconv_dot(...)
                    the linear and conv heads under the dot-product inner loss -(1/N) sum <f(k), v>
  linear_minibatch(...)
                    the linear head trained by mini-batch gradient descent over consecutive token
                    batches (prefix: causal prefix sums inside a batch; epoch: one mean step per batch)
  linear_backward(...), dwconv_backward(...), mlp_backward(...)
                    the chain rule through the full-batch linear / depthwise-conv / MLP step: dQ, dK,
                    dV, the weights' gradients, deta
  gelu_tanh(u), gelu_tanh_deriv(u), gelu_tanh_deriv2(u)

Parity status: every function here is pinned by tests/test_oracle_pins.py (closed forms,
invariants, exact finite differences, autograd and library special cases).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        i = ctypes.c_int
        d = ctypes.c_double
        lib.oracle_linear.argtypes = [i, i, i, i, dp, dp, dp, dp, d, dp, dp, i]
        lib.oracle_linear_gram.argtypes = [i, i, i, i, dp, dp, dp, dp, d, dp, dp, i]
        lib.oracle_linear_dot.argtypes = [i, i, i, i, dp, dp, dp, dp, d, dp, dp, i]
        lib.oracle_linear_minibatch.argtypes = [i, i, i, i, i, i, dp, dp, dp, dp, d, dp, dp, i]
        lib.oracle_linear_backward.argtypes = [i, i, i, i, dp, dp, dp, dp, d, dp, dp, dp, dp, dp, dp, i]
        lib.oracle_dwconv.argtypes = [i, i, i, i, i, dp, dp, dp, dp, d, dp, dp, i]
        lib.oracle_dwconv_dot.argtypes = [i, i, i, i, i, dp, dp, dp, dp, d, dp, dp, i]
        lib.oracle_conv3x3.argtypes = [i, i, i, i, i, dp, dp, dp, dp, d, dp, dp, i]
        lib.oracle_dwconv_backward.argtypes = [i, i, i, i, i, dp, dp, dp, dp, d, dp, dp, dp, dp, dp, dp, i]
        lib.oracle_mlp_backward.argtypes = [i, i, i, i, i, dp, dp, dp, dp, dp, d, dp, dp, dp, dp, dp, dp, dp, i]
        lib.oracle_mlp.argtypes = [i, i, i, i, i, dp, dp, dp, dp, dp, d, dp, dp, dp, i]
        for f in (lib.oracle_linear, lib.oracle_linear_gram, lib.oracle_linear_dot, lib.oracle_linear_minibatch,
                  lib.oracle_linear_backward,
                  lib.oracle_dwconv,
                  lib.oracle_dwconv_dot, lib.oracle_conv3x3, lib.oracle_dwconv_backward, lib.oracle_mlp_backward,
                  lib.oracle_mlp):
            f.restype = ctypes.c_int
        lib.oracle_gelu_tanh.argtypes = [d]
        lib.oracle_gelu_tanh.restype = d
        lib.oracle_gelu_tanh_deriv.argtypes = [d]
        lib.oracle_gelu_tanh_deriv.restype = d
        lib.oracle_gelu_tanh_deriv2.argtypes = [d]
        lib.oracle_gelu_tanh_deriv2.restype = d
        lib.oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x):
    """Exact widening to a contiguous float64 array (bf16 / fp32 values are representable)."""
    if hasattr(x, "detach"):  # a torch tensor: widen through torch, then hand over to numpy
        x = x.detach().to("cpu").double().contiguous().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def default_threads():
    return max(1, len(os.sched_getaffinity(0)))


def _check(status, name):
    if status != 0:
        raise RuntimeError(f"oracle {name} failed with status {status}")


def linear(Q, K, V, W0, eta, threads=None, gram=False):
    """Returns (Z [B][h][N][d], W1 [B][h][d][d]) in float64."""
    Q, K, V, W0 = _f64(Q), _f64(K), _f64(V), _f64(W0)
    B, H, N, d = Q.shape
    assert K.shape == Q.shape and V.shape == Q.shape and W0.shape == (H, d, d)
    Z = np.empty_like(Q)
    W1 = np.empty((B, H, d, d))
    fn = _load().oracle_linear_gram if gram else _load().oracle_linear
    _check(fn(B, H, N, d, _p(Q), _p(K), _p(V), _p(W0), float(eta), _p(W1), _p(Z),
              threads or default_threads()), "linear")
    return Z, W1


def linear_gram(Q, K, V, W0, eta, threads=None):
    return linear(Q, K, V, W0, eta, threads=threads, gram=True)


def linear_dot(Q, K, V, W0, eta, threads=None):
    """Linear inner model with the dot-product inner loss L(W) = -(1/N) sum <W k, v>.
    Returns (Z [B][h][N][d], W1 [B][h][d][d]) in float64."""
    Q, K, V, W0 = _f64(Q), _f64(K), _f64(V), _f64(W0)
    B, H, N, d = Q.shape
    assert K.shape == Q.shape and V.shape == Q.shape and W0.shape == (H, d, d)
    Z = np.empty_like(Q)
    W1 = np.empty((B, H, d, d))
    _check(_load().oracle_linear_dot(B, H, N, d, _p(Q), _p(K), _p(V), _p(W0), float(eta), _p(W1), _p(Z),
                                     threads or default_threads()), "linear_dot")
    return Z, W1


def linear_minibatch(Q, K, V, W0, eta, b, mode, threads=None):
    """Linear inner model trained by mini-batch gradient descent over consecutive batches of b
    tokens.  mode "prefix": causal prefix sums inside a batch, z_t = W_t q_t; mode "epoch": one
    mean-gradient step per batch, every query read out with the final weights.
    Returns (Z [B][h][N][d], W1 [B][h][d][d]: the weights after the last batch) in float64."""
    Q, K, V, W0 = _f64(Q), _f64(K), _f64(V), _f64(W0)
    B, H, N, d = Q.shape
    assert K.shape == Q.shape and V.shape == Q.shape and W0.shape == (H, d, d)
    m = {"prefix": 0, "epoch": 1}[mode]
    Z = np.empty_like(Q)
    W1 = np.empty((B, H, d, d))
    _check(_load().oracle_linear_minibatch(B, H, N, d, int(b), m, _p(Q), _p(K), _p(V), _p(W0), float(eta),
                                           _p(W1), _p(Z), threads or default_threads()), "linear_minibatch")
    return Z, W1


def linear_backward(Q, K, V, W0, eta, dZ, threads=None):
    """Backward pass of the full-batch linear head (L2 loss) for the upstream gradient dZ.
    Returns (dQ, dK, dV [B][h][N][d], dW0 [h][d][d] summed over images, deta: a float summed over
    every unit) in float64."""
    Q, K, V, W0, dZ = _f64(Q), _f64(K), _f64(V), _f64(W0), _f64(dZ)
    B, H, N, d = Q.shape
    assert K.shape == Q.shape and V.shape == Q.shape and dZ.shape == Q.shape and W0.shape == (H, d, d)
    dQ, dK, dV = np.empty_like(Q), np.empty_like(Q), np.empty_like(Q)
    dW0 = np.empty((H, d, d))
    deta = np.zeros(1)
    _check(_load().oracle_linear_backward(B, H, N, d, _p(Q), _p(K), _p(V), _p(W0), float(eta), _p(dZ), _p(dQ),
                                          _p(dK), _p(dV), _p(dW0), _p(deta), threads or default_threads()),
           "linear_backward")
    return dQ, dK, dV, dW0, float(deta[0])


def dwconv_backward(Q, K, V, W0, eta, dZ, Hg, Wg, threads=None):
    """Backward pass of the depthwise-conv head (L2 loss) for the upstream gradient dZ.
    Returns (dQ, dK, dV [B][h][N][d], dW0 [h][d][3][3] summed over images, deta: a float summed over
    every unit) in float64."""
    Q, K, V, W0, dZ = _f64(Q), _f64(K), _f64(V), _f64(W0), _f64(dZ)
    B, H, N, d = Q.shape
    assert N == Hg * Wg and K.shape == Q.shape and V.shape == Q.shape and dZ.shape == Q.shape
    assert W0.shape == (H, d, 3, 3)
    dQ, dK, dV = np.empty_like(Q), np.empty_like(Q), np.empty_like(Q)
    dW0 = np.empty((H, d, 3, 3))
    deta = np.zeros(1)
    _check(_load().oracle_dwconv_backward(B, H, Hg, Wg, d, _p(Q), _p(K), _p(V), _p(W0), float(eta), _p(dZ), _p(dQ),
                                          _p(dK), _p(dV), _p(dW0), _p(deta), threads or default_threads()),
           "dwconv_backward")
    return dQ, dK, dV, dW0, float(deta[0])


def dwconv(Q, K, V, W0, eta, Hg, Wg, threads=None):
    """Q, K, V: [B][h][Hg*Wg][d]; W0: [h][d][3][3].  Returns (Z, W1 [B][h][d][3][3])."""
    Q, K, V, W0 = _f64(Q), _f64(K), _f64(V), _f64(W0)
    B, H, N, d = Q.shape
    assert N == Hg * Wg and K.shape == Q.shape and V.shape == Q.shape and W0.shape == (H, d, 3, 3)
    Z = np.empty_like(Q)
    W1 = np.empty((B, H, d, 3, 3))
    _check(_load().oracle_dwconv(B, H, Hg, Wg, d, _p(Q), _p(K), _p(V), _p(W0), float(eta), _p(W1),
                                 _p(Z), threads or default_threads()), "dwconv")
    return Z, W1


def conv3x3(Q, K, V, W0, eta, Hg, Wg, threads=None):
    """Full 3x3 conv inner model.  Q, K, V: [B][h][Hg*Wg][d]; W0: [h][d][d][3][3].
    Returns (Z, W1 [B][h][d][d][3][3])."""
    Q, K, V, W0 = _f64(Q), _f64(K), _f64(V), _f64(W0)
    B, H, N, d = Q.shape
    assert N == Hg * Wg and K.shape == Q.shape and V.shape == Q.shape and W0.shape == (H, d, d, 3, 3)
    Z = np.empty_like(Q)
    W1 = np.empty((B, H, d, d, 3, 3))
    _check(_load().oracle_conv3x3(B, H, Hg, Wg, d, _p(Q), _p(K), _p(V), _p(W0), float(eta), _p(W1),
                                  _p(Z), threads or default_threads()), "conv3x3")
    return Z, W1


def dwconv_dot(Q, K, V, W0, eta, Hg, Wg, threads=None):
    """Conv inner model with the dot-product inner loss L(W) = -(1/N) sum <f(K;W), V>.
    Q, K, V: [B][h][Hg*Wg][d]; W0: [h][d][3][3].  Returns (Z, W1 [B][h][d][3][3])."""
    Q, K, V, W0 = _f64(Q), _f64(K), _f64(V), _f64(W0)
    B, H, N, d = Q.shape
    assert N == Hg * Wg and K.shape == Q.shape and V.shape == Q.shape and W0.shape == (H, d, 3, 3)
    Z = np.empty_like(Q)
    W1 = np.empty((B, H, d, 3, 3))
    _check(_load().oracle_dwconv_dot(B, H, Hg, Wg, d, _p(Q), _p(K), _p(V), _p(W0), float(eta), _p(W1),
                                     _p(Z), threads or default_threads()), "dwconv_dot")
    return Z, W1


def mlp_backward(Q, K, V, Wa, Wb, eta, dZ, threads=None):
    """Backward pass of the MLP head (L2 loss) for the upstream gradient dZ.  Returns (dQ, dK, dV
    [B][h][N][d], dWa [h][hidden][d], dWb [h][d][hidden] summed over images, deta: a float summed over
    every unit) in float64."""
    Q, K, V, Wa, Wb, dZ = _f64(Q), _f64(K), _f64(V), _f64(Wa), _f64(Wb), _f64(dZ)
    B, H, N, d = Q.shape
    hidden = Wa.shape[1]
    assert Wa.shape == (H, hidden, d) and Wb.shape == (H, d, hidden) and dZ.shape == Q.shape
    dQ, dK, dV = np.empty_like(Q), np.empty_like(Q), np.empty_like(Q)
    dWa, dWb = np.empty((H, hidden, d)), np.empty((H, d, hidden))
    deta = np.zeros(1)
    _check(_load().oracle_mlp_backward(B, H, N, d, hidden, _p(Q), _p(K), _p(V), _p(Wa), _p(Wb), float(eta), _p(dZ),
                                       _p(dQ), _p(dK), _p(dV), _p(dWa), _p(dWb), _p(deta),
                                       threads or default_threads()), "mlp_backward")
    return dQ, dK, dV, dWa, dWb, float(deta[0])


def gelu_tanh_deriv2(u):
    return _load().oracle_gelu_tanh_deriv2(float(u))


def mlp(Q, K, V, Wa, Wb, eta, threads=None):
    """Wa: [h][hidden][d], Wb: [h][d][hidden].  Returns (Z, Wa1 [B][h][hidden][d], Wb1 [B][h][d][hidden])."""
    Q, K, V, Wa, Wb = _f64(Q), _f64(K), _f64(V), _f64(Wa), _f64(Wb)
    B, H, N, d = Q.shape
    hidden = Wa.shape[1]
    assert Wa.shape == (H, hidden, d) and Wb.shape == (H, d, hidden)
    Z = np.empty_like(Q)
    Wa1 = np.empty((B, H, hidden, d))
    Wb1 = np.empty((B, H, d, hidden))
    _check(_load().oracle_mlp(B, H, N, d, hidden, _p(Q), _p(K), _p(V), _p(Wa), _p(Wb), float(eta),
                              _p(Wa1), _p(Wb1), _p(Z), threads or default_threads()), "mlp")
    return Z, Wa1, Wb1


def gelu_tanh(u):
    return _load().oracle_gelu_tanh(float(u))


def gelu_tanh_deriv(u):
    return _load().oracle_gelu_tanh_deriv(float(u))


def max_threads():
    return _load().oracle_max_threads()
