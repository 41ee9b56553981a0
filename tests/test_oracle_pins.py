"""Pins for the fp64 oracle: each check ties it to something other than itself.

* exact finite differences: the loss is quadratic in the weights of the linear and conv heads, so a
  central difference computed in rational arithmetic IS the gradient, with no truncation error;
* closed forms: with orthogonal keys and eta = N / (2 s) the step lands on the least-squares
  solution (numpy.linalg.lstsq) whatever W0 is;
* invariants: eta = 0 gives z = f(q; W0); values that the initial model already reproduces give a
  zero update; the identity conv kernel with V = K reproduces Q;
* library special cases: torch conv2d (groups=d for the depthwise head, groups=1 for the full 3x3
  head), torch gelu(approximate="tanh") and torch float64 autograd of the pages' L2 loss;
* reductions between heads: a channel-diagonal full 3x3 kernel is the depthwise head, and a full 3x3
  kernel on a one-token grid is the linear head;
* planted mistakes (a transposed gradient, a flipped sign, a 1/N instead of 2/N factor, a dropped
  update) are shown to fail the pins.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

RNG = np.random.default_rng(1234)


# ------------------------------------------------------------------------------------------------
# helpers: the loss as the pages define it (L2 reconstruction over all pairs, mean over tokens)
# ------------------------------------------------------------------------------------------------
def _frac_loss_linear(W, K, V):
    """(1/N) sum_n ||W k_n - v_n||^2 in exact rational arithmetic."""
    N, d = len(K), len(K[0])
    tot = Fraction(0)
    for n in range(N):
        for i in range(d):
            r = sum(W[i][j] * K[n][j] for j in range(d)) - V[n][i]
            tot += r * r
    return tot / N


def _frac_conv(Wc, X, Hg, Wg, c, y, x):
    s = Fraction(0)
    for a in range(3):
        for b in range(3):
            yy, xx = y + a - 1, x + b - 1
            if 0 <= yy < Hg and 0 <= xx < Wg:
                s += Wc[a][b] * X[yy * Wg + xx][c]
    return s


def _frac_loss_conv(W, K, V, Hg, Wg):
    d = len(K[0])
    tot = Fraction(0)
    for c in range(d):
        for y in range(Hg):
            for x in range(Wg):
                r = _frac_conv(W[c], K, Hg, Wg, c, y, x) - V[y * Wg + x][c]
                tot += r * r
    return tot / (Hg * Wg)


def _small_ints(shape, lo=-3, hi=4):
    return RNG.integers(lo, hi, size=shape).astype(np.float64)


def _torch_conv_f(X, W, Hg, Wg):
    """Depthwise 3x3 cross-correlation through torch.conv2d: X [N][d] -> [N][d]."""
    N, d = X.shape
    img = X.T.reshape(1, d, Hg, Wg)
    out = F.conv2d(img, W.reshape(d, 1, 3, 3), padding=1, groups=d)
    return out.reshape(d, N).T


# ------------------------------------------------------------------------------------------------
# linear head
# ------------------------------------------------------------------------------------------------
def test_linear_gradient_exact_rational_fd():
    d, N, eta = 3, 5, 1.0
    K = _small_ints((N, d)); V = _small_ints((N, d)); W0 = _small_ints((d, d)); Q = _small_ints((N, d))
    _, W1 = oracle.linear(Q[None, None], K[None, None], V[None, None], W0[None], eta)
    grad = (W0 - W1[0, 0]) / eta
    Kf = [[Fraction(int(v)) for v in row] for row in K]
    Vf = [[Fraction(int(v)) for v in row] for row in V]
    Wf = [[Fraction(int(v)) for v in row] for row in W0]
    for i in range(d):
        for j in range(d):
            Wp = [r[:] for r in Wf]; Wm = [r[:] for r in Wf]
            Wp[i][j] += 1; Wm[i][j] -= 1
            exact = (_frac_loss_linear(Wp, Kf, Vf) - _frac_loss_linear(Wm, Kf, Vf)) / 2
            assert abs(grad[i, j] - float(exact)) <= 1e-12 * max(1.0, abs(float(exact)))


@pytest.mark.parametrize("d,reps", [(8, 2), (16, 3)])
def test_linear_least_squares_closed_form(d, reps):
    """K stacked from `reps` orthogonal d x d bases => sum_n k_n k_n^T = reps * I.  With
    eta = N / (2 reps) the step gives W1 = V^T K / reps, the least-squares minimiser, for any W0."""
    blocks = [np.linalg.qr(RNG.standard_normal((d, d)))[0] for _ in range(reps)]
    K = np.concatenate(blocks, axis=0)                      # [N][d]
    N = K.shape[0]
    V = RNG.standard_normal((N, d))
    W0 = RNG.standard_normal((d, d))
    Q = RNG.standard_normal((N, d))
    eta = N / (2.0 * reps)
    _, W1 = oracle.linear(Q[None, None], K[None, None], V[None, None], W0[None], eta)
    X, *_ = np.linalg.lstsq(K, V, rcond=None)               # K X ~= V, W = X^T
    np.testing.assert_allclose(W1[0, 0], X.T, atol=1e-12, rtol=0)


def test_linear_eta_zero_is_plain_readout():
    B, H, N, d = 2, 3, 37, 16
    Q, K, V = (RNG.standard_normal((B, H, N, d)) for _ in range(3))
    W0 = RNG.standard_normal((H, d, d))
    Z, W1 = oracle.linear(Q, K, V, W0, 0.0)
    np.testing.assert_array_equal(W1, np.broadcast_to(W0, W1.shape))
    ref = np.einsum("bhnj,hij->bhni", Q, W0)
    np.testing.assert_allclose(Z, ref, atol=1e-13, rtol=0)


def test_linear_reproduced_values_give_no_update():
    B, H, N, d = 1, 2, 50, 8
    Q, K = RNG.standard_normal((B, H, N, d)), RNG.standard_normal((B, H, N, d))
    W0 = RNG.standard_normal((H, d, d))
    V = np.einsum("bhnj,hij->bhni", K, W0)                  # v_n = W0 k_n
    Z, W1 = oracle.linear(Q, K, V, W0, 1.0)
    np.testing.assert_allclose(W1, np.broadcast_to(W0, W1.shape), atol=1e-13, rtol=0)


def test_linear_matches_torch_autograd():
    B, H, N, d, eta = 2, 2, 29, 12, 0.7
    Q, K, V = (RNG.standard_normal((B, H, N, d)) for _ in range(3))
    W0 = RNG.standard_normal((H, d, d))
    Z, W1 = oracle.linear(Q, K, V, W0, eta)
    for b in range(B):
        for h in range(H):
            W = torch.tensor(W0[h], requires_grad=True)
            Kt, Vt = torch.tensor(K[b, h]), torch.tensor(V[b, h])
            loss = ((Kt @ W.T - Vt) ** 2).sum(-1).mean()
            loss.backward()
            W1_ref = (W - eta * W.grad).detach().numpy()
            np.testing.assert_allclose(W1[b, h], W1_ref, atol=1e-12, rtol=0)
            np.testing.assert_allclose(Z[b, h], Q[b, h] @ W1_ref.T, atol=1e-12, rtol=0)


def test_linear_gram_form_equals_pair_form():
    B, H, N, d = 2, 2, 101, 16
    Q, K, V = (RNG.standard_normal((B, H, N, d)) for _ in range(3))
    W0 = RNG.standard_normal((H, d, d))
    Z1, W1 = oracle.linear(Q, K, V, W0, 0.9)
    Z2, W2 = oracle.linear_gram(Q, K, V, W0, 0.9)
    np.testing.assert_allclose(W1, W2, atol=1e-12, rtol=0)
    np.testing.assert_allclose(Z1, Z2, atol=1e-11, rtol=0)


def _ls_pin_holds(W1_candidate, K, V, reps):
    X, *_ = np.linalg.lstsq(K, V, rcond=None)
    return np.allclose(W1_candidate, X.T, atol=1e-9, rtol=0)


@pytest.mark.parametrize("mistake", ["transpose", "sign", "one_over_n", "no_update"])
def test_planted_mistakes_fail_the_linear_pins(mistake):
    """Plant a plausible mistake in the oracle's result (on the CPU) and check a pin catches it."""
    d, reps = 8, 2
    K = np.concatenate([np.linalg.qr(RNG.standard_normal((d, d)))[0] for _ in range(reps)], axis=0)
    N = K.shape[0]
    V = RNG.standard_normal((N, d)); W0 = RNG.standard_normal((d, d)); Q = RNG.standard_normal((N, d))
    eta = N / (2.0 * reps)
    _, W1 = oracle.linear(Q[None, None], K[None, None], V[None, None], W0[None], eta)
    W1 = W1[0, 0]
    assert _ls_pin_holds(W1, K, V, reps)
    grad = (W0 - W1) / eta
    bad = {"transpose": W0 - eta * grad.T, "sign": W0 + eta * grad,
           "one_over_n": W0 - eta * grad / 2, "no_update": W0}[mistake]
    assert not _ls_pin_holds(bad, K, V, reps)


# ------------------------------------------------------------------------------------------------
# linear head, dot-product inner loss  L(W) = -(1/N) sum_n <W k_n, v_n>
# ------------------------------------------------------------------------------------------------
def _frac_loss_dot(W, K, V):
    """-(1/N) sum_n <W k_n, v_n> in exact rational arithmetic."""
    N, d = len(K), len(K[0])
    tot = Fraction(0)
    for n in range(N):
        for i in range(d):
            tot += sum(W[i][j] * K[n][j] for j in range(d)) * V[n][i]
    return -tot / N


def _dot_fd_grad(W0, K, V):
    Kf = [[Fraction(int(v)) for v in row] for row in K]
    Vf = [[Fraction(int(v)) for v in row] for row in V]
    Wf = [[Fraction(int(v)) for v in row] for row in W0]
    d = len(Wf)
    g = np.zeros((d, d))
    for i in range(d):
        for j in range(d):
            Wp = [r[:] for r in Wf]; Wm = [r[:] for r in Wf]
            Wp[i][j] += 1; Wm[i][j] -= 1
            g[i, j] = float((_frac_loss_dot(Wp, Kf, Vf) - _frac_loss_dot(Wm, Kf, Vf)) / 2)
    return g


def test_linear_dot_gradient_exact_rational_fd():
    d, N, eta = 3, 5, 1.0
    K = _small_ints((N, d)); V = _small_ints((N, d)); W0 = _small_ints((d, d)); Q = _small_ints((N, d))
    _, W1 = oracle.linear_dot(Q[None, None], K[None, None], V[None, None], W0[None], eta)
    grad = (W0 - W1[0, 0]) / eta
    np.testing.assert_allclose(grad, _dot_fd_grad(W0, K, V), atol=1e-12, rtol=0)


@pytest.mark.parametrize("mistake", ["sign", "two_over_n", "transpose", "l2_gram"])
def test_planted_mistakes_fail_the_dot_pin(mistake):
    """A plausible mistake planted in the oracle's gradient (on the CPU) fails the exact-FD pin."""
    d, N = 3, 5
    K = _small_ints((N, d)); V = _small_ints((N, d)); W0 = _small_ints((d, d)); Q = _small_ints((N, d))
    _, W1 = oracle.linear_dot(Q[None, None], K[None, None], V[None, None], W0[None], 1.0)
    grad = W0 - W1[0, 0]
    bad = {"sign": -grad, "two_over_n": 2 * grad, "transpose": grad.T,
           "l2_gram": grad + (W0 @ (K.T @ K)) * 2 / N}[mistake]
    assert not np.allclose(bad, _dot_fd_grad(W0, K, V), atol=1e-9, rtol=0)


def test_linear_dot_eta_zero_and_w0_independent_update():
    B, H, N, d = 2, 3, 41, 16
    Q, K, V = (RNG.standard_normal((B, H, N, d)) for _ in range(3))
    W0a, W0b = RNG.standard_normal((H, d, d)), RNG.standard_normal((H, d, d))
    Z, W1 = oracle.linear_dot(Q, K, V, W0a, 0.0)
    np.testing.assert_array_equal(W1, np.broadcast_to(W0a, W1.shape))
    np.testing.assert_allclose(Z, np.einsum("bhnj,hij->bhni", Q, W0a), atol=1e-13, rtol=0)
    _, W1a = oracle.linear_dot(Q, K, V, W0a, 0.8)
    _, W1b = oracle.linear_dot(Q, K, V, W0b, 0.8)
    np.testing.assert_allclose(W1a - W0a[None], W1b - W0b[None], atol=1e-12, rtol=0)


def test_linear_dot_matches_torch_autograd():
    B, H, N, d, eta = 2, 2, 23, 12, 1.0
    Q, K, V = (RNG.standard_normal((B, H, N, d)) for _ in range(3))
    W0 = RNG.standard_normal((H, d, d))
    Z, W1 = oracle.linear_dot(Q, K, V, W0, eta)
    for b in range(B):
        for h in range(H):
            W = torch.tensor(W0[h], requires_grad=True)
            Kt, Vt = torch.tensor(K[b, h]), torch.tensor(V[b, h])
            loss = -((Kt @ W.T) * Vt).sum(-1).mean()
            loss.backward()
            W1_ref = (W - eta * W.grad).detach().numpy()
            np.testing.assert_allclose(W1[b, h], W1_ref, atol=1e-12, rtol=0)
            np.testing.assert_allclose(Z[b, h], Q[b, h] @ W1_ref.T, atol=1e-12, rtol=0)


# ------------------------------------------------------------------------------------------------
# linear head, mini-batch gradient descent over consecutive token batches
# ------------------------------------------------------------------------------------------------
def _per_token_ttt(Q, K, V, W0, eta):
    """Brute force of per-token sequential TTT (each token one step at the current weights):
    W_t = W_{t-1} - eta * 2 (W_{t-1} k_t - v_t) k_t^T,  z_t = W_t q_t."""
    W = W0.copy()
    Z = np.empty_like(Q)
    for t in range(Q.shape[0]):
        W = W - eta * 2.0 * np.outer(W @ K[t] - V[t], K[t])
        Z[t] = W @ Q[t]
    return Z, W


def test_minibatch_prefix_b1_is_per_token_ttt():
    """With one token per mini-batch the prefix form is per-token sequential TTT."""
    N, d, eta = 37, 8, 0.1
    Q, K, V = (RNG.standard_normal((1, 1, N, d)) for _ in range(3))
    W0 = RNG.standard_normal((1, d, d)) / np.sqrt(d)
    Z, W1 = oracle.linear_minibatch(Q, K, V, W0, eta, 1, "prefix")
    Zr, Wr = _per_token_ttt(Q[0, 0], K[0, 0], V[0, 0], W0[0], eta)
    np.testing.assert_allclose(Z[0, 0], Zr, atol=1e-12, rtol=0)
    np.testing.assert_allclose(W1[0, 0], Wr, atol=1e-12, rtol=0)


def test_minibatch_prefix_single_batch_matches_full_batch_on_every_prefix():
    """With b = N every gradient is taken at W0, so W_t is the full-batch step over tokens 0..t with
    the mean's factor 2/(t+1) absorbed into eta: z_t = W1_full(prefix t, eta (t+1)) q_t."""
    N, d, eta = 23, 8, 0.05
    Q, K, V = (RNG.standard_normal((1, 1, N, d)) for _ in range(3))
    W0 = RNG.standard_normal((1, d, d)) / np.sqrt(d)
    Z, W1 = oracle.linear_minibatch(Q, K, V, W0, eta, N, "prefix")
    for t in range(N):
        _, Wp = oracle.linear(Q[:, :, :t + 1], K[:, :, :t + 1], V[:, :, :t + 1], W0, eta * (t + 1))
        np.testing.assert_allclose(Z[0, 0, t], Wp[0, 0] @ Q[0, 0, t], atol=1e-12, rtol=0)
    np.testing.assert_allclose(W1[0, 0], Wp[0, 0], atol=1e-12, rtol=0)


@pytest.mark.parametrize("N,b", [(40, 40), (40, 64), (41, 21), (30, 10), (7, 3)])
def test_minibatch_epoch_chains_full_batch_steps(N, b):
    """Epoch mode = one full-batch step per consecutive mini-batch (the pinned full-batch oracle run
    on each chunk in turn from the previous chunk's weights), then the readout of every query with
    the final weights.  b >= N is exactly the full-batch layer."""
    d, eta = 8, 0.7
    Q, K, V = (RNG.standard_normal((2, 1, N, d)) for _ in range(3))
    W0 = RNG.standard_normal((1, d, d)) / np.sqrt(d)
    Z, W1 = oracle.linear_minibatch(Q, K, V, W0, eta, b, "epoch")
    for img in range(2):
        W = W0.copy()
        for s0 in range(0, N, b):
            sl = slice(s0, min(N, s0 + b))
            _, Wn = oracle.linear(Q[img:img + 1, :, sl], K[img:img + 1, :, sl], V[img:img + 1, :, sl], W, eta)
            W = Wn[0]
        np.testing.assert_allclose(W1[img, 0], W[0], atol=1e-12, rtol=0)
        np.testing.assert_allclose(Z[img, 0], Q[img, 0] @ W[0].T, atol=1e-12, rtol=0)
    if b >= N:
        Zf, W1f = oracle.linear(Q, K, V, W0, eta)
        np.testing.assert_allclose(Z, Zf, atol=1e-12, rtol=0)


@pytest.mark.parametrize("mode", ["prefix", "epoch"])
def test_minibatch_invariants(mode):
    """eta = 0 reads out through W0; values that W0 reproduces exactly give no update at all.  Keys
    are unit rows (as in the layer's inputs), so that the prefix recurrence contracts and the
    rounding left in V - W0 K is not amplified from batch to batch."""
    N, d, b = 45, 8, 16
    Q, K = RNG.standard_normal((1, 2, N, d)), RNG.standard_normal((1, 2, N, d))
    K /= np.linalg.norm(K, axis=-1, keepdims=True)
    W0 = RNG.standard_normal((2, d, d))
    V = np.einsum("hij,bhnj->bhni", W0, K)
    for eta, V_ in ((0.0, RNG.standard_normal((1, 2, N, d))), (0.2, V)):
        Z, W1 = oracle.linear_minibatch(Q, K, V_, W0, eta, b, mode)
        np.testing.assert_allclose(W1, np.broadcast_to(W0, W1.shape), atol=1e-12, rtol=0)
        np.testing.assert_allclose(Z, np.einsum("hij,bhnj->bhni", W0, Q), atol=1e-12, rtol=0)


@pytest.mark.parametrize("mistake", ["running_weights", "mean_scale"])
def test_planted_mistakes_fail_the_minibatch_pins(mistake):
    """A plausible mistake planted in a CPU copy of the prefix recurrence fails the pins above:
    gradients taken at the running weights instead of the batch's start weights (fails the b = N
    prefix pin), or a mean instead of a sum inside the batch (fails the b = 1 pin unless b = 1,
    so it is checked at b = N)."""
    N, d, eta = 12, 6, 0.05
    Q, K, V = (RNG.standard_normal((N, d)) for _ in range(3))
    W0 = RNG.standard_normal((d, d)) / np.sqrt(d)
    W = W0.copy()
    Wt = W0.copy()
    Z = np.empty_like(Q)
    for t in range(N):
        Wg = Wt if mistake == "running_weights" else W
        scale = eta / N if mistake == "mean_scale" else eta
        Wt = Wt - scale * 2.0 * np.outer(Wg @ K[t] - V[t], K[t])
        Z[t] = Wt @ Q[t]
    Zo, _ = oracle.linear_minibatch(Q[None, None], K[None, None], V[None, None], W0[None], eta, N, "prefix")
    assert not np.allclose(Z, Zo[0, 0], atol=1e-9, rtol=0)


# ------------------------------------------------------------------------------------------------
# backward pass of the linear head
# ------------------------------------------------------------------------------------------------
def _bwd_case(B=2, H=2, N=9, d=5, seed=0):
    r = np.random.default_rng(100 + seed)
    Q, K, V, dZ = (r.standard_normal((B, H, N, d)) for _ in range(4))
    W0 = r.standard_normal((H, d, d)) / np.sqrt(d)
    return Q, K, V, W0, dZ


def _fwd_loss(Q, K, V, W0, eta, dZ):
    """L = sum dZ * Z with Z from the pinned forward oracle."""
    Z, _ = oracle.linear(Q, K, V, W0, eta)
    return float(np.sum(dZ * Z))


def test_linear_backward_matches_central_differences_of_the_forward_oracle():
    """Every gradient the backward oracle returns equals the central difference of the pinned
    forward oracle's L = sum dZ * Z, on a few entries of each input and on eta."""
    Q, K, V, W0, dZ = _bwd_case()
    eta, h = 0.7, 1e-5
    dQ, dK, dV, dW0, deta = oracle.linear_backward(Q, K, V, W0, eta, dZ)
    grads = {"Q": dQ, "K": dK, "V": dV, "W0": dW0}
    args = {"Q": Q, "K": K, "V": V, "W0": W0}
    r = np.random.default_rng(5)
    for name, g in grads.items():
        for _ in range(6):
            idx = tuple(int(r.integers(0, n)) for n in args[name].shape)
            plus = {k: v.copy() for k, v in args.items()}
            minus = {k: v.copy() for k, v in args.items()}
            plus[name][idx] += h
            minus[name][idx] -= h
            fd = (_fwd_loss(plus["Q"], plus["K"], plus["V"], plus["W0"], eta, dZ) -
                  _fwd_loss(minus["Q"], minus["K"], minus["V"], minus["W0"], eta, dZ)) / (2 * h)
            assert abs(g[idx] - fd) <= 1e-6 * max(1.0, abs(fd)), (name, idx, g[idx], fd)
    fd = (_fwd_loss(Q, K, V, W0, eta + h, dZ) - _fwd_loss(Q, K, V, W0, eta - h, dZ)) / (2 * h)
    assert abs(deta - fd) <= 1e-6 * max(1.0, abs(fd))


def test_linear_backward_matches_torch_autograd():
    Q, K, V, W0, dZ = _bwd_case(B=2, H=3, N=17, d=8, seed=1)
    eta = 0.4
    dQ, dK, dV, dW0, deta = oracle.linear_backward(Q, K, V, W0, eta, dZ)
    tQ, tK, tV, tW = (torch.tensor(a, requires_grad=True) for a in (Q, K, V, W0))
    te = torch.tensor(eta, dtype=torch.float64, requires_grad=True)
    N = Q.shape[2]
    r = (tK @ tW.transpose(-1, -2)[None]) - tV                       # [B][H][N][d]: W0 k - v
    grad = 2.0 / N * (r.transpose(-1, -2) @ tK)                      # (2/N) sum (W0 k - v) k^T
    W1 = tW[None] - te * grad
    Z = tQ @ W1.transpose(-1, -2)
    (Z * torch.tensor(dZ)).sum().backward()
    np.testing.assert_allclose(dQ, tQ.grad.numpy(), atol=1e-10, rtol=0)
    np.testing.assert_allclose(dK, tK.grad.numpy(), atol=1e-10, rtol=0)
    np.testing.assert_allclose(dV, tV.grad.numpy(), atol=1e-10, rtol=0)
    np.testing.assert_allclose(dW0, tW.grad.numpy(), atol=1e-10, rtol=0)
    assert abs(deta - te.grad.item()) <= 1e-10 * max(1.0, abs(deta))


def test_linear_backward_special_cases():
    """dZ = 0 gives zero gradients; eta = 0 makes the layer z = W0 q, so dQ = W0^T dz, dK = dV = 0
    and dW0 = sum over images of dZ^T Q."""
    Q, K, V, W0, dZ = _bwd_case(B=3, H=2, N=11, d=6, seed=2)
    out = oracle.linear_backward(Q, K, V, W0, 0.9, np.zeros_like(dZ))
    for a in out[:4]:
        assert np.all(a == 0.0)
    assert out[4] == 0.0
    dQ, dK, dV, dW0, _ = oracle.linear_backward(Q, K, V, W0, 0.0, dZ)
    np.testing.assert_allclose(dQ, np.einsum("hij,bhni->bhnj", W0, dZ), atol=1e-12, rtol=0)
    assert np.all(dK == 0.0) and np.all(dV == 0.0)
    np.testing.assert_allclose(dW0, np.einsum("bhni,bhnj->hij", dZ, Q), atol=1e-12, rtol=0)


def test_planted_mistake_fails_the_backward_pin():
    """Dropping the transposed half of the Gram gradient (dG k instead of (dG + dG^T) k), planted in
    a CPU copy of the key gradient, disagrees with the central differences."""
    Q, K, V, W0, dZ = _bwd_case(B=1, H=1, N=7, d=4, seed=3)
    eta, h = 0.7, 1e-5
    dQ, dK, dV, _, _ = oracle.linear_backward(Q, K, V, W0, eta, dZ)
    N = Q.shape[2]
    s = 2 * eta / N
    dW1 = dZ[0, 0].T @ Q[0, 0]
    dG = -s * W0[0].T @ dW1
    bad = dK[0, 0] - (K[0, 0] @ dG)                      # remove the dG^T k half
    idx = (0, 0, 3, 2)
    plus, minus = K.copy(), K.copy()
    plus[idx] += h
    minus[idx] -= h
    fd = (_fwd_loss(Q, plus, V, W0, eta, dZ) - _fwd_loss(Q, minus, V, W0, eta, dZ)) / (2 * h)
    assert abs(dK[idx] - fd) <= 1e-6 * max(1.0, abs(fd))
    assert abs(bad[3, 2] - fd) > 1e-4


# ------------------------------------------------------------------------------------------------
# backward pass of the depthwise-conv head
# ------------------------------------------------------------------------------------------------
def _cbwd_case(B=2, H=2, Hg=4, Wg=5, d=3, seed=0):
    r = np.random.default_rng(200 + seed)
    N = Hg * Wg
    Q, K, V, dZ = (r.standard_normal((B, H, N, d)) for _ in range(4))
    W0 = r.standard_normal((H, d, 3, 3)) / 3.0
    return Q, K, V, W0, dZ


def _cfwd_loss(Q, K, V, W0, eta, dZ, Hg, Wg):
    """L = sum dZ * Z with Z from the pinned forward oracle of the depthwise-conv head."""
    Z, _ = oracle.dwconv(Q, K, V, W0, eta, Hg, Wg)
    return float(np.sum(dZ * Z))


@pytest.mark.parametrize("Hg,Wg", [(4, 5), (1, 6), (3, 1)])
def test_dwconv_backward_matches_central_differences_of_the_forward_oracle(Hg, Wg):
    Q, K, V, W0, dZ = _cbwd_case(Hg=Hg, Wg=Wg)
    eta, h = 0.7, 1e-5
    dQ, dK, dV, dW0, deta = oracle.dwconv_backward(Q, K, V, W0, eta, dZ, Hg, Wg)
    grads = {"Q": dQ, "K": dK, "V": dV, "W0": dW0}
    args = {"Q": Q, "K": K, "V": V, "W0": W0}
    r = np.random.default_rng(7)
    for name, g in grads.items():
        for _ in range(8):
            idx = tuple(int(r.integers(0, n)) for n in args[name].shape)
            plus = {k: v.copy() for k, v in args.items()}
            minus = {k: v.copy() for k, v in args.items()}
            plus[name][idx] += h
            minus[name][idx] -= h
            fd = (_cfwd_loss(plus["Q"], plus["K"], plus["V"], plus["W0"], eta, dZ, Hg, Wg) -
                  _cfwd_loss(minus["Q"], minus["K"], minus["V"], minus["W0"], eta, dZ, Hg, Wg)) / (2 * h)
            assert abs(g[idx] - fd) <= 1e-6 * max(1.0, abs(fd)), (name, idx, g[idx], fd)
    fd = (_cfwd_loss(Q, K, V, W0, eta + h, dZ, Hg, Wg) - _cfwd_loss(Q, K, V, W0, eta - h, dZ, Hg, Wg)) / (2 * h)
    assert abs(deta - fd) <= 1e-6 * max(1.0, abs(fd))


def test_dwconv_backward_matches_torch_autograd():
    Hg, Wg = 6, 7
    Q, K, V, W0, dZ = _cbwd_case(B=2, H=2, Hg=Hg, Wg=Wg, d=5, seed=1)
    eta = 0.4
    dQ, dK, dV, dW0, deta = oracle.dwconv_backward(Q, K, V, W0, eta, dZ, Hg, Wg)
    tQ, tK, tV, tW = (torch.tensor(a, requires_grad=True) for a in (Q, K, V, W0))
    te = torch.tensor(eta, dtype=torch.float64, requires_grad=True)
    B, H, N, d = Q.shape
    tot = 0.0
    for b in range(B):
        for hh in range(H):
            r = _torch_conv_f(tK[b, hh], tW[hh], Hg, Wg) - tV[b, hh]
            Wv = tW[hh]
            g = torch.stack([torch.stack([
                (r * _shifted(tK[b, hh], a, bb, Hg, Wg)).sum(0) for bb in range(3)], -1) for a in range(3)], -2)
            W1 = Wv - te * (2.0 / N) * g
            Z = _torch_conv_f(tQ[b, hh], W1, Hg, Wg)
            tot = tot + (Z * torch.tensor(dZ[b, hh])).sum()
    tot.backward()
    np.testing.assert_allclose(dQ, tQ.grad.numpy(), atol=1e-10, rtol=0)
    np.testing.assert_allclose(dK, tK.grad.numpy(), atol=1e-10, rtol=0)
    np.testing.assert_allclose(dV, tV.grad.numpy(), atol=1e-10, rtol=0)
    np.testing.assert_allclose(dW0, tW.grad.numpy(), atol=1e-10, rtol=0)
    assert abs(deta - te.grad.item()) <= 1e-10 * max(1.0, abs(deta))


def _shifted(X, a, b, Hg, Wg):
    """X [N][d] read at grid offset (a-1, b-1) with zero padding: row p holds X[p + s]."""
    N, d = X.shape
    img = X.T.reshape(d, Hg, Wg)
    pad = F.pad(img, (1, 1, 1, 1))
    return pad[:, a:a + Hg, b:b + Wg].reshape(d, N).T


def test_dwconv_backward_special_cases():
    """dZ = 0 gives zero gradients; eta = 0 makes the head Z = f(Q; W0): dK = dV = 0, dQ is the
    transposed depthwise conv of dZ (torch conv_transpose2d) and dW0 = sum dZ Q[shifted]."""
    Hg, Wg = 5, 6
    Q, K, V, W0, dZ = _cbwd_case(B=3, H=2, Hg=Hg, Wg=Wg, d=4, seed=2)
    out = oracle.dwconv_backward(Q, K, V, W0, 0.9, np.zeros_like(dZ), Hg, Wg)
    for a in out[:4]:
        assert np.all(a == 0.0)
    assert out[4] == 0.0
    dQ, dK, dV, dW0, deta = oracle.dwconv_backward(Q, K, V, W0, 0.0, dZ, Hg, Wg)
    assert np.all(dK == 0.0) and np.all(dV == 0.0)
    d = Q.shape[3]
    for b in range(3):
        for h in range(2):
            img = torch.tensor(dZ[b, h].T.reshape(1, d, Hg, Wg))
            ref = F.conv_transpose2d(img, torch.tensor(W0[h]).reshape(d, 1, 3, 3), padding=1, groups=d)
            np.testing.assert_allclose(dQ[b, h], ref.reshape(d, Hg * Wg).T.numpy(), atol=1e-12, rtol=0)
    ref_w = np.zeros_like(W0)
    for b in range(3):
        for h in range(2):
            for a in range(3):
                for bb in range(3):
                    ref_w[h, :, a, bb] += (dZ[b, h] * _shifted(torch.tensor(Q[b, h]), a, bb, Hg, Wg).numpy()).sum(0)
    np.testing.assert_allclose(dW0, ref_w, atol=1e-12, rtol=0)


def test_planted_mistake_fails_the_conv_backward_pin():
    """Dropping the term of dK that flows through the gradient's own K factor ((2/N) dg r[q - s]),
    planted in a CPU copy, disagrees with the central differences."""
    Hg, Wg = 4, 4
    Q, K, V, W0, dZ = _cbwd_case(B=1, H=1, Hg=Hg, Wg=Wg, d=2, seed=3)
    eta, h = 0.7, 1e-5
    dQ, dK, dV, _, _ = oracle.dwconv_backward(Q, K, V, W0, eta, dZ, Hg, Wg)
    N = Hg * Wg
    c, qy, qx = 1, 2, 1
    Kt = torch.tensor(K[0, 0])
    r = (_torch_conv_f(Kt, torch.tensor(W0[0]), Hg, Wg) - torch.tensor(V[0, 0])).numpy()
    dW1 = np.array([[(dZ[0, 0][:, c] * _shifted(torch.tensor(Q[0, 0]), a, b, Hg, Wg).numpy()[:, c]).sum()
                     for b in range(3)] for a in range(3)])
    dg = -eta * dW1
    term = 0.0
    for a in range(3):
        for b in range(3):
            yy, xx = qy - (a - 1), qx - (b - 1)
            if 0 <= yy < Hg and 0 <= xx < Wg:
                term += (2.0 / N) * dg[a, b] * r[yy * Wg + xx, c]
    idx = (0, 0, qy * Wg + qx, c)
    bad = dK[idx] - term
    plus, minus = K.copy(), K.copy()
    plus[idx] += h
    minus[idx] -= h
    fd = (_cfwd_loss(Q, plus, V, W0, eta, dZ, Hg, Wg) - _cfwd_loss(Q, minus, V, W0, eta, dZ, Hg, Wg)) / (2 * h)
    assert abs(dK[idx] - fd) <= 1e-6 * max(1.0, abs(fd))
    assert abs(bad - fd) > 1e-4


# ------------------------------------------------------------------------------------------------
# depthwise 3x3 conv head
# ------------------------------------------------------------------------------------------------
def test_dwconv_gradient_exact_rational_fd():
    Hg, Wg, d, eta = 3, 4, 2, 1.0
    N = Hg * Wg
    K = _small_ints((N, d)); V = _small_ints((N, d)); Q = _small_ints((N, d))
    W0 = _small_ints((d, 3, 3))
    _, W1 = oracle.dwconv(Q[None, None], K[None, None], V[None, None], W0[None], eta, Hg, Wg)
    grad = (W0 - W1[0, 0]) / eta
    Kf = [[Fraction(int(v)) for v in row] for row in K]
    Vf = [[Fraction(int(v)) for v in row] for row in V]
    Wf = [[[Fraction(int(v)) for v in r] for r in W0[c]] for c in range(d)]
    for c in range(d):
        for a in range(3):
            for b in range(3):
                Wp = [[r[:] for r in ch] for ch in Wf]; Wm = [[r[:] for r in ch] for ch in Wf]
                Wp[c][a][b] += 1; Wm[c][a][b] -= 1
                exact = (_frac_loss_conv(Wp, Kf, Vf, Hg, Wg) - _frac_loss_conv(Wm, Kf, Vf, Hg, Wg)) / 2
                assert abs(grad[c, a, b] - float(exact)) <= 1e-12 * max(1.0, abs(float(exact)))


@pytest.mark.parametrize("Hg,Wg", [(5, 7), (1, 6), (6, 1), (1, 1)])
def test_dwconv_eta_zero_is_torch_conv2d(Hg, Wg):
    d = 8
    N = Hg * Wg
    Q, K, V = (RNG.standard_normal((1, 2, N, d)) for _ in range(3))
    W0 = RNG.standard_normal((2, d, 3, 3))
    Z, W1 = oracle.dwconv(Q, K, V, W0, 0.0, Hg, Wg)
    for h in range(2):
        ref = _torch_conv_f(torch.tensor(Q[0, h]), torch.tensor(W0[h]), Hg, Wg).numpy()
        np.testing.assert_allclose(Z[0, h], ref, atol=1e-13, rtol=0)


@pytest.mark.parametrize("Hg,Wg", [(6, 5), (1, 9), (4, 1)])
def test_dwconv_matches_torch_autograd(Hg, Wg):
    d, eta = 6, 0.5
    N = Hg * Wg
    Q, K, V = (RNG.standard_normal((1, 1, N, d)) for _ in range(3))
    W0 = RNG.standard_normal((1, d, 3, 3))
    Z, W1 = oracle.dwconv(Q, K, V, W0, eta, Hg, Wg)
    W = torch.tensor(W0[0], requires_grad=True)
    r = _torch_conv_f(torch.tensor(K[0, 0]), W, Hg, Wg) - torch.tensor(V[0, 0])
    loss = (r ** 2).sum(-1).mean()
    loss.backward()
    W1_ref = (W - eta * W.grad).detach()
    np.testing.assert_allclose(W1[0, 0], W1_ref.numpy(), atol=1e-12, rtol=0)
    Zref = _torch_conv_f(torch.tensor(Q[0, 0]), W1_ref, Hg, Wg).numpy()
    np.testing.assert_allclose(Z[0, 0], Zref, atol=1e-12, rtol=0)


def test_dwconv_identity_kernel_reproduces_queries():
    Hg, Wg, d = 7, 5, 8
    N = Hg * Wg
    Q, K = RNG.standard_normal((2, 1, N, d)), RNG.standard_normal((2, 1, N, d))
    W0 = np.zeros((1, d, 3, 3)); W0[:, :, 1, 1] = 1.0
    Z, W1 = oracle.dwconv(Q, K, K.copy(), W0, 1.0, Hg, Wg)
    np.testing.assert_array_equal(W1, np.broadcast_to(W0, W1.shape))
    np.testing.assert_array_equal(Z, Q)


def test_dwconv_degenerate_grids_zero_out_missing_taps():
    d = 4
    Q, K, V = (RNG.standard_normal((1, 1, 1, d)) for _ in range(3))
    W0 = RNG.standard_normal((1, d, 3, 3))
    _, W1 = oracle.dwconv(Q, K, V, W0, 1.0, 1, 1)
    delta = W1[0, 0] - W0[0]
    mask = np.ones((3, 3), bool); mask[1, 1] = False
    assert np.all(delta[:, mask] == 0.0) and np.any(delta[:, 1, 1] != 0.0)
    Q, K, V = (RNG.standard_normal((1, 1, 9, d)) for _ in range(3))
    _, W1 = oracle.dwconv(Q, K, V, W0, 1.0, 1, 9)           # a single row: no vertical neighbours
    delta = W1[0, 0] - W0[0]
    assert np.all(delta[:, 0, :] == 0.0) and np.all(delta[:, 2, :] == 0.0)


def test_dwconv_centre_tap_matches_diagonal_linear_gradient():
    """A kernel with only the centre tap is the diagonal linear map W = diag(w); the centre-tap
    gradient must equal the diagonal of the linear head's gradient at that W."""
    Hg, Wg, d, eta = 6, 6, 8, 1.0
    N = Hg * Wg
    Q, K, V = (RNG.standard_normal((1, 1, N, d)) for _ in range(3))
    w = RNG.standard_normal(d)
    Wc = np.zeros((1, d, 3, 3)); Wc[0, :, 1, 1] = w
    _, W1c = oracle.dwconv(Q, K, V, Wc, eta, Hg, Wg)
    _, W1l = oracle.linear(Q, K, V, np.diag(w)[None], eta)
    np.testing.assert_allclose((Wc[0, :, 1, 1] - W1c[0, 0, :, 1, 1]),
                               np.diag(np.diag(w) - W1l[0, 0]), atol=1e-12, rtol=0)


# ------------------------------------------------------------------------------------------------
# full 3x3 conv head: f(X;W)[c,y,x] = sum_{c',a,b} W[c][c'][a][b] X[c', y+a-1, x+b-1]
# ------------------------------------------------------------------------------------------------
def _frac_loss_conv3x3(W, K, V, Hg, Wg):
    """(1/N) sum_{c,y,x} (f(K;W)[c,y,x] - V[c,y,x])^2 in exact rational arithmetic, the dense
    cross-correlation written from its definition (every output channel reads every input one)."""
    d = len(K[0])
    tot = Fraction(0)
    for c in range(d):
        for y in range(Hg):
            for x in range(Wg):
                f = Fraction(0)
                for cp in range(d):
                    for a in range(3):
                        for b in range(3):
                            yy, xx = y + a - 1, x + b - 1
                            if 0 <= yy < Hg and 0 <= xx < Wg:
                                f += W[c][cp][a][b] * K[yy * Wg + xx][cp]
                r = f - V[y * Wg + x][c]
                tot += r * r
    return tot / (Hg * Wg)


def _conv3x3_fd_grad(W0, K, V, Hg, Wg, entries):
    """Exact central differences (step 1; the loss is quadratic in W) at the listed entries."""
    Kf = [[Fraction(int(v)) for v in row] for row in K]
    Vf = [[Fraction(int(v)) for v in row] for row in V]
    Wf = [[[[Fraction(int(v)) for v in r] for r in W0[c][cp]] for cp in range(W0.shape[1])] for c in range(W0.shape[0])]
    out = {}
    for (c, cp, a, b) in entries:
        Wp = [[[r[:] for r in k] for k in ch] for ch in Wf]
        Wm = [[[r[:] for r in k] for k in ch] for ch in Wf]
        Wp[c][cp][a][b] += 1
        Wm[c][cp][a][b] -= 1
        out[(c, cp, a, b)] = float((_frac_loss_conv3x3(Wp, Kf, Vf, Hg, Wg) - _frac_loss_conv3x3(Wm, Kf, Vf, Hg, Wg)) / 2)
    return out


def _torch_conv3x3_f(X, W, Hg, Wg):
    """Full 3x3 cross-correlation through torch.conv2d (groups=1): X [N][d] -> [N][d]."""
    N, d = X.shape
    img = X.T.reshape(1, d, Hg, Wg)
    return F.conv2d(img, W, padding=1).reshape(W.shape[0], N).T


def test_conv3x3_gradient_exact_rational_fd():
    Hg, Wg, d, eta = 3, 4, 2, 1.0
    N = Hg * Wg
    K = _small_ints((N, d)); V = _small_ints((N, d)); Q = _small_ints((N, d))
    W0 = _small_ints((d, d, 3, 3))
    _, W1 = oracle.conv3x3(Q[None, None], K[None, None], V[None, None], W0[None], eta, Hg, Wg)
    grad = (W0 - W1[0, 0]) / eta
    entries = [(c, cp, a, b) for c in range(d) for cp in range(d) for a in range(3) for b in range(3)]
    fd = _conv3x3_fd_grad(W0, K, V, Hg, Wg, entries)
    for e, exact in fd.items():
        assert abs(grad[e] - exact) <= 1e-12 * max(1.0, abs(exact)), e


@pytest.mark.parametrize("mistake", ["sign", "transposed_channels", "flipped_taps", "half_scale"])
def test_planted_mistakes_fail_the_conv3x3_pin(mistake):
    """A copy of the oracle's gradient with a planted mistake must disagree with the exact
    differences: the pin detects sign, channel-transpose, tap-flip and scale errors."""
    Hg, Wg, d, eta = 3, 4, 2, 1.0
    N = Hg * Wg
    K = _small_ints((N, d)); V = _small_ints((N, d)); Q = _small_ints((N, d))
    W0 = _small_ints((d, d, 3, 3))
    _, W1 = oracle.conv3x3(Q[None, None], K[None, None], V[None, None], W0[None], eta, Hg, Wg)
    grad = (W0 - W1[0, 0]) / eta
    bad = {"sign": -grad, "transposed_channels": grad.transpose(1, 0, 2, 3),
           "flipped_taps": grad[:, :, ::-1, ::-1], "half_scale": grad / 2}[mistake]
    entries = [(c, cp, a, b) for c in range(d) for cp in range(d) for a in range(3) for b in range(3)]
    fd = _conv3x3_fd_grad(W0, K, V, Hg, Wg, entries)
    assert max(abs(bad[e] - v) for e, v in fd.items()) > 1e-6


@pytest.mark.parametrize("Hg,Wg", [(5, 7), (1, 6), (6, 1), (1, 1)])
def test_conv3x3_eta_zero_is_torch_conv2d(Hg, Wg):
    d = 6
    N = Hg * Wg
    Q, K, V = (RNG.standard_normal((1, 2, N, d)) for _ in range(3))
    W0 = RNG.standard_normal((2, d, d, 3, 3))
    Z, W1 = oracle.conv3x3(Q, K, V, W0, 0.0, Hg, Wg)
    for h in range(2):
        ref = _torch_conv3x3_f(torch.tensor(Q[0, h]), torch.tensor(W0[h]), Hg, Wg).numpy()
        np.testing.assert_allclose(Z[0, h], ref, atol=1e-12, rtol=0)
        np.testing.assert_array_equal(W1[0, h], W0[h])


@pytest.mark.parametrize("Hg,Wg", [(6, 5), (1, 9), (4, 1)])
def test_conv3x3_matches_torch_autograd(Hg, Wg):
    d, eta = 5, 0.5
    N = Hg * Wg
    Q, K, V = (RNG.standard_normal((1, 1, N, d)) for _ in range(3))
    W0 = RNG.standard_normal((1, d, d, 3, 3)) * 0.3
    Z, W1 = oracle.conv3x3(Q, K, V, W0, eta, Hg, Wg)
    W = torch.tensor(W0[0], requires_grad=True)
    r = _torch_conv3x3_f(torch.tensor(K[0, 0]), W, Hg, Wg) - torch.tensor(V[0, 0])
    loss = (r ** 2).sum(-1).mean()
    loss.backward()
    W1_ref = (W - eta * W.grad).detach()
    np.testing.assert_allclose(W1[0, 0], W1_ref.numpy(), atol=1e-12, rtol=0)
    Zref = _torch_conv3x3_f(torch.tensor(Q[0, 0]), W1_ref, Hg, Wg).numpy()
    np.testing.assert_allclose(Z[0, 0], Zref, atol=1e-12, rtol=0)


def test_conv3x3_channel_diagonal_kernel_reduces_to_depthwise_head():
    """With W0[c][c'] = 0 for c != c', the residual is the depthwise head's, so the diagonal of the
    dense update equals the depthwise update (the off-diagonal entries move too)."""
    Hg, Wg, d, eta = 6, 5, 6, 0.7
    N = Hg * Wg
    Q, K, V = (RNG.standard_normal((2, 1, N, d)) for _ in range(3))
    Wdw = RNG.standard_normal((1, d, 3, 3))
    Wfull = np.zeros((1, d, d, 3, 3))
    for c in range(d):
        Wfull[0, c, c] = Wdw[0, c]
    _, W1f = oracle.conv3x3(Q, K, V, Wfull, eta, Hg, Wg)
    _, W1d = oracle.dwconv(Q, K, V, Wdw, eta, Hg, Wg)
    for c in range(d):
        np.testing.assert_allclose(W1f[:, 0, c, c], W1d[:, 0, c], atol=1e-12, rtol=0)
    off = W1f[:, 0] - Wfull[0][None]
    assert np.abs(off[:, 0, 1]).max() > 0.0


def test_conv3x3_single_token_grid_is_the_linear_head():
    """On a 1 x 1 grid only the centre tap sees a token: the centre taps are the linear head's W
    (same update, same readout) and every other tap gets no update."""
    d, eta = 6, 0.8
    Q, K, V = (RNG.standard_normal((3, 1, 1, d)) for _ in range(3))
    W0 = RNG.standard_normal((1, d, d, 3, 3))
    Z, W1 = oracle.conv3x3(Q, K, V, W0, eta, 1, 1)
    Zl, W1l = oracle.linear(Q, K, V, W0[:, :, :, 1, 1], eta)
    np.testing.assert_allclose(W1[:, 0, :, :, 1, 1], W1l[:, 0], atol=1e-12, rtol=0)
    np.testing.assert_allclose(Z, Zl, atol=1e-12, rtol=0)
    mask = np.ones((3, 3), bool); mask[1, 1] = False
    assert np.all(W1[:, 0][..., mask] == np.broadcast_to(W0[0][..., mask], W1[:, 0][..., mask].shape))


def test_conv3x3_reproduced_values_give_no_update():
    Hg, Wg, d = 5, 6, 4
    N = Hg * Wg
    Q, K = RNG.standard_normal((1, 1, N, d)), RNG.standard_normal((1, 1, N, d))
    W0 = RNG.standard_normal((1, d, d, 3, 3))
    V = _torch_conv3x3_f(torch.tensor(K[0, 0]), torch.tensor(W0[0]), Hg, Wg).numpy()[None, None]
    _, W1 = oracle.conv3x3(Q, K, V, W0, 1.0, Hg, Wg)
    np.testing.assert_allclose(W1[0, 0], W0[0], atol=1e-12, rtol=0)


# ------------------------------------------------------------------------------------------------
# depthwise 3x3 conv head, dot-product inner loss  L(W) = -(1/N) sum <f(K;W), V>
# ------------------------------------------------------------------------------------------------
def _frac_loss_conv_dot(W, K, V, Hg, Wg):
    d = len(K[0])
    tot = Fraction(0)
    for c in range(d):
        for y in range(Hg):
            for x in range(Wg):
                tot += _frac_conv(W[c], K, Hg, Wg, c, y, x) * V[y * Wg + x][c]
    return -tot / (Hg * Wg)


def _conv_dot_fd_grad(W0, K, V, Hg, Wg):
    d = W0.shape[0]
    Kf = [[Fraction(int(v)) for v in row] for row in K]
    Vf = [[Fraction(int(v)) for v in row] for row in V]
    Wf = [[[Fraction(int(v)) for v in r] for r in W0[c]] for c in range(d)]
    g = np.zeros((d, 3, 3))
    for c in range(d):
        for a in range(3):
            for b in range(3):
                Wp = [[r[:] for r in ch] for ch in Wf]; Wm = [[r[:] for r in ch] for ch in Wf]
                Wp[c][a][b] += 1; Wm[c][a][b] -= 1
                g[c, a, b] = float((_frac_loss_conv_dot(Wp, Kf, Vf, Hg, Wg) -
                                    _frac_loss_conv_dot(Wm, Kf, Vf, Hg, Wg)) / 2)
    return g


def test_dwconv_dot_gradient_exact_rational_fd():
    Hg, Wg, d, eta = 3, 4, 2, 1.0
    N = Hg * Wg
    K = _small_ints((N, d)); V = _small_ints((N, d)); Q = _small_ints((N, d))
    W0 = _small_ints((d, 3, 3))
    _, W1 = oracle.dwconv_dot(Q[None, None], K[None, None], V[None, None], W0[None], eta, Hg, Wg)
    grad = (W0 - W1[0, 0]) / eta
    np.testing.assert_allclose(grad, _conv_dot_fd_grad(W0, K, V, Hg, Wg), atol=1e-12, rtol=0)


@pytest.mark.parametrize("mistake", ["sign", "two_over_n", "flipped_taps", "l2_residual"])
def test_planted_mistakes_fail_the_conv_dot_pin(mistake):
    """A plausible mistake planted in the oracle's conv gradient (on the CPU) fails the exact-FD pin."""
    Hg, Wg, d = 3, 4, 2
    N = Hg * Wg
    K = _small_ints((N, d)); V = _small_ints((N, d)); Q = _small_ints((N, d))
    W0 = _small_ints((d, 3, 3))
    _, W1 = oracle.dwconv_dot(Q[None, None], K[None, None], V[None, None], W0[None], 1.0, Hg, Wg)
    grad = W0 - W1[0, 0]
    _, W1l2 = oracle.dwconv(Q[None, None], K[None, None], V[None, None], W0[None], 1.0, Hg, Wg)
    bad = {"sign": -grad, "two_over_n": 2 * grad, "flipped_taps": grad[:, ::-1, ::-1],
           "l2_residual": W0 - W1l2[0, 0]}[mistake]
    assert not np.allclose(bad, _conv_dot_fd_grad(W0, K, V, Hg, Wg), atol=1e-9, rtol=0)


@pytest.mark.parametrize("Hg,Wg", [(6, 5), (1, 9), (4, 1)])
def test_dwconv_dot_matches_torch_autograd(Hg, Wg):
    d, eta = 6, 1.0
    N = Hg * Wg
    Q, K, V = (RNG.standard_normal((1, 1, N, d)) for _ in range(3))
    W0 = RNG.standard_normal((1, d, 3, 3))
    Z, W1 = oracle.dwconv_dot(Q, K, V, W0, eta, Hg, Wg)
    W = torch.tensor(W0[0], requires_grad=True)
    loss = -(_torch_conv_f(torch.tensor(K[0, 0]), W, Hg, Wg) * torch.tensor(V[0, 0])).sum(-1).mean()
    loss.backward()
    W1_ref = (W - eta * W.grad).detach()
    np.testing.assert_allclose(W1[0, 0], W1_ref.numpy(), atol=1e-12, rtol=0)
    Zref = _torch_conv_f(torch.tensor(Q[0, 0]), W1_ref, Hg, Wg).numpy()
    np.testing.assert_allclose(Z[0, 0], Zref, atol=1e-12, rtol=0)


def test_dwconv_dot_centre_tap_matches_linear_dot_diagonal_and_update_ignores_w0():
    Hg, Wg, d, eta = 5, 7, 8, 0.9
    N = Hg * Wg
    Q, K, V = (RNG.standard_normal((1, 1, N, d)) for _ in range(3))
    Wa, Wb = RNG.standard_normal((1, d, 3, 3)), RNG.standard_normal((1, d, 3, 3))
    _, W1a = oracle.dwconv_dot(Q, K, V, Wa, eta, Hg, Wg)
    _, W1b = oracle.dwconv_dot(Q, K, V, Wb, eta, Hg, Wg)
    np.testing.assert_allclose(W1a[0, 0] - Wa[0], W1b[0, 0] - Wb[0], atol=1e-12, rtol=0)
    _, W1l = oracle.linear_dot(Q, K, V, np.zeros((1, d, d)), eta)
    np.testing.assert_allclose(W1a[0, 0, :, 1, 1] - Wa[0, :, 1, 1], np.diag(W1l[0, 0]), atol=1e-12, rtol=0)
    _, W1 = oracle.dwconv_dot(Q[:, :, :1], K[:, :, :1], V[:, :, :1], Wa, eta, 1, 1)   # one token
    delta = W1[0, 0] - Wa[0]
    mask = np.ones((3, 3), bool); mask[1, 1] = False
    assert np.all(delta[:, mask] == 0.0)


# ------------------------------------------------------------------------------------------------
# MLP head
# ------------------------------------------------------------------------------------------------
def test_gelu_tanh_matches_torch():
    us = np.concatenate([np.linspace(-8, 8, 401), RNG.standard_normal(200) * 3])
    ut = torch.tensor(us, requires_grad=True)
    gt = F.gelu(ut, approximate="tanh")
    gt.sum().backward()
    for u, g, dg in zip(us, gt.detach().numpy(), ut.grad.numpy()):
        assert abs(oracle.gelu_tanh(u) - g) <= 1e-14 * max(1.0, abs(g))
        assert abs(oracle.gelu_tanh_deriv(u) - dg) <= 1e-13


def _torch_mlp(X, Wa, Wb):
    return F.gelu(X @ Wa.T, approximate="tanh") @ Wb.T


def test_mlp_eta_zero_is_plain_readout():
    B, H, N, d, hid = 1, 2, 23, 8, 32
    Q, K, V = (RNG.standard_normal((B, H, N, d)) for _ in range(3))
    Wa, Wb = RNG.standard_normal((H, hid, d)) / 3, RNG.standard_normal((H, d, hid)) / 6
    Z, Wa1, Wb1 = oracle.mlp(Q, K, V, Wa, Wb, 0.0)
    for h in range(H):
        ref = _torch_mlp(torch.tensor(Q[0, h]), torch.tensor(Wa[h]), torch.tensor(Wb[h])).numpy()
        np.testing.assert_allclose(Z[0, h], ref, atol=1e-13, rtol=0)


def test_mlp_matches_torch_autograd():
    B, H, N, d, hid, eta = 2, 1, 31, 8, 32, 0.5
    Q, K, V = (RNG.standard_normal((B, H, N, d)) for _ in range(3))
    Wa, Wb = RNG.standard_normal((H, hid, d)) / 3, RNG.standard_normal((H, d, hid)) / 6
    Z, Wa1, Wb1 = oracle.mlp(Q, K, V, Wa, Wb, eta)
    for b in range(B):
        A = torch.tensor(Wa[0], requires_grad=True)
        Bm = torch.tensor(Wb[0], requires_grad=True)
        r = _torch_mlp(torch.tensor(K[b, 0]), A, Bm) - torch.tensor(V[b, 0])
        loss = (r ** 2).sum(-1).mean()
        loss.backward()
        A1, B1 = (A - eta * A.grad).detach(), (Bm - eta * Bm.grad).detach()
        np.testing.assert_allclose(Wa1[b, 0], A1.numpy(), atol=1e-12, rtol=0)
        np.testing.assert_allclose(Wb1[b, 0], B1.numpy(), atol=1e-12, rtol=0)
        np.testing.assert_allclose(Z[b, 0], _torch_mlp(torch.tensor(Q[b, 0]), A1, B1).numpy(),
                                   atol=1e-12, rtol=0)


def test_mlp_central_differences():
    N, d, hid, eta = 17, 4, 8, 1.0
    Q, K, V = (RNG.standard_normal((1, 1, N, d)) for _ in range(3))
    Wa, Wb = RNG.standard_normal((1, hid, d)) / 2, RNG.standard_normal((1, d, hid)) / 3
    _, Wa1, Wb1 = oracle.mlp(Q, K, V, Wa, Wb, eta)
    gA, gB = (Wa[0] - Wa1[0, 0]) / eta, (Wb[0] - Wb1[0, 0]) / eta

    def loss(A, Bm):
        H = K[0, 0] @ A.T
        Aact = 0.5 * H * (1 + np.tanh(np.sqrt(2 / np.pi) * (H + 0.044715 * H ** 3)))
        return np.mean(np.sum((Aact @ Bm.T - V[0, 0]) ** 2, axis=-1))

    h = 1e-6
    for (i, j) in [(0, 0), (3, 2), (7, 1), (5, 3)]:
        Ap, Am = Wa[0].copy(), Wa[0].copy(); Ap[i, j] += h; Am[i, j] -= h
        assert abs((loss(Ap, Wb[0]) - loss(Am, Wb[0])) / (2 * h) - gA[i, j]) < 1e-7
    for (i, j) in [(0, 0), (2, 7), (3, 4)]:
        Bp, Bmm = Wb[0].copy(), Wb[0].copy(); Bp[i, j] += h; Bmm[i, j] -= h
        assert abs((loss(Wa[0], Bp) - loss(Wa[0], Bmm)) / (2 * h) - gB[i, j]) < 1e-7


def test_mlp_reproduced_values_give_no_update():
    N, d, hid = 40, 8, 32
    Q, K = RNG.standard_normal((1, 1, N, d)), RNG.standard_normal((1, 1, N, d))
    Wa, Wb = RNG.standard_normal((1, hid, d)) / 3, RNG.standard_normal((1, d, hid)) / 6
    V = _torch_mlp(torch.tensor(K[0, 0]), torch.tensor(Wa[0]), torch.tensor(Wb[0])).numpy()[None, None]
    _, Wa1, Wb1 = oracle.mlp(Q, K, V, Wa, Wb, 1.0)
    np.testing.assert_allclose(Wa1[0], Wa, atol=1e-13, rtol=0)
    np.testing.assert_allclose(Wb1[0], Wb, atol=1e-13, rtol=0)


# ------------------------------------------------------------------------------------------------
# backward pass of the MLP head
# ------------------------------------------------------------------------------------------------
def test_gelu_tanh_second_derivative_matches_torch():
    us = np.concatenate([np.linspace(-8, 8, 201), RNG.standard_normal(100) * 3])
    for u in us:
        ut = torch.tensor(u, dtype=torch.float64, requires_grad=True)
        (g1,) = torch.autograd.grad(F.gelu(ut, approximate="tanh"), ut, create_graph=True)
        (g2,) = torch.autograd.grad(g1, ut)
        assert abs(oracle.gelu_tanh_deriv2(u) - g2.item()) <= 1e-12 * max(1.0, abs(g2.item()))


def _mbwd_case(B=2, H=2, N=7, d=4, hid=8, seed=0):
    r = np.random.default_rng(300 + seed)
    Q, K, V, dZ = (r.standard_normal((B, H, N, d)) for _ in range(4))
    Wa = r.standard_normal((H, hid, d)) / np.sqrt(d)
    Wb = r.standard_normal((H, d, hid)) / np.sqrt(hid)
    return Q, K, V, Wa, Wb, dZ


def _mfwd_loss(Q, K, V, Wa, Wb, eta, dZ):
    """L = sum dZ * Z with Z from the pinned forward oracle of the MLP head."""
    Z, _, _ = oracle.mlp(Q, K, V, Wa, Wb, eta)
    return float(np.sum(dZ * Z))


def test_mlp_backward_matches_central_differences_of_the_forward_oracle():
    Q, K, V, Wa, Wb, dZ = _mbwd_case()
    eta, h = 0.6, 1e-5
    dQ, dK, dV, dWa, dWb, deta = oracle.mlp_backward(Q, K, V, Wa, Wb, eta, dZ)
    grads = {"Q": dQ, "K": dK, "V": dV, "Wa": dWa, "Wb": dWb}
    args = {"Q": Q, "K": K, "V": V, "Wa": Wa, "Wb": Wb}
    r = np.random.default_rng(11)
    for name, g in grads.items():
        for _ in range(8):
            idx = tuple(int(r.integers(0, n)) for n in args[name].shape)
            plus = {k: v.copy() for k, v in args.items()}
            minus = {k: v.copy() for k, v in args.items()}
            plus[name][idx] += h
            minus[name][idx] -= h
            fd = (_mfwd_loss(plus["Q"], plus["K"], plus["V"], plus["Wa"], plus["Wb"], eta, dZ) -
                  _mfwd_loss(minus["Q"], minus["K"], minus["V"], minus["Wa"], minus["Wb"], eta, dZ)) / (2 * h)
            assert abs(g[idx] - fd) <= 1e-6 * max(1.0, abs(fd)), (name, idx, g[idx], fd)
    fd = (_mfwd_loss(Q, K, V, Wa, Wb, eta + h, dZ) - _mfwd_loss(Q, K, V, Wa, Wb, eta - h, dZ)) / (2 * h)
    assert abs(deta - fd) <= 1e-6 * max(1.0, abs(fd))


def test_mlp_backward_matches_torch_autograd():
    Q, K, V, Wa, Wb, dZ = _mbwd_case(B=2, H=2, N=13, d=6, hid=12, seed=1)
    eta = 0.4
    dQ, dK, dV, dWa, dWb, deta = oracle.mlp_backward(Q, K, V, Wa, Wb, eta, dZ)
    tQ, tK, tV, tA, tB = (torch.tensor(a, requires_grad=True) for a in (Q, K, V, Wa, Wb))
    te = torch.tensor(eta, dtype=torch.float64, requires_grad=True)
    N = Q.shape[2]
    tot = 0.0
    for b in range(Q.shape[0]):
        for hh in range(Q.shape[1]):
            A, Bm = tA[hh], tB[hh]
            r = _torch_mlp(tK[b, hh], A, Bm) - tV[b, hh]
            loss = (r ** 2).sum(-1).mean()
            gA, gB = torch.autograd.grad(loss, (A, Bm), create_graph=True)
            Z = _torch_mlp(tQ[b, hh], A - te * gA, Bm - te * gB)
            tot = tot + (Z * torch.tensor(dZ[b, hh])).sum()
    tot.backward()
    for got, t in ((dQ, tQ), (dK, tK), (dV, tV), (dWa, tA), (dWb, tB)):
        np.testing.assert_allclose(got, t.grad.numpy(), atol=1e-10, rtol=0)
    assert abs(deta - te.grad.item()) <= 1e-10 * max(1.0, abs(deta))


def test_mlp_backward_special_cases():
    """dZ = 0 gives zero gradients; eta = 0 makes the head z = Wb gelu(Wa q): dK = dV = 0 and dQ,
    dWa, dWb are the plain MLP's gradients (torch autograd)."""
    Q, K, V, Wa, Wb, dZ = _mbwd_case(B=2, H=1, N=9, d=4, hid=8, seed=2)
    out = oracle.mlp_backward(Q, K, V, Wa, Wb, 0.8, np.zeros_like(dZ))
    for a in out[:5]:
        assert np.all(a == 0.0)
    assert out[5] == 0.0
    dQ, dK, dV, dWa, dWb, _ = oracle.mlp_backward(Q, K, V, Wa, Wb, 0.0, dZ)
    assert np.all(dK == 0.0) and np.all(dV == 0.0)
    tQ, tA, tB = (torch.tensor(a, requires_grad=True) for a in (Q, Wa[0], Wb[0]))
    (_torch_mlp(tQ[:, 0], tA, tB) * torch.tensor(dZ[:, 0])).sum().backward()
    np.testing.assert_allclose(dQ[:, 0], tQ.grad.numpy()[:, 0], atol=1e-12, rtol=0)
    np.testing.assert_allclose(dWa[0], tA.grad.numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dWb[0], tB.grad.numpy(), atol=1e-12, rtol=0)


def test_planted_mistake_fails_the_mlp_backward_pin():
    """Dropping the gelu'' term of dh (the path through gelu' inside the inner gradient) changes
    the key gradient by more than the central differences allow."""
    Q, K, V, Wa, Wb, dZ = _mbwd_case(B=1, H=1, N=5, d=3, hid=6, seed=3)
    eta, h = 0.9, 1e-5
    dQ, dK, _, _, _, _ = oracle.mlp_backward(Q, K, V, Wa, Wb, eta, dZ)
    N, s = Q.shape[2], 2.0 / Q.shape[2]
    _, Wa1, Wb1 = oracle.mlp(Q, K, V, Wa, Wb, eta)
    # the readout's dWa1, then the dropped term for key token n
    gel = lambda u: 0.5 * u * (1 + np.tanh(np.sqrt(2 / np.pi) * (u + 0.044715 * u ** 3)))
    d1 = np.vectorize(oracle.gelu_tanh_deriv)
    d2 = np.vectorize(oracle.gelu_tanh_deriv2)
    Hq = Q[0, 0] @ Wa1[0, 0].T
    dHq = (dZ[0, 0] @ Wb1[0, 0]) * d1(Hq)
    dWa1 = dHq.T @ Q[0, 0]
    n, i = 2, 1
    k, v = K[0, 0, n], V[0, 0, n]
    hvec = Wa[0] @ k
    rvec = Wb[0] @ gel(hvec) - v
    bvec = Wb[0].T @ rvec
    de = s * (-eta * dWa1) @ k
    dropped = (de * bvec * d2(hvec)) @ Wa[0][:, i]
    bad = dK[0, 0, n, i] - dropped
    plus, minus = K.copy(), K.copy()
    plus[0, 0, n, i] += h
    minus[0, 0, n, i] -= h
    fd = (_mfwd_loss(Q, plus, V, Wa, Wb, eta, dZ) - _mfwd_loss(Q, minus, V, Wa, Wb, eta, dZ)) / (2 * h)
    assert abs(dK[0, 0, n, i] - fd) <= 1e-6 * max(1.0, abs(fd))
    assert abs(bad - fd) > 1e-5


def test_threads_do_not_change_results():
    B, H, N, d = 3, 2, 40, 8
    Q, K, V = (RNG.standard_normal((B, H, N, d)) for _ in range(3))
    W0 = RNG.standard_normal((H, d, d))
    Z1, W1 = oracle.linear(Q, K, V, W0, 1.0, threads=1)
    Z4, W4 = oracle.linear(Q, K, V, W0, 1.0, threads=4)
    np.testing.assert_array_equal(Z1, Z4)
    np.testing.assert_array_equal(W1, W4)
