"""Pins for the oracle's expert FFN, combine and backward (CPU only).

  * E=1, k=1 reduces the layer to a dense SwiGLU FFN: compared with torch
    float64 ops, forward and autograd backward.
  * Identity experts: y[t] = (sum_j w[t, j]) x[t].
  * Forced one-hot routing: y[t] = w[t] * FFN_e(x[t]) from a dense
    per-token torch computation.
  * Central finite differences of loss = sum(y * dY) for every input the
    backward differentiates (x, W_r, W_gu, W_d, router bias), with and
    without renormalisation and with forced routing.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import moe_ref as R


def _draw(T, d, f, E, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, d))
    w_r = rng.standard_normal((E, d)) / np.sqrt(d)
    w_gu = rng.standard_normal((E, 2 * f, d)) / np.sqrt(d)
    w_d = rng.standard_normal((E, d, f)) / np.sqrt(d)
    dy = rng.standard_normal((T, d))
    return x, w_r, w_gu, w_d, dy


def test_single_expert_is_dense_swiglu_fwd_bwd():
    T, d, f = 9, 16, 12
    x, w_r, w_gu, w_d, dy = _draw(T, d, f, 1, 0)
    fwd = R.layer_fwd(x, w_r, w_gu, w_d, 1, rnd=None)
    xt = torch.tensor(x, requires_grad=True)
    wg = torch.tensor(w_gu[0, :f], requires_grad=True)
    wu = torch.tensor(w_gu[0, f:], requires_grad=True)
    wd = torch.tensor(w_d[0], requires_grad=True)
    y = (F.silu(xt @ wg.T) * (xt @ wu.T)) @ wd.T
    np.testing.assert_allclose(fwd["y"], y.detach().numpy(), rtol=1e-12, atol=1e-13)
    (y * torch.tensor(dy)).sum().backward()
    bwd = R.layer_bwd(fwd, dy, x, w_r, w_gu, w_d, rnd=None)
    np.testing.assert_allclose(bwd["dx"], xt.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(bwd["dW_gu"][0, :f], wg.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(bwd["dW_gu"][0, f:], wu.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(bwd["dW_d"][0], wd.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(bwd["dw_r"], 0.0, atol=1e-14)


def test_identity_experts_return_gate_weighted_input():
    T, d, f, E, k = 40, 8, 4, 6, 3
    x, w_r, w_gu, w_d, _ = _draw(T, d, f, E, 1)
    fwd = R.layer_fwd(x, w_r, w_gu, w_d, k, rnd=None, expert_fn=lambda e, X: X)
    np.testing.assert_allclose(fwd["y"], fwd["w"].sum(axis=1)[:, None] * x,
                               rtol=1e-13, atol=1e-14)


def test_forced_one_hot_routing_matches_dense_per_token():
    T, d, f, E = 20, 8, 6, 5
    x, w_r, w_gu, w_d, _ = _draw(T, d, f, E, 2)
    route = (np.arange(T) * 3 % E)[:, None]
    fwd = R.layer_fwd(x, w_r, w_gu, w_d, 1, route=route, rnd=None)
    p = torch.softmax(torch.tensor(x @ w_r.T), dim=1).numpy()
    for t in range(T):
        e = route[t, 0]
        xt = torch.tensor(x[t])
        h = F.silu(torch.tensor(w_gu[e, :f]) @ xt) * (torch.tensor(w_gu[e, f:]) @ xt)
        ref = p[t, e] * (torch.tensor(w_d[e]) @ h).numpy()
        np.testing.assert_allclose(fwd["y"][t], ref, rtol=1e-12, atol=1e-13)


def test_empty_experts_and_zero_gradients():
    T, d, f, E = 6, 8, 4, 5
    x, w_r, w_gu, w_d, dy = _draw(T, d, f, E, 3)
    route = np.tile(np.array([[1, 3]]), (T, 1))
    fwd = R.layer_fwd(x, w_r, w_gu, w_d, 2, route=route)
    assert fwd["counts"].tolist() == [0, T, 0, T, 0]
    bwd = R.layer_bwd(fwd, dy, x, w_r, w_gu, w_d)
    for e in (0, 2, 4):
        assert np.all(bwd["dW_gu"][e] == 0) and np.all(bwd["dW_d"][e] == 0)


def _loss(x, w_r, w_gu, w_d, bias, dy, k, renorm, route):
    fwd = R.layer_fwd(x, w_r, w_gu, w_d, k, bias=bias, renorm=renorm, route=route, rnd=None)
    return float(np.sum(fwd["y"] * dy)), fwd


def _fd(fun, arr, eps=1e-6):
    g = np.zeros_like(arr)
    it = np.nditer(arr, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = arr[i]
        arr[i] = old + eps
        lp = fun()
        arr[i] = old - eps
        lm = fun()
        arr[i] = old
        g[i] = (lp - lm) / (2 * eps)
    return g


def _margin_ok(fwd, k):
    L = np.sort(fwd["logits"], axis=1)[:, ::-1]
    return k >= L.shape[1] or np.min(L[:, k - 1] - L[:, k]) > 1e-3


@pytest.mark.parametrize("renorm,use_bias,forced", [(False, False, False), (True, False, False),
                                                    (False, True, False), (True, True, True)])
def test_backward_matches_finite_differences(renorm, use_bias, forced):
    T, d, f, E, k = 7, 6, 4, 4, 2
    x, w_r, w_gu, w_d, dy = _draw(T, d, f, E, 10)
    bias = np.array([0.3, -0.2, 0.1, 0.0]) if use_bias else None
    route = np.array([[(t + 1) % E, (t + 3) % E] for t in range(T)]) if forced else None
    _, fwd = _loss(x, w_r, w_gu, w_d, bias, dy, k, renorm, route)
    assert forced or _margin_ok(fwd, k)
    bwd = R.layer_bwd(fwd, dy, x, w_r, w_gu, w_d, renorm=renorm, rnd=None)

    def L():
        return _loss(x, w_r, w_gu, w_d, bias, dy, k, renorm, route)[0]

    checks = [(x, bwd["dx"]), (w_r, bwd["dw_r"]), (w_gu, bwd["dW_gu"]), (w_d, bwd["dW_d"])]
    if use_bias:
        checks.append((bias, bwd["db"]))
    for arr, g in checks:
        num = _fd(L, arr)
        err = np.max(np.abs(num - g)) / max(np.max(np.abs(num)), 1e-30)
        assert err < 1e-6, err


def test_rounding_points_are_bf16():
    T, d, f, E, k = 16, 8, 8, 4, 2
    x, w_r, w_gu, w_d, dy = _draw(T, d, f, E, 11)
    fwd = R.layer_fwd(x, w_r, w_gu, w_d, k)
    bwd = R.layer_bwd(fwd, dy, x, w_r, w_gu, w_d)
    for name, a in [("x_perm", fwd["x_perm"]), ("AU", fwd["AU"]), ("H", fwd["H"]),
                    ("O", fwd["O"]), ("y", fwd["y"]), ("dO", bwd["dO"]),
                    ("dAU", bwd["dAU"]), ("dX_perm", bwd["dX_perm"]), ("dx", bwd["dx"]),
                    ("dW_gu", bwd["dW_gu"]), ("dW_d", bwd["dW_d"]), ("dw_r", bwd["dw_r"])]:
        np.testing.assert_array_equal(a, R.bf16_round(a), err_msg=name)
    # and close to the unrounded layer
    ex = R.layer_fwd(x, w_r, w_gu, w_d, k, rnd=None)
    assert np.max(np.abs(fwd["y"] - ex["y"])) / np.max(np.abs(ex["y"])) < 2e-2


# ---------------------------------------------------------------- shared expert
def test_shared_expert_alone_is_dense_swiglu():
    """With every routed expert's down projection zero, the layer's output
    and input gradient are those of the shared expert alone: a dense SwiGLU
    over all tokens, checked against torch float64 ops and autograd."""
    T, d, f, E, k, fs = 11, 16, 8, 4, 2, 12
    x, w_r, w_gu, w_d, dy = _draw(T, d, f, E, 20)
    w_d = np.zeros_like(w_d)
    rng = np.random.default_rng(21)
    w_gu_s = rng.standard_normal((2 * fs, d)) / np.sqrt(d)
    w_d_s = rng.standard_normal((d, fs)) / np.sqrt(fs)
    fwd = R.layer_fwd(x, w_r, w_gu, w_d, k, rnd=None, w_gu_s=w_gu_s, w_d_s=w_d_s)
    xt = torch.tensor(x, requires_grad=True)
    wg = torch.tensor(w_gu_s[:fs], requires_grad=True)
    wu = torch.tensor(w_gu_s[fs:], requires_grad=True)
    wd = torch.tensor(w_d_s, requires_grad=True)
    y = (F.silu(xt @ wg.T) * (xt @ wu.T)) @ wd.T
    np.testing.assert_allclose(fwd["y"], y.detach().numpy(), rtol=1e-12, atol=1e-13)
    (y * torch.tensor(dy)).sum().backward()
    bwd = R.layer_bwd(fwd, dy, x, w_r, w_gu, w_d, rnd=None, w_gu_s=w_gu_s, w_d_s=w_d_s)
    np.testing.assert_allclose(bwd["dx"], xt.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(bwd["dW_gu_s"][:fs], wg.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(bwd["dW_gu_s"][fs:], wu.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(bwd["dW_d_s"], wd.grad.numpy(), rtol=1e-11, atol=1e-12)


def test_shared_expert_backward_matches_finite_differences():
    T, d, f, E, k, fs = 6, 6, 4, 4, 2, 5
    x, w_r, w_gu, w_d, dy = _draw(T, d, f, E, 30)
    rng = np.random.default_rng(31)
    w_gu_s = rng.standard_normal((2 * fs, d)) / np.sqrt(d)
    w_d_s = rng.standard_normal((d, fs)) / np.sqrt(fs)

    def L():
        fwd = R.layer_fwd(x, w_r, w_gu, w_d, k, rnd=None, w_gu_s=w_gu_s, w_d_s=w_d_s)
        return float(np.sum(fwd["y"] * dy))

    fwd = R.layer_fwd(x, w_r, w_gu, w_d, k, rnd=None, w_gu_s=w_gu_s, w_d_s=w_d_s)
    assert _margin_ok(fwd, k)
    bwd = R.layer_bwd(fwd, dy, x, w_r, w_gu, w_d, rnd=None, w_gu_s=w_gu_s, w_d_s=w_d_s)
    for arr, g in [(x, bwd["dx"]), (w_gu_s, bwd["dW_gu_s"]), (w_d_s, bwd["dW_d_s"]),
                   (w_gu, bwd["dW_gu"]), (w_r, bwd["dw_r"])]:
        num = _fd(L, arr)
        err = np.max(np.abs(num - g)) / max(np.max(np.abs(num)), 1e-30)
        assert err < 1e-6, err
