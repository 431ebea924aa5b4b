"""Pins for the oracle's MLP-half backward: each check compares it with
something other than itself.

Sources of truth: central finite differences of the forward composition,
torch autograd (fp64) through F.layer_norm and F.gelu(approximate='tanh'),
closed forms of GELU's derivative and of LayerNorm's invariances, and a
plain-loop restatement of the weight gradients on a tiny input.  Planted
mistakes in the oracle (on the CPU) must make one of them fail.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as Fn

from oracle import tsp_oracle as O

EPS = 1e-5


def _tiny(seed=0, n=6, h=8, F=16):
    rng = np.random.default_rng(seed)
    y1 = rng.normal(size=(n, h)) * 1.5 + 0.3
    dy = rng.normal(size=(n, h))
    w = {"w1": rng.normal(size=(h, F)) * 0.4, "w2": rng.normal(size=(F, h)) * 0.4}
    return y1, dy, w


def _loss(y1, w1, w2, dy):
    """sum(dY * Y) for Y = Y1 + GELU(LN(Y1) W1) W2, written with numpy."""
    mu = y1.mean(axis=1, keepdims=True)
    var = ((y1 - mu) ** 2).mean(axis=1, keepdims=True)
    xn = (y1 - mu) / np.sqrt(var + EPS)
    u = xn @ w1
    hh = 0.5 * u * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (u + 0.044715 * u ** 3)))
    return float((dy * (y1 + hh @ w2)).sum())


def _central(f, x, step=1e-6):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        a = x.copy(); a[i] += step
        b = x.copy(); b[i] -= step
        g[i] = (f(a) - f(b)) / (2 * step)
    return g


def test_gelu_grad_closed_forms_and_differences():
    assert O.gelu_tanh_grad(0.0) == pytest.approx(0.5, abs=1e-15)
    x = np.linspace(-6, 6, 121)
    # GELU(x) - GELU(-x) = x, so GELU'(x) + GELU'(-x) = 1
    np.testing.assert_allclose(O.gelu_tanh_grad(x) + O.gelu_tanh_grad(-x), 1.0, atol=1e-14)
    num = (O.gelu_tanh(x + 1e-6) - O.gelu_tanh(x - 1e-6)) / 2e-6
    np.testing.assert_allclose(O.gelu_tanh_grad(x), num, atol=1e-8)
    # far tails: GELU -> x (slope 1) and -> 0 (slope 0)
    assert O.gelu_tanh_grad(30.0) == pytest.approx(1.0, abs=1e-12)
    assert O.gelu_tanh_grad(-30.0) == pytest.approx(0.0, abs=1e-12)


def test_layer_norm_backward_invariances_and_autograd():
    rng = np.random.default_rng(1)
    x = rng.normal(size=(5, 12)) * 2 + 1
    g = rng.normal(size=(5, 12))
    dx = O.layer_norm_backward(x, g, EPS)
    # LN(x + c) = LN(x): the gradient sums to zero along each row
    np.testing.assert_allclose(dx.sum(axis=1), 0.0, atol=1e-12)
    xt = torch.tensor(x, requires_grad=True)
    (Fn.layer_norm(xt, (12,), eps=EPS) * torch.tensor(g)).sum().backward()
    np.testing.assert_allclose(dx, xt.grad.numpy(), rtol=1e-12, atol=1e-12)


def test_mlp_backward_matches_finite_differences():
    y1, dy, w = _tiny()
    r = O.mlp_backward(y1, dy, w, EPS, storage=None, grad_storage=None)
    g_y1 = _central(lambda a: _loss(a, w["w1"], w["w2"], dy), y1)
    g_w1 = _central(lambda a: _loss(y1, a, w["w2"], dy), w["w1"])
    g_w2 = _central(lambda a: _loss(y1, w["w1"], a, dy), w["w2"])
    np.testing.assert_allclose(r["dy1"], g_y1, atol=1e-7)
    np.testing.assert_allclose(r["dw1"], g_w1, atol=1e-7)
    np.testing.assert_allclose(r["dw2"], g_w2, atol=1e-7)


def test_mlp_backward_matches_torch_autograd():
    y1, dy, w = _tiny(seed=3, n=9, h=16, F=40)
    r = O.mlp_backward(y1, dy, w, EPS, storage=None, grad_storage=None)
    yt = torch.tensor(y1, requires_grad=True)
    w1t = torch.tensor(w["w1"], requires_grad=True)
    w2t = torch.tensor(w["w2"], requires_grad=True)
    y = yt + Fn.gelu(Fn.layer_norm(yt, (16,), eps=EPS) @ w1t, approximate="tanh") @ w2t
    (y * torch.tensor(dy)).sum().backward()
    np.testing.assert_allclose(r["dy1"], yt.grad.numpy(), rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(r["dw1"], w1t.grad.numpy(), rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(r["dw2"], w2t.grad.numpy(), rtol=1e-11, atol=1e-11)


def test_weight_gradients_by_loops():
    """dW1[i, j] = sum_t Xn2[t, i] dU[t, j] and dW2[f, o] = sum_t H[t, f] dY[t, o],
    in plain loops, with the rounded storage."""
    y1, dy, w = _tiny(seed=5, n=4, h=4, F=8)
    r = O.mlp_backward(y1, dy, w, EPS, storage="fp16", grad_storage="bf16")
    xn2 = O.round_fp16(O.layer_norm(y1, EPS))
    xb = O.round_bf16(xn2)
    hb = O.round_bf16(O.gelu_tanh(r["u"]))
    du = r["du"]
    for i in range(4):
        for j in range(8):
            assert r["dw1"][i, j] == pytest.approx(sum(xb[t, i] * du[t, j] for t in range(4)), abs=1e-12)
    for f in range(8):
        for o in range(4):
            assert r["dw2"][f, o] == pytest.approx(sum(hb[t, f] * dy[t, o] for t in range(4)), abs=1e-12)


@pytest.mark.parametrize("storage,grad_storage", [(None, None), ("fp16", "bf16")])
def test_sampled_backward_equals_full(storage, grad_storage):
    rng = np.random.default_rng(7)
    n, h, F = 24, 32, 64
    y1 = rng.normal(size=(n, h))
    dy = O.round_bf16(rng.normal(size=(n, h)))
    w = {"w1": O.round_bf16(rng.normal(size=(h, F)) * 0.05), "w2": O.round_bf16(rng.normal(size=(F, h)) * 0.05)}
    full = O.mlp_backward(y1, dy, w, EPS, storage, grad_storage)
    rows, c1, r2 = [0, 5, 23], [1, 17, 63], [0, 30, 62]
    s = O.mlp_backward_sampled(y1, dy, w, rows, c1, r2, EPS, storage, grad_storage)
    np.testing.assert_allclose(s["dy1"], full["dy1"][rows], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s["dw1"], full["dw1"][:, c1], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s["dw2"], full["dw2"][r2, :], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mistake", ["grad_sign", "ln_mean_term", "transposed_w2"])
def test_planted_backward_mistakes_are_caught(monkeypatch, mistake):
    """Each plausible bug, planted in the oracle, must break the autograd pin."""
    if mistake == "grad_sign":
        good = O.gelu_tanh_grad
        monkeypatch.setattr(O, "gelu_tanh_grad", lambda x: 1.0 - good(x))
    elif mistake == "ln_mean_term":
        def bad(x, g, eps=EPS):
            x = np.asarray(x, dtype=np.float64)
            c = x - x.mean(axis=-1, keepdims=True)
            rstd = 1.0 / np.sqrt((c * c).mean(axis=-1, keepdims=True) + eps)
            return rstd * (g - (c * rstd) * (g * c * rstd).mean(axis=-1, keepdims=True))
        monkeypatch.setattr(O, "layer_norm_backward", bad)
    else:
        orig = O.mlp_backward

        def bad_mlp(y1, dy, w, *a, **k):
            return orig(y1, dy, {"w1": w["w1"], "w2": w["w2"][::-1].copy()}, *a, **k)
        monkeypatch.setattr(O, "mlp_backward", bad_mlp)
    with pytest.raises(AssertionError):
        test_mlp_backward_matches_torch_autograd()


@pytest.mark.parametrize("mistake", ["gelu_grad_first_term_only", "ln_backward_without_mean", "dw2_from_u"])
def test_gpu_parity_bound_rejects_plausible_mistakes(monkeypatch, mistake):
    """The GPU parity bound for the backward (rel-L2 <= 1e-3, max-abs <=
    1e-2 max|ref|) is far tighter than what a plausible bug changes: each
    planted mistake below moves some output beyond it (CPU only)."""
    rng = np.random.default_rng(9)
    n, h, F = 64, 32, 128
    y1 = rng.normal(size=(n, h))
    dy = O.round_bf16(rng.normal(size=(n, h)))
    w = {"w1": O.round_bf16(rng.normal(size=(h, F)) * 0.1), "w2": O.round_bf16(rng.normal(size=(F, h)) * 0.1)}
    ref = O.mlp_backward(y1, dy, w)
    if mistake == "gelu_grad_first_term_only":
        monkeypatch.setattr(O, "gelu_tanh_grad",
                            lambda x: 0.5 * (1.0 + np.tanh(np.sqrt(2 / np.pi) * (x + 0.044715 * x ** 3))))
    elif mistake == "ln_backward_without_mean":
        def bad(x, g, eps=EPS):
            c = x - x.mean(axis=-1, keepdims=True)
            rstd = 1.0 / np.sqrt((c * c).mean(axis=-1, keepdims=True) + eps)
            return rstd * (g - (c * rstd) * (g * c * rstd).mean(axis=-1, keepdims=True))
        monkeypatch.setattr(O, "layer_norm_backward", bad)
    else:
        monkeypatch.setattr(O, "gelu_tanh", lambda x: np.asarray(x, dtype=np.float64))
    got = O.mlp_backward(y1, dy, w)

    def within(a, b):
        return (np.abs(a - b).max() <= 1e-2 * np.abs(b).max()
                and np.linalg.norm(a - b) <= 1e-3 * np.linalg.norm(b))
    assert not all(within(got[k], ref[k]) for k in ("dy1", "dw1", "dw2"))
