"""Pins for the oracle's causal-attention backward (the attention half of the
layer's backward is not built in CUDA yet; its oracle comes first).

Sources of truth: central finite differences, torch autograd in fp64 through
F.scaled_dot_product_attention with an explicit position mask, the softmax's
invariances, and the sum over zigzag ranks against the whole sequence."""
import numpy as np
import pytest
import torch
import torch.nn.functional as Fn

from oracle import tsp_oracle as O


def _inputs(seed, n, T, H, d, pos=None):
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(n, H * d))
    k = rng.normal(size=(T, H * d))
    v = rng.normal(size=(T, H * d))
    dout = rng.normal(size=(n, H * d))
    if pos is None:
        pos = np.sort(rng.choice(T, size=n, replace=False))
    return q, k, v, np.asarray(pos), dout


def _loss(q, k, v, pos, dout, H, scale):
    return float((dout * O.causal_attention(q, k, v, pos, H, scale)).sum())


def _central(f, x, step=1e-6):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        a = x.copy(); a[i] += step
        b = x.copy(); b[i] -= step
        g[i] = (f(a) - f(b)) / (2 * step)
    return g


def test_attention_backward_matches_finite_differences():
    H, d, T = 2, 3, 7
    q, k, v, pos, dout = _inputs(0, 4, T, H, d, pos=[0, 2, 5, 6])
    s = 0.6
    dq, dk, dv = O.causal_attention_backward(q, k, v, pos, dout, H, s)
    np.testing.assert_allclose(dq, _central(lambda a: _loss(a, k, v, pos, dout, H, s), q), atol=1e-7)
    np.testing.assert_allclose(dk, _central(lambda a: _loss(q, a, v, pos, dout, H, s), k), atol=1e-7)
    np.testing.assert_allclose(dv, _central(lambda a: _loss(q, k, a, pos, dout, H, s), v), atol=1e-7)


def test_attention_backward_matches_torch_autograd():
    H, d, T = 3, 8, 40
    q, k, v, pos, dout = _inputs(1, 12, T, H, d)
    s = 1.0 / np.sqrt(d)
    dq, dk, dv = O.causal_attention_backward(q, k, v, pos, dout, H, s)
    qt, kt, vt = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    mask = torch.tensor(np.arange(T)[None, :] <= pos[:, None])
    split = lambda t: t.view(t.shape[0], H, d).transpose(0, 1)
    o = Fn.scaled_dot_product_attention(split(qt), split(kt), split(vt), attn_mask=mask, scale=s)
    (o.transpose(0, 1).reshape(len(pos), H * d) * torch.tensor(dout)).sum().backward()
    np.testing.assert_allclose(dq, qt.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, kt.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv, vt.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_attention_backward_invariants():
    """Rows of P sum to 1, so the key-summed dV equals the query-summed dO;
    softmax ignores a common shift of the scores, so the key-summed dK of each
    head is zero; keys past the last query position get no gradient."""
    H, d, T = 2, 4, 30
    q, k, v, pos, dout = _inputs(2, 9, T, H, d)
    dq, dk, dv = O.causal_attention_backward(q, k, v, pos, dout, H, 0.5)
    np.testing.assert_allclose(dv.sum(axis=0), dout.sum(axis=0), atol=1e-12)
    np.testing.assert_allclose(dk.sum(axis=0), 0.0, atol=1e-12)
    assert not dk[pos.max() + 1:].any() and not dv[pos.max() + 1:].any()
    # position 0 attends only to key 0: its query gets no gradient
    q0, k0, v0, p0, do0 = _inputs(3, 3, 10, 1, 4, pos=[0, 4, 9])
    g0 = O.causal_attention_backward(q0, k0, v0, p0, do0, 1, 0.5)[0]
    assert not g0[0].any()


@pytest.mark.parametrize("T,D", [(16, 2), (24, 3)])
def test_zigzag_ranks_sum_to_the_whole_sequence(T, D):
    """Each rank back-propagates its own zigzag rows against the full K/V; the
    sum of the ranks' dK, dV is the whole sequence's, and the ranks' dQ rows
    are the whole sequence's rows at their positions."""
    H, d = 2, 4
    q, k, v, _, dout = _inputs(4, T, T, H, d, pos=np.arange(T))
    s = 0.4
    full = O.causal_attention_backward(q, k, v, np.arange(T), dout, H, s)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for r in range(D):
        idx = O.zigzag_index(T, D, r)
        dq_r, dk_r, dv_r = O.causal_attention_backward(q[idx], k, v, idx, dout[idx], H, s)
        np.testing.assert_allclose(dq_r, full[0][idx], atol=1e-12)
        dk += dk_r
        dv += dv_r
    np.testing.assert_allclose(dk, full[1], atol=1e-12)
    np.testing.assert_allclose(dv, full[2], atol=1e-12)


def test_planted_softmax_backward_mistake_is_caught(monkeypatch):
    """A backward that drops the row-sum term of dS (dS = P * dP) must break
    the autograd pin."""
    def bad(q, k, v, q_pos, dout, n_heads, scale):
        q = np.asarray(q, dtype=np.float64)
        n, hd = q.shape
        d = hd // n_heads
        dq, dk, dv = np.zeros((n, hd)), np.zeros(k.shape), np.zeros(v.shape)
        _, probs = O.causal_attention(q, k, v, q_pos, n_heads, scale, return_probs=True)
        km = probs[0].shape[1]
        for j in range(n_heads):
            c = slice(j * d, (j + 1) * d)
            p = probs[j]
            ds = p * (dout[:, c] @ v[:km, c].T)
            dv[:km, c] = p.T @ dout[:, c]
            dq[:, c] = scale * (ds @ k[:km, c])
            dk[:km, c] = scale * (ds.T @ q[:, c])
        return dq, dk, dv
    monkeypatch.setattr(O, "causal_attention_backward", bad)
    with pytest.raises(AssertionError):
        test_attention_backward_matches_torch_autograd()


def _rank_sum(T, D, x, w, dy, H, s, **prec):
    """dX and the six weight gradients summed over the D ranks' shares, with
    dK, dV summed over ranks (the reduce-scatter) and each owner's K/V
    backward added."""
    h = x.shape[1]
    dx = np.zeros((T, h))
    grads = {n: np.zeros_like(w[n]) for n in w}
    dk = np.zeros((T, h))
    dv = np.zeros((T, h))
    for r in range(D):
        idx = O.zigzag_index(T, D, r)
        g = O.rank_layer_backward(r, D, x, w, dy[idx], H, scale=s, **prec)
        dx[idx] += g["dx_partial"]
        for n in ("wq", "wo", "w1", "w2"):
            grads[n] += g["d" + n]
        dk += g["dk_full"]
        dv += g["dv_full"]
    for r in range(D):   # each owner's K/V backward for its own rows
        idx = O.zigzag_index(T, D, r)
        kv = O.kv_backward_rows(x[idx], dk[idx], dv[idx], w, **prec)
        dx[idx] += kv["dx"]
        grads["wk"] += kv["dwk"]
        grads["wv"] += kv["dwv"]
    return dx, grads


def _small_layer(T, seed=11):
    h, H, F = 8, 2, 16
    rng = np.random.default_rng(seed)
    x = rng.normal(size=(T, h))
    w = {n: rng.normal(size=s) * 0.3 for n, s in (("wq", (h, h)), ("wk", (h, h)), ("wv", (h, h)), ("wo", (h, h)),
                                                    ("w1", (h, F)), ("w2", (F, h)))}
    dy = rng.normal(size=(T, h))
    return x, w, dy, h, H, F


@pytest.mark.parametrize("T,D", [(8, 2), (12, 3)])
def test_rank_backwards_sum_to_the_whole_layer_gradient(T, D):
    """The D ranks' shares, with dK, dV summed over ranks (the reduce-scatter)
    and each owner's K/V backward added, equal torch autograd of the whole
    unsharded layer (fp64) for every input row and all six weights."""
    x, w, dy, h, H, F = _small_layer(T)
    s = 1.0 / np.sqrt(h // H)
    dx, grads = _rank_sum(T, D, x, w, dy, H, s)
    xt = torch.tensor(x, requires_grad=True)
    wt = {n: torch.tensor(a, requires_grad=True) for n, a in w.items()}
    xn = Fn.layer_norm(xt, (h,), eps=O.LN_EPS)
    split = lambda t: t.view(T, H, h // H).transpose(0, 1)
    att = Fn.scaled_dot_product_attention(split(xn @ wt["wq"]), split(xn @ wt["wk"]), split(xn @ wt["wv"]),
                                          is_causal=True, scale=s)
    y1 = xt + att.transpose(0, 1).reshape(T, h) @ wt["wo"]
    y = y1 + Fn.gelu(Fn.layer_norm(y1, (h,), eps=O.LN_EPS) @ wt["w1"], approximate="tanh") @ wt["w2"]
    (y * torch.tensor(dy)).sum().backward()
    np.testing.assert_allclose(dx, xt.grad.numpy(), rtol=1e-9, atol=1e-11)
    for n in w:
        np.testing.assert_allclose(grads[n], wt[n].grad.numpy(), rtol=1e-9, atol=1e-11, err_msg=n)


def test_stored_layer_backward_is_the_plain_one_up_to_16_bit_rounding():
    """With the kernels' precision model (fp16 forward storage and dA, bf16
    gradient operands) the rank-summed gradients stay within 16-bit rounding
    of the plain ones (pinned to autograd above), and the rounding really
    happens.  A transposed operand, a dropped term or a wrong index in the
    stored branch would move them by O(1)."""
    T, D = 64, 2
    x, w, dy, h, H, F = _small_layer(T, seed=12)
    w = {n: O.round_bf16(a) for n, a in w.items()}   # bf16 model weights
    s = 1.0 / np.sqrt(h // H)
    dx0, g0 = _rank_sum(T, D, x, w, dy, H, s)
    dx1, g1 = _rank_sum(T, D, x, w, dy, H, s, storage="fp16", grad_storage="bf16")
    rel = lambda a, b: np.linalg.norm(a - b) / np.linalg.norm(b)
    assert 1e-6 < rel(dx1, dx0) < 2e-2, rel(dx1, dx0)
    for n in w:
        assert 1e-6 < rel(g1[n], g0[n]) < 2e-2, (n, rel(g1[n], g0[n]))


# --------------------------------------------------------------------------
# the stored-value form (what a 16-bit tensor-core pipeline computes)
# --------------------------------------------------------------------------
def test_logsumexp_closed_form_and_library():
    """attention_logsumexp against torch.logsumexp of the masked scores, and
    exp(score - lse) against the oracle's own probabilities."""
    H, d, T = 2, 4, 25
    q, k, v, pos, _ = _inputs(5, 7, T, H, d)
    s = 0.7
    lse = O.attention_logsumexp(q, k, pos, H, s)
    _, probs = O.causal_attention(q, k, v, pos, H, s, return_probs=True)
    for j in range(H):
        cols = slice(j * d, (j + 1) * d)
        sc = torch.tensor(s * q[:, cols] @ k[:, cols].T)
        sc = sc.masked_fill(torch.tensor(np.arange(T)[None, :] > pos[:, None]), -np.inf)
        np.testing.assert_allclose(lse[:, j], torch.logsumexp(sc, dim=1).numpy(), rtol=1e-13)
        kmax = probs[j].shape[1]
        p = np.exp(s * q[:, cols] @ k[:kmax, cols].T - lse[:, j:j + 1]) * (np.arange(kmax)[None, :] <= pos[:, None])
        np.testing.assert_allclose(p, probs[j], atol=1e-14)
    # one key: lse is that key's score
    one = O.attention_logsumexp(q[:1], k, [0], H, s)
    np.testing.assert_allclose(one[0], [s * q[0, :d] @ k[0, :d], s * q[0, d:] @ k[0, d:]], rtol=1e-13)


def test_stored_backward_without_rounding_is_the_plain_backward():
    """storage=None with the exact output o = P v: Delta = rowsum(dO * o)
    equals rowsum(dP * P), so the stored form reduces to the pinned plain
    backward (the scale folded into dS changes nothing either)."""
    H, d, T = 3, 8, 40
    q, k, v, pos, dout = _inputs(6, 12, T, H, d)
    s = 1.0 / np.sqrt(d)
    o = O.causal_attention(q, k, v, pos, H, s)
    got = O.attention_backward_stored(q, k, v, o, pos, dout, H, s, storage=None)
    ref = O.causal_attention_backward(q, k, v, pos, dout, H, s)
    for g, r in zip(got, ref):
        np.testing.assert_allclose(g, r, rtol=1e-11, atol=1e-13)


def _torch_stored_backward(q, k, v, o, pos, dout, H, s):
    """The stored-value backward written independently with torch ops: the
    probabilities from torch.softmax, 16-bit rounding by a cast to float16."""
    f16 = lambda t: t.to(torch.float16).to(torch.float64)
    q, k, v, o, dout = (torch.tensor(a) for a in (q, k, v, o, dout))
    n, hd = q.shape
    d = hd // H
    T = k.shape[0]
    mask = torch.tensor(np.arange(T)[None, :] > np.asarray(pos)[:, None])
    do = f16(dout)
    dq, dk, dv = torch.zeros(n, hd, dtype=torch.float64), torch.zeros(T, hd, dtype=torch.float64), \
        torch.zeros(T, hd, dtype=torch.float64)
    for j in range(H):
        c = slice(j * d, (j + 1) * d)
        p = torch.softmax((s * q[:, c] @ k[:, c].T).masked_fill(mask, -float("inf")), dim=1)
        delta = (do[:, c] * o[:, c]).sum(dim=1, keepdim=True)
        ds = f16(s * p * (do[:, c] @ v[:, c].T - delta))
        dv[:, c] = f16(p).T @ do[:, c]
        dq[:, c] = ds @ k[:, c]
        dk[:, c] = ds.T @ q[:, c]
    return dq.numpy(), dk.numpy(), dv.numpy()


def test_stored_backward_matches_torch_composition():
    H, d, T = 2, 16, 48
    q, k, v, pos, dout = _inputs(7, 14, T, H, d)
    q, k, v = (O.round_fp16(a) for a in (q, k, v))
    s = 1.0 / np.sqrt(d)
    o = O.round_fp16(O.causal_attention(q, k, v, pos, H, s))
    got = O.attention_backward_stored(q, k, v, o, pos, dout, H, s)
    ref = _torch_stored_backward(q, k, v, o, pos, dout, H, s)
    for g, r in zip(got, ref):
        np.testing.assert_allclose(g, r, rtol=1e-12, atol=1e-14)
    # and it stays within fp16 rounding of the plain backward
    plain = O.causal_attention_backward(q, k, v, pos, dout, H, s)
    for g, r in zip(got, plain):
        assert np.linalg.norm(g - r) <= 5e-3 * np.linalg.norm(r)
