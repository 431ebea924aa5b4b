"""Oracle for the TSP per-rank dense-layer forward: plain, slow, CPU, fp64.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or
executes this module: only the tests, the smoke check and the benchmark's
CPU-baseline leg do.  It shares no code with the CUDA library and imports
nothing from it.

Source of the method: the zubnet.ai news item "Zyphra TSP folds TP+SP onto
one GPU axis" (four paragraphs, cited below as [TSP ¶n]):

* [TSP ¶1] Tensor and sequence parallelism are folded onto one device-mesh
  axis of size D: every GPU holds 1/D of the weights *and* 1/D of the
  sequence tokens.  The validated model is a dense decoder (h=4096, 32 Q/KV
  heads, FFN = 4h, bf16) at 128K tokens with D=8.
* [TSP ¶2] Attention: weight shards are broadcast one after another, each GPU
  applies every shard to its own tokens, and K/V are all-gathered with a
  zigzag sequence partition for load balance.  MLP: a ring passes the weight
  shards point to point, which removes tensor parallelism's all-reduce.
* [TSP ¶4] The MLP-without-all-reduce step stands on its own.

The pages give no layer internals.  The layer form used here is the one the
workload states: pre-LayerNorm (eps 1e-5, gamma=1, beta=0, biased variance),
GELU with the tanh approximation, no biases, no positional encoding, causal
softmax with scale 1/sqrt(head_dim), multi-head attention with as many K/V
heads as Q heads.

Because re-partitioning weights and tokens does not change what a layer
computes, the per-rank TSP output is exactly (up to summation order) the
rows, at that rank's token positions, of the plain unsharded layer.  So the
reference for parity is that plain definition (``layer_forward`` and, given
the all-gathered K/V, ``rank_rows_forward``).  ``rank_forward_sharded`` and
``kv_all_gather_sharded`` restate the pages' shard-by-shard schedule; tests
pin them to the plain definition (the sum over shards equals the unsharded
contraction).

Precision: every product and sum is fp64.  The layer holds the operands
of its matmuls in a 16-bit float, so the oracle rounds exactly those values
(round to nearest even) at the points where the layer stores them: the
weights, the LN1 output, Q, K, V, the attention output, the LN2 output and
the GELU output H.  The residual stream (X + attention, and the layer
output) stays unrounded.  The pages give the model's dtype as bf16; inputs X
and weights arrive in bf16.  The storage format of the matmul operands is
``storage``: "fp16" (11 significant bits, the default, what the CUDA path
uses), "bf16" (8 bits) or None (no rounding: the pure fp64 layer).  fp16
holds every value this pre-LayerNorm layer produces exactly as bf16 would
(same 16 bits) but with three more significand bits; bf16 weights convert
to fp16 exactly down to |w| = 2^-14 and within 2^-25 below that.

Zigzag partition: the sequence is cut into 2D equal chunks of c = T/(2D)
tokens, and rank r holds chunks r and 2D-1-r, in that order.

Parity status: every function here is pinned by tests/test_oracle_pins.py
and, for the backward, tests/test_oracle_backward_pins.py (MLP half) and
tests/test_oracle_attention_backward_pins.py (causal attention) (closed
forms, invariants, brute force, finite differences and independent library
routines).
"""
from __future__ import annotations

import numpy as np

LN_EPS = 1e-5


# ----------------------------------------------------------------------------
# 16-bit storage rounding
# ----------------------------------------------------------------------------
def round_bf16(x) -> np.ndarray:
    """Round each value to the nearest bf16 number (ties to even), kept as fp64.

    bf16 keeps 8 significant bits.  frexp gives x = m * 2**e with
    0.5 <= |m| < 1, so m*256 carries exactly 8 integer bits and rint (which
    rounds half to even) performs the rounding; ldexp scales back.  Valid for
    the normal range, which is all the layer produces.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


def round_fp16(x) -> np.ndarray:
    """Round each value to the nearest IEEE binary16 number (ties to even),
    subnormals included, kept as fp64.  numpy's float64 -> float16 cast rounds
    once, directly from the fp64 value."""
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def _rounder(storage):
    if storage is None:
        return lambda a: np.asarray(a, dtype=np.float64)
    if storage == "fp16":
        return round_fp16
    if storage == "bf16":
        return round_bf16
    raise ValueError(f"unknown storage format {storage!r}")


# ----------------------------------------------------------------------------
# token partition  [TSP ¶2: "zigzag partition"]
# ----------------------------------------------------------------------------
def zigzag_index(T: int, D: int, rank: int) -> np.ndarray:
    """Global positions of rank `rank`'s tokens, in rank-local order.

    T tokens are cut into 2D chunks of c = T/(2D); rank r holds chunk r, then
    chunk 2D-1-r.  Returned as int64 [2c].
    """
    if T % (2 * D) != 0:
        raise ValueError("T must be a multiple of 2D")
    if not 0 <= rank < D:
        raise ValueError("rank out of range")
    c = T // (2 * D)
    first = np.arange(rank * c, (rank + 1) * c, dtype=np.int64)
    second = np.arange((2 * D - 1 - rank) * c, (2 * D - rank) * c, dtype=np.int64)
    return np.concatenate([first, second])


# ----------------------------------------------------------------------------
# elementwise pieces of the layer
# ----------------------------------------------------------------------------
def layer_norm(x, eps: float = LN_EPS) -> np.ndarray:
    """Row-wise (x - mean) / sqrt(var + eps), biased variance, gamma=1, beta=0."""
    x = np.asarray(x, dtype=np.float64)
    mean = x.mean(axis=-1, keepdims=True)
    centred = x - mean
    var = (centred * centred).mean(axis=-1, keepdims=True)
    return centred / np.sqrt(var + eps)


def gelu_tanh(x) -> np.ndarray:
    """GELU, tanh form: 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))."""
    x = np.asarray(x, dtype=np.float64)
    inner = np.sqrt(2.0 / np.pi) * (x + 0.044715 * x * x * x)
    return 0.5 * x * (1.0 + np.tanh(inner))


def causal_attention(q, k, v, q_pos, n_heads: int, scale: float,
                     return_probs: bool = False):
    """Multi-head causal attention of query rows at global positions `q_pos`.

    q: [n, H*d] query rows; k, v: [T, H*d] full-sequence keys/values in
    natural order, head j in columns j*d .. (j+1)*d.  Row i attends to the
    keys at positions 0 .. q_pos[i] inclusive, with weights
    softmax(scale * q.k).  Returns [n, H*d] (and the per-head probability
    matrices when asked).
    """
    q = np.asarray(q, dtype=np.float64)
    q_pos = np.asarray(q_pos, dtype=np.int64)
    n, hd = q.shape
    d = hd // n_heads
    kmax = int(q_pos.max()) + 1 if n else 0
    out = np.zeros((n, hd), dtype=np.float64)
    probs = []
    if n == 0:
        return (out, probs) if return_probs else out
    key_pos = np.arange(kmax, dtype=np.int64)
    allowed = key_pos[None, :] <= q_pos[:, None]            # [n, kmax]
    for j in range(n_heads):
        cols = slice(j * d, (j + 1) * d)
        kj = np.asarray(k[:kmax, cols], dtype=np.float64)
        vj = np.asarray(v[:kmax, cols], dtype=np.float64)
        scores = scale * (q[:, cols] @ kj.T)                 # [n, kmax]
        scores = np.where(allowed, scores, -np.inf)
        scores -= scores.max(axis=1, keepdims=True)
        w = np.exp(scores)
        w /= w.sum(axis=1, keepdims=True)
        out[:, cols] = w @ vj
        if return_probs:
            probs.append(w)
    return (out, probs) if return_probs else out


# ----------------------------------------------------------------------------
# the plain (unsharded) layer
# ----------------------------------------------------------------------------
class StoredWeights(dict):
    """Weights already rounded to a storage format (what ``stored_weights``
    returns).  Rounding to nearest is idempotent, so handing these to the
    layer functions computes exactly what the raw weights give; it only
    skips re-rounding every matrix on every call."""

    def __init__(self, w: dict, storage):
        super().__init__(w)
        self.storage = storage


def stored_weights(w: dict, storage="fp16") -> StoredWeights:
    """The weights rounded once to `storage` (fp64 arrays), for repeated calls."""
    rnd = _rounder(storage)
    return StoredWeights({n: rnd(np.asarray(a, dtype=np.float64)) for n, a in w.items()}, storage)


def _weights(w: dict, rnd, storage="fp16") -> dict:
    """The weights as the layer holds them for its matmuls."""
    if isinstance(w, StoredWeights) and w.storage == storage:
        return w
    return {n: rnd(np.asarray(a, dtype=np.float64)) for n, a in w.items()}


def kv_project(x_rows, w: dict, eps: float = LN_EPS, storage="fp16"):
    """K and V rows of tokens `x_rows`: LN1(x) @ Wk and LN1(x) @ Wv."""
    rnd = _rounder(storage)
    w = _weights(w, rnd, storage)
    xn = rnd(layer_norm(x_rows, eps))
    return rnd(xn @ w["wk"]), rnd(xn @ w["wv"])


def rank_rows_forward(x_rows, q_pos, k_full, v_full, w: dict, n_heads: int,
                      eps: float = LN_EPS, scale: float | None = None,
                      storage="fp16") -> dict:
    """Layer output for tokens `x_rows` at global positions `q_pos`.

    `k_full`, `v_full` [T, h] are the keys and values of the whole sequence
    (what every rank holds after the all-gather).  Every step is row-local
    except attention, so any subset of a rank's rows can be computed alone.
    Returns the output and the stored intermediates.
    """
    rnd = _rounder(storage)
    w = _weights(w, rnd, storage)
    x = np.asarray(x_rows, dtype=np.float64)
    h = x.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(h // n_heads)
    xn1 = rnd(layer_norm(x, eps))
    q = rnd(xn1 @ w["wq"])
    a = rnd(causal_attention(q, k_full, v_full, q_pos, n_heads, scale))
    y1 = x + a @ w["wo"]
    xn2 = rnd(layer_norm(y1, eps))
    hh = rnd(gelu_tanh(xn2 @ w["w1"]))
    y = y1 + hh @ w["w2"]
    return {"xn1": xn1, "q": q, "a": a, "y1": y1, "xn2": xn2, "h": hh, "y": y}


def layer_forward(x, w: dict, n_heads: int, eps: float = LN_EPS,
                  scale: float | None = None, storage="fp16") -> dict:
    """The whole unsharded layer over a full sequence x [T, h] (natural order)."""
    x = np.asarray(x, dtype=np.float64)
    k, v = kv_project(x, w, eps, storage)
    out = rank_rows_forward(x, np.arange(x.shape[0]), k, v, w, n_heads, eps,
                            scale, storage)
    out["k"], out["v"] = k, v
    return out


# ----------------------------------------------------------------------------
# the pages' shard-by-shard schedule  [TSP ¶1, ¶2]
# ----------------------------------------------------------------------------
def kv_all_gather_sharded(x_full, D: int, w: dict, eps: float = LN_EPS,
                          storage="fp16"):
    """Full-sequence K/V as TSP builds it.

    Every rank r projects its own zigzag tokens with every attention shard
    k (head group k = columns k*h/D .. (k+1)*h/D of Wk, Wv); the all-gather
    places each rank's rows back at their global positions.
    """
    rnd = _rounder(storage)
    w = _weights(w, rnd, storage)
    x_full = np.asarray(x_full, dtype=np.float64)
    T, h = x_full.shape
    hs = h // D
    K = np.zeros((T, h))
    V = np.zeros((T, h))
    for rank in range(D):
        idx = zigzag_index(T, D, rank)
        xn = rnd(layer_norm(x_full[idx], eps))
        for s in range(D):
            cols = slice(s * hs, (s + 1) * hs)
            K[idx, cols] = rnd(xn @ w["wk"][:, cols])
            V[idx, cols] = rnd(xn @ w["wv"][:, cols])
    return K, V


def rank_forward_sharded(rank: int, D: int, x_local, k_full, v_full, w: dict,
                         n_heads: int, eps: float = LN_EPS,
                         scale: float | None = None,
                         storage="fp16") -> np.ndarray:
    """Rank `rank`'s output computed the way TSP schedules it.

    Attention: shard k (heads k*H/D .. (k+1)*H/D of Wq and Wo) is applied to
    the local tokens in turn and its output projection is accumulated.
    MLP: at ring step s the rank holds W1/W2 shard (rank+s) mod D (FFN columns
    of W1, rows of W2) and adds GELU(x W1_k) W2_k; the sum over shards is
    local, so no all-reduce is needed.
    """
    rnd = _rounder(storage)
    w = _weights(w, rnd, storage)
    x = np.asarray(x_local, dtype=np.float64)
    L, h = x.shape
    T = np.asarray(k_full).shape[0]
    F = w["w1"].shape[1]
    hs, Fs, Hs = h // D, F // D, n_heads // D
    if scale is None:
        scale = 1.0 / np.sqrt(h // n_heads)
    pos = zigzag_index(T, D, rank)
    xn1 = rnd(layer_norm(x, eps))
    y1 = x.copy()
    for s in range(D):
        cols = slice(s * hs, (s + 1) * hs)
        q_s = rnd(xn1 @ w["wq"][:, cols])
        a_s = rnd(causal_attention(q_s, np.asarray(k_full)[:, cols],
                                   np.asarray(v_full)[:, cols], pos, Hs, scale))
        y1 = y1 + a_s @ w["wo"][cols, :]
    xn2 = rnd(layer_norm(y1, eps))
    y = y1.copy()
    for step in range(D):
        s = (rank + step) % D
        cols = slice(s * Fs, (s + 1) * Fs)
        h_s = rnd(gelu_tanh(xn2 @ w["w1"][:, cols]))
        y = y + h_s @ w["w2"][cols, :]
    return y


# ----------------------------------------------------------------------------
# work accounting
# ----------------------------------------------------------------------------
def causal_pairs(T: int, D: int, rank: int) -> int:
    """Number of (query, key) pairs rank `rank` scores: sum over its tokens of pos+1."""
    return int((zigzag_index(T, D, rank) + 1).sum())


# ----------------------------------------------------------------------------
# backward of the MLP half of the layer  [TSP ¶1: the validated workload is
# training; ¶2, ¶4: the MLP is a sum over weight shards with no all-reduce]
# ----------------------------------------------------------------------------
# The pages give no backward; it is the chain rule applied to the forward
# above.  For rows Y1 of the residual stream the MLP half is
#     Xn2 = LN(Y1),  U = Xn2 W1,  H = GELU(U),  Y = Y1 + H W2,
# and for a loss gradient dY the gradients are
#     dH = dY W2^T,  dU = dH * GELU'(U),  dXn2 = dU W1^T,
#     dY1 = dY + LN'(Y1)^T dXn2,  dW1 = Xn2^T dU,  dW2 = H^T dY.
# Over shards, dW1 and dW2 split by FFN columns / rows exactly as W1 and W2
# do, and dXn2 = sum_k dU_k W1_k^T is again a sum over shards.

def gelu_tanh_grad(x) -> np.ndarray:
    """Derivative of gelu_tanh: with s = sqrt(2/pi), a = 0.044715 and
    t = tanh(s (x + a x^3)),  0.5 (1 + t) + 0.5 x (1 - t^2) s (1 + 3 a x^2)."""
    x = np.asarray(x, dtype=np.float64)
    s = np.sqrt(2.0 / np.pi)
    t = np.tanh(s * (x + 0.044715 * x * x * x))
    return 0.5 * (1.0 + t) + 0.5 * x * (1.0 - t * t) * s * (1.0 + 3.0 * 0.044715 * x * x)


def layer_norm_backward(x, g, eps: float = LN_EPS) -> np.ndarray:
    """Gradient with respect to x of sum(g * layer_norm(x)), row-wise:
    rstd * (g - mean(g) - xhat * mean(g * xhat)), xhat = layer_norm(x),
    rstd = 1 / sqrt(var + eps) (biased variance, gamma=1, beta=0)."""
    x = np.asarray(x, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    mean = x.mean(axis=-1, keepdims=True)
    centred = x - mean
    var = (centred * centred).mean(axis=-1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + eps)
    xhat = centred * rstd
    return rstd * (g - g.mean(axis=-1, keepdims=True) - xhat * (g * xhat).mean(axis=-1, keepdims=True))


def mlp_backward(y1, dy, w: dict, eps: float = LN_EPS, storage="fp16", grad_storage="bf16") -> dict:
    """Gradients of the MLP half for rows y1 [n, h] given dY [n, h]:
    {"dy1": [n, h], "dw1": [h, F], "dw2": [F, h]} (weights in the math
    orientation [in, out]).

    Precision model (the values the layer keeps in 16 bits, rounded to
    nearest even; every product and sum in fp64):
    * forward part, as in rank_rows_forward with `storage`: the weights, the
      LN2 output Xn2 and the pre-activation U = Xn2 W1 are stored in
      `storage`;
    * backward part, in `grad_storage`: dU, and the copies of Xn2 and
      H = GELU(U) that feed the weight-gradient products, are stored in
      `grad_storage`; dY and the bf16 weights enter as given.  dH, dXn2, dY1,
      dW1 and dW2 stay unrounded.
    storage=None and grad_storage=None give the plain fp64 chain rule.
    """
    rnd, grnd = _rounder(storage), _rounder(grad_storage)
    y1 = np.asarray(y1, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    w1 = np.asarray(w["w1"], dtype=np.float64)
    w2 = np.asarray(w["w2"], dtype=np.float64)
    xn2 = rnd(layer_norm(y1, eps))
    u = rnd(xn2 @ rnd(w1))
    hh = grnd(gelu_tanh(u))
    dh = dy @ w2.T
    du = grnd(dh * gelu_tanh_grad(u))
    dxn2 = du @ w1.T
    dy1 = dy + layer_norm_backward(y1, dxn2, eps)
    dw1 = grnd(xn2).T @ du
    dw2 = hh.T @ dy
    return {"dy1": dy1, "dw1": dw1, "dw2": dw2, "du": du, "u": u}


def mlp_backward_sampled(y1, dy, w: dict, rows, w1_cols, w2_rows, eps: float = LN_EPS,
                         storage="fp16", grad_storage="bf16") -> dict:
    """The outputs of mlp_backward at sampled places, each computed alone
    with the same precision model: dY1 at rows `rows` (row-local), dW1 at
    columns `w1_cols` (column j needs U[:, j] and dU[:, j] over all rows) and
    dW2 at rows `w2_rows` (row f needs H[:, f]).  For sizes where the full
    products are too slow on a CPU."""
    rnd, grnd = _rounder(storage), _rounder(grad_storage)
    y1 = np.asarray(y1, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    w1 = np.asarray(w["w1"], dtype=np.float64)
    w2 = np.asarray(w["w2"], dtype=np.float64)
    w1r = rnd(w1)
    xn2 = rnd(layer_norm(y1, eps))
    out = {}
    # dY1 rows
    r = np.asarray(rows)
    u_r = rnd(xn2[r] @ w1r)
    du_r = grnd((dy[r] @ w2.T) * gelu_tanh_grad(u_r))
    out["dy1"] = dy[r] + layer_norm_backward(y1[r], du_r @ w1.T, eps)
    # dW1 columns
    c = np.asarray(w1_cols)
    u_c = rnd(xn2 @ w1r[:, c])
    du_c = grnd((dy @ w2[c, :].T) * gelu_tanh_grad(u_c))
    out["dw1"] = grnd(xn2).T @ du_c
    # dW2 rows
    f = np.asarray(w2_rows)
    h_f = grnd(gelu_tanh(rnd(xn2 @ w1r[:, f])))
    out["dw2"] = h_f.T @ dy
    return out


# ----------------------------------------------------------------------------
# backward of causal attention  [TSP ¶1 (training), ¶2 (each rank's queries
# against the all-gathered K/V)]
# ----------------------------------------------------------------------------
def causal_attention_backward(q, k, v, q_pos, dout, n_heads: int, scale: float):
    """Gradients of sum(dout * causal_attention(q, k, v, q_pos)) with respect
    to q [n, H*d] and to the full-sequence k, v [T, H*d], per head:
        S = scale q k^T (keys past q_pos masked), P = softmax(S), O = P v,
        dV = P^T dO,  dP = dO v^T,  dS = P * (dP - rowsum(dP * P)),
        dQ = scale dS k,  dK = scale dS^T q.
    Keys no query row reaches get zero gradient.  A rank's dK, dV are its
    queries' contributions; summed over the ranks they give the gradients of
    the whole sequence (what a reduce-scatter back to the key owners adds)."""
    q = np.asarray(q, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    q_pos = np.asarray(q_pos, dtype=np.int64)
    n, hd = q.shape
    T = np.asarray(k).shape[0]
    d = hd // n_heads
    dq = np.zeros((n, hd))
    dk = np.zeros((T, hd))
    dv = np.zeros((T, hd))
    if n == 0:
        return dq, dk, dv
    _, probs = causal_attention(q, k, v, q_pos, n_heads, scale, return_probs=True)
    kmax = probs[0].shape[1]
    for j in range(n_heads):
        cols = slice(j * d, (j + 1) * d)
        kj = np.asarray(k[:kmax, cols], dtype=np.float64)
        vj = np.asarray(v[:kmax, cols], dtype=np.float64)
        p = probs[j]
        do = dout[:, cols]
        dv[:kmax, cols] = p.T @ do
        dp = do @ vj.T
        ds = p * (dp - (dp * p).sum(axis=1, keepdims=True))
        dq[:, cols] = scale * (ds @ kj)
        dk[:kmax, cols] = scale * (ds.T @ q[:, cols])
    return dq, dk, dv


def attention_logsumexp(q, k, q_pos, n_heads: int, scale: float) -> np.ndarray:
    """Per row and head, the log-sum-exp (natural log) of the row's causal
    scores: lse[i, j] = log sum_{key <= q_pos[i]} exp(scale q_ij . k_j).  The
    softmax probabilities are exp(scale q.k - lse).  Returns [n, H]."""
    q = np.asarray(q, dtype=np.float64)
    q_pos = np.asarray(q_pos, dtype=np.int64)
    n, hd = q.shape
    d = hd // n_heads
    out = np.zeros((n, n_heads))
    if n == 0:
        return out
    kmax = int(q_pos.max()) + 1
    allowed = np.arange(kmax)[None, :] <= q_pos[:, None]
    for j in range(n_heads):
        cols = slice(j * d, (j + 1) * d)
        sc = scale * (q[:, cols] @ np.asarray(k[:kmax, cols], dtype=np.float64).T)
        sc = np.where(allowed, sc, -np.inf)
        m = sc.max(axis=1, keepdims=True)
        out[:, j] = (m + np.log(np.exp(sc - m).sum(axis=1, keepdims=True)))[:, 0]
    return out


def attention_backward_stored(q, k, v, o, q_pos, dout, n_heads: int, scale: float, storage="fp16"):
    """causal_attention_backward with the values a 16-bit tensor-core pipeline
    holds rounded at the points where it stores them.  Per head:
        dO = rnd(dout),  P = softmax of the causal scores (exact),
        Delta = rowsum(dO * o)   (o: the stored attention output),
        dP = dO v^T,  dS = rnd(scale P * (dP - Delta)),
        dV = rnd(P)^T dO,  dK = dS^T q,  dQ = dS k.
    With the exact output o = P v, Delta equals rowsum(dP * P), so with
    storage=None this is causal_attention_backward.  q, k, v and o enter as
    given (already 16-bit in the layer)."""
    rnd = _rounder(storage)
    q = np.asarray(q, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    dout = rnd(dout)
    q_pos = np.asarray(q_pos, dtype=np.int64)
    n, hd = q.shape
    T = np.asarray(k).shape[0]
    d = hd // n_heads
    dq = np.zeros((n, hd))
    dk = np.zeros((T, hd))
    dv = np.zeros((T, hd))
    if n == 0:
        return dq, dk, dv
    _, probs = causal_attention(q, k, v, q_pos, n_heads, scale, return_probs=True)
    kmax = probs[0].shape[1]
    for j in range(n_heads):
        cols = slice(j * d, (j + 1) * d)
        kj = np.asarray(k[:kmax, cols], dtype=np.float64)
        vj = np.asarray(v[:kmax, cols], dtype=np.float64)
        p = probs[j]
        do = dout[:, cols]
        delta = (do * o[:, cols]).sum(axis=1, keepdims=True)
        ds = rnd(scale * p * (do @ vj.T - delta))
        dv[:kmax, cols] = rnd(p).T @ do
        dq[:, cols] = ds @ kj
        dk[:kmax, cols] = ds.T @ q[:, cols]
    return dq, dk, dv


def rank_layer_backward(rank: int, D: int, x_full, w: dict, dy_local, n_heads: int,
                        eps: float = LN_EPS, scale: float | None = None,
                        storage=None, grad_storage=None) -> dict:
    """One TSP rank's share of the whole layer's backward for the loss
    gradient dy_local [L, h] of its own output rows (rank-local order).
    x_full [T, h] is the sequence in natural order.

    The rank computes, from its own rows and the all-gathered K/V:
      the MLP half (mlp_backward): dY1, and its dW1, dW2 contributions;
      the attention half: dA = dY1 Wo^T, dWo = A^T dY1, then the attention
      backward gives dQ for its rows and dK, dV for all T keys;
      dWq = Xn1^T dQ; dXn1 = dQ Wq^T; dX = dY1 + LN1'^T dXn1.
    What crosses ranks: "dk_full", "dv_full" (every rank's contributions,
    summed by a reduce-scatter back to the key owners).  After that sum, each
    owner adds LN1'^T (dK Wk^T + dV Wv^T) to its rows' dX and forms dWk, dWv
    (kv_backward_rows).  Weight-gradient entries are this rank's
    contributions over its tokens; summed over ranks they give the layer's.

    Precision: storage=None and grad_storage=None (the defaults) give the
    plain fp64 chain rule.  Otherwise the forward values are stored as in
    rank_rows_forward(storage) (the weights, LN outputs, Q, K, V, A, H), the
    MLP half follows mlp_backward(storage, grad_storage), the attention
    backward follows attention_backward_stored(storage) with dA stored in
    `storage`, and the gradient products take their operands rounded to
    `grad_storage`: dY1 (for dA and dWo), A (for dWo), dQ and LN1(X) (for
    dWq, dXn1); the bf16 model weights enter those products as given."""
    x_full = np.asarray(x_full, dtype=np.float64)
    T, h = x_full.shape
    if scale is None:
        scale = 1.0 / np.sqrt(h // n_heads)
    rnd, grnd = _rounder(storage), _rounder(grad_storage)
    w_raw = {n: np.asarray(a, dtype=np.float64) for n, a in w.items()}
    w16 = _weights(w_raw, rnd, storage)
    pos = zigzag_index(T, D, rank)
    x = x_full[pos]
    xn_full = rnd(layer_norm(x_full, eps))
    k_full, v_full = rnd(xn_full @ w16["wk"]), rnd(xn_full @ w16["wv"])
    xn1 = xn_full[pos]
    q = rnd(xn1 @ w16["wq"])
    a = rnd(causal_attention(q, k_full, v_full, pos, n_heads, scale))
    y1 = x + a @ w16["wo"]
    mlp = mlp_backward(y1, dy_local, w_raw, eps, storage=storage, grad_storage=grad_storage)
    dy1 = mlp["dy1"]
    dy1_g = grnd(dy1)
    da = rnd(dy1_g @ w_raw["wo"].T)
    dwo = grnd(a).T @ dy1_g
    if storage is None:
        dq, dk_full, dv_full = causal_attention_backward(q, k_full, v_full, pos, da, n_heads, scale)
    else:
        dq, dk_full, dv_full = attention_backward_stored(q, k_full, v_full, a, pos, da, n_heads, scale, storage)
    dq_g = grnd(dq)
    dwq = grnd(xn1).T @ dq_g
    dx = dy1 + layer_norm_backward(x, dq_g @ w_raw["wq"].T, eps)
    return {"dx_partial": dx, "dwq": dwq, "dwo": dwo, "dw1": mlp["dw1"], "dw2": mlp["dw2"],
            "dk_full": dk_full, "dv_full": dv_full}


def kv_backward_rows(x_rows, dk_rows, dv_rows, w: dict, eps: float = LN_EPS,
                     storage=None, grad_storage=None) -> dict:
    """For rows whose keys/values are K = LN1(x) Wk, V = LN1(x) Wv and whose
    summed gradients are dK, dV: the rows' extra input gradient
    LN1'^T (dK Wk^T + dV Wv^T) and their dWk = LN1(x)^T dK, dWv = LN1(x)^T dV.
    With grad_storage, dK, dV and LN1(x) (itself stored in `storage`) enter
    the products rounded to grad_storage; the weights as given."""
    rnd, grnd = _rounder(storage), _rounder(grad_storage)
    x_rows = np.asarray(x_rows, dtype=np.float64)
    xn = grnd(rnd(layer_norm(x_rows, eps)))
    dk = grnd(np.asarray(dk_rows, dtype=np.float64))
    dv = grnd(np.asarray(dv_rows, dtype=np.float64))
    wk = np.asarray(w["wk"], dtype=np.float64)
    wv = np.asarray(w["wv"], dtype=np.float64)
    return {"dx": layer_norm_backward(x_rows, dk @ wk.T + dv @ wv.T, eps),
            "dwk": xn.T @ dk, "dwv": xn.T @ dv}
