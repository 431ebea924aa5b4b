"""Python binding of libtsp_b200.so (the C ABI in include/tsp.h).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity, then their pointers and the current CUDA stream are passed to the
C functions.  Every step of the layer runs in the library's CUDA kernels;
there is no fallback.  If the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import torch

MAX_D = 16
N_STEP_EVENTS = 8
N_WS_OFFSETS = 9
OUT_BF16, OUT_F32 = 0, 1
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "CUDA error",
          4: "device wait timed out", 5: "workspace too small", 6: "fp16 conversion saturated",
          7: "device index check failed"}
(TSP_OK, TSP_ERR_INVALID_ARG, TSP_ERR_UNSUPPORTED, TSP_ERR_CUDA, TSP_ERR_TIMEOUT, TSP_ERR_WORKSPACE,
 TSP_ERR_SATURATED, TSP_ERR_BOUNDS) = range(8)
DEVICE_STATUSES = (TSP_OK, TSP_ERR_TIMEOUT, TSP_ERR_SATURATED, TSP_ERR_BOUNDS)

# TSP_LIBRARY selects another build of the library (the -DTSP_DEBUG one).
LIB_PATH = os.environ.get("TSP_LIBRARY") or os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtsp_b200.so")
WEIGHT_NAMES = ("wq", "wk", "wv", "wo", "w1", "w2")


class TSPError(RuntimeError):
    def __init__(self, code: int, what: str, detail: str = ""):
        self.code = code
        msg = f"{what}: {STATUS.get(code, code)}"
        if detail:
            msg += f" ({detail})"
        super().__init__(msg)


class Dims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("h", ctypes.c_int32), ("n_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("ffn", ctypes.c_int32), ("ln_eps", ctypes.c_float),
                ("softmax_scale", ctypes.c_float)]


class Weights(ctypes.Structure):
    _fields_ = [("D", ctypes.c_int32)] + [(n, ctypes.c_void_p * MAX_D) for n in WEIGHT_NAMES]


_lib = None


def lib() -> ctypes.CDLL:
    """Loads the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m folded_tensor_sequence_rank_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    pd, pw = ctypes.POINTER(Dims), ctypes.POINTER(Weights)
    sig = {
        "tsp_status_string": (ctypes.c_char_p, [i32]),
        "tsp_last_cuda_error": (ctypes.c_char_p, []),
        "tsp_check_dims": (i32, [pd, i32]),
        "tsp_zigzag_index": (i32, [i64, i32, i32, vp, vp]),
        "tsp_shard_buffer_bytes": (sz, [pd, i32]),
        "tsp_pack_shards": (i32, [pd, i32, ctypes.POINTER(vp), vp, sz, pw, vp]),
        "tsp_workspace_bytes": (sz, [pd, i32]),
        "tsp_workspace_offsets": (i32, [pd, i32, ctypes.POINTER(sz)]),
        "tsp_reset_device_status": (i32, [vp, vp]),
        "tsp_get_device_status": (i32, [vp, vp]),
        "tsp_kv_project": (i32, [pd, pw, i32, vp, vp, vp, vp, sz, vp]),
        "tsp_kv_project_noalloc": (i32, [pd, pw, i32, vp, vp, vp, vp]),
        "tsp_kv_project_noalloc_status": (i32, [vp]),
        "tsp_layer_forward": (i32, [pd, pw, i32, vp, vp, vp, vp, i32, vp, sz, vp, ctypes.POINTER(vp)]),
        "tsp_rank_step": (i32, [pd, pw, i32, vp, vp, vp, vp, i32, vp, sz, vp, ctypes.POINTER(vp)]),
        "tsp_rank_step_host": (i32, [pd, pw, i32, vp, vp, vp, vp, vp, vp, i32, vp, sz, vp, vp, vp]),
        "tsp_selftest_wait_timeout": (i32, [vp, ctypes.c_uint64, vp]),
        "tsp_attn_backward_workspace_bytes": (sz, [pd, i32]),
        "tsp_attn_backward": (i32, [pd, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "tsp_layer_backward_workspace_bytes": (sz, [pd, i32]),
        "tsp_layer_backward": (i32, [pd, pw, ctypes.POINTER(vp), i32, vp, vp, sz, vp, vp, vp, vp, vp, vp, vp, vp,
                                     vp, vp, vp, sz, vp, ctypes.POINTER(vp)]),
        "tsp_kv_backward_workspace_bytes": (sz, [pd, i32]),
        "tsp_kv_backward": (i32, [pd, i32, ctypes.POINTER(vp), i32, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "tsp_shard_workspace_bytes": (sz, []),
        "tsp_layernorm": (i32, [i64, i32, ctypes.c_float, vp, i32, vp, vp]),
        "tsp_shard_qkv": (i32, [pd, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "tsp_shard_attention": (i32, [pd, i32, i32, vp, vp, vp, vp, vp, vp]),
        "tsp_shard_ffn_up": (i32, [pd, i32, vp, vp, vp, vp, vp]),
        "tsp_shard_accumulate": (i32, [pd, i32, vp, i32, vp, vp, vp, vp]),
        "tsp_tp_workspace_bytes": (sz, [pd, i32]),
        "tsp_tp_attention_partial": (i32, [pd, pw, i32, vp, vp, vp, sz, vp]),
        "tsp_tp_mlp_partial": (i32, [pd, pw, i32, vp, vp, vp, sz, vp]),
        "tsp_tp_all_reduce": (i32, [pd, i32, ctypes.POINTER(vp), vp, i32, vp, i32, vp]),
        "tsp_mlp_backward_workspace_bytes": (sz, [pd, i32]),
        "tsp_mlp_backward": (i32, [pd, pw, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, ctypes.POINTER(vp)]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def _check(rc: int, what: str):
    if rc != TSP_OK:
        detail = lib().tsp_last_cuda_error().decode() if rc == TSP_ERR_CUDA else ""
        raise TSPError(rc, what, detail)


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t: torch.Tensor | None, name: str, dtype=None, shape=None, cuda=True):
    if t is None:
        raise ValueError(f"{name} is required")
    if cuda and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


# ---------------------------------------------------------------------------
def make_dims(T: int, h: int, n_heads: int, ffn: int, ln_eps: float = 1e-5,
              softmax_scale: float | None = None) -> Dims:
    d = h // n_heads
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    return Dims(T, h, n_heads, d, ffn, ln_eps, softmax_scale)


def check_dims(dims: Dims, D: int) -> int:
    return lib().tsp_check_dims(ctypes.byref(dims), D)


def local_tokens(dims: Dims, D: int) -> int:
    return dims.T // D


def zigzag_index(T: int, D: int, rank: int, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty(T // D, dtype=torch.int32, device="cuda")
    _check(lib().tsp_zigzag_index(T, D, rank, _ptr(out, "out", torch.int32, (T // D,)), _stream(stream)),
           "tsp_zigzag_index")
    return out


def shard_buffer_bytes(dims: Dims, D: int) -> int:
    return lib().tsp_shard_buffer_bytes(ctypes.byref(dims), D)


@dataclass
class ShardedWeights:
    """Per-shard weight pointers plus the buffer that owns them."""
    D: int
    buf: torch.Tensor
    struct: Weights

    def shard(self, name: str, k: int, shape) -> torch.Tensor:
        """A view of shard k of weight `name` (for inspection)."""
        base = self.buf.data_ptr()
        ptr = getattr(self.struct, name)[k]
        n = int(torch.tensor(shape).prod())
        off = ptr - base
        return self.buf[off: off + 2 * n].view(torch.float16).view(*shape)


def pack_shards(dims: Dims, D: int, w_full: dict, stream=None) -> ShardedWeights:
    """Splits full math-orientation bf16 weights ([in, out], CUDA) into D fp16 shards."""
    h, F = dims.h, dims.ffn
    shapes = {"wq": (h, h), "wk": (h, h), "wv": (h, h), "wo": (h, h), "w1": (h, F), "w2": (F, h)}
    ptrs = (ctypes.c_void_p * 6)(*[_ptr(w_full[n], n, torch.bfloat16, shapes[n]) for n in WEIGHT_NAMES])
    nbytes = shard_buffer_bytes(dims, D)
    if nbytes == 0:
        _check(check_dims(dims, D) or TSP_ERR_INVALID_ARG, "tsp_shard_buffer_bytes")
    buf = torch.empty(nbytes, dtype=torch.uint8, device=w_full["wq"].device)
    ws = Weights()
    _check(lib().tsp_pack_shards(ctypes.byref(dims), D, ptrs, buf.data_ptr(), nbytes, ctypes.byref(ws),
                                 _stream(stream)), "tsp_pack_shards")
    return ShardedWeights(D, buf, ws)


def workspace_bytes(dims: Dims, D: int) -> int:
    return lib().tsp_workspace_bytes(ctypes.byref(dims), D)


def workspace_offsets(dims: Dims, D: int) -> list:
    off = (ctypes.c_size_t * N_WS_OFFSETS)()
    _check(lib().tsp_workspace_offsets(ctypes.byref(dims), D, off), "tsp_workspace_offsets")
    return list(off)


def alloc_workspace(dims: Dims, D: int, device="cuda") -> torch.Tensor:
    n = workspace_bytes(dims, D)
    if n == 0:
        _check(check_dims(dims, D) or TSP_ERR_INVALID_ARG, "tsp_workspace_bytes")
    ws = torch.zeros(n, dtype=torch.uint8, device=device)
    return ws


def workspace_view(ws: torch.Tensor, dims: Dims, D: int, name: str) -> torch.Tensor:
    """Views of the per-rank intermediates left in the workspace."""
    off = workspace_offsets(dims, D)
    L, h, F = dims.T // D, dims.h, dims.ffn
    table = {"xn": (1, torch.float16, (L, h)), "q": (2, torch.float16, (L, h)),
             "a": (3, torch.float16, (L, h)), "y1": (4, torch.float32, (L, h)),
             "h": (5, torch.float16, (L, F)), "lse": (8, torch.float32, (dims.n_heads, 2, stash_rows(dims, D)))}
    i, dt, shape = table[name]
    nb = int(torch.tensor(shape).prod()) * (4 if dt == torch.float32 else 2)
    return ws[off[i]: off[i] + nb].view(dt).view(*shape)


def stash_rows(dims: Dims, D: int) -> int:
    """Rows per chunk of the per-head stashes [H][2][c_pad]: c rounded up to 128."""
    c = dims.T // (2 * D)
    return (c + 127) // 128 * 128


def lse_rows(lse_stash: torch.Tensor, dims: Dims, D: int) -> torch.Tensor:
    """The forward's log-sum-exp stash [H][2][c_pad] as [T/D, H] in rank-local order."""
    c = dims.T // (2 * D)
    return torch.cat([lse_stash[:, 0, :c], lse_stash[:, 1, :c]], dim=1).t()


def reset_device_status(ws: torch.Tensor, stream=None):
    _check(lib().tsp_reset_device_status(_ptr(ws, "ws"), _stream(stream)), "tsp_reset_device_status")


def get_device_status(ws: torch.Tensor, stream=None) -> int:
    """Reads a status section (a workspace, an MLP backward workspace or a
    packed shard buffer): TSP_OK, TSP_ERR_TIMEOUT or TSP_ERR_SATURATED."""
    rc = lib().tsp_get_device_status(_ptr(ws, "ws"), _stream(stream))
    if rc not in DEVICE_STATUSES:
        _check(rc, "tsp_get_device_status")
    return rc


def kv_project_noalloc_status(stream=None) -> int:
    """Status section of tsp_kv_project_noalloc's static scratch (its last call)."""
    rc = lib().tsp_kv_project_noalloc_status(_stream(stream))
    if rc not in DEVICE_STATUSES:
        _check(rc, "tsp_kv_project_noalloc_status")
    return rc


def _rank_io(dims: Dims, w: ShardedWeights, x_local, k_full, v_full, y_local, ws):
    L, h, T = dims.T // w.D, dims.h, dims.T
    px = _ptr(x_local, "x_local", torch.bfloat16, (L, h))
    pk = _ptr(k_full, "k_full", torch.float16, (T, h))
    pv = _ptr(v_full, "v_full", torch.float16, (T, h))
    if y_local is not None and y_local.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("y_local must be bf16 or fp32")
    py = _ptr(y_local, "y_local", None, (L, h)) if y_local is not None else None
    pws = _ptr(ws, "ws", torch.uint8)
    return px, pk, pv, py, pws


def _events(events):
    if events is None:
        return None
    if len(events) != N_STEP_EVENTS:
        raise ValueError(f"need {N_STEP_EVENTS} events")
    for e in events:
        if not e.cuda_event:  # torch creates the CUDA event on its first record
            e.record()
    return (ctypes.c_void_p * N_STEP_EVENTS)(*[e.cuda_event for e in events])


def kv_project(dims: Dims, w: ShardedWeights, rank: int, x_local, k_full, v_full, ws, stream=None):
    px, pk, pv, _, pws = _rank_io(dims, w, x_local, k_full, v_full, None, ws)
    _check(lib().tsp_kv_project(ctypes.byref(dims), ctypes.byref(w.struct), rank, px, pk, pv, pws, ws.numel(),
                                _stream(stream)), "tsp_kv_project")


def kv_project_noalloc(dims: Dims, w: ShardedWeights, rank: int, x_local, k_full, v_full, stream=None):
    """tsp_kv_project without a workspace (for callers that cannot allocate):
    its scratch is a fixed 64 MiB device array inside the library."""
    ws_dummy = torch.empty(0, dtype=torch.uint8, device=x_local.device)
    px, pk, pv, _, _ = _rank_io(dims, w, x_local, k_full, v_full, None, ws_dummy)
    _check(lib().tsp_kv_project_noalloc(ctypes.byref(dims), ctypes.byref(w.struct), rank, px, pk, pv,
                                        _stream(stream)), "tsp_kv_project_noalloc")


def layer_forward(dims: Dims, w: ShardedWeights, rank: int, x_local, k_full, v_full, y_local, ws,
                  stream=None, events=None):
    px, pk, pv, py, pws = _rank_io(dims, w, x_local, k_full, v_full, y_local, ws)
    yd = OUT_F32 if y_local.dtype == torch.float32 else OUT_BF16
    _check(lib().tsp_layer_forward(ctypes.byref(dims), ctypes.byref(w.struct), rank, px, pk, pv, py, yd, pws,
                                   ws.numel(), _stream(stream), _events(events)), "tsp_layer_forward")


def rank_step(dims: Dims, w: ShardedWeights, rank: int, x_local, k_full, v_full, y_local, ws,
              stream=None, events=None):
    px, pk, pv, py, pws = _rank_io(dims, w, x_local, k_full, v_full, y_local, ws)
    yd = OUT_F32 if y_local.dtype == torch.float32 else OUT_BF16
    _check(lib().tsp_rank_step(ctypes.byref(dims), ctypes.byref(w.struct), rank, px, pk, pv, py, yd, pws,
                               ws.numel(), _stream(stream), _events(events)), "tsp_rank_step")


def attn_backward_workspace_bytes(dims: Dims, D: int) -> int:
    return lib().tsp_attn_backward_workspace_bytes(ctypes.byref(dims), D)


def alloc_attn_backward_workspace(dims: Dims, D: int, device="cuda") -> torch.Tensor:
    n = attn_backward_workspace_bytes(dims, D)
    if n == 0:
        _check(check_dims(dims, D) or TSP_ERR_INVALID_ARG, "tsp_attn_backward_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def attn_backward(dims: Dims, D: int, rank: int, q, k_full, v_full, o, lse, d_o, dq, dk_full, dv_full, aws,
                  stream=None):
    """Backward of rank `rank`'s causal attention: dq [T/D, h] fp32 (overwritten),
    dk_full, dv_full [T, h] fp32 (added to), from the forward's Q, A (o) and
    log-sum-exp stash, the all-gathered K/V and the gradient d_o of A (fp16)."""
    L, h, T = dims.T // D, dims.h, dims.T
    args = [_ptr(q, "q", torch.float16, (L, h)), _ptr(k_full, "k_full", torch.float16, (T, h)),
            _ptr(v_full, "v_full", torch.float16, (T, h)), _ptr(o, "o", torch.float16, (L, h)),
            _ptr(lse, "lse", torch.float32, (dims.n_heads, 2, stash_rows(dims, D))),
            _ptr(d_o, "d_o", torch.float16, (L, h)), _ptr(dq, "dq", torch.float32, (L, h)),
            _ptr(dk_full, "dk_full", torch.float32, (T, h)), _ptr(dv_full, "dv_full", torch.float32, (T, h))]
    _check(lib().tsp_attn_backward(ctypes.byref(dims), D, rank, *args, _ptr(aws, "aws", torch.uint8), aws.numel(),
                                   _stream(stream)), "tsp_attn_backward")


def _alloc_ws(fn_name: str, dims: Dims, D: int, device="cuda") -> torch.Tensor:
    n = getattr(lib(), fn_name)(ctypes.byref(dims), D)
    if n == 0:
        _check(check_dims(dims, D) or TSP_ERR_INVALID_ARG, fn_name)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def alloc_layer_backward_workspace(dims: Dims, D: int, device="cuda") -> torch.Tensor:
    return _alloc_ws("tsp_layer_backward_workspace_bytes", dims, D, device)


def alloc_kv_backward_workspace(dims: Dims, D: int, device="cuda") -> torch.Tensor:
    return _alloc_ws("tsp_kv_backward_workspace_bytes", dims, D, device)


def _w_full_ptrs(dims: Dims, w_full: dict):
    h, F = dims.h, dims.ffn
    shapes = {"wq": (h, h), "wk": (h, h), "wv": (h, h), "wo": (h, h), "w1": (h, F), "w2": (F, h)}
    return (ctypes.c_void_p * 6)(*[_ptr(w_full[n], n, torch.bfloat16, shapes[n]) for n in WEIGHT_NAMES])


def layer_backward(dims: Dims, w: ShardedWeights, w_full: dict, rank: int, x_local, fwd_ws, k_full, v_full, dy,
                   dx, grads: dict, dk_full, dv_full, bws, stream=None, events=None):
    """One rank's share of the layer's backward (see tsp_layer_backward):
    dx [T/D, h] fp32, grads["wq"|"wo"|"w1"|"w2"] fp32 in the math orientation
    (overwritten); dk_full, dv_full [T, h] fp32 added to.  fwd_ws is this
    rank's forward workspace; w_full the bf16 model weights [in, out]."""
    L, h, F, T = dims.T // w.D, dims.h, dims.ffn, dims.T
    args = [_ptr(x_local, "x_local", torch.bfloat16, (L, h)), _ptr(fwd_ws, "fwd_ws", torch.uint8), fwd_ws.numel(),
            _ptr(k_full, "k_full", torch.float16, (T, h)), _ptr(v_full, "v_full", torch.float16, (T, h)),
            _ptr(dy, "dy", torch.bfloat16, (L, h)), _ptr(dx, "dx", torch.float32, (L, h)),
            _ptr(grads["wq"], "dwq", torch.float32, (h, h)), _ptr(grads["wo"], "dwo", torch.float32, (h, h)),
            _ptr(grads["w1"], "dw1", torch.float32, (h, F)), _ptr(grads["w2"], "dw2", torch.float32, (F, h)),
            _ptr(dk_full, "dk_full", torch.float32, (T, h)), _ptr(dv_full, "dv_full", torch.float32, (T, h))]
    _check(lib().tsp_layer_backward(ctypes.byref(dims), ctypes.byref(w.struct), _w_full_ptrs(dims, w_full), rank,
                                    *args, _ptr(bws, "bws", torch.uint8), bws.numel(), _stream(stream),
                                    _events(events)), "tsp_layer_backward")


def kv_backward(dims: Dims, D: int, w_full: dict, rank: int, x_local, dk_full, dv_full, dx, dwk, dwv, kws,
                stream=None):
    """The key owner's step after the dK/dV sum (see tsp_kv_backward): dx added
    to, dwk, dwv [h, h] fp32 overwritten."""
    L, h, T = dims.T // D, dims.h, dims.T
    args = [_ptr(x_local, "x_local", torch.bfloat16, (L, h)), _ptr(dk_full, "dk_full", torch.float32, (T, h)),
            _ptr(dv_full, "dv_full", torch.float32, (T, h)), _ptr(dx, "dx", torch.float32, (L, h)),
            _ptr(dwk, "dwk", torch.float32, (h, h)), _ptr(dwv, "dwv", torch.float32, (h, h))]
    _check(lib().tsp_kv_backward(ctypes.byref(dims), D, _w_full_ptrs(dims, w_full), rank, *args,
                                 _ptr(kws, "kws", torch.uint8), kws.numel(), _stream(stream)), "tsp_kv_backward")


def alloc_tp_workspace(dims: Dims, D: int, device="cuda") -> torch.Tensor:
    return _alloc_ws("tsp_tp_workspace_bytes", dims, D, device)


def tp_attention_partial(dims: Dims, w: ShardedWeights, k: int, x, part, ws, stream=None):
    """Tensor-parallel rank k's attention partial A_k Wo_k^T over all T tokens
    (x bf16 [T, h]; part fp32 [T, h])."""
    T, h = dims.T, dims.h
    _check(lib().tsp_tp_attention_partial(ctypes.byref(dims), ctypes.byref(w.struct), k,
                                          _ptr(x, "x", torch.bfloat16, (T, h)), _ptr(part, "part", torch.float32, (T, h)),
                                          _ptr(ws, "ws", torch.uint8), ws.numel(), _stream(stream)),
           "tsp_tp_attention_partial")


def tp_mlp_partial(dims: Dims, w: ShardedWeights, k: int, y1, part, ws, stream=None):
    """Tensor-parallel rank k's MLP partial GELU(LN2(Y1) W1_k^T) W2_k^T (y1, part fp32 [T, h])."""
    T, h = dims.T, dims.h
    _check(lib().tsp_tp_mlp_partial(ctypes.byref(dims), ctypes.byref(w.struct), k,
                                    _ptr(y1, "y1", torch.float32, (T, h)), _ptr(part, "part", torch.float32, (T, h)),
                                    _ptr(ws, "ws", torch.uint8), ws.numel(), _stream(stream)), "tsp_tp_mlp_partial")


def tp_all_reduce(dims: Dims, parts: list, resid, out, stream=None):
    """out = resid + sum(parts): the tensor-parallel all-reduce, on one GPU."""
    T, h = dims.T, dims.h
    ptrs = (ctypes.c_void_p * len(parts))(*[_ptr(t, "part", torch.float32, (T, h)) for t in parts])
    if resid.dtype not in (torch.float32, torch.bfloat16) or out.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("resid and out must be fp32 or bf16")
    _check(lib().tsp_tp_all_reduce(ctypes.byref(dims), len(parts), ptrs, _ptr(resid, "resid", None, (T, h)),
                                   int(resid.dtype == torch.float32), _ptr(out, "out", None, (T, h)),
                                   OUT_F32 if out.dtype == torch.float32 else OUT_BF16, _stream(stream)),
           "tsp_tp_all_reduce")


def mlp_backward_workspace_bytes(dims: Dims, D: int) -> int:
    return lib().tsp_mlp_backward_workspace_bytes(ctypes.byref(dims), D)


def alloc_mlp_backward_workspace(dims: Dims, D: int, device="cuda") -> torch.Tensor:
    n = mlp_backward_workspace_bytes(dims, D)
    if n == 0:
        _check(check_dims(dims, D) or TSP_ERR_INVALID_ARG, "tsp_mlp_backward_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def mlp_backward(dims: Dims, w: ShardedWeights, w1_full, w2_full, y1, dy, dy1, dw1, dw2, bws,
                 stream=None, events=None):
    """Backward of the MLP half for one rank's rows: dy1 = dL/dY1, dw1 = dL/dW1 [h, F],
    dw2 = dL/dW2 [F, h] (fp32), from y1 (fp32) and dy (bf16) [T/D, h], rank-local order.
    w1_full [h, F] and w2_full [F, h] are the full bf16 weights in the math orientation."""
    L, h, F = dims.T // w.D, dims.h, dims.ffn
    args = [_ptr(w1_full, "w1_full", torch.bfloat16, (h, F)), _ptr(w2_full, "w2_full", torch.bfloat16, (F, h)),
            _ptr(y1, "y1", torch.float32, (L, h)) if L else None, _ptr(dy, "dy", torch.bfloat16, (L, h)) if L else None,
            _ptr(dy1, "dy1", torch.float32, (L, h)) if L else None, _ptr(dw1, "dw1", torch.float32, (h, F)),
            _ptr(dw2, "dw2", torch.float32, (F, h))]
    _check(lib().tsp_mlp_backward(ctypes.byref(dims), ctypes.byref(w.struct), *args, _ptr(bws, "bws", torch.uint8),
                                  bws.numel(), _stream(stream), _events(events)), "tsp_mlp_backward")


def _event(e):
    """A torch.cuda.Event as a CUDA event handle (created on first use), or None."""
    if e is None:
        return None
    if not e.cuda_event:
        e.record()  # torch creates the CUDA event on its first record
    return e.cuda_event


def rank_step_host(dims: Dims, w: ShardedWeights, rank: int, h_x_local, x_staging, k_full, v_full,
                   y_staging, h_y_local, ws, stream=None, compute_after=None, compute_done=None):
    """rank_step with host (ideally pinned) token buffers; copies run on the stream.
    compute_after / compute_done: optional torch.cuda.Event objects that order
    this step's kernels after another step's and mark their end (see the C
    header)."""
    L, h = dims.T // w.D, dims.h
    if h_x_local.is_cuda or h_y_local.is_cuda:
        raise ValueError("h_x_local and h_y_local must be host tensors")
    phx = _ptr(h_x_local, "h_x_local", torch.bfloat16, (L, h), cuda=False)
    phy = _ptr(h_y_local, "h_y_local", y_staging.dtype, (L, h), cuda=False)
    pxs = _ptr(x_staging, "x_staging", torch.bfloat16, (L, h))
    pys = _ptr(y_staging, "y_staging", None, (L, h))
    pk = _ptr(k_full, "k_full", torch.float16, (dims.T, h))
    pv = _ptr(v_full, "v_full", torch.float16, (dims.T, h))
    yd = OUT_F32 if y_staging.dtype == torch.float32 else OUT_BF16
    _check(lib().tsp_rank_step_host(ctypes.byref(dims), ctypes.byref(w.struct), rank, phx, pxs, pk, pv, pys, phy,
                                    yd, _ptr(ws, "ws", torch.uint8), ws.numel(), _stream(stream),
                                    _event(compute_after), _event(compute_done)),
           "tsp_rank_step_host")


def selftest_wait_timeout(ws: torch.Tensor | None, timeout_ns: int, stream=None):
    """ws=None targets the status section of tsp_kv_project_noalloc's scratch."""
    _check(lib().tsp_selftest_wait_timeout(None if ws is None else _ptr(ws, "ws"), timeout_ns, _stream(stream)),
           "tsp_selftest_wait_timeout")
