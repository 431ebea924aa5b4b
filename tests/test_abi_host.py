"""Host-side checks of the C ABI: the library loads without a GPU, exports every
function include/tsp.h declares, and rejects bad arguments before touching
the device.  No compute call is made here."""
import ctypes
import os
import re

import pytest

from folded_tensor_sequence_rank_b200 import build as tsp_build
from folded_tensor_sequence_rank_b200 import tsp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tsp.h")


@pytest.fixture(scope="module")
def L():
    tsp_build.build()
    return tsp.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tsp_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("tsp_zigzag_index", "tsp_kv_project", "tsp_layer_forward", "tsp_rank_step",
                     "tsp_pack_shards", "tsp_workspace_bytes", "tsp_get_device_status"):
        assert required in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_struct_layouts_match_header():
    # tsp_dims: int64 + 4 x int32 + 2 x float; tsp_weights: int32 D + 6 x 16 pointers
    assert ctypes.sizeof(tsp.Dims) == 32
    assert ctypes.sizeof(tsp.Weights) == 8 + 6 * 16 * 8


def test_status_strings(L):
    for code in range(8):
        assert L.tsp_status_string(code).decode() == tsp.STATUS[code]


def dims(T=512, h=256, H=4, F=1024):
    return tsp.make_dims(T, h, H, F)


@pytest.mark.parametrize("kw,D,expect", [
    (dict(), 2, tsp.TSP_OK),
    (dict(T=0), 2, tsp.TSP_OK),
    (dict(T=800), 2, tsp.TSP_OK),             # ragged chunk (c = 200)
    (dict(T=131072, h=4096, H=32, F=16384), 8, tsp.TSP_OK),
    (dict(T=32768, h=4096, H=32, F=16384), 16, tsp.TSP_OK),
    (dict(T=510), 2, tsp.TSP_ERR_INVALID_ARG),   # T % 2D
    (dict(), 3, tsp.TSP_ERR_INVALID_ARG),        # H % D
    (dict(), 0, tsp.TSP_ERR_INVALID_ARG),
    (dict(), 32, tsp.TSP_ERR_UNSUPPORTED),       # D > TSP_MAX_D
    (dict(h=384, H=4), 2, tsp.TSP_ERR_UNSUPPORTED),   # head_dim 96
    (dict(T=768, h=192, H=3, F=768), 3, tsp.TSP_OK),       # D = 3: h/D = 64, F/D = 256
    (dict(T=768, h=192, H=3, F=768), 2, tsp.TSP_ERR_INVALID_ARG),  # H % D
    (dict(h=256, H=4, F=1024), 4, tsp.TSP_OK),   # h/D = 64
    (dict(h=256, H=4, F=96), 2, tsp.TSP_ERR_UNSUPPORTED),  # F/D = 48
    (dict(T=256, h=8192, H=64, F=16384), 2, tsp.TSP_OK),     # the widest rows the LayerNorm kernels hold
    (dict(T=256, h=8320, H=65, F=16640), 1, tsp.TSP_ERR_UNSUPPORTED),  # h > 8192
])
def test_check_dims(L, kw, D, expect):
    d = dims(**kw)
    assert tsp.check_dims(d, D) == expect


def test_workspace_sizes_and_offsets(L):
    d = dims(T=131072, h=4096, H=32, F=16384)
    off = tsp.workspace_offsets(d, 8)
    assert off[7] == tsp.workspace_bytes(d, 8)
    L_tok = 131072 // 8
    assert off[5] + L_tok * 16384 * 2 <= off[7]
    assert all(o % 1024 == 0 for o in off)
    # shard buffer: a 1 KiB status section, then all six weights once
    assert tsp.shard_buffer_bytes(d, 8) == 1024 + 2 * (4 * 4096 * 4096 + 2 * 4096 * 16384)


def test_bad_arguments_fail_before_any_device_work(L):
    d = dims()
    w = tsp.Weights()
    w.D = 2
    # null weight pointers
    rc = L.tsp_layer_forward(ctypes.byref(d), ctypes.byref(w), 0, None, None, None, None, 0, None, 0, None, None)
    assert rc == tsp.TSP_ERR_INVALID_ARG
    for name in tsp.WEIGHT_NAMES:
        arr = getattr(w, name)
        for k in range(2):
            arr[k] = 0x10000 * (k + 1)
    # rank out of range
    rc = L.tsp_layer_forward(ctypes.byref(d), ctypes.byref(w), 2, 16, 16, 16, 16, 0, 256, 1 << 30, None, None)
    assert rc == tsp.TSP_ERR_INVALID_ARG
    # workspace too small
    rc = L.tsp_layer_forward(ctypes.byref(d), ctypes.byref(w), 0, 16, 16, 16, 16, 0, 256, 1024, None, None)
    assert rc == tsp.TSP_ERR_WORKSPACE
    # misaligned workspace
    rc = L.tsp_kv_project(ctypes.byref(d), ctypes.byref(w), 0, 16, 16, 16, 257, 1 << 30, None)
    assert rc == tsp.TSP_ERR_INVALID_ARG
    # bad output dtype
    rc = L.tsp_rank_step(ctypes.byref(d), ctypes.byref(w), 0, 16, 16, 16, 16, 7, 256, 1 << 30, None, None)
    assert rc == tsp.TSP_ERR_INVALID_ARG
    # zigzag argument checks
    assert L.tsp_zigzag_index(510, 2, 0, None, None) == tsp.TSP_ERR_INVALID_ARG
    assert L.tsp_zigzag_index(512, 2, 2, None, None) == tsp.TSP_ERR_INVALID_ARG
    assert L.tsp_zigzag_index(0, 2, 0, None, None) == tsp.TSP_OK
    # self-test limits
    assert L.tsp_selftest_wait_timeout(256, 0, None) == tsp.TSP_ERR_INVALID_ARG
    assert L.tsp_selftest_wait_timeout(None, 0, None) == tsp.TSP_ERR_INVALID_ARG
    assert L.tsp_selftest_wait_timeout(256, 3 * 10 ** 9, None) == tsp.TSP_ERR_INVALID_ARG


def test_rank_step_host_checks_everything_before_its_first_copy(L):
    """tsp_rank_step_host validates every argument tsp_rank_step would, before
    it enqueues the host-to-device copy: without a GPU, any CUDA call would
    return TSP_ERR_CUDA, so an INVALID_ARG here shows nothing was enqueued."""
    d = dims()
    w = tsp.Weights()
    w.D = 2
    for name in tsp.WEIGHT_NAMES:
        arr = getattr(w, name)
        for k in range(2):
            arr[k] = 0x10000 * (k + 1)
    ws, nws = 256, 1 << 30
    ok = dict(hx=0x1000, xs=0x2000, k=0x3000, v=0x4000, ys=0x5000, hy=0x6000)

    def call(y_dtype=0, **kw):
        a = dict(ok, **kw)
        return L.tsp_rank_step_host(ctypes.byref(d), ctypes.byref(w), 0, a["hx"], a["xs"], a["k"], a["v"], a["ys"],
                                    a["hy"], y_dtype, ws, nws, None, None, None)
    assert call(y_dtype=7) == tsp.TSP_ERR_INVALID_ARG      # output dtype
    assert call(k=None) == tsp.TSP_ERR_INVALID_ARG         # K
    assert call(v=0x4008) == tsp.TSP_ERR_INVALID_ARG       # V misaligned
    assert call(xs=0x2004) == tsp.TSP_ERR_INVALID_ARG      # token staging misaligned
    assert call(ys=None) == tsp.TSP_ERR_INVALID_ARG        # result staging
    assert call(hx=None) == tsp.TSP_ERR_INVALID_ARG        # host tokens
    # with valid arguments the first CUDA call is reached and fails for want
    # of a GPU (on a GPU machine it would copy from the fake host address)
    import torch
    if not torch.cuda.is_available():
        assert call() == tsp.TSP_ERR_CUDA


def test_empty_sequence_is_a_no_op(L):
    d = dims(T=0)
    w = tsp.Weights()
    w.D = 2
    for name in tsp.WEIGHT_NAMES:
        arr = getattr(w, name)
        for k in range(2):
            arr[k] = 0x10000 * (k + 1)
    ws = tsp.workspace_bytes(d, 2)
    assert ws > 0
    rc = L.tsp_layer_forward(ctypes.byref(d), ctypes.byref(w), 1, None, None, None, None, 0, 1024, ws, None, None)
    assert rc == tsp.TSP_OK


def test_binding_refuses_cpu_tensors(L):
    import torch
    d = dims()
    with pytest.raises(ValueError):
        tsp.pack_shards(d, 2, {n: torch.zeros(1, dtype=torch.bfloat16) for n in tsp.WEIGHT_NAMES})


def test_memory_account_7b_forward():
    """Per-GPU bytes of a 32-layer forward of the 7B layer at 128K on D = 8
    GPUs, against the formula written out here: 384 MiB of fp16 weights per
    layer, 1/D of them owned, one layer's other shards in flight, the rank's
    tokens in and out, the all-gathered K/V, and the layer workspace."""
    from folded_tensor_sequence_rank_b200 import stack
    dims = tsp.make_dims(131072, 4096, 32, 16384)
    acc = stack.memory_account(dims, 8, 32)
    MiB = 1 << 20
    assert acc["weights_own_shards"] == 32 * 384 * MiB // 8
    assert acc["weights_receive_buffer"] == 384 * MiB * 7 // 8
    assert acc["tokens_in_out"] == 2 * 16384 * 4096 * 2
    assert acc["kv_all_gathered"] == 2 * 131072 * 4096 * 2
    assert acc["workspace"] == tsp.workspace_bytes(dims, 8) > 0
    assert acc["total"] == sum(v for k, v in acc.items() if k != "total")
    assert 5.0 < acc["total"] / 2**30 < 6.0


def test_mlp_backward_argument_checks(L):
    d = dims()
    w = tsp.Weights()
    w.D = 2
    for name in tsp.WEIGHT_NAMES:
        arr = getattr(w, name)
        for k in range(2):
            arr[k] = 0x10000 * (k + 1)
    n = L.tsp_mlp_backward_workspace_bytes(ctypes.byref(d), 2)
    L_tok, h, F = 256, 256, 1024
    # the backward workspace holds at least the recomputed and transposed activations
    assert n >= L_tok * (h * 2 + F * 2 * 4 + h * 4 + h * 2 * 2)
    assert L.tsp_mlp_backward_workspace_bytes(ctypes.byref(dims(T=510)), 2) == 0
    ok = [16] * 7
    # a null or misaligned pointer
    for i in range(7):
        args = list(ok)
        args[i] = None
        assert L.tsp_mlp_backward(ctypes.byref(d), ctypes.byref(w), *args, 256, n, None, None) == tsp.TSP_ERR_INVALID_ARG
        args[i] = 24
        assert L.tsp_mlp_backward(ctypes.byref(d), ctypes.byref(w), *args, 256, n, None, None) == tsp.TSP_ERR_INVALID_ARG
    # workspace: misaligned, then too small
    assert L.tsp_mlp_backward(ctypes.byref(d), ctypes.byref(w), *ok, 272, n, None, None) == tsp.TSP_ERR_INVALID_ARG
    assert L.tsp_mlp_backward(ctypes.byref(d), ctypes.byref(w), *ok, 256, n - 1, None, None) == tsp.TSP_ERR_WORKSPACE
    # ragged token count: T/D = 400 is not a multiple of 128
    d3 = dims(T=800)
    n3 = L.tsp_mlp_backward_workspace_bytes(ctypes.byref(d3), 2)
    assert L.tsp_mlp_backward(ctypes.byref(d3), ctypes.byref(w), *ok, 256, n3, None, None) == tsp.TSP_ERR_UNSUPPORTED
    # h not a multiple of 256
    d2 = dims(T=768, h=192, H=3, F=768)
    w.D = 3
    for name in tsp.WEIGHT_NAMES:
        getattr(w, name)[2] = 0x30000
    n2 = L.tsp_mlp_backward_workspace_bytes(ctypes.byref(d2), 3)
    assert L.tsp_mlp_backward(ctypes.byref(d2), ctypes.byref(w), *ok, 256, n2, None, None) == tsp.TSP_ERR_UNSUPPORTED


def test_mlp_backward_binding_checks_shapes_before_the_call(L):
    import torch
    d = dims()
    w = tsp.ShardedWeights(D=2, buf=torch.zeros(1, dtype=torch.uint8), struct=tsp.Weights())
    cpu = torch.zeros(4, dtype=torch.bfloat16)
    with pytest.raises(ValueError):  # CPU tensors are refused before the library is called
        tsp.mlp_backward(d, w, cpu, cpu, cpu, cpu, cpu, cpu, cpu, torch.zeros(16, dtype=torch.uint8))


def test_attn_backward_checks_arguments_first(L):
    d = dims()
    n = L.tsp_attn_backward_workspace_bytes(ctypes.byref(d), 2)
    assert n > 0
    ok = [0x1000 * (i + 1) for i in range(9)]

    def call(rank=0, D=2, ws=256, nws=n, ptrs=ok):
        return L.tsp_attn_backward(ctypes.byref(d), D, rank, *ptrs, ws, nws, None)
    assert call(rank=2) == tsp.TSP_ERR_INVALID_ARG                 # rank out of range
    assert call(D=3) == tsp.TSP_ERR_INVALID_ARG                    # H % D
    assert call(ws=257) == tsp.TSP_ERR_INVALID_ARG                 # misaligned workspace
    assert call(nws=n - 1) == tsp.TSP_ERR_WORKSPACE
    for i in range(9):                                             # each pointer: null, then misaligned
        assert call(ptrs=ok[:i] + [None] + ok[i + 1:]) == tsp.TSP_ERR_INVALID_ARG, i
        assert call(ptrs=ok[:i] + [ok[i] + 8] + ok[i + 1:]) == tsp.TSP_ERR_INVALID_ARG, i
    e = dims(T=0)
    assert L.tsp_attn_backward(ctypes.byref(e), 2, 0, *ok, 256, 1 << 20, None) == tsp.TSP_OK  # no tokens


def test_debug_build_exports_the_same_abi():
    """The -DTSP_DEBUG build (device index checks that report TSP_ERR_BOUNDS)
    exports every declared function too."""
    lib = tsp_build.build(debug=True)
    Ld = ctypes.CDLL(lib)
    for name in declared_functions():
        assert hasattr(Ld, name), name
    Ld.tsp_status_string.restype = ctypes.c_char_p
    assert Ld.tsp_status_string(tsp.TSP_ERR_BOUNDS).decode() == tsp.STATUS[tsp.TSP_ERR_BOUNDS]
