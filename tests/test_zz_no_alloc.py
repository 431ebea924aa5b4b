"""The allocation-free K/V projection (tsp_kv_project_noalloc), called through
the C ABI, against the workspace-taking tsp_kv_project.

Some callers cannot allocate device memory (a plugin handed only its input
and output buffers, or a hot path where cudaMalloc could synchronise or
fail), so the library offers this one entry point whose scratch is a fixed
device array inside the library.  It must give the same K and V as the
regular entry point - the same kernels run, so bit for bit - on two calls in
a row, which share that array.  This file is collected last so that a run
stopping at its first failure has already run every other test; it also
passes alone in a fresh process (it builds and loads the library itself).
"""
import ctypes

import pytest
import torch

from folded_tensor_sequence_rank_b200 import build as tsp_build
from folded_tensor_sequence_rank_b200 import inputs
from folded_tensor_sequence_rank_b200 import tsp

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    tsp_build.build()
    return tsp.lib()


def _setup(T, h, H, F, D, seed):
    raw = {k: v.cuda() for k, v in inputs.layer_inputs(T, h, F, seed).items()}
    dims = tsp.make_dims(T, h, H, F)
    sw = tsp.pack_shards(dims, D, raw)
    xs = [raw["x"].index_select(0, tsp.zigzag_index(T, D, r).long()).contiguous() for r in range(D)]
    return dims, sw, xs


def _call_noalloc(L, dims, sw, rank, x, K, V):
    stream = torch.cuda.current_stream().cuda_stream
    return L.tsp_kv_project_noalloc(ctypes.byref(dims), ctypes.byref(sw.struct), rank, x.data_ptr(), K.data_ptr(),
                                    V.data_ptr(), stream)


@pytest.mark.parametrize("T,h,H,F,D", [(1024, 256, 4, 1024, 2), (8192, 4096, 32, 16384, 8)])
def test_noalloc_matches_workspace_entry_on_two_calls(L, T, h, H, F, D):
    dims, sw, xs = _setup(T, h, H, F, D, 21)
    ws = tsp.alloc_workspace(dims, D)
    for rank in (0, D - 1):          # two calls in a row, different ranks
        Kr = torch.zeros(T, h, dtype=torch.float16, device="cuda")
        Vr = torch.zeros_like(Kr)
        tsp.kv_project(dims, sw, rank, xs[rank], Kr, Vr, ws)
        Kn = torch.zeros_like(Kr)
        Vn = torch.zeros_like(Kr)
        assert _call_noalloc(L, dims, sw, rank, xs[rank], Kn, Vn) == tsp.TSP_OK
        torch.cuda.synchronize()
        assert torch.equal(Kn.view(torch.int16), Kr.view(torch.int16)), rank
        assert torch.equal(Vn.view(torch.int16), Vr.view(torch.int16)), rank
        assert Kn.abs().sum() > 0


def test_noalloc_rejects_sizes_beyond_its_scratch(L):
    T, h, H, F, D = 16384, 4096, 32, 16384, 1     # T/D * h * 2 = 128 MiB > 64 MiB
    dims = tsp.make_dims(T, h, H, F)
    w = tsp.Weights()
    w.D = D
    for name in tsp.WEIGHT_NAMES:
        getattr(w, name)[0] = 0x10000
    rc = L.tsp_kv_project_noalloc(ctypes.byref(dims), ctypes.byref(w), 0, 16, 16, 16, None)
    assert rc == tsp.TSP_ERR_WORKSPACE
    assert b"exceeds" in L.tsp_last_cuda_error()


def test_noalloc_status_reports_a_timeout_and_the_next_call_clears_it(L):
    """A device-side timeout inside the allocation-free call lands in the
    static scratch's status section, which tsp_kv_project_noalloc_status
    reads.  The bounded-wait self test, aimed at that section, stands in for a
    wait that runs out (it waits on a barrier nothing completes, then returns
    normally); the next call starts by clearing the section."""
    tsp.selftest_wait_timeout(None, 20_000_000)  # 20 ms
    assert tsp.kv_project_noalloc_status() == tsp.TSP_ERR_TIMEOUT
    T, h, H, F, D = 1024, 256, 4, 1024, 2
    dims, sw, xs = _setup(T, h, H, F, D, 22)
    K = torch.zeros(T, h, dtype=torch.float16, device="cuda")
    V = torch.zeros_like(K)
    assert _call_noalloc(L, dims, sw, 1, xs[1], K, V) == tsp.TSP_OK
    assert tsp.kv_project_noalloc_status() == tsp.TSP_OK
    assert K.abs().sum() > 0
