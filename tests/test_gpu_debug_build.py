"""The -DTSP_DEBUG build of the library on the small configurations: its
device index checks (output rows and columns of every GEMM epilogue, the
attention's output rows and log-sum-exp stash, the backward's bulk
reductions, statistics copies and dK/dV rows) must all pass - a failed check
would show as TSP_ERR_BOUNDS - and the results must keep their parity with
the oracle.  The debug library is loaded in a child process (TSP_LIBRARY),
so the normal build this session has loaded is untouched."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu


def _child():
    import numpy as np
    import torch
    sys.path.insert(0, ROOT)
    from folded_tensor_sequence_rank_b200 import inputs, tp, tsp
    from oracle import tsp_oracle as O
    assert tsp.LIB_PATH.endswith("libtsp_b200_debug.so")
    out = []
    for (T, h, H, F, D, seed) in [(512, 256, 4, 1024, 2, 70), (800, 256, 4, 1024, 2, 71), (960, 320, 5, 1280, 5, 72),
                                  (2048, 512, 4, 2048, 2, 73), (8, 256, 4, 1024, 4, 74)]:
        raw = inputs.layer_inputs(T, h, F, seed)
        dev = {k: v.cuda() for k, v in raw.items()}
        dims = tsp.make_dims(T, h, H, F)
        sw = tsp.pack_shards(dims, D, dev)
        ws = tsp.alloc_workspace(dims, D)
        aws = tsp.alloc_attn_backward_workspace(dims, D)
        K = torch.zeros(T, h, dtype=torch.float16, device="cuda")
        V = torch.zeros_like(K)
        idx = [tsp.zigzag_index(T, D, r).long() for r in range(D)]
        xs = [dev["x"].index_select(0, i).contiguous() for i in idx]
        for r in range(D):
            tsp.kv_project(dims, sw, r, xs[r], K, V, ws)
        Y = torch.zeros(T, h, device="cuda")
        dK = torch.zeros(T, h, device="cuda")
        dV = torch.zeros_like(dK)
        statuses = []
        for r in range(D):
            y = torch.empty(T // D, h, device="cuda")
            tsp.layer_forward(dims, sw, r, xs[r], K, V, y, ws)
            Y[idx[r]] = y
            d_o = inputs.attention_grad_inputs(T // D, h, seed + r).cuda()
            dq = torch.empty(T // D, h, device="cuda")
            tsp.attn_backward(dims, D, r, tsp.workspace_view(ws, dims, D, "q"), K, V,
                              tsp.workspace_view(ws, dims, D, "a"), tsp.workspace_view(ws, dims, D, "lse"), d_o, dq,
                              dK, dV, aws)
            statuses += [tsp.get_device_status(ws), tsp.get_device_status(aws)]
        tws = tsp.alloc_tp_workspace(dims, D)
        yt = tp.tp_layer_forward(dims, sw, dev["x"], tws, y_dtype=torch.float32)
        statuses += [tsp.get_device_status(tws), tsp.get_device_status(sw.buf)]
        x = raw["x"].double().numpy()
        ref = O.layer_forward(x, {n: raw[n].double().numpy() for n in inputs.WEIGHT_NAMES}, H)["y"]
        rel = lambda a: float(np.linalg.norm(a - ref) / np.linalg.norm(ref))
        out.append({"shape": [T, h, H, F, D], "statuses": statuses, "rel_tsp": rel(Y.double().cpu().numpy()),
                    "rel_tp": rel(yt.double().cpu().numpy())})
    print("RESULT " + json.dumps(out), flush=True)


def test_debug_build_checks_pass_on_small_configs():
    from folded_tensor_sequence_rank_b200 import build as tsp_build
    lib = tsp_build.build(debug=True)
    env = dict(os.environ, TSP_LIBRARY=lib)
    res = subprocess.run([sys.executable, os.path.abspath(__file__), "--child"], env=env, capture_output=True,
                         text=True, timeout=600)
    assert res.returncode == 0, res.stdout[-2000:] + res.stderr[-2000:]
    line = [ln for ln in res.stdout.splitlines() if ln.startswith("RESULT ")][-1]
    for case in json.loads(line[len("RESULT "):]):
        print(case)
        assert all(st == 0 for st in case["statuses"]), case
        assert case["rel_tsp"] <= 5e-3 and case["rel_tp"] <= 5e-3, case


if __name__ == "__main__" and "--child" in sys.argv:
    _child()
