"""The workspace-free selection entry point, checked against the workspace one.

scope_build_lut_and_select_noalloc exists for callers that cannot call cudaMalloc (a
host application that owns every device allocation, or a loop that must not let
cudaMalloc / cudaFree synchronise the device): it keeps its scratch in a fixed device
array of the library.  This file is collected last on purpose, and it must pass both in
a fresh process (the first call on the device also loads the device code there) and after
the other tests.  Two calls in a row check that the array's leftover contents from the
previous call do not leak into the next one.
"""
import ctypes

import numpy as np
import pytest
import torch

from free_sparse_attention_b200 import capi, synth
from free_sparse_attention_b200.workloads import COGVIDEOX, Workload

pytestmark = pytest.mark.gpu

MID = Workload("mid", 1, 2, 5, 16, 20, 44, 42, 42, "bf16", 50, 60, seed=6)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from free_sparse_attention_b200.build import build
    build()
    capi.lib()


def _clustered(w):
    x = synth.layer_inputs(w)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    Q, K = (torch.from_numpy(x[n]).reshape(w.B, w.H, w.N, w.d).to("cuda", dt) for n in "qk")
    qi = torch.from_numpy(x["q_init"]).reshape(w.B, w.H, w.Cq).cuda()
    ki = torch.from_numpy(x["k_init"]).reshape(w.B, w.H, 3, w.Cm).cuda()
    p = capi.Params.from_workload(w)
    ws = capi.alloc_workspace(p)
    qc, _, qs = capi.cluster_queries(p, Q, init_idx=qi, ws=ws)
    kc, kk = capi.cluster_keys(p, K, init_idx=ki, ws=ws)
    ref = capi.build_lut_and_select(p, qc, qs, kc, kk, ws=ws)
    torch.cuda.synchronize()
    return p, (qc, qs, kc, kk), ref


@pytest.mark.parametrize("w", [MID, COGVIDEOX.with_(H=3)], ids=lambda w: w.name)
def test_noalloc_selection_matches_workspace_selection_twice(w):
    p, args, ref = _clustered(w)
    for call in range(2):
        got = capi.build_lut_and_select_noalloc(p, *args)
        torch.cuda.synchronize()
        for k in ref:
            np.testing.assert_array_equal(got[k].cpu().numpy(), ref[k].cpu().numpy(),
                                          err_msg=f"{k}, call {call}")


def test_noalloc_rejects_layers_beyond_its_array():
    # B*H*Cq above the fixed array's capacity is refused before anything is enqueued
    w = MID.with_(H=400)
    p = capi.Params.from_workload(w)
    assert w.B * w.H * w.Cq > 16384
    fake = ctypes.c_void_p(1 << 20)
    rc = capi.lib().scope_build_lut_and_select_noalloc(ctypes.byref(p), *([fake] * 9), None)
    assert rc == 2
