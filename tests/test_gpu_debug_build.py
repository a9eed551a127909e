"""The debug build (-DSCOPE_DEBUG): internal index checks that report in the status word.

The library is rebuilt with -DSCOPE_DEBUG, which checks the token rows the kernels take from
permutations and key lists and the cluster indices they store; an index out of range would
set SCOPE_DEV_DEBUG_CHECK and be replaced by 0 instead of faulting.  A child process runs the
layer (and the dense branch) with each build on the same inputs: the debug build must report a
clean status word and produce the release build's outputs bit for bit.
"""
import json
import os
import subprocess
import sys
import textwrap

import pytest
import torch

from free_sparse_attention_b200 import build as B

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

CHILD = textwrap.dedent("""
    import hashlib, json
    import torch
    from free_sparse_attention_b200 import capi, synth
    from free_sparse_attention_b200.workloads import COGVIDEOX, Workload
    out = {}
    cases = [Workload("ragged", 1, 2, 3, 9, 11, 16, 24, 24, "bf16", 13, 17, seed=5),
             Workload("mid", 1, 2, 5, 16, 20, 44, 42, 42, "bf16", 50, 60, seed=6),
             COGVIDEOX.with_(H=1)]
    for w in cases:
        x = synth.layer_inputs(w)
        Q, K, V = (torch.from_numpy(x[n]).reshape(w.B, w.H, w.N, w.d).to("cuda", torch.bfloat16) for n in "qkv")
        qi = torch.from_numpy(x["q_init"]).reshape(w.B, w.H, w.Cq).cuda()
        ki = torch.from_numpy(x["k_init"]).reshape(w.B, w.H, 3, w.Cm).cuda()
        p = capi.Params.from_workload(w)
        ws = capi.alloc_workspace(p)
        O, it = capi.forward(p, Q, K, V, qi, ki, ws=ws, intermediates=True)
        Od = capi.dense_attention(p, Q, K, V, ws=ws)
        torch.cuda.synchronize()
        st = capi.get_device_status(ws)
        h = {k: hashlib.sha1(v.cpu().numpy().tobytes()).hexdigest() for k, v in it.items()}
        h["O"] = hashlib.sha1(O.cpu().float().numpy().tobytes()).hexdigest()
        h["O_dense"] = hashlib.sha1(Od.cpu().float().numpy().tobytes()).hexdigest()
        out[w.name] = {"status": st, "hashes": h}
    print(json.dumps(out))
""")


def _run(lib):
    env = dict(os.environ, SCOPE_LIB_PATH=lib, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


def test_debug_build_is_clean_and_matches_release():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    release = B.build()
    debug = B.build(debug=True)
    a, b = _run(release), _run(debug)
    for name in a:
        assert a[name]["status"] == 0, name
        assert b[name]["status"] == 0, (name, b[name]["status"])
        assert a[name]["hashes"] == b[name]["hashes"], name
