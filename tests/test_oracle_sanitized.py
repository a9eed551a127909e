"""The CPU oracle under AddressSanitizer and UndefinedBehaviorSanitizer.

The oracle's C library is rebuilt with -fsanitize=address,undefined (no recovery: the first
report aborts the process) and loaded by a child Python process with the sanitizer runtimes
preloaded; the child runs the whole per-head path (k-means of queries and key subspaces,
selection, sparse attention) and the dense layer on small workloads, including ragged grids,
d = 64 and 128, and Cq = 1.  The test passes when the child exits 0 with no sanitizer report.
"""
import os
import subprocess
import sys
import textwrap

import pytest

from oracle import build as obuild

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

CHILD = textwrap.dedent("""
    import numpy as np
    import oracle
    from free_sparse_attention_b200 import synth
    from free_sparse_attention_b200.workloads import TINY, Workload
    cases = [TINY,
             Workload("ragged", 1, 2, 3, 9, 11, 16, 24, 24, "bf16", 13, 17, seed=5),
             Workload("mid128", 1, 1, 2, 7, 9, 44, 42, 42, "bf16", 1, 20, seed=8)]
    for w in cases:
        x = synth.layer_inputs(w)
        for i in range(w.B * w.H):
            for dense in (False, True):
                r = oracle.layer(x["q"][i], x["k"][i], x["v"][i], w, x["q_init"][i], x["k_init"][i], dense)
                assert np.isfinite(r["O"]).all()
    print("sanitized oracle ok")
""")


def _runtime(name):
    path = subprocess.run(["gcc", f"-print-file-name={name}"], capture_output=True, text=True).stdout.strip()
    return path if os.path.isabs(path) and os.path.exists(path) else None


def test_oracle_under_asan_and_ubsan():
    asan, ubsan = _runtime("libasan.so"), _runtime("libubsan.so")
    if not asan or not ubsan:
        pytest.skip("gcc's sanitizer runtimes are not installed")
    lib = obuild.build_sanitized(os.path.join(ROOT, "oracle", "liboracle_san.so"))   # gitignored
    env = dict(os.environ, SCOPE_ORACLE_LIB=lib, LD_PRELOAD=f"{asan}:{ubsan}",
               ASAN_OPTIONS="detect_leaks=0:abort_on_error=1", UBSAN_OPTIONS="print_stacktrace=1",
               OMP_NUM_THREADS="2", PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    report = r.stdout[-2000:] + r.stderr[-4000:]
    assert r.returncode == 0, report
    assert "sanitized oracle ok" in r.stdout, report
    assert "runtime error" not in r.stderr and "AddressSanitizer" not in r.stderr, report
