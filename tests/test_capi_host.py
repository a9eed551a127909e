"""Host-side tests of the C ABI: no GPU needed, no kernel is launched.

The library links the CUDA runtime statically, so it loads on a machine without a
GPU; argument validation runs before anything is enqueued, so every rejection below
returns its status without touching the device.
"""
import ctypes
import os
import re

import pytest

from free_sparse_attention_b200 import capi
from free_sparse_attention_b200.build import build
from free_sparse_attention_b200.workloads import ALL, HUNYUAN720, TINY

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build()
    return capi.lib()


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "scope.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(scope_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = _declared_functions()
    assert len(names) >= 8
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(capi.EXPORTS)


def test_status_strings(L):
    for code, name in capi.STATUS.items():
        assert L.scope_status_string(code).decode() == name


@pytest.mark.parametrize("name", sorted(ALL))
def test_workspace_bytes_for_every_workload(L, name):
    p = capi.Params.from_workload(ALL[name])
    n = capi.workspace_bytes(p)
    assert n > 0 and n % 256 == 0


def test_workspace_fits_hbm_at_118800_tokens(L):
    # dominated by the attention gather lists: 4 B x B*H*Cq*N (3.4 GB here)
    n = capi.workspace_bytes(capi.Params.from_workload(HUNYUAN720))
    assert n < 6 * 1024 ** 3


BAD = [
    dict(d_t=10),                 # split does not sum to d
    dict(Cq=0), dict(Cm=0),
    dict(Cq=300),                 # more centroids than tokens (N = 256)
    dict(rho=0.0), dict(rho=1.5), dict(rho=float("nan")),
    dict(alpha=-0.1), dict(alpha=1.1),
    dict(iters=0), dict(B=0), dict(T=0), dict(dtype=7),
]


@pytest.mark.parametrize("over", BAD)
def test_invalid_params_rejected(L, over):
    p = capi.Params.from_workload(TINY, **over)
    assert capi.workspace_bytes(p) == 0
    fake = ctypes.c_void_p(1 << 20)
    rc = L.scope_cluster_queries(ctypes.byref(p), fake, fake, None, fake, fake, fake, fake,
                                 1 << 30, None)
    assert rc == 1 or rc == 2


def test_unsupported_shapes(L):
    for over in (dict(d=96, d_t=32, d_h=32, d_w=32), dict(Cq=4096, T=64)):
        p = capi.Params.from_workload(TINY, **over)
        assert L.scope_workspace_bytes(ctypes.byref(p)) == 0


def test_small_workspace_and_bad_pointers_rejected(L):
    p = capi.Params.from_workload(TINY)
    need = capi.workspace_bytes(p)
    fake = ctypes.c_void_p(1 << 20)
    args = (fake, fake, None, fake, fake, fake, fake)
    assert L.scope_cluster_queries(ctypes.byref(p), *args, need - 256, None) == 3
    # misaligned workspace
    assert L.scope_cluster_queries(ctypes.byref(p), *args[:6], ctypes.c_void_p((1 << 20) + 8),
                                   need, None) == 1
    # missing init
    assert L.scope_cluster_queries(ctypes.byref(p), fake, None, None, fake, fake, fake, fake,
                                   need, None) == 1
    # misaligned tensor
    assert L.scope_sparse_attention(ctypes.byref(p), ctypes.c_void_p((1 << 20) + 4), fake, fake,
                                    fake, fake, fake, fake, fake, need, None) == 1
    assert L.scope_forward(ctypes.byref(p), fake, fake, fake, None, fake, fake, None, fake,
                           need, None) == 1
    assert L.scope_build_lut_and_select(ctypes.byref(p), fake, fake, fake, fake, None, fake,
                                        fake, None, fake, fake, need, None) == 1


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(capi, "_lib", None)
    monkeypatch.setattr(capi, "LIB_PATH", "/nonexistent/libscope.so")
    with pytest.raises(RuntimeError):
        capi.lib()
