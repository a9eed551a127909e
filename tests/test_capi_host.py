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
    return sorted(set(re.findall(r"\b(scope_[a-z0-9_]+)\s*\(", text)))


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
    assert n < 5 * 1024 ** 3


BAD = [
    dict(d_t=10),                 # split does not sum to d
    dict(Cq=0), dict(Cm=0),
    dict(Cq=300),                 # more centroids than tokens (N = 256)
    dict(rho=0.0), dict(rho=1.5), dict(rho=float("nan")),
    dict(alpha=-0.1), dict(alpha=1.1),
    dict(iters=0), dict(B=0), dict(T=0), dict(dtype=7),
    dict(khead_mode=2), dict(key_clustering=2), dict(key_clustering=-1),
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


def test_layer_schedule_decision_matches_oracle(L):
    """scope_layer_is_dense (host logic in the library) against the oracle's reading of
    the dense-prefix schedule."""
    import oracle
    for layer in range(3):
        for step in range(12):
            for dense_layers in (0, 1, 2):
                for dense_steps in (0, 5, 10):
                    s = capi.Schedule(layer=layer, step=step, dense_layers=dense_layers,
                                      dense_steps=dense_steps, rope=0, rope_base=10000.0)
                    assert capi.layer_is_dense(s) == oracle.layer_is_dense(layer, step, dense_layers,
                                                                            dense_steps)
    assert L.scope_layer_is_dense(None) == -1
    bad = capi.Schedule(layer=-1, step=0, dense_layers=1, dense_steps=0, rope=0, rope_base=1e4)
    assert L.scope_layer_is_dense(ctypes.byref(bad)) == -1


def test_rope_and_layer_rejections(L):
    fake = ctypes.c_void_p(1 << 20)
    p = capi.Params.from_workload(TINY)
    # odd channel ranges, bad base, K without its output
    odd = capi.Params.from_workload(TINY, d_t=TINY.d_t - 1, d_h=TINY.d_h + 1)
    assert L.scope_rope3d(ctypes.byref(odd), 1e4, fake, fake, fake, fake, None) == 1
    for base in (0.0, -2.0, float("nan"), float("inf")):
        assert L.scope_rope3d(ctypes.byref(p), base, fake, fake, fake, fake, None) == 1
    assert L.scope_rope3d(ctypes.byref(p), 1e4, fake, fake, fake, None, None) == 1
    assert L.scope_rope3d(ctypes.byref(p), 1e4, None, None, fake, None, None) == 1
    # a cos/sin table larger than shared memory allows: 24 B x (1*8 + 1*12 + 1100*12) pairs
    wide = capi.Params.from_workload(TINY, T=1, Hg=1, Wg=1100)
    assert L.scope_rope3d(ctypes.byref(wide), 1e4, fake, fake, fake, fake, None) == 2
    # the layer: everything validated up front
    need = capi.workspace_bytes(p)
    sp = capi.Schedule(layer=3, step=20, dense_layers=1, dense_steps=5, rope=1, rope_base=1e4)
    assert L.scope_attention_layer(ctypes.byref(p), ctypes.byref(sp), fake, fake, fake, fake, fake, fake,
                                   None, fake, fake, need, None) == 1            # no Qr
    assert L.scope_attention_layer(ctypes.byref(p), ctypes.byref(sp), fake, fake, fake, None, fake, fake,
                                   fake, fake, fake, need, None) == 1            # sparse, no init
    assert L.scope_attention_layer(ctypes.byref(p), ctypes.byref(sp), fake, fake, fake, fake, fake, fake,
                                   fake, fake, fake, need - 256, None) == 3      # workspace
    assert L.scope_attention_layer(ctypes.byref(p), None, fake, fake, fake, fake, fake, fake,
                                   fake, fake, fake, need, None) == 1            # no schedule
    assert L.scope_dense_attention(ctypes.byref(p), fake, fake, fake, fake, fake, need - 256, None) == 3
    assert L.scope_dense_attention(ctypes.byref(p), fake, None, fake, fake, fake, need, None) == 1


@pytest.mark.parametrize("name", sorted(ALL))
def test_dense_layout_fits_the_layer_workspace(L, name):
    """The dense branch carves a one-cluster layout out of the layer's workspace."""
    p = capi.Params.from_workload(ALL[name])
    p1 = capi.Params.from_workload(ALL[name], Cq=1)
    assert 0 < capi.workspace_bytes(p1) <= capi.workspace_bytes(p)


def test_rank_correlation_rejections(L):
    """Validation of scope_rank_correlation happens before any device work."""
    fake = ctypes.c_void_p(1 << 20)
    p = capi.Params.from_workload(TINY)
    args = [fake] * 6
    # no samples: nothing to do
    assert L.scope_rank_correlation(ctypes.byref(p), *args, None, 0, None, fake, 0, None) == 0
    assert L.scope_rank_correlation(ctypes.byref(p), *args, fake, -1, fake, fake, 1 << 30, None) == 1
    assert L.scope_rank_correlation(ctypes.byref(p), *args, None, 3, fake, fake, 1 << 30, None) == 1   # no samples
    assert L.scope_rank_correlation(ctypes.byref(p), *args, fake, 3, None, fake, 1 << 30, None) == 1   # no output
    assert L.scope_rank_correlation(ctypes.byref(p), ctypes.c_void_p((1 << 20) + 4), *args[1:], fake, 3, fake,
                                    fake, 1 << 30, None) == 1   # misaligned Q
    big = capi.Params.from_workload(TINY, Cm=1100, T=8, Hg=16, Wg=16)
    assert L.scope_rank_correlation(ctypes.byref(big), *args, fake, 3, fake, fake, 1 << 30, None) == 2
    assert L.scope_rank_correlation_scratch_bytes(ctypes.byref(p), 0) == 0
    bad = capi.Params.from_workload(TINY, rho=2.0)
    assert L.scope_rank_correlation_scratch_bytes(ctypes.byref(bad), 4) == 0


def test_cluster_keys_rejections(L):
    p = capi.Params.from_workload(TINY)
    need = capi.workspace_bytes(p)
    fake = ctypes.c_void_p(1 << 20)
    # workspace too small, misaligned workspace, no initial centroids, misaligned K
    assert L.scope_cluster_keys(ctypes.byref(p), fake, fake, None, fake, fake, fake, need - 256, None) == 3
    assert L.scope_cluster_keys(ctypes.byref(p), fake, fake, None, fake, fake,
                                ctypes.c_void_p((1 << 20) + 8), need, None) == 1
    assert L.scope_cluster_keys(ctypes.byref(p), fake, None, None, fake, fake, fake, need, None) == 1
    assert L.scope_cluster_keys(ctypes.byref(p), ctypes.c_void_p((1 << 20) + 2), fake, None, fake, fake,
                                fake, need, None) == 1
    bad = capi.Params.from_workload(TINY, key_clustering=3)
    assert L.scope_cluster_keys(ctypes.byref(bad), fake, fake, None, fake, fake, fake, need, None) == 1


def test_permute_channels_rejections(L):
    p = capi.Params.from_workload(TINY)
    fake, other = ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 21)
    assert L.scope_permute_channels(ctypes.byref(p), fake, fake, fake, None) == 1        # in place
    assert L.scope_permute_channels(ctypes.byref(p), fake, None, other, None) == 1       # no permutation
    assert L.scope_permute_channels(ctypes.byref(p), ctypes.c_void_p((1 << 20) + 4), fake, other, None) == 1
    bad = capi.Params.from_workload(TINY, d_t=10)
    assert L.scope_permute_channels(ctypes.byref(bad), fake, fake, other, None) == 1


def test_selection_recall_rejections(L):
    p = capi.Params.from_workload(TINY)
    fake = ctypes.c_void_p(1 << 20)
    f = L.scope_selection_recall

    def call(params, n, frac, scratch_bytes, samples=fake):
        return f(ctypes.byref(params), fake, fake, fake, fake, fake, fake, fake, samples, n,
                 ctypes.c_double(frac), fake, fake, fake, scratch_bytes, None)

    per = 16 * TINY.N                       # scratch bytes the recall pass needs
    for frac in (0.0, -0.5, 1.5, float("nan")):
        assert call(p, 1, frac, per) == 1
    assert call(p, -1, 0.1, per) == 1
    assert call(p, 1, 0.1, per, samples=None) == 1
    assert call(p, 0, 0.1, per - 16) == 3   # scratch too small
    assert call(p, 0, 0.1, per) == 0        # nothing to do: no launch
    # a valid layer with more key centroids than the fidelity kernels hold
    from free_sparse_attention_b200.workloads import COGVIDEOX
    big = capi.Params.from_workload(COGVIDEOX, Cm=1500)
    assert capi.workspace_bytes(big) > 0
    assert call(big, 1, 0.1, 16 * COGVIDEOX.N) == 2


def test_device_status_rejections(L):
    out = ctypes.c_int32(0)
    assert L.scope_get_device_status(None, None, ctypes.byref(out)) == 1
    assert L.scope_get_device_status(ctypes.c_void_p(1 << 20), None, None) == 1


def test_selection_stats_rejections(L):
    """scope_get_selection_stats validates before touching the device."""
    from free_sparse_attention_b200.workloads import COGVIDEOX
    p = capi.Params.from_workload(COGVIDEOX)
    out = (ctypes.c_int32 * 4)()
    f = L.scope_get_selection_stats
    assert f(ctypes.byref(p), None, None, out) == 1
    assert f(ctypes.byref(p), ctypes.c_void_p(1 << 20), None, None) == 1
    bad = capi.Params.from_workload(COGVIDEOX, rho=0.0)
    assert f(ctypes.byref(bad), ctypes.c_void_p(1 << 20), None, out) == 1


def test_wait_timeout_check_rejections(L):
    """scope_check_wait_timeout validates on the host before launching anything."""
    from free_sparse_attention_b200.workloads import COGVIDEOX
    p = capi.Params.from_workload(COGVIDEOX)
    n = capi.workspace_bytes(p)
    ws = ctypes.c_void_p(1 << 20)
    f = L.scope_check_wait_timeout
    assert f(ctypes.byref(p), 1000, None, n, None) == 1                  # no workspace
    assert f(ctypes.byref(p), 1000, ws, n - 256, None) == 3             # workspace too small
    assert f(ctypes.byref(p), 0, ws, n, None) == 1                      # no limit
    assert f(ctypes.byref(p), 10 ** 10 + 1, ws, n, None) == 1           # limit above 10 s
    p32 = capi.Params.from_workload(TINY)
    assert f(ctypes.byref(p32), 1000, ws, capi.workspace_bytes(p32), None) == 2   # fp32: no tensor-core kernel
    assert L.scope_status_string(6).decode() == "SCOPE_ERR_TIMEOUT"
