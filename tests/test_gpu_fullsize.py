"""Parity at the full workload sizes, in the launch configuration the benchmark times.

The whole layer runs on the GPU for every head (scope_forward with intermediates); the
oracle recomputes a sample of heads end to end (clustering and selection in full,
attention for a sample of query rows).  Clustering must match exactly, selection
exactly except at a near tie the oracle logs, attention within the bf16 tolerance.
"""
import numpy as np
import pytest
import torch

import oracle
from free_sparse_attention_b200 import capi, synth
from free_sparse_attention_b200.workloads import HUNYUAN720, WAN480, WAN720

from gpu_common import check_selection, compare_attention, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from free_sparse_attention_b200.build import build
    build()
    capi.lib()


def _device(w, x):
    dt = torch.bfloat16
    t = {n: torch.from_numpy(x[n]).reshape(w.B, w.H, w.N, w.d).to("cuda", dt) for n in "qkv"}
    t["qi"] = torch.from_numpy(x["q_init"]).reshape(w.B, w.H, w.Cq).cuda()
    t["ki"] = torch.from_numpy(x["k_init"]).reshape(w.B, w.H, 3, w.Cm).cuda()
    return t


def _check_head(w, x, i, O, it, rng, rho):
    b, h = divmod(i, w.H)
    rq = oracle.kmeans(x["q"][i], 0, w.d, w.Cq, w.iters, init_idx=x["q_init"][i])
    rk = oracle.cluster_keys(x["k"][i], (w.d_t, w.d_h, w.d_w), w.Cm, w.iters, init_idx3=x["k_init"][i])
    np.testing.assert_array_equal(it["q_assign"][b, h], rq["assign"])
    np.testing.assert_array_equal(it["q_centroids"][b, h], rq["centroids"])
    np.testing.assert_array_equal(it["q_sizes"][b, h], rq["sizes"])
    np.testing.assert_array_equal(it["k_codes"][b, h], rk["codes"])
    np.testing.assert_array_equal(it["k_centroids"][b, h], rk["centroids"])
    args = (rq["centroids"], rq["sizes"], rk["centroids"], rk["codes"], (w.d_t, w.d_h, w.d_w), rho, w.alpha)
    sel = oracle.select(*args)
    gi = {k: it[k][b, h] for k in ("topp_counts", "base_counts", "final_counts", "k_head", "sel_mask")}
    ties = check_selection(w, gi, sel, rq["sizes"], lambda: oracle.select(*args, want_scores=True))
    # attention on sampled rows, on the oracle's own selection; after a near tie (the GPU's
    # selection validated above) only rows whose cluster kept the oracle's exact set
    rows = np.sort(rng.choice(w.N, 96, replace=False))
    if ties:
        same = (gi["sel_mask"].view(np.uint32) == sel["mask"]).all(axis=1)
        rows = rows[same[rq["assign"][rows]]]
    ref = oracle.attention(x["q"][i], x["k"][i], x["v"][i], rq["assign"], sel["mask"], rows=rows)
    compare_attention(w, O[i][rows], ref)
    return ties


def _run(w, heads_to_check, rhos=None):
    x = synth.layer_inputs(w)
    t = _device(w, x)
    rng = np.random.default_rng(7)
    densities = {}
    for rho in (rhos or (w.rho,)):
        p = capi.Params.from_workload(w, rho=rho)
        ws = capi.alloc_workspace(p)
        O, it = capi.forward(p, t["q"], t["k"], t["v"], t["qi"], t["ki"], ws=ws, intermediates=True)
        torch.cuda.synchronize()
        assert capi.get_device_status(ws) == 0
        # the selection's own count of Top-p decisions near a tie (every unit decides once)
        st = capi.get_selection_stats(p, ws)
        assert st["decisions"] == (w.B * w.H * w.Cq if rho < 1.0 else 0), st
        assert 0 <= st["margin_below_3e-7"] <= st["margin_below_1e-6"] <= st["decisions"], st
        print(f"rho={rho}: Top-p decisions {st}")
        n = it["q_sizes"].double()
        r = it["final_counts"].double()
        densities[rho] = float((n * r).sum() / (w.B * w.H * w.N * w.N))
        O = O.float().cpu().numpy().reshape(w.B * w.H, w.N, w.d)
        g = {k: to_np(v) for k, v in it.items()}
        del it
        ties = sum(_check_head(w, x, i, O, g, rng, rho) for i in heads_to_check)
        # the committed seeds give no near tie; a nonzero count (every value still
        # validated) means a change of input or arithmetic reached one
        assert ties == 0, f"rho={rho}: {ties} clusters took the near-tie branch"
        del ws
        torch.cuda.empty_cache()
    return densities


def test_hunyuan720p_full_size():
    _run(HUNYUAN720, heads_to_check=[0, 17])


def test_wan480p_full_size():
    _run(WAN480, heads_to_check=[5, 39])


def test_wan720p_rho_sweep_full_size():
    d = _run(WAN720, heads_to_check=[11], rhos=WAN720.rho_sweep)
    print("realised density per rho:", {k: round(v, 4) for k, v in d.items()})
    vals = [d[r] for r in WAN720.rho_sweep]
    assert all(a < b for a, b in zip(vals, vals[1:])), vals   # monotone in rho
