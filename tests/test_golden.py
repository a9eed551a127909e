"""The configuration values the SCOPE pages print (tests/golden/implementation_details.txt,
with its citations) against the workload shapes, the oracle's dense-prefix schedule and the
schedule decision of the C ABI."""
import os

import pytest

import oracle
from free_sparse_attention_b200 import capi
from free_sparse_attention_b200.workloads import HUNYUAN720, WAN480, WAN720

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "implementation_details.txt")


def _golden():
    vals = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, val = (t.strip() for t in line.split("=", 1))
            nums = [float(x) for x in val.split()]
            vals[key] = nums if len(nums) > 1 else nums[0]
    return vals


def test_golden_file_holds_the_printed_values():
    g = _golden()
    assert set(g) == {"Cq", "Cm", "alpha", "dense_layers", "dense_step_fraction.wan",
                      "dense_step_fraction.hunyuan", "rho_sweep"}


@pytest.mark.parametrize("w", [HUNYUAN720, WAN480, WAN720], ids=lambda w: w.name)
def test_model_family_workloads_use_the_printed_hyperparameters(w):
    """The shapes of the pages' model families take the implementation details' Cq, the
    per-subspace C_T = C_H = C_W and alpha; the Wan 720p shape carries the rho sweep."""
    g = _golden()
    assert (w.Cq, w.Cm, w.alpha) == (g["Cq"], g["Cm"], g["alpha"])
    assert list(WAN720.rho_sweep) == g["rho_sweep"]


@pytest.mark.parametrize("family,n_steps", [("wan", 50), ("hunyuan", 50), ("wan", 40), ("hunyuan", 30)])
def test_dense_prefix_schedule_from_the_printed_fractions(family, n_steps):
    """Read through the oracle's schedule, the printed values give: the first layer dense at
    every step, and exactly the printed share of the steps dense for every other layer."""
    g = _golden()
    dense_layers = int(g["dense_layers"])
    dense_steps = round(g[f"dense_step_fraction.{family}"] * n_steps)
    assert all(oracle.layer_is_dense(0, s, dense_layers, dense_steps) for s in range(n_steps))
    for layer in (1, 2, 17):
        dense = [oracle.layer_is_dense(layer, s, dense_layers, dense_steps) for s in range(n_steps)]
        assert sum(dense) == dense_steps and all(dense[:dense_steps]), (layer, dense_steps)


@pytest.mark.parametrize("name,family", [("hunyuan720p", "hunyuan"), ("wan720p", "wan"), ("wan480p", "wan")])
def test_bench_schedule_is_the_printed_schedule(name, family):
    """The schedule bench.py --schedule measures is the printed one for the shape's family."""
    import bench
    g = _golden()
    for n_steps in (50, 30):
        assert bench.dense_prefix_schedule(name, n_steps) == (
            int(g["dense_layers"]), round(g[f"dense_step_fraction.{family}"] * n_steps))


def test_c_abi_schedule_decision_on_the_printed_schedule():
    """scope_layer_is_dense on HunyuanVideo's printed schedule (10 % of 50 steps, layer 0)."""
    from free_sparse_attention_b200.build import build
    build()
    g = _golden()
    steps = round(g["dense_step_fraction.hunyuan"] * 50)
    for layer, step, want in [(0, 49, 1), (1, 0, 1), (1, steps - 1, 1), (1, steps, 0), (7, 49, 0)]:
        sch = capi.Schedule(layer=layer, step=step, dense_layers=int(g["dense_layers"]), dense_steps=steps)
        assert capi.layer_is_dense(sch) == want
