"""Shared helpers of the GPU tests: seeded inputs on the device, oracle per head, and
the comparison rules.

Parity rules (SCOPE hot path):
  - cluster assignments, member counts, centroids: identical to the binary64 oracle
    (the CUDA path certifies its fp32 distances and sums members in token order);
  - p_c, b_c, k_head, r_c and the selected sets: identical, except where the oracle
    logs the Top-p decision as a near tie (|prefix mass - rho Z| / Z < 1e-6);
  - attention output on the same selection: max-abs <= 2e-2 and relative RMS <= 5e-3
    for bf16 inputs, both <= 1e-4 for fp32 inputs.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from free_sparse_attention_b200 import capi, synth
from free_sparse_attention_b200.workloads import Workload

NEAR_TIE = 1e-6


def tol(w: Workload):
    return (2e-2, 5e-3) if w.dtype == "bf16" else (1e-4, 1e-4)


def device_inputs(w: Workload, x):
    """float32 numpy [BH, N, d] -> device tensors [B, H, N, d] in the workload dtype."""
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    out = {}
    for name in ("q", "k", "v"):
        t = torch.from_numpy(x[name]).reshape(w.B, w.H, w.N, w.d)
        out[name] = t.to(device="cuda", dtype=dt).contiguous()
    out["q_init"] = torch.from_numpy(x["q_init"]).reshape(w.B, w.H, w.Cq).cuda()
    out["k_init"] = torch.from_numpy(x["k_init"]).reshape(w.B, w.H, 3, w.Cm).cuda()
    return out


def oracle_head(w: Workload, x, i, rows=None, rho=None):
    return oracle.forward_head(x["q"][i], x["k"][i], x["v"][i], w, x["q_init"][i], x["k_init"][i],
                               rows=rows, logs=True, rho=rho)


def mask_bits(mask_row_u32, N):
    m = np.ascontiguousarray(mask_row_u32).view(np.uint32)
    return np.unpackbits(m.view(np.uint8), axis=-1, bitorder="little")[..., :N]


def compare_attention(w, O_gpu, O_ref):
    O_gpu = np.asarray(O_gpu, np.float64)
    err = np.abs(O_gpu - O_ref)
    rel_rms = np.sqrt(np.mean(err ** 2)) / max(np.sqrt(np.mean(O_ref ** 2)), 1e-30)
    mabs, rrms = tol(w)
    assert err.max() <= mabs, f"max-abs {err.max():.3e} > {mabs}"
    assert rel_rms <= rrms, f"rel-RMS {rel_rms:.3e} > {rrms}"
    return float(err.max()), float(rel_rms)


def selection_mismatch_ok(sel_ref, p_gpu, c):
    """A p_c mismatch is tolerated only at a near tie logged by the oracle."""
    return sel_ref["topp_margin"][c] < NEAR_TIE


def to_np(t):
    return t.detach().cpu().numpy()
