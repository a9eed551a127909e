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


def pack_mask(bits):
    """bool [..., N] -> uint32 [..., ceil(N/32)], key j at bit j % 32 of word j // 32."""
    bits = np.asarray(bits, bool)
    N = bits.shape[-1]
    nw = (N + 31) // 32
    pad = np.zeros(bits.shape[:-1] + (nw * 32,), bool)
    pad[..., :N] = bits
    return np.packbits(pad, axis=-1, bitorder="little").view(np.uint32)


def check_selection(w, g, sel, sizes, rerun_with_scores, khead_off=False):
    """Selection of one head against the oracle; returns the number of clusters whose
    Top-p count p_c differs from the oracle's at a near tie the oracle logged.

    g: the GPU's topp_counts, base_counts, final_counts [Cq], k_head (int), sel_mask
    [Cq, nw] (uint32); sel: oracle.select() on the same inputs; sizes: the oracle's n_c.
    Every value is checked: with no near tie everything must be identical; at a near tie
    the tied clusters' p_c may differ, and then every other cluster's p_c and b_c must
    still be identical, b_c, k_head and r_c must follow from the GPU's p_c by Eqs. 8-10
    (exact integers), and every S_c must be the first r_c keys of the oracle's own ranking
    (logit descending, key index ascending), which rerun_with_scores() supplies."""
    p = np.asarray(g["topp_counts"])
    bad = np.nonzero(p != sel["p"])[0]
    assert all(sel["topp_margin"][c] < NEAR_TIE for c in bad), \
        ("p_c differs away from a logged near tie", bad, p[bad], sel["p"][bad])
    agree = np.ones(p.shape[0], bool)
    agree[bad] = False
    b = np.asarray(g["base_counts"])
    np.testing.assert_array_equal(b[agree], sel["b"][agree])
    mask = np.asarray(g["sel_mask"]).view(np.uint32)
    if len(bad) == 0:
        assert int(g["k_head"]) == sel["k_head"]
        np.testing.assert_array_equal(g["final_counts"], sel["r"])
        np.testing.assert_array_equal(mask, sel["mask"])
        return 0
    N = w.N
    kfix = oracle.kfix(w.alpha, N)
    np.testing.assert_array_equal(b, np.maximum(p, kfix))                          # Eq. 8
    n = np.asarray(sizes, np.int64)
    kh = -(-int((n * b.astype(np.int64)).sum()) // int(n.sum()))                   # Eq. 9
    assert int(g["k_head"]) == kh
    r = b if khead_off else np.maximum(b, kh)                                      # Eq. 10
    np.testing.assert_array_equal(g["final_counts"], r)
    scores = rerun_with_scores()["scores"]
    idx = np.arange(N)
    for c in range(p.shape[0]):
        order = np.lexsort((idx, -scores[c]))
        want = np.zeros(N, bool)
        want[order[:r[c]]] = True
        np.testing.assert_array_equal(mask[c], pack_mask(want))
    return len(bad)


def to_np(t):
    return t.detach().cpu().numpy()
