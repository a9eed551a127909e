"""Seeded synthetic inputs for the SCOPE hot path (generator "G").

This module holds no part of the SCOPE method: it only draws the post-RoPE Q, K, V
activations and the random initial centroid indices that both the CUDA path and the
CPU oracle consume.  The real inputs behind the paper's numbers are activations of
Wan2.1/2.2 and HunyuanVideo DiTs (SCOPE abstract; "Implementation details"), which
are not available; a smooth spatiotemporal field plus noise stands in for them.

Recipe, per (batch b, head h) and per tensor x in {q, k, v}, token (t, h, w):

    x[t,h,w,:] = sum_{i=1..8} a_i * cos(2*pi*(omega_i . (t/T, h/Hg, w/Wg)) + phi_i) * u_i
                 + 0.5 * eps[t,h,w,:]

with a_i ~ N(0,1), omega_i uniform in {0..3}^3, phi_i ~ U[0, 2*pi),
u_i ~ N(0, I_d)/sqrt(d) and eps ~ N(0, I_d).  q and k then get 3D rotary embedding
(RoFormer pairs (2i, 2i+1) inside each of the temporal / height / width channel
blocks, theta_i = 10000^(-2i/d_axis), integer positions t, h, w), unless pre-RoPE
inputs are asked for; that rotation is the generator's own, shared with neither the
oracle nor the CUDA path, which each implement RoPE separately.  Values are built in
float64, rounded to float32 (round-to-nearest-even) and, for bf16 workloads, to bf16
(round-to-nearest-even).  Token index n = t*Hg*Wg + h*Wg + w.

Every (b, h, tensor) draws from its own numpy stream
``default_rng(SeedSequence(seed, spawn_key=(b, h, tensor_id)))`` (q=0, k=1, v=2), so
any head can be regenerated alone.  Draw order in a stream: a (8), omega (8x3),
phi (8), u (8 x d), eps (N x d).  Initial centroid indices for clustering role
r in {0: queries, 1: key-T, 2: key-H, 3: key-W} are ``rng.choice(N, C, replace=False)``
from the stream with spawn_key (b, h, 10 + r).
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from .workloads import Workload

N_COMPONENTS = 8
TENSOR_IDS = {"q": 0, "k": 1, "v": 2}


def _stream(seed: int, *key: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence(entropy=seed, spawn_key=tuple(key)))


def round_to_bf16(x32: np.ndarray) -> np.ndarray:
    """float32 -> nearest bf16 (ties to even), returned as float32 holding bf16 values."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    u = (u + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)
    return u.view(np.float32)


def _grid_positions(w: Workload):
    t = np.arange(w.T)[:, None, None]
    hh = np.arange(w.Hg)[None, :, None]
    ww = np.arange(w.Wg)[None, None, :]
    shape = (w.T, w.Hg, w.Wg)
    return (np.broadcast_to(t, shape).reshape(-1).astype(np.float64),
            np.broadcast_to(hh, shape).reshape(-1).astype(np.float64),
            np.broadcast_to(ww, shape).reshape(-1).astype(np.float64))


def _rope3d_inplace(x: np.ndarray, w: Workload, pos) -> None:
    c0 = 0
    for d_a, p in zip((w.d_t, w.d_h, w.d_w), pos):
        half = d_a // 2
        theta = 10000.0 ** (-2.0 * np.arange(half) / d_a)
        ang = p[:, None] * theta[None, :]
        cs, sn = np.cos(ang), np.sin(ang)
        x0 = x[:, c0:c0 + d_a:2].copy()
        x1 = x[:, c0 + 1:c0 + d_a:2].copy()
        x[:, c0:c0 + d_a:2] = x0 * cs - x1 * sn
        x[:, c0 + 1:c0 + d_a:2] = x0 * sn + x1 * cs
        c0 += d_a


def head_tensor(w: Workload, b: int, h: int, which: str, rope: bool = True,
                raw: bool = False) -> np.ndarray:
    """One head's q, k or v as a float32 [N, d] array holding values of w.dtype.

    rope=False leaves q and k pre-RoPE (the same draws, no rotation): the inputs of the
    layer variant that applies 3D RoPE on the device.  raw=True returns the float64
    values before any rounding."""
    rng = _stream(w.seed, b, h, TENSOR_IDS[which])
    d, N = w.d, w.N
    a = rng.standard_normal(N_COMPONENTS)
    omega = rng.integers(0, 4, size=(N_COMPONENTS, 3))
    phi = rng.uniform(0.0, 2.0 * np.pi, size=N_COMPONENTS)
    u = rng.standard_normal((N_COMPONENTS, d)) / np.sqrt(d)
    eps = rng.standard_normal((N, d))
    pt, ph, pw = _grid_positions(w)
    arg = 2.0 * np.pi * (np.outer(pt / w.T, omega[:, 0]) + np.outer(ph / w.Hg, omega[:, 1])
                         + np.outer(pw / w.Wg, omega[:, 2])) + phi[None, :]
    x = (a[None, :] * np.cos(arg)) @ u
    x += 0.5 * eps
    if rope and which in ("q", "k"):
        _rope3d_inplace(x, w, (pt, ph, pw))
    if raw:
        return x
    x32 = x.astype(np.float32)
    if w.dtype == "bf16":
        x32 = round_to_bf16(x32)
    return x32


def init_indices(w: Workload, b: int, h: int, role: int) -> np.ndarray:
    """Seeded distinct token indices used as initial centroids (int32 [C])."""
    C = w.Cq if role == 0 else w.Cm
    rng = _stream(w.seed, b, h, 10 + role)
    return rng.choice(w.N, size=C, replace=False).astype(np.int32)


def layer_inputs(w: Workload, heads=None, rope: bool = True):
    """Q, K, V as float32 [B, H', N, d] plus init indices, for the listed (b, h) heads.

    rope=False gives pre-RoPE q and k (see head_tensor).

    ``heads`` is a list of (b, h); None means every head.  Returns a dict with
    "q", "k", "v" ([B*H' heads stacked as given], N, d), "q_init" [heads, Cq] and
    "k_init" [heads, 3, Cm].
    """
    if heads is None:
        heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    out = {name: np.empty((len(heads), w.N, w.d), np.float32) for name in ("q", "k", "v")}
    q_init = np.empty((len(heads), w.Cq), np.int32)
    k_init = np.empty((len(heads), 3, w.Cm), np.int32)

    def fill(job):
        i, (b, h), name = job
        out[name][i] = head_tensor(w, b, h, name, rope=rope)

    jobs = [(i, bh, name) for i, bh in enumerate(heads) for name in ("q", "k", "v")]
    # numpy's generators and ufuncs release the GIL, so threads overlap the draws
    with ThreadPoolExecutor(max_workers=max(1, min(len(jobs), os.cpu_count() or 1))) as ex:
        list(ex.map(fill, jobs))
    for i, (b, h) in enumerate(heads):
        q_init[i] = init_indices(w, b, h, 0)
        for r in range(3):
            k_init[i, r] = init_indices(w, b, h, 1 + r)
    out["q_init"] = q_init
    out["k_init"] = k_init
    out["heads"] = heads
    return out
