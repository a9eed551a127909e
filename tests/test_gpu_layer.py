"""3D RoPE, the dense branch and the layer wrapper under the dense-prefix schedule on the
GPU, against the binary64 oracle.

RoPE rule: both sides evaluate the rotation in binary64 and round once to the element
type, but their cos and sin may differ in the last binary64 bits.  So the rotated value
must equal the oracle's rounded value, except where the oracle's binary64 value lies
within (|x0| + |x1|) * 2^-45 of a rounding boundary of the element type; there either
neighbour is accepted (and counted)."""
import numpy as np
import pytest
import torch

import oracle
from free_sparse_attention_b200 import capi, synth
from free_sparse_attention_b200.workloads import HUNYUAN720, Workload

from gpu_common import compare_attention, to_np

pytestmark = pytest.mark.gpu

W = Workload("layer", 1, 2, 3, 12, 10, 44, 42, 42, "bf16", 16, 12, seed=23)    # N = 360, d = 128
W64 = Workload("layer64", 2, 1, 5, 7, 9, 20, 22, 22, "f32", 8, 8, seed=24)     # N = 315, d = 64


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from free_sparse_attention_b200.build import build
    build()
    capi.lib()


def _round(v, dtype):
    """binary64 -> the element type, to nearest with ties to even (exact in binary64)."""
    if dtype == "f32":
        return v.astype(np.float32).astype(np.float64)
    m, e = np.frexp(v)
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


def _check_rope(Y, X, w, rows=None):
    """Y: the GPU's rotated rows (float64), X: the pre-RoPE rows it was given."""
    ref = oracle.rope3d(X, (w.T, w.Hg, w.Wg), (w.d_t, w.d_h, w.d_w), rows=rows)
    mag = np.abs(X)
    delta = np.repeat(mag[:, 0::2] + mag[:, 1::2], 2, axis=1) * 2.0 ** -45
    mid, lo, hi = _round(ref, w.dtype), _round(ref - delta, w.dtype), _round(ref + delta, w.dtype)
    exact = Y == mid
    near = (lo != hi) & ((Y == lo) | (Y == hi))
    assert np.all(exact | near), np.argwhere(~(exact | near))[:5]
    return int((~exact).sum())


def _dev(w, a):
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    return torch.from_numpy(np.ascontiguousarray(a)).reshape(w.B, w.H, w.N, w.d).to("cuda", dt)


def _np(t, w):
    return t.double().cpu().numpy().reshape(w.B * w.H, w.N, w.d)


@pytest.mark.parametrize("w", [W, W.with_(dtype="f32"), W64, W64.with_(dtype="bf16")], ids=lambda w: f"{w.name}-{w.dtype}")
def test_rope3d_matches_oracle(w):
    x = synth.layer_inputs(w, rope=False)
    p = capi.Params.from_workload(w)
    Q, K = _dev(w, x["q"]), _dev(w, x["k"])
    Qr, Kr = capi.rope3d(p, Q, K)
    torch.cuda.synchronize()
    near = 0
    for name, Y in (("q", Qr), ("k", Kr)):
        Yn = _np(Y, w)
        for i in range(w.B * w.H):
            near += _check_rope(Yn[i], x[name][i].astype(np.float64), w)
    assert near <= 2
    # in place, Q only: the same values
    Qi = Q.clone()
    capi.rope3d(p, Qi, None, out_q=Qi)
    torch.cuda.synchronize()
    assert torch.equal(Qi, Qr)
    # the post-RoPE inputs the rest of the path is tested on come from the generator's own
    # rotation before rounding: the two agree to about one unit of the element type
    post = synth.layer_inputs(w)
    ulp = 2.0 ** -7 if w.dtype == "bf16" else 2.0 ** -22
    diff = np.abs(_np(Qr, w) - post["q"])
    assert diff.max() <= ulp * np.abs(post["q"]).max()


def test_rope3d_full_size_sampled_rows():
    """HunyuanVideo's 24 heads of 118800 tokens in one launch; sampled rows of three heads
    (first, middle, last) against the oracle."""
    w = HUNYUAN720
    p = capi.Params.from_workload(w)
    heads = [0, 11, w.H - 1]
    Q = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.bfloat16, device="cuda")
    pre = {}
    for h in range(w.H):
        a = synth.head_tensor(w, 0, h, "q", rope=False)
        Q[0, h] = torch.from_numpy(a).to("cuda", torch.bfloat16)
        if h in heads:
            pre[h] = a
    Qr, _ = capi.rope3d(p, Q, None)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    rows = np.sort(np.concatenate([rng.choice(w.N, 500, replace=False), [0, w.N - 1]]))
    for h in heads:
        Y = Qr[0, h][torch.from_numpy(rows).cuda()].double().cpu().numpy()
        assert _check_rope(Y, pre[h][rows].astype(np.float64), w, rows=rows) <= 1


@pytest.mark.parametrize("w", [W, W64], ids=lambda w: f"{w.name}-{w.dtype}")
def test_dense_attention_matches_oracle(w):
    x = synth.layer_inputs(w)
    p = capi.Params.from_workload(w)
    ws = capi.alloc_workspace(p)
    O = capi.dense_attention(p, _dev(w, x["q"]), _dev(w, x["k"]), _dev(w, x["v"]), ws=ws)
    torch.cuda.synchronize()
    assert capi.get_device_status(ws) == 0
    On = O.float().cpu().numpy().reshape(w.B * w.H, w.N, w.d)
    for i in range(w.B * w.H):
        compare_attention(w, On[i], oracle.dense_attention(x["q"][i], x["k"][i], x["v"][i]))


def test_dense_attention_full_size_sampled_rows():
    """The dense branch at HunyuanVideo's 118800 tokens (4 of its 24 heads), sampled rows."""
    w = HUNYUAN720.with_(H=4)
    x = synth.layer_inputs(w)
    p = capi.Params.from_workload(w)
    ws = capi.alloc_workspace(p)
    O = capi.dense_attention(p, _dev(w, x["q"]), _dev(w, x["k"]), _dev(w, x["v"]), ws=ws)
    torch.cuda.synchronize()
    assert capi.get_device_status(ws) == 0
    rng = np.random.default_rng(6)
    for i in (0, 3):
        rows = np.sort(rng.choice(w.N, 48, replace=False))
        ref = oracle.dense_attention(x["q"][i], x["k"][i], x["v"][i], rows=rows)
        got = O[0, i][torch.from_numpy(rows).cuda()].float().cpu().numpy()
        compare_attention(w, got, ref)


@pytest.mark.parametrize("layer,step", [(0, 30), (4, 2), (4, 30)])
@pytest.mark.parametrize("rope", [1, 0])
def test_attention_layer_under_the_schedule(layer, step, rope):
    """scope_attention_layer = [RoPE] + the branch the schedule picks (dense_layers = 1,
    dense_steps = 5), each against the oracle's layer on the generator's inputs."""
    w = W
    x = synth.layer_inputs(w, rope=not rope)
    p = capi.Params.from_workload(w)
    sched = capi.Schedule(layer=layer, step=step, dense_layers=1, dense_steps=5, rope=rope, rope_base=10000.0)
    dense = oracle.layer_is_dense(layer, step, 1, 5)
    assert capi.layer_is_dense(sched) == dense
    ws = capi.alloc_workspace(p)
    qi = torch.from_numpy(x["q_init"]).reshape(w.B, w.H, w.Cq).cuda()
    ki = torch.from_numpy(x["k_init"]).reshape(w.B, w.H, 3, w.Cm).cuda()
    Qr = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.bfloat16, device="cuda")
    Kr = torch.empty_like(Qr)
    O = capi.attention_layer(p, sched, _dev(w, x["q"]), _dev(w, x["k"]), _dev(w, x["v"]), qi, ki, ws=ws,
                             out_q=Qr, out_k=Kr)
    torch.cuda.synchronize()
    assert capi.get_device_status(ws) == 0
    On = O.float().cpu().numpy().reshape(w.B * w.H, w.N, w.d)
    for i in range(w.B * w.H):
        ref = oracle.layer(x["q"][i], x["k"][i], x["v"][i], w, x["q_init"][i], x["k_init"][i], dense,
                           rope_base=10000.0 if rope else None, round_rope=lambda a: _round(a, w.dtype))
        if rope:
            assert _check_rope(_np(Qr, w)[i], x["q"][i].astype(np.float64), w) == 0
            assert _check_rope(_np(Kr, w)[i], x["k"][i].astype(np.float64), w) == 0
        compare_attention(w, On[i], ref["O"])


def test_rope3d_bf16_near_rounding_boundaries():
    """Pairs whose rotated value lies within 2^-22 (|x0| + |x1|) of a bf16 rounding
    boundary: the binary32 evaluation cannot decide them, so the kernel must fall back to
    binary64 and still round like the oracle.  Temporal pair 0 of tokens with t = 1 turns
    by exactly 1 rad."""
    w = Workload("rope_edge", 1, 1, 2, 12, 10, 44, 42, 42, "bf16", 4, 4, seed=25)
    rng = np.random.default_rng(9)
    c, s = np.cos(1.0), np.sin(1.0)
    found = []
    while len(found) < 120:
        e = rng.integers(-6, 6, size=(4096, 2))
        m = rng.integers(128, 256, size=(4096, 2)) * rng.choice([-1, 1], size=(4096, 2))
        x = np.ldexp(m.astype(np.float64), e - 7)            # bf16 values
        S = np.abs(x).sum(axis=1)
        for y in (x[:, 0] * c - x[:, 1] * s, x[:, 0] * s + x[:, 1] * c):
            mid = _round(y, "bf16")
            # nearest boundary: half a bf16 unit from the rounded value, on y's side
            ulp = np.ldexp(1.0, np.frexp(np.abs(mid))[1] - 8)
            dist = np.abs(np.abs(y - mid) - ulp / 2)
            hit = np.nonzero(dist < S * 2.0 ** -22)[0]
            found.extend(x[hit].tolist())
    X = np.zeros((w.N, w.d), np.float32)
    rows = np.arange(w.Hg * w.Wg, 2 * w.Hg * w.Wg)                  # tokens with t = 1
    X[rows, 0:2] = np.asarray(found[:len(rows)], np.float32)
    p = capi.Params.from_workload(w)
    Qr, _ = capi.rope3d(p, _dev(w, X[None]), None)
    torch.cuda.synchronize()
    assert _check_rope(_np(Qr, w)[0], X.astype(np.float64), w) == 0
