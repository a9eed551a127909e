"""Edge cases of the SCOPE path on the GPU, each against the binary64 oracle or a closed
form: empty clusters, a single centroid, rho = 1 (dense attention), explicit initial
centroids (warm start), and the device status word for an out-of-range init index."""
import numpy as np
import pytest
import torch

import oracle
from free_sparse_attention_b200 import capi, synth
from free_sparse_attention_b200.workloads import Workload

from gpu_common import check_selection, compare_attention, to_np

pytestmark = pytest.mark.gpu

W = Workload("edge", 1, 2, 3, 12, 10, 44, 42, 42, "bf16", 16, 12, seed=21)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from free_sparse_attention_b200.build import build
    build()
    capi.lib()


def _dev(w, x, q_init=None, k_init=None):
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    t = {n: torch.from_numpy(x[n]).reshape(w.B, w.H, w.N, w.d).to("cuda", dt) for n in "qkv"}
    qi = x["q_init"] if q_init is None else q_init
    ki = x["k_init"] if k_init is None else k_init
    t["qi"] = torch.from_numpy(np.ascontiguousarray(qi)).reshape(w.B, w.H, w.Cq).cuda()
    t["ki"] = torch.from_numpy(np.ascontiguousarray(ki)).reshape(w.B, w.H, 3, w.Cm).cuda()
    return t


def _forward_and_compare(w, x, t, q_init, k_init, rho=None, khead_off=False, key_full=False):
    over = {} if rho is None else {"rho": rho}
    if khead_off:
        over["khead_mode"] = capi.SCOPE_KHEAD_OFF
    if key_full:
        over["key_clustering"] = capi.SCOPE_KEYS_FULL
    p = capi.Params.from_workload(w, **over)
    ws = capi.alloc_workspace(p)
    O, it = capi.forward(p, t["q"], t["k"], t["v"], t["qi"], t["ki"], ws=ws, intermediates=True)
    torch.cuda.synchronize()
    assert capi.get_device_status(ws) == 0
    g = {k: to_np(v) for k, v in it.items()}
    O = O.float().cpu().numpy().reshape(w.B * w.H, w.N, w.d)
    for i in range(w.B * w.H):
        ref = oracle.forward_head(x["q"][i], x["k"][i], x["v"][i], w, q_init[i], k_init[i], rho=rho,
                                  khead_off=khead_off, key_full=key_full)
        np.testing.assert_array_equal(g["q_assign"][0, i], ref["q"]["assign"])
        np.testing.assert_array_equal(g["q_centroids"][0, i], ref["q"]["centroids"])
        np.testing.assert_array_equal(g["k_codes"][0, i], ref["k"]["codes"])
        np.testing.assert_array_equal(g["k_centroids"][0, i], ref["k"]["centroids"])
        np.testing.assert_array_equal(g["final_counts"][0, i], ref["sel"]["r"])
        assert int(g["k_head"][0, i]) == ref["sel"]["k_head"]
        np.testing.assert_array_equal(g["sel_mask"][0, i].view(np.uint32), ref["sel"]["mask"])
        compare_attention(w, O[i], ref["O"])
    return g, O


def test_duplicate_init_rows_give_empty_clusters():
    """Two initial centroids on the same token tie everywhere: after the first iteration
    the higher index has no member and keeps its centroid; the whole layer (where the
    stale duplicate may win members again later) still matches the oracle."""
    x = synth.layer_inputs(W)
    qi = x["q_init"].copy()
    ki = x["k_init"].copy()
    qi[:, 5] = qi[:, 2]
    ki[:, 1, 7] = ki[:, 1, 3]
    t = _dev(W, x, qi, ki)
    _forward_and_compare(W, x, t, qi, ki)
    p1 = capi.Params.from_workload(W, iters=1)
    qc, qa, qs = capi.cluster_queries(p1, t["q"], init_idx=t["qi"])
    torch.cuda.synchronize()
    assert np.all(to_np(qs)[0, :, 5] == 0)
    first = np.stack([x["q"][h][qi[h, 2]] for h in range(W.H)]).astype(np.float64)
    np.testing.assert_array_equal(to_np(qc)[0, :, 5], first)


@pytest.mark.parametrize("grid,Cq,Cm", [((1, 1, 1), 1, 1), ((1, 2, 3), 2, 3), ((1, 3, 11), 5, 4)],
                         ids=["N1", "N6", "N33"])
def test_tiny_token_counts(grid, Cq, Cm):
    """Layers of 1, 6 and 33 tokens: fewer keys than one 64-key attention tile, than one
    32-bit mask word or one 8-key row of saved bins (33: one word and one key more).  The
    whole layer must equal the oracle's."""
    w = Workload("tiny_n", 1, 2, *grid, 44, 42, 42, "bf16", Cq, Cm, seed=27)
    x = synth.layer_inputs(w)
    t = _dev(w, x)
    _forward_and_compare(w, x, t, x["q_init"], x["k_init"])
    _forward_and_compare(w, x, t, x["q_init"], x["k_init"], rho=0.5)


def test_single_centroid_everywhere():
    w = W.with_(Cq=1, Cm=1)
    x = synth.layer_inputs(w)
    t = _dev(w, x)
    g, _ = _forward_and_compare(w, x, t, x["q_init"], x["k_init"])
    assert np.all(g["k_head"] == g["base_counts"][..., 0])


def test_rho_one_is_dense_attention():
    x = synth.layer_inputs(W)
    t = _dev(W, x)
    p = capi.Params.from_workload(W, rho=1.0)
    O, it = capi.forward(p, t["q"], t["k"], t["v"], t["qi"], t["ki"], intermediates=True)
    dense = torch.nn.functional.scaled_dot_product_attention(t["q"].float(), t["k"].float(), t["v"].float())
    torch.cuda.synchronize()
    assert torch.all(it["final_counts"] == W.N)
    err = (O.float() - dense).abs()
    assert err.max().item() <= 2e-2
    assert (err.pow(2).mean().sqrt() / dense.pow(2).mean().sqrt()).item() <= 5e-3


def test_explicit_initial_centroids_warm_start():
    """Clustering started from caller centroids (e.g. the previous step's) equals the
    oracle started from the same centroids."""
    x = synth.layer_inputs(W)
    t = _dev(W, x)
    p = capi.Params.from_workload(W)
    rng = np.random.default_rng(3)
    qc0 = rng.standard_normal((W.B, W.H, W.Cq, W.d))
    kc0 = rng.standard_normal((W.B, W.H, W.Cm, W.d))
    qc, qa, qs = capi.cluster_queries(p, t["q"], init_cent=torch.from_numpy(qc0).cuda())
    kc, kk = capi.cluster_keys(p, t["k"], init_cent=torch.from_numpy(kc0).cuda())
    torch.cuda.synchronize()
    for h in range(W.H):
        rq = oracle.kmeans(x["q"][h], 0, W.d, W.Cq, W.iters, init_cent=qc0[0, h])
        rk = oracle.cluster_keys(x["k"][h], (W.d_t, W.d_h, W.d_w), W.Cm, W.iters, init_cent=kc0[0, h])
        np.testing.assert_array_equal(to_np(qa)[0, h], rq["assign"])
        np.testing.assert_array_equal(to_np(qc)[0, h], rq["centroids"])
        np.testing.assert_array_equal(to_np(kk)[0, h], rk["codes"])
        np.testing.assert_array_equal(to_np(kc)[0, h], rk["centroids"])


def test_equal_logits_with_spread_tables_and_a_topup():
    """Every key carries the same three codes, so inside a cluster all logits are equal,
    while the memberless centroids keep each table spread (its bounds differ).  The Top-p
    pass then sees one logit value and bins nothing by value; with rho below alpha every
    cluster is topped up to k_fix keys (Eq. 10), which the ranking by index makes the first
    k_fix keys.  An earlier call on the same workspace leaves real first-level counts
    behind, which the mask kernel must not take for this call's."""
    w = W
    rho = 0.0513   # rho N = 18.47: the Top-p count is 19 keys, far from a mass tie
    p = capi.Params.from_workload(w, rho=rho)
    ws = capi.alloc_workspace(p)
    rng = np.random.default_rng(8)
    BH = w.B * w.H
    qc = rng.standard_normal((BH, w.Cq, w.d))
    qs = (1 + rng.multinomial(w.N - w.Cq, np.full(w.Cq, 1.0 / w.Cq), size=BH)).astype(np.int32)
    kc = rng.standard_normal((BH, w.Cm, w.d))
    spread = rng.integers(0, w.Cm, (BH, 3, w.N)).astype(np.uint16)
    equal = np.zeros((BH, 3, w.N), np.uint16)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).reshape((w.B, w.H) + a.shape[1:]).cuda()
    capi.build_lut_and_select(p, dev(qc), dev(qs), dev(kc), dev(spread), ws=ws)
    out = capi.build_lut_and_select(p, dev(qc), dev(qs), dev(kc), dev(equal), ws=ws)
    torch.cuda.synchronize()
    assert capi.get_device_status(ws) == 0
    g = {k: to_np(v).reshape((BH,) + tuple(v.shape[2:])) for k, v in out.items()}
    for i in range(BH):
        ref = oracle.select(qc[i], qs[i], kc[i], equal[i], (w.d_t, w.d_h, w.d_w), rho, w.alpha)
        assert np.all(g["topp_counts"][i] == 19)
        kfix = int(ref["r"][0])
        assert kfix > 19 and np.all(ref["r"] == kfix)
        first = np.zeros(p.nw, np.uint32)
        for j in range(kfix):
            first[j >> 5] |= np.uint32(1 << (j & 31))
        assert np.all(ref["mask"] == first)
        np.testing.assert_array_equal(g["final_counts"][i], ref["r"])
        np.testing.assert_array_equal(g["sel_mask"][i].view(np.uint32), ref["mask"])


@pytest.mark.parametrize("rho", [0.3, 0.75])
def test_two_logit_values_in_bins_larger_than_the_gather_capacity(rho):
    """The keys take only two codes in the temporal subspace and one in the others, so every
    cluster sees two logit values, each shared by ~3456 keys: the Top-p crossing and the
    top-up boundary both fall inside a bin of more keys than one gather holds (2048), where
    the ranking among equal logits is by key index.  Selection must equal the oracle's (a
    logged near tie excepted, as everywhere)."""
    w = Workload("twovalues", 1, 1, 3, 48, 48, 44, 42, 42, "bf16", 16, 4, seed=23)
    p = capi.Params.from_workload(w, rho=rho)
    rng = np.random.default_rng(12)
    BH = w.B * w.H
    qc = rng.standard_normal((BH, w.Cq, w.d))
    qs = (1 + rng.multinomial(w.N - w.Cq, np.full(w.Cq, 1.0 / w.Cq), size=BH)).astype(np.int32)
    kc = rng.standard_normal((BH, w.Cm, w.d))
    codes = np.zeros((BH, 3, w.N), np.uint16)
    codes[:, 0] = rng.integers(0, 2, (BH, w.N))
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).reshape((w.B, w.H) + a.shape[1:]).cuda()
    ws = capi.alloc_workspace(p)
    out = capi.build_lut_and_select(p, dev(qc), dev(qs), dev(kc), dev(codes), ws=ws)
    torch.cuda.synchronize()
    assert capi.get_device_status(ws) == 0
    g = {k: to_np(v).reshape((BH,) + tuple(v.shape[2:])) for k, v in out.items()}
    split = (w.d_t, w.d_h, w.d_w)
    for i in range(BH):
        args = (qc[i], qs[i], kc[i], codes[i], split, rho, w.alpha)
        sel = oracle.select(*args)
        gi = {k: g[k][i] for k in g}
        check_selection(w, gi, sel, qs[i], lambda: oracle.select(*args, want_scores=True))
        # each logit value is shared by more than 2048 keys, and some clusters are topped up
        assert min((codes[i, 0] == 0).sum(), (codes[i, 0] == 1).sum()) > 2048
        assert np.any(sel["r"] != sel["p"]) and np.all(sel["r"] < w.N)


def test_bad_init_index_sets_status():
    x = synth.layer_inputs(W)
    qi = x["q_init"].copy()
    qi[0, 0] = W.N + 5
    t = _dev(W, x, qi, x["k_init"])
    p = capi.Params.from_workload(W)
    ws = capi.alloc_workspace(p)
    capi.cluster_queries(p, t["q"], init_idx=t["qi"], ws=ws)
    assert capi.get_device_status(ws) & capi.DEV_BAD_INIT_INDEX
    # the next call on the same workspace starts clean
    capi.cluster_queries(p, t["q"], init_idx=_dev(W, x)["qi"], ws=ws)
    assert capi.get_device_status(ws) == 0


def test_fp32_and_bf16_paths_agree_on_selection():
    """The same values as fp32 and as bf16 give identical clustering and selection
    (the inputs are bf16-exact), and attention within tolerance of each other."""
    x = synth.layer_inputs(W)
    w32 = W.with_(dtype="f32")
    t16, t32 = _dev(W, x), _dev(w32, x)
    O16, i16 = capi.forward(capi.Params.from_workload(W), t16["q"], t16["k"], t16["v"], t16["qi"],
                            t16["ki"], intermediates=True)
    O32, i32 = capi.forward(capi.Params.from_workload(w32), t32["q"], t32["k"], t32["v"], t32["qi"],
                            t32["ki"], intermediates=True)
    torch.cuda.synchronize()
    for k in ("q_assign", "k_codes", "final_counts", "sel_mask", "k_head"):
        assert torch.equal(i16[k], i32[k]), k
    assert (O16.float() - O32).abs().max().item() <= 2e-2


def _bf16_exact(a):
    """Rounds float64 values to bf16 and returns them as float32 (exact copies)."""
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16).float().numpy()


@pytest.mark.parametrize("wide", [False, True])
def test_member_sums_with_and_without_the_exact_parallel_path(wide):
    """Centroid means of bf16 members are summed in parallel only when every partial sum is
    exactly representable (sum |x| <= 2^52 * the smallest ulp among the members); otherwise
    in token order.  With `wide`, half of the channels mix values near 2^40 and 2^-30 inside
    one cluster, so those channels take the in-order path and the others the parallel one.
    Either way the centroids must equal the oracle's in-order binary64 means bit for bit."""
    w = Workload("sums", 1, 2, 4, 16, 16, 44, 42, 42, "bf16", 3, 5, seed=31)
    rng = np.random.default_rng(5)
    q = rng.standard_normal((w.H, w.N, w.d))
    if wide:
        big = rng.random((w.H, w.N)) < 0.05
        q[:, :, 64:] = np.where(big[..., None], 2.0 ** 40, 2.0 ** -30) * (1.0 + rng.random((w.H, w.N, 64)))
    q = _bf16_exact(q)
    init = np.stack([rng.choice(w.N, w.Cq, replace=False) for _ in range(w.H)]).astype(np.int32)
    Q = torch.from_numpy(q).reshape(w.B, w.H, w.N, w.d).to("cuda", torch.bfloat16)
    p = capi.Params.from_workload(w)
    qc, qa, qs = capi.cluster_queries(p, Q, init_idx=torch.from_numpy(init).reshape(w.B, w.H, w.Cq).cuda())
    torch.cuda.synchronize()
    for h in range(w.H):
        ref = oracle.kmeans(q[h].astype(np.float32), 0, w.d, w.Cq, w.iters, init_idx=init[h])
        np.testing.assert_array_equal(to_np(qa)[0, h], ref["assign"])
        np.testing.assert_array_equal(to_np(qs)[0, h], ref["sizes"])
        np.testing.assert_array_equal(to_np(qc)[0, h], ref["centroids"])


def test_khead_off_ablation_matches_oracle():
    """The review page's ablation with the online k_head disabled: the whole layer (r_c =
    b_c, no top-up) against the oracle run with the same switch."""
    w = W.with_(Cq=20, Cm=16)
    x = synth.layer_inputs(w)
    t = _dev(w, x)
    g, _ = _forward_and_compare(w, x, t, x["q_init"], x["k_init"], khead_off=True)
    np.testing.assert_array_equal(g["final_counts"], g["base_counts"])


def test_warm_start_from_previous_step_with_one_iteration():
    """Warm start across denoising steps (review page, pith_inferences): the next step's
    layer (the same inputs plus small noise) clusters from the previous step's centroids
    with a single Lloyd iteration, then selects and attends through the stage entry
    points; every stage equals the oracle run from the same centroids."""
    w = W.with_(Cq=12, Cm=10)
    x = synth.layer_inputs(w)
    t = _dev(w, x)
    p = capi.Params.from_workload(w)
    _, it = capi.forward(p, t["q"], t["k"], t["v"], t["qi"], t["ki"], intermediates=True)
    qc0, kc0 = it["q_centroids"].clone(), it["k_centroids"].clone()
    rng = np.random.default_rng(9)
    x2 = dict(x)
    for n in "qkv":
        x2[n] = _bf16_exact(x[n] + 0.05 * rng.standard_normal(x[n].shape))
    t2 = _dev(w, x2)
    p1 = capi.Params.from_workload(w, iters=1)
    qc, qa, qs = capi.cluster_queries(p1, t2["q"], init_cent=qc0)
    kc, kk = capi.cluster_keys(p1, t2["k"], init_cent=kc0)
    sel = capi.build_lut_and_select(p, qc, qs, kc, kk)
    O = capi.sparse_attention(p, t2["q"], t2["k"], t2["v"], qa, sel["sel_mask"], sel["final_counts"])
    torch.cuda.synchronize()
    O = O.float().cpu().numpy().reshape(w.H, w.N, w.d)
    for h in range(w.H):
        # step A by the oracle itself (equal to the GPU's, whose centroids started step B)
        qa0 = oracle.kmeans(x["q"][h], 0, w.d, w.Cq, w.iters, init_idx=x["q_init"][h])["centroids"]
        ka0 = oracle.cluster_keys(x["k"][h], (w.d_t, w.d_h, w.d_w), w.Cm, w.iters,
                                  init_idx3=x["k_init"][h])["centroids"]
        np.testing.assert_array_equal(to_np(qc0)[0, h], qa0)
        np.testing.assert_array_equal(to_np(kc0)[0, h], ka0)
        rq = oracle.kmeans(x2["q"][h], 0, w.d, w.Cq, 1, init_cent=qa0)
        rk = oracle.cluster_keys(x2["k"][h], (w.d_t, w.d_h, w.d_w), w.Cm, 1, init_cent=ka0)
        np.testing.assert_array_equal(to_np(qa)[0, h], rq["assign"])
        np.testing.assert_array_equal(to_np(qc)[0, h], rq["centroids"])
        np.testing.assert_array_equal(to_np(kk)[0, h], rk["codes"])
        np.testing.assert_array_equal(to_np(kc)[0, h], rk["centroids"])
        rs = oracle.select(rq["centroids"], rq["sizes"], rk["centroids"], rk["codes"],
                           (w.d_t, w.d_h, w.d_w), w.rho, w.alpha)
        np.testing.assert_array_equal(to_np(sel["final_counts"])[0, h], rs["r"])
        np.testing.assert_array_equal(to_np(sel["sel_mask"])[0, h].view(np.uint32), rs["mask"])
        ref = oracle.attention(x2["q"][h], x2["k"][h], x2["v"][h], rq["assign"], rs["mask"])
        compare_attention(w, O[h], ref)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_random_channel_partition_ablation(dtype):
    """scope_permute_channels equals numpy indexing, and the layer run on Q and K permuted
    alike (key subspaces = random channel subsets; review page, significance) equals the
    oracle run on the same permuted inputs."""
    w = W.with_(dtype=dtype, Cq=10, Cm=8)
    x = synth.layer_inputs(w)
    perm = np.random.default_rng(44).permutation(w.d).astype(np.int32)
    t = _dev(w, x)
    p = capi.Params.from_workload(w)
    pd = torch.from_numpy(perm).cuda()
    qp = capi.permute_channels(p, t["q"], pd)
    kp = capi.permute_channels(p, t["k"], pd)
    torch.cuda.synchronize()
    xp = dict(x)
    xp["q"] = np.ascontiguousarray(x["q"][..., perm])
    xp["k"] = np.ascontiguousarray(x["k"][..., perm])
    tp = _dev(w, xp)
    assert torch.equal(qp, tp["q"]) and torch.equal(kp, tp["k"])
    _forward_and_compare(w, xp, tp, x["q_init"], x["k_init"])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_full_d_key_clustering_ablation(dtype):
    """The review page's full-dimensional cluster scoring (significance; falsifier): one
    k-means of the keys over all d channels; code rows 1 and 2 are zero and the proxy is
    the cluster-level dot product.  Whole layer against the oracle, at Cm and at 3 Cm
    (the same number of key centroids as the three subspaces)."""
    for Cm in (W.Cm, 3 * W.Cm):
        w = W.with_(dtype=dtype, Cm=Cm)
        x = synth.layer_inputs(w)
        t = _dev(w, x)
        g, _ = _forward_and_compare(w, x, t, x["q_init"], x["k_init"], key_full=True)
        assert not g["k_codes"][:, :, 1:].any()


def test_wait_timeout_is_reported_and_the_context_survives():
    """Failure detection without a GPU fault: scope_check_wait_timeout holds the attention
    kernel's scheduler back, so the first wait of every warp runs out after 2 ms, before
    any copy or tensor-core product is issued.  The kernel returns with SCOPE_DEV_TIMEOUT in
    the status word (scope_get_device_status: SCOPE_ERR_TIMEOUT), and the next layer on the
    same workspace runs normally and matches the oracle."""
    x = synth.layer_inputs(W)
    t = _dev(W, x)
    p = capi.Params.from_workload(W)
    ws = capi.alloc_workspace(p)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    capi.check_wait_timeout(p, 2_000_000, ws=ws)
    e1.record()
    code, word = capi.device_status_code(ws)
    assert code == 6 and word == 0x8, (code, word)          # SCOPE_ERR_TIMEOUT, SCOPE_DEV_TIMEOUT only
    assert 2.0 <= e0.elapsed_time(e1) < 1000.0               # gave up after the limit, not hung
    O = capi.forward(p, t["q"], t["k"], t["v"], t["qi"], t["ki"], ws=ws)
    assert capi.device_status_code(ws) == (0, 0)             # the same workspace, clean again
    g, O2 = _forward_and_compare(W, x, t, x["q_init"], x["k_init"])
    np.testing.assert_array_equal(O.float().cpu().numpy().reshape(O2.shape), O2)
