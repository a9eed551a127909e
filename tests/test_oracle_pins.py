"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test ties one oracle function to an independent source: a library routine that
implements the same textbook step (scipy's Lloyd k-means, torch's attention), exact
rational arithmetic, a closed form that the SCOPE equations imply for a special
input, or brute force over all subsets of a tiny input.  A dropped term, a wrong sign
or index, or a transposed operand in the oracle fails at least one of them.
"""
import itertools
import math
import warnings
from fractions import Fraction

import numpy as np
import pytest
import scipy.cluster.vq as vq
import torch

import oracle
from free_sparse_attention_b200 import synth
from free_sparse_attention_b200.workloads import TINY


def _blobs(rng, N, dm, C, spread=0.05):
    centers = rng.standard_normal((C, dm)) * 3.0
    lab = rng.integers(0, C, size=N)
    X = centers[lab] + spread * rng.standard_normal((N, dm))
    return X.astype(np.float32)


# ----------------------------------------------------------------------------- k-means
@pytest.mark.parametrize("iters", [1, 2, 5])
@pytest.mark.parametrize("dm,C", [(4, 3), (16, 8), (24, 13)])
def test_kmeans_matches_scipy_lloyd(iters, dm, C):
    """Eq. 3 by Lloyd's iteration == scipy.cluster.vq.kmeans2 with the same init."""
    rng = np.random.default_rng(1000 + 17 * dm + C + iters)
    X = rng.standard_normal((300, dm)).astype(np.float32)
    init = rng.choice(300, size=C, replace=False).astype(np.int32)
    res = oracle.kmeans(X, 0, dm, C, iters, init_idx=init)
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")
        cb, lab = vq.kmeans2(X.astype(np.float64), X[init].astype(np.float64), iter=iters,
                             minit="matrix", missing="warn")
    np.testing.assert_array_equal(res["assign"].astype(np.int64), lab)
    np.testing.assert_allclose(res["centroids"], cb, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(res["sizes"], np.bincount(lab, minlength=C))


def test_kmeans_subspace_channels_match_scipy():
    """A channel range of a wider row is clustered on exactly those channels."""
    rng = np.random.default_rng(7)
    X = rng.standard_normal((257, 64)).astype(np.float32)
    for ch0, dm in [(0, 16), (16, 24), (40, 24)]:
        init = rng.choice(257, size=8, replace=False).astype(np.int32)
        res = oracle.kmeans(X, ch0, dm, 8, 5, init_idx=init)
        sub = X[:, ch0:ch0 + dm].astype(np.float64)
        with warnings.catch_warnings():
            warnings.simplefilter("ignore")
            cb, lab = vq.kmeans2(sub, sub[init], iter=5, minit="matrix", missing="warn")
        np.testing.assert_array_equal(res["assign"].astype(np.int64), lab)
        np.testing.assert_allclose(res["centroids"], cb, rtol=1e-12, atol=1e-12)


def test_kmeans_one_iteration_brute_force():
    """One iteration: every row goes to its nearest init centroid (lowest index on a
    tie) and every centroid becomes its members' mean (numpy mean)."""
    rng = np.random.default_rng(3)
    X = _blobs(rng, 200, 10, 6)
    init = rng.choice(200, size=6, replace=False).astype(np.int32)
    res = oracle.kmeans(X, 0, 10, 6, 1, init_idx=init)
    X64 = X.astype(np.float64)
    d2 = ((X64[:, None, :] - X64[init][None, :, :]) ** 2).sum(-1)
    np.testing.assert_array_equal(res["assign"], np.argmin(d2, axis=1))
    for c in range(6):
        members = X64[res["assign"] == c]
        expect = members.mean(0) if len(members) else X64[init[c]]
        np.testing.assert_allclose(res["centroids"][c], expect, rtol=1e-13, atol=1e-13)


def test_kmeans_tie_goes_to_lowest_index_and_empty_keeps_centroid():
    X = np.array([[0.0], [2.0], [10.0]], np.float32)
    # centroids -1 and 1 are equidistant from row 0; centroid 100 gets no member
    res = oracle.kmeans(X, 0, 1, 3, 1, init_cent=np.array([[1.0], [-1.0], [100.0]]))
    assert list(res["assign"]) == [0, 0, 0]
    np.testing.assert_allclose(res["centroids"][:, 0], [4.0, -1.0, 100.0])
    assert list(res["sizes"]) == [3, 0, 0]


def test_kmeans_objective_non_increasing():
    """Lloyd never increases the squared error: assign and update each lower it."""
    rng = np.random.default_rng(11)
    X = rng.standard_normal((500, 24)).astype(np.float32)
    init = rng.choice(500, size=12, replace=False).astype(np.int32)
    res = oracle.kmeans(X, 0, 24, 12, 8, init_idx=init, logs=True)
    seq = np.stack([res["obj_assign"], res["obj_update"]], 1).reshape(-1)
    assert np.all(np.diff(seq) <= 1e-9 * seq[0])
    # the logged margin is the relative gap to the second-nearest centroid
    assert np.all(res["margin"] >= 0)


# ----------------------------------------------------------------------------- selection
def _random_select_inputs(rng, N=97, d=16, split=(4, 6, 6), Cq=5, Cm=7):
    qcent = rng.standard_normal((Cq, d))
    kcent = rng.standard_normal((Cm, d))
    codes = rng.integers(0, Cm, size=(3, N)).astype(np.uint16)
    qsizes = rng.integers(0, 40, size=Cq).astype(np.int32)
    qsizes[0] = max(qsizes[0], 1)
    return qcent, qsizes, kcent, codes, split


def test_proxy_logit_equals_product_code_inner_product():
    """Eq. 27: the LUT sum equals <q_c, k_hat_j>/sqrt(d), k_hat_j the concatenation of
    key j's three subspace centroids."""
    rng = np.random.default_rng(5)
    qcent, qsizes, kcent, codes, split = _random_select_inputs(rng)
    sel = oracle.select(qcent, qsizes, kcent, codes, split, 0.9, 0.1, want_scores=True)
    d = qcent.shape[1]
    b = [0, split[0], split[0] + split[1], d]
    khat = np.empty((codes.shape[1], d))
    for m in range(3):
        khat[:, b[m]:b[m + 1]] = kcent[codes[m], b[m]:b[m + 1]]
    expect = qcent @ khat.T / math.sqrt(d)
    np.testing.assert_allclose(sel["scores"], expect, rtol=1e-12, atol=1e-13)


def _ranking(scores_row):
    N = scores_row.shape[0]
    return np.lexsort((np.arange(N), -scores_row))


def test_topp_is_minimal_subset_by_brute_force():
    """Eq. 7: p_c is the least number of keys whose softmax mass reaches rho; over ALL
    subsets of a tiny key set, no smaller subset reaches it, and the selected keys are
    the highest-scoring ones (index order on equal scores)."""
    rng = np.random.default_rng(9)
    for trial in range(6):
        N = 11
        qcent, qsizes, kcent, codes, split = _random_select_inputs(rng, N=N, Cq=3, Cm=3)
        rho = [0.3, 0.5, 0.7, 0.8, 0.9, 0.95][trial]
        sel = oracle.select(qcent, qsizes, kcent, codes, split, rho, 0.0, want_scores=True)
        for c in range(3):
            s = sel["scores"][c]
            w = np.exp(s - s.max())
            Z = w.sum()
            best = min(len(S) for k in range(1, N + 1) for S in itertools.combinations(range(N), k)
                       if w[list(S)].sum() >= rho * Z * (1 + 1e-12))
            assert sel["p"][c] == best, (trial, c)


def test_uniform_logits_give_ceil_rho_n():
    """All keys equal => every key carries mass 1/N => p_c = ceil(rho*N) (closed form)."""
    N, Cq, Cm, d = 1000, 4, 3, 16
    rng = np.random.default_rng(2)
    codes = np.zeros((3, N), np.uint16)
    for rho in (0.3337, 0.5001, 0.9003, 0.0149):
        sel = oracle.select(rng.standard_normal((Cq, d)), np.full(Cq, 10, np.int32),
                            rng.standard_normal((Cm, d)), codes, (4, 6, 6), rho, 0.0)
        assert np.all(sel["p"] == math.ceil(rho * N))


def test_rho_one_keeps_every_key():
    rng = np.random.default_rng(4)
    qcent, qsizes, kcent, codes, split = _random_select_inputs(rng, N=70)
    sel = oracle.select(qcent, qsizes, kcent, codes, split, 1.0, 0.1)
    assert np.all(sel["p"] == 70) and np.all(sel["r"] == 70) and sel["k_head"] == 70
    bits = np.unpackbits(sel["mask"].view(np.uint8), bitorder="little").reshape(len(qsizes), -1)
    assert np.all(bits[:, :70] == 1) and np.all(bits[:, 70:] == 0)


def test_tiny_rho_gives_fixed_topk_floor():
    """rho -> 0 keeps one key by Top-p, so b_c = k_fix = ceil(alpha*N) everywhere and
    k_head = k_fix; with one query cluster, k_head = b_1."""
    rng = np.random.default_rng(6)
    qcent, qsizes, kcent, codes, split = _random_select_inputs(rng, N=200)
    sel = oracle.select(qcent, qsizes, kcent, codes, split, 1e-12, 0.1)
    assert np.all(sel["p"] == 1)
    assert np.all(sel["b"] == 20) and sel["k_head"] == 20 and np.all(sel["r"] == 20)
    sel1 = oracle.select(qcent[:1], qsizes[:1], kcent, codes, split, 0.6, 0.0)
    assert sel1["k_head"] == sel1["b"][0]


def test_khead_is_exact_weighted_mean_ceiling_and_topup_invariants():
    """Eq. 9 against exact rationals, Eq. 10 invariants, and the selected sets are
    prefixes of each cluster's ranking of the sizes r_c."""
    rng = np.random.default_rng(8)
    for trial in range(5):
        qcent, qsizes, kcent, codes, split = _random_select_inputs(rng, N=150, Cq=9, Cm=5)
        sel = oracle.select(qcent, qsizes, kcent, codes, split, [0.5, 0.7, 0.9, 0.95, 0.99][trial],
                            0.1, want_scores=True)
        b, r, kh = sel["b"].astype(int), sel["r"].astype(int), sel["k_head"]
        expect = math.ceil(Fraction(int(np.dot(qsizes.astype(int), b)), int(qsizes.sum())))
        assert kh == expect
        kfix = math.ceil(Fraction(1, 10) * 150)
        assert np.all(b >= kfix) and np.all(b >= sel["p"]) and kh >= kfix
        nz = qsizes > 0
        assert b[nz].min() <= kh <= b[nz].max()
        assert np.all(r >= kh) and np.all(r[b >= kh] == b[b >= kh]) and np.all(r == np.maximum(b, kh))
        bits = np.unpackbits(sel["mask"].view(np.uint8), bitorder="little").reshape(9, -1)[:, :150]
        for c in range(9):
            top = _ranking(sel["scores"][c])[:r[c]]
            expect_bits = np.zeros(150, np.uint8)
            expect_bits[top] = 1
            np.testing.assert_array_equal(bits[c], expect_bits)


def test_khead_off_ablation_keeps_the_hybrid_counts():
    """The ablation with the online k_head disabled (review page, significance): p_c, b_c and
    k_head are those of the method, r_c = b_c, and every S_c is the b_c-key prefix of the
    cluster's ranking, so it sits inside the method's set (equal where b_c >= k_head)."""
    rng = np.random.default_rng(18)
    for trial in range(4):
        qcent, qsizes, kcent, codes, split = _random_select_inputs(rng, N=160, Cq=11, Cm=6)
        rho = [0.5, 0.8, 0.9, 0.97][trial]
        on = oracle.select(qcent, qsizes, kcent, codes, split, rho, 0.1, want_scores=True)
        off = oracle.select(qcent, qsizes, kcent, codes, split, rho, 0.1, want_scores=True, khead_off=True)
        np.testing.assert_array_equal(off["p"], on["p"])
        np.testing.assert_array_equal(off["b"], on["b"])
        assert off["k_head"] == on["k_head"]
        np.testing.assert_array_equal(off["r"], off["b"])
        bon = np.unpackbits(on["mask"].view(np.uint8), bitorder="little").reshape(11, -1)[:, :160]
        boff = np.unpackbits(off["mask"].view(np.uint8), bitorder="little").reshape(11, -1)[:, :160]
        for c in range(11):
            top = _ranking(off["scores"][c])[:off["b"][c]]
            expect_bits = np.zeros(160, np.uint8)
            expect_bits[top] = 1
            np.testing.assert_array_equal(boff[c], expect_bits)
            assert np.all(boff[c] <= bon[c])
            if on["b"][c] >= on["k_head"]:
                np.testing.assert_array_equal(boff[c], bon[c])


def test_lossless_codebook_gives_exact_logits():
    """Keys whose subspace parts take at most Cm distinct values, clustered from those
    values, are reproduced exactly (k_hat = k), so the proxy is the true logit."""
    rng = np.random.default_rng(12)
    N, d, split, Cm = 120, 16, (4, 6, 6), 5
    b = [0, 4, 10, 16]
    K = np.empty((N, d), np.float32)
    vals = []
    for m in range(3):
        v = rng.standard_normal((Cm, b[m + 1] - b[m])).astype(np.float32)
        pick = rng.integers(0, Cm, size=N)
        pick[:Cm] = np.arange(Cm)          # every value occurs
        K[:, b[m]:b[m + 1]] = v[pick]
        vals.append(pick)
    init = np.stack([np.arange(Cm, dtype=np.int32)] * 3)
    kc = oracle.cluster_keys(K, split, Cm, 3, init_idx3=init)
    for m in range(3):
        np.testing.assert_array_equal(kc["codes"][m], vals[m])
    q = rng.standard_normal((2, d))
    sel = oracle.select(q, np.array([3, 4], np.int32), kc["centroids"], kc["codes"], split,
                        0.9, 0.1, want_scores=True)
    np.testing.assert_allclose(sel["scores"], q @ K.astype(np.float64).T / 4.0, rtol=1e-14, atol=1e-14)


# ----------------------------------------------------------------------------- attention
def _sdpa64(Q, K, V, allowed):
    q = torch.from_numpy(Q.astype(np.float64))[None, None]
    k = torch.from_numpy(K.astype(np.float64))[None, None]
    v = torch.from_numpy(V.astype(np.float64))[None, None]
    m = torch.from_numpy(allowed)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=m)[0, 0].numpy()


def test_attention_equals_masked_sdpa():
    """Sparse attention over S_c == torch SDPA (float64) with -inf on unselected keys."""
    rng = np.random.default_rng(13)
    N, d, Cq = 90, 32, 4
    Q, K, V = (rng.standard_normal((N, d)).astype(np.float32) for _ in range(3))
    qassign = rng.integers(0, Cq, size=N).astype(np.uint16)
    bits = rng.random((Cq, 96)) < 0.4
    bits[:, 90:] = False
    bits[:, 0] = True
    mask = np.packbits(bits.astype(np.uint8), axis=1, bitorder="little").view(np.uint32)
    O = oracle.attention(Q, K, V, qassign, mask)
    np.testing.assert_allclose(O, _sdpa64(Q, K, V, bits[qassign][:, :N]), rtol=1e-12, atol=1e-12)
    rows = np.array([5, 0, 77], np.int64)
    np.testing.assert_allclose(oracle.attention(Q, K, V, qassign, mask, rows=rows), O[rows],
                               rtol=0, atol=0)


def test_rho_one_forward_is_dense_attention():
    """With rho = 1 every cluster keeps every key, so the whole hot path reduces to
    dense softmax attention over the original Q, K, V."""
    x = synth.layer_inputs(TINY)
    q, k, v = x["q"][0], x["k"][0], x["v"][0]
    res = oracle.forward_head(q, k, v, TINY, x["q_init"][0], x["k_init"][0], rho=1.0)
    dense = _sdpa64(q, k, v, np.ones((TINY.N, TINY.N), bool))
    np.testing.assert_allclose(res["O"], dense, rtol=1e-12, atol=1e-12)


def test_tiny_forward_invariants():
    x = synth.layer_inputs(TINY)
    res = oracle.forward_head(x["q"][0], x["k"][0], x["v"][0], TINY, x["q_init"][0],
                              x["k_init"][0], logs=True)
    sel = res["sel"]
    assert res["q"]["sizes"].sum() == TINY.N
    assert np.all(sel["r"] >= sel["k_head"]) and sel["k_head"] >= oracle.kfix(TINY.alpha, TINY.N)
    assert np.all(np.isfinite(res["O"]))


def test_selection_recall_closed_forms_and_brute_force():
    """Proxy-ranking fidelity (review page, falsifier): frac = 1 gives |S| / N and 1; a proxy
    equal to the true logits recalls everything; selecting exactly the true top set recalls
    everything; and a tiny case with tied logits against brute-force enumeration of the
    ranking (value descending, index ascending)."""
    rng = np.random.default_rng(21)
    N, d = 97, 12
    q = rng.standard_normal(d)
    K = rng.standard_normal((N, d))
    proxy = rng.standard_normal(N)
    sel = rng.random(N) < 0.4
    rs, rp = oracle.selection_recall(q, K, proxy, sel, 1.0)
    assert rs == sel.sum() / N and rp == 1.0
    exact = K @ q
    for frac in (0.05, 0.1, 0.33, 0.7):
        _, rp = oracle.selection_recall(q, K, exact, sel, frac)
        assert rp == 1.0
        k = math.ceil(frac * N)
        top = np.argsort(-exact, kind="stable")[:k]
        only = np.zeros(N, bool)
        only[top] = True
        rs, _ = oracle.selection_recall(q, K, exact, only, frac)
        assert rs == 1.0
    # ties: integer-valued keys so that many logits coincide exactly
    Kt = rng.integers(-2, 3, size=(40, 3)).astype(np.float64)
    qt = np.array([1.0, 1.0, 0.0])
    pt = rng.integers(0, 4, size=40).astype(np.float64)
    st = rng.random(40) < 0.5
    for frac in (0.1, 0.25, 0.5):
        k = math.ceil(frac * 40)
        lt = [(-(qt @ Kt[j]), j) for j in range(40)]
        T = {j for _, j in sorted(lt)[:k]}
        P = {j for _, j in sorted((-pt[j], j) for j in range(40))[:k]}
        rs, rp = oracle.selection_recall(qt, Kt, pt, st, frac)
        assert rs == sum(st[j] for j in T) / k
        assert rp == len(T & P) / k


def test_common_channel_permutation_leaves_attention_unchanged():
    """The random-channel-partition ablation permutes the channels of q and k alike: every
    logit q.k, hence attention over any selection, is unchanged (up to summation order)."""
    rng = np.random.default_rng(33)
    N, d = 60, 16
    q = rng.standard_normal((N, d)).astype(np.float32)
    k = rng.standard_normal((N, d)).astype(np.float32)
    v = rng.standard_normal((N, d)).astype(np.float32)
    assign = rng.integers(0, 3, N).astype(np.uint16)
    mask = rng.integers(0, 2 ** 32, size=(3, (N + 31) // 32), dtype=np.uint64).astype(np.uint32)
    mask[:, 0] |= 1
    perm = rng.permutation(d)
    a = oracle.attention(q, k, v, assign, mask)
    b = oracle.attention(np.ascontiguousarray(q[:, perm]), np.ascontiguousarray(k[:, perm]), v, assign, mask)
    np.testing.assert_allclose(b, a, rtol=1e-12, atol=1e-14)


# ----------------------------------------------------------------------------- 3D RoPE
_GRID, _SPLIT = (3, 4, 6), (16, 56, 56)   # HunyuanVideo's channel split on a small grid


def _token(t, h, w):
    return (t * _GRID[1] + h) * _GRID[2] + w


def test_rope3d_closed_form_angles_per_axis():
    """RoFormer's rotation on unit vectors at angles with closed forms: with base 10000,
    pair i of a range of width d_a turns by p * 10^(-8i/d_a).  t = 1 turns temporal pair 0
    by exactly 1 rad and temporal pair 4 by 10^-2; h = 3 turns height pair 14 by 3*10^-2;
    w = 5 turns width pair 7 by 5*10^-1; every other pair of the token stays put.  (1, 0)
    goes to (cos, sin) and (0, 1) to (-sin, cos): the counter-clockwise sense."""
    N, d = int(np.prod(_GRID)), sum(_SPLIT)
    cases = [  # (token, first channel of the pair, angle in rad)
        (_token(1, 0, 0), 0, 1.0),
        (_token(1, 0, 0), 8, 0.01),
        (_token(0, 3, 0), 16 + 28, 0.03),
        (_token(0, 0, 5), 72 + 14, 0.5),
    ]
    # the printed decimal values of cos and sin at those angles
    table = {1.0: (0.5403023058681398, 0.8414709848078965),
             0.01: (0.9999500004166653, 0.009999833334166664),
             0.03: (0.9995500337489875, 0.029995500202495664),
             0.5: (0.8775825618903728, 0.479425538604203)}
    for tok, c, ang in cases:
        cs, sn = table[ang]
        for x0, x1, e0, e1 in ((1.0, 0.0, cs, sn), (0.0, 1.0, -sn, cs)):
            X = np.zeros((N, d))
            X[tok, c], X[tok, c + 1] = x0, x1
            Y = oracle.rope3d(X, _GRID, _SPLIT)
            assert abs(Y[tok, c] - e0) < 1e-15 and abs(Y[tok, c + 1] - e1) < 1e-15, (tok, c)
            # channels outside the pair and other tokens are untouched
            Y[tok, c] = Y[tok, c + 1] = 0.0
            assert not Y.any()


def test_rope3d_origin_identity_and_pair_norms():
    rng = np.random.default_rng(71)
    N, d = int(np.prod(_GRID)), sum(_SPLIT)
    X = rng.standard_normal((N, d))
    Y = oracle.rope3d(X, _GRID, _SPLIT)
    np.testing.assert_array_equal(Y[0], X[0])   # token (0, 0, 0): every angle is 0
    nx = X[:, 0::2] ** 2 + X[:, 1::2] ** 2
    ny = Y[:, 0::2] ** 2 + Y[:, 1::2] ** 2
    np.testing.assert_allclose(ny, nx, rtol=1e-13, atol=1e-15)
    assert np.abs(Y - X).max() > 0.5             # it does rotate


def test_rope3d_relative_position_property():
    """RoPE's defining property: the dot product of a rotated query and a rotated key
    depends only on their displacement (dt, dh, dw), not on where the pair sits."""
    rng = np.random.default_rng(72)
    N, d = int(np.prod(_GRID)), sum(_SPLIT)
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    Rq = oracle.rope3d(np.tile(q, (N, 1)), _GRID, _SPLIT)
    Rk = oracle.rope3d(np.tile(k, (N, 1)), _GRID, _SPLIT)
    for (a1, b1), (a2, b2) in [(((0, 0, 0), (1, 2, 3)), ((1, 1, 2), (2, 3, 5))),
                               (((2, 3, 5), (0, 1, 1)), ((2, 2, 4), (0, 0, 0))),
                               (((1, 0, 4), (1, 3, 0)), ((0, 0, 5), (0, 3, 1)))]:
        s1 = Rq[_token(*a1)] @ Rk[_token(*b1)]
        s2 = Rq[_token(*a2)] @ Rk[_token(*b2)]
        assert abs(s1 - s2) < 1e-12 * (np.abs(q) @ np.abs(k))
    # and the plain (unrotated) score is not what it gives off the diagonal
    assert abs(Rq[_token(0, 0, 0)] @ Rk[_token(1, 2, 3)] - q @ k) > 1e-3


@pytest.mark.parametrize("which", ["q", "k"])
def test_rope3d_matches_generator_rotation(which):
    """The generator rotates its own q and k (separate code, same RoFormer reading); the
    oracle applied to the generator's pre-RoPE draws reproduces them in binary64."""
    pre = synth.head_tensor(TINY, 0, 0, which, rope=False, raw=True)
    post = synth.head_tensor(TINY, 0, 0, which, rope=True, raw=True)
    got = oracle.rope3d(pre, (TINY.T, TINY.Hg, TINY.Wg), (TINY.d_t, TINY.d_h, TINY.d_w))
    np.testing.assert_allclose(got, post, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- dense branch
def test_dense_attention_equals_sdpa():
    rng = np.random.default_rng(73)
    N, d = 75, 32
    Q, K, V = (rng.standard_normal((N, d)).astype(np.float32) for _ in range(3))
    O = oracle.dense_attention(Q, K, V)
    np.testing.assert_allclose(O, _sdpa64(Q, K, V, np.ones((N, N), bool)), rtol=1e-12, atol=1e-12)


def test_dense_prefix_schedule_cases():
    """The paper's schedule: the first layer dense at every step; every layer dense for the
    first 20 % of 50 steps (Wan, 10 steps) or 10 % (HunyuanVideo, 5 steps)."""
    for dense_steps in (10, 5):
        for step in range(50):
            for layer in range(4):
                want = layer == 0 or step < dense_steps
                assert oracle.layer_is_dense(layer, step, 1, dense_steps) == want


# ----------------------------------------------------------------------------- full-d keys
def test_full_d_key_proxy_is_the_cluster_level_dot_product():
    """Full-d key clustering read as a one-subspace code with split (d, 0, 0): the Eq. 6
    proxy reduces to q_c . mu_{z_j} / sqrt d (numpy matmul), the empty subspaces adding
    nothing; with every key its own centroid the selection ranks the exact logits."""
    rng = np.random.default_rng(81)
    N, d, Cq, Cm = 70, 24, 3, 9
    K = rng.standard_normal((N, d)).astype(np.float32)
    qcent = rng.standard_normal((Cq, d))
    kc = oracle.cluster_keys(K, (8, 8, 8), Cm, 3, init_idx3=np.tile(np.arange(Cm, dtype=np.int32), (3, 1)),
                             full=True)
    assert not kc["codes"][1:].any()
    ref = oracle.kmeans(K, 0, d, Cm, 3, init_idx=np.arange(Cm, dtype=np.int32))
    np.testing.assert_array_equal(kc["codes"][0], ref["assign"])
    sel = oracle.select(qcent, np.full(Cq, N // Cq, np.int32), kc["centroids"], kc["codes"], (d, 0, 0), 0.9, 0.1,
                        want_scores=True)
    want = (qcent @ kc["centroids"].T)[:, kc["codes"][0]] / math.sqrt(d)
    np.testing.assert_allclose(sel["scores"], want, rtol=1e-12, atol=1e-12)
    # lossless: Cm = N, centroid j = key j
    codes = np.zeros((3, N), np.uint16)
    codes[0] = np.arange(N)
    sel = oracle.select(qcent, np.full(Cq, 10, np.int32), K.astype(np.float64), codes, (d, 0, 0), 0.9, 0.1,
                        want_scores=True)
    np.testing.assert_allclose(sel["scores"], qcent @ K.astype(np.float64).T / math.sqrt(d), rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- rank correlation
def test_rank_correlation_pins():
    """Spearman's rho: scipy's spearmanr (average ranks for ties), +-1 under monotone maps,
    a hand-worked case with ties, and invariance under a common permutation of the keys."""
    import scipy.stats
    rng = np.random.default_rng(91)
    N, d = 200, 16
    q = rng.standard_normal(d).astype(np.float32)
    K = rng.standard_normal((N, d)).astype(np.float32)
    logit = K.astype(np.float64) @ q.astype(np.float64)
    proxy = np.round(logit + 0.8 * rng.standard_normal(N), 1)          # with many ties
    rho = oracle.rank_correlation(q, K, proxy)
    assert abs(rho - scipy.stats.spearmanr(logit, proxy).statistic) < 1e-12
    assert abs(oracle.rank_correlation(q, K, np.exp(logit)) - 1.0) < 1e-12
    assert abs(oracle.rank_correlation(q, K, -logit ** 3) + 1.0) < 1e-12
    perm = rng.permutation(N)
    assert abs(oracle.rank_correlation(q, K[perm], proxy[perm]) - rho) < 1e-12
    # hand-worked: ranks (1, 2.5, 2.5, 4) and (1, 3, 2, 4), centred (-1.5, 0, 0, 1.5) and
    # (-1.5, 0.5, -0.5, 1.5): rho = 4.5 / sqrt(4.5 * 5)
    np.testing.assert_array_equal(oracle.average_ranks([1.0, 2.0, 2.0, 3.0]), [1.0, 2.5, 2.5, 4.0])
    q1 = np.ones(1, np.float32)
    K1 = np.array([[1.0], [2.0], [2.0], [3.0]], np.float32)
    assert abs(oracle.rank_correlation(q1, K1, np.array([1.0, 3.0, 2.0, 4.0])) - 4.5 / math.sqrt(22.5)) < 1e-15


def test_equal_scores_rank_by_ascending_index():
    """The ranking is (proxy descending, key index ascending): with every key on the same
    code triple all proxies are equal, so S_c is exactly keys 0 .. r_c - 1; with two code
    groups, the higher-scoring group comes first and each group is cut in index order."""
    N, Cq, Cm, d = 300, 3, 2, 16
    rng = np.random.default_rng(21)
    qcent = rng.standard_normal((Cq, d))
    kcent = rng.standard_normal((Cm, d))
    codes = np.zeros((3, N), np.uint16)
    sel = oracle.select(qcent, np.full(Cq, 5, np.int32), kcent, codes, (4, 6, 6), 0.5, 0.0)
    bits = np.unpackbits(sel["mask"].view(np.uint8), bitorder="little").reshape(Cq, -1)[:, :N]
    for c in range(Cq):
        r = int(sel["r"][c])
        assert np.all(bits[c, :r] == 1) and np.all(bits[c, r:] == 0), c
    # two groups of keys, interleaved: even keys on centroid 0, odd keys on centroid 1
    codes2 = np.zeros((3, N), np.uint16)
    codes2[:, 1::2] = 1
    sel2 = oracle.select(qcent, np.full(Cq, 5, np.int32), kcent, codes2, (4, 6, 6), 0.5, 0.0,
                         want_scores=True)
    bits2 = np.unpackbits(sel2["mask"].view(np.uint8), bitorder="little").reshape(Cq, -1)[:, :N]
    for c in range(Cq):
        s = sel2["scores"][c]
        assert s[0] != s[1]
        hi = 0 if s[0] > s[1] else 1          # the group whose proxy is larger
        order = np.concatenate([np.arange(hi, N, 2), np.arange(1 - hi, N, 2)])
        r = int(sel2["r"][c])
        expect = np.zeros(N, np.uint8)
        expect[order[:r]] = 1
        assert np.array_equal(bits2[c], expect), c
