"""fp64 CPU oracle of the SCOPE per-layer hot path -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this package.  It shares no code with the CUDA library; both sides only share
the seeded input generator.  Each function works on one (batch, head) slice and
follows the SCOPE equations as cited in ``scope_oracle.c``.

Parity status of each function (what pins it, in tests/test_oracle_pins.py):
  kmeans     -- pinned: scipy.cluster.vq.kmeans2 (same Lloyd reading), brute-force
                nearest-centroid, member means, non-increasing objective.
  select     -- pinned: Eq. 27 closed form (numpy dot with the product-code key),
                rho=1 keeps everything, uniform logits give ceil(rho*N), rho->0 gives
                k_fix, k_head against exact rational arithmetic, Eq. 10 invariants,
                lossless codebook.
  attention  -- pinned: torch scaled_dot_product_attention (float64, CPU) with the
                selection as a boolean mask; rho=1 equals dense attention.
  rope3d     -- pinned: closed-form angles (base^(-2i/d_a) at exact powers of ten) on unit
                vectors per axis, identity at the origin token, pair norms, the relative-
                position property, and the input generator's own post-RoPE tensors.
  dense_attention -- pinned: torch scaled_dot_product_attention (float64, CPU).
  rank_correlation -- pinned: scipy.stats.spearmanr, +-1 for monotone maps, a hand-worked
                case with ties, invariance under a common permutation of the keys.
  layer      -- the schedule's choice between dense_attention and forward_head, after
                rope3d; pinned through its parts.
"""
from __future__ import annotations

import ctypes
import os

import math

import numpy as np

from .build import build as _build

_lib = None

_f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(np.int64, flags="C_CONTIGUOUS")
_u16p = np.ctypeslib.ndpointer(np.uint16, flags="C_CONTIGUOUS")
_u32p = np.ctypeslib.ndpointer(np.uint32, flags="C_CONTIGUOUS")
_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int
_dbl = ctypes.c_double


def lib():
    global _lib
    if _lib is None:
        path = _build()
        L = ctypes.CDLL(path)
        L.oracle_num_threads.restype = _int
        L.oracle_kfix.restype = _i64
        L.oracle_kfix.argtypes = [_dbl, _i64]
        L.oracle_kmeans.restype = _int
        L.oracle_kmeans.argtypes = [_f32p, _i64, _i64, _int, _int, _int, _vp, _vp, _int,
                                    _f64p, _u16p, _i32p, _vp, _vp, _vp]
        L.oracle_select.restype = _int
        L.oracle_select.argtypes = [_f64p, _i32p, _f64p, _u16p, _i64, _int, _int, _int, _int,
                                    _int, _int, _dbl, _dbl, _vp, _i32p, _i32p, _i32p, _i32p,
                                    _u32p, _vp, _int]
        L.oracle_attention.restype = _int
        L.oracle_attention.argtypes = [_f32p, _f32p, _f32p, _i64, _int, _u16p, _u32p, _int,
                                       _vp, _i64, _f64p]
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return lib().oracle_num_threads()


def kfix(alpha: float, N: int) -> int:
    return int(lib().oracle_kfix(float(alpha), int(N)))


def kmeans(X, ch0, dm, C, iters, init_idx=None, init_cent=None, logs=False):
    """Lloyd k-means on channels [ch0, ch0+dm) of the rows of X (float32 [N, ld])."""
    X = np.ascontiguousarray(X, np.float32)
    N, ld = X.shape
    if init_idx is not None:
        init_idx = np.ascontiguousarray(init_idx, np.int32)
    if init_cent is not None:
        init_cent = np.ascontiguousarray(init_cent, np.float64)
    cent = np.empty((C, dm), np.float64)
    assign = np.empty(N, np.uint16)
    sizes = np.empty(C, np.int32)
    margin = np.empty(N, np.float64) if logs else None
    oa = np.empty(iters, np.float64) if logs else None
    ou = np.empty(iters, np.float64) if logs else None
    rc = lib().oracle_kmeans(X, N, ld, ch0, dm, C, _ptr(init_idx), _ptr(init_cent), iters,
                             cent, assign, sizes, _ptr(margin), _ptr(oa), _ptr(ou))
    if rc:
        raise ValueError(f"oracle_kmeans failed ({rc})")
    out = {"centroids": cent, "assign": assign, "sizes": sizes}
    if logs:
        out.update(margin=margin, obj_assign=oa, obj_update=ou)
    return out


def select(qcent, qsizes, kcent, codes, d_split, rho, alpha, want_scores=False, khead_off=False):
    """Eqs. 6-10 for one head.  qcent [Cq, d], kcent [Cm, d], codes [3, N] uint16.
    khead_off: the review page's ablation (online k_head disabled): r_c = b_c."""
    qcent = np.ascontiguousarray(qcent, np.float64)
    kcent = np.ascontiguousarray(kcent, np.float64)
    qsizes = np.ascontiguousarray(qsizes, np.int32)
    codes = np.ascontiguousarray(codes, np.uint16)
    Cq, d = qcent.shape
    Cm = kcent.shape[0]
    N = codes.shape[1]
    dt, dh, dw = d_split
    nw = (N + 31) // 32
    scores = np.empty((Cq, N), np.float64) if want_scores else None
    p = np.empty(Cq, np.int32)
    b = np.empty(Cq, np.int32)
    r = np.empty(Cq, np.int32)
    kh = np.empty(1, np.int32)
    mask = np.empty((Cq, nw), np.uint32)
    margin = np.empty(Cq, np.float64)
    rc = lib().oracle_select(qcent, qsizes, kcent, codes, N, d, dt, dh, dw, Cq, Cm, float(rho),
                             float(alpha), _ptr(scores), p, b, kh, r, mask, _ptr(margin),
                             1 if khead_off else 0)
    if rc:
        raise ValueError(f"oracle_select failed ({rc})")
    out = {"p": p, "b": b, "k_head": int(kh[0]), "r": r, "mask": mask, "topp_margin": margin}
    if want_scores:
        out["scores"] = scores
    return out


def attention(Q, K, V, qassign, mask, rows=None):
    """Sparse attention of the listed query rows (all when None); float64 [nrows, d]."""
    Q = np.ascontiguousarray(Q, np.float32)
    K = np.ascontiguousarray(K, np.float32)
    V = np.ascontiguousarray(V, np.float32)
    qassign = np.ascontiguousarray(qassign, np.uint16)
    mask = np.ascontiguousarray(mask, np.uint32)
    N, d = Q.shape
    Cq = mask.shape[0]
    if rows is not None:
        rows = np.ascontiguousarray(rows, np.int64)
    nrows = N if rows is None else rows.shape[0]
    O = np.empty((nrows, d), np.float64)
    rc = lib().oracle_attention(Q, K, V, N, d, qassign, mask, Cq, _ptr(rows), nrows, O)
    if rc:
        raise ValueError(f"oracle_attention failed ({rc})")
    return O


def cluster_keys(K, d_split, Cm, iters, init_idx3=None, init_cent=None, logs=False, full=False):
    """The three subspace k-means of one head's keys.

    Returns centroids [Cm, d] (subspace m's centroid in m's channel range), codes
    [3, N] uint16 and per-subspace logs.  init_idx3 is [3, Cm]; init_cent is [Cm, d].
    full=True: the review page's ablation (full-dimensional cluster scoring): one k-means
    over all d channels (initial indices init_idx3[0]); codes row 0 holds the clusters and
    rows 1, 2 are zero, to be read with the split (d, 0, 0) (see key_split).
    """
    N, d = K.shape
    if full:
        res = kmeans(K, 0, d, Cm, iters, init_idx=None if init_idx3 is None else init_idx3[0],
                     init_cent=init_cent, logs=logs)
        codes = np.zeros((3, N), np.uint16)
        codes[0] = res["assign"]
        sizes = np.zeros((3, Cm), np.int32)
        sizes[0] = res["sizes"]
        return {"centroids": res["centroids"], "codes": codes, "sizes": sizes, "per_subspace": [res]}
    bounds = [0, d_split[0], d_split[0] + d_split[1], d]
    cent = np.zeros((Cm, d), np.float64)
    codes = np.empty((3, N), np.uint16)
    sizes = np.empty((3, Cm), np.int32)
    extra = []
    for m in range(3):
        ch0, dm = bounds[m], bounds[m + 1] - bounds[m]
        res = kmeans(K, ch0, dm, Cm, iters,
                     init_idx=None if init_idx3 is None else init_idx3[m],
                     init_cent=None if init_cent is None else init_cent[:, ch0:ch0 + dm],
                     logs=logs)
        cent[:, ch0:ch0 + dm] = res["centroids"]
        codes[m] = res["assign"]
        sizes[m] = res["sizes"]
        extra.append(res)
    return {"centroids": cent, "codes": codes, "sizes": sizes, "per_subspace": extra}


def key_split(wl, full=False):
    """Channel split the proxy of Eq. 6 reads the key codes with: the three RoPE ranges,
    or, for full-d key clustering, one subspace of all d channels and two empty ones."""
    return (wl.d, 0, 0) if full else (wl.d_t, wl.d_h, wl.d_w)


def forward_head(q, k, v, wl, q_init, k_init, rows=None, logs=False, rho=None, khead_off=False,
                 key_full=False):
    """The whole hot path for one head: clustering, selection, sparse attention."""
    rho = wl.rho if rho is None else rho
    qc = kmeans(q, 0, wl.d, wl.Cq, wl.iters, init_idx=q_init, logs=logs)
    kc = cluster_keys(k, (wl.d_t, wl.d_h, wl.d_w), wl.Cm, wl.iters, init_idx3=k_init, logs=logs,
                      full=key_full)
    sel = select(qc["centroids"], qc["sizes"], kc["centroids"], kc["codes"],
                 key_split(wl, key_full), rho, wl.alpha, khead_off=khead_off)
    O = attention(q, k, v, qc["assign"], sel["mask"], rows=rows)
    return {"q": qc, "k": kc, "sel": sel, "O": O}


def selection_recall(q, K, proxy, selected, frac):
    """Proxy-ranking fidelity of one query (review page, falsifier and skeptic's concrete
    test), from the definition: the query's exact logits l_j = q . k_j in binary64 with the
    channels summed in order, T = its ceil(frac N) keys of largest logit (ties to the lower
    index), P = the ceil(frac N) keys of largest proxy logit (ties to the lower index).
    q [d], K [N, d], proxy [N] (Eq. 6 logits of the query's cluster), selected [N] bool.
    Returns (|T n S| / |T|, |T n P| / |T|)."""
    q = np.asarray(q, np.float64)
    K = np.asarray(K, np.float64)
    N = K.shape[0]
    logit = np.zeros(N, np.float64)
    for e in range(q.shape[0]):
        logit = logit + q[e] * K[:, e]
    k = min(max(int(math.ceil(frac * N)), 1), N)
    idx = np.arange(N)
    top_true = np.lexsort((idx, -logit))[:k]
    top_proxy = np.lexsort((idx, -np.asarray(proxy, np.float64)))[:k]
    sel = np.asarray(selected, bool)
    return float(sel[top_true].sum()) / k, float(np.isin(top_true, top_proxy).sum()) / k


def rope3d(X, grid, d_split, base=10000.0, rows=None):
    """3D rotary position embedding of one head's [N, d] tensor, binary64.

    SCOPE clusters post-RoPE queries and keys whose channels fall into the temporal,
    height and width ranges of 3D RoPE (SCOPE abstract; the rotation is RoFormer's, the
    page's reference [31]).  Token n = t*Hg*Wg + h*Wg + w.  In channel range a (start c_a,
    width d_a, position p_a in (t, h, w)), pair i = channels (c_a + 2i, c_a + 2i + 1) turns
    counter-clockwise by phi = p_a * base**(-2i/d_a):
        y0 = x0 cos(phi) - x1 sin(phi),   y1 = x0 sin(phi) + x1 cos(phi),
    each product rounded to binary64, then the sum (no fused multiply-add).
    grid = (T, Hg, Wg); d_split = (d_t, d_h, d_w), each even.  rows: the token index of
    each row of X (all tokens in order when None)."""
    X = np.asarray(X, np.float64)
    T, Hg, Wg = grid
    N, d = X.shape
    n = np.arange(N) if rows is None else np.asarray(rows, np.int64)
    positions = (n // (Hg * Wg), (n // Wg) % Hg, n % Wg)
    Y = X.copy()
    c_a = 0
    for d_a, p_a in zip(d_split, positions):
        for i in range(d_a // 2):
            theta = base ** ((-2.0 * i) / d_a)
            phi = p_a.astype(np.float64) * theta
            cs, sn = np.cos(phi), np.sin(phi)
            x0, x1 = X[:, c_a + 2 * i], X[:, c_a + 2 * i + 1]
            Y[:, c_a + 2 * i] = x0 * cs - x1 * sn
            Y[:, c_a + 2 * i + 1] = x0 * sn + x1 * cs
        c_a += d_a
    return Y


def dense_attention(Q, K, V, rows=None):
    """Softmax attention of the listed query rows over all N keys: the sparse attention
    with one query cluster that keeps every key.  float64 [nrows, d]."""
    N = np.asarray(Q).shape[0]
    nw = (N + 31) // 32
    mask = np.zeros((1, nw), np.uint32)
    for j in range(N):
        mask[0, j // 32] |= np.uint32(1 << (j % 32))
    return attention(Q, K, V, np.zeros(N, np.uint16), mask, rows=rows)


def layer_is_dense(layer, step, dense_layers, dense_steps):
    """Dense-prefix schedule (review page, major_comments: "§4, Implementation details"):
    the first dense_layers layers at every step, and every layer during the first
    dense_steps denoising steps, run dense attention."""
    return layer < dense_layers or step < dense_steps


def layer(q, k, v, wl, q_init, k_init, dense, rope_base=None, rows=None, round_rope=None):
    """One layer: [3D RoPE of q and k, then round_rope (the rounding to the path's element
    type)], then dense attention or the SCOPE path.  Returns the forward_head dict (with
    "O", plus "q", "k" post-RoPE when rope_base is given)."""
    extra = {}
    if rope_base is not None:
        grid, split = (wl.T, wl.Hg, wl.Wg), (wl.d_t, wl.d_h, wl.d_w)
        q = rope3d(q, grid, split, rope_base)
        k = rope3d(k, grid, split, rope_base)
        if round_rope is not None:
            q, k = round_rope(q), round_rope(k)
        extra = {"q_rot": q, "k_rot": k}
    if dense:
        out = {"O": dense_attention(q, k, v, rows=rows)}
    else:
        out = forward_head(q, k, v, wl, q_init, k_init, rows=rows)
    out.update(extra)
    return out


def average_ranks(v):
    """1-based ranks of v in ascending order; tied values share the mean of their ranks."""
    v = np.asarray(v, np.float64)
    order = np.argsort(v, kind="stable")
    sv = v[order]
    ranks = np.empty(v.shape[0], np.float64)
    lo = 0
    n = v.shape[0]
    while lo < n:
        hi = lo + 1
        while hi < n and sv[hi] == sv[lo]:
            hi += 1
        ranks[order[lo:hi]] = 0.5 * (lo + 1 + hi)
        lo = hi
    return ranks


def rank_correlation(q, K, proxy):
    """Spearman's rho of one query's exact logits (binary64, channels summed in order) with
    the Eq. 6 proxy logits of its cluster (review page, the skeptic's concrete test): the
    Pearson correlation of the two vectors of average ranks."""
    q = np.asarray(q, np.float64)
    K = np.asarray(K, np.float64)
    logit = np.zeros(K.shape[0], np.float64)
    for e in range(q.shape[0]):
        logit = logit + q[e] * K[:, e]
    rx = average_ranks(logit) - 0.5 * (K.shape[0] + 1)
    ry = average_ranks(proxy) - 0.5 * (K.shape[0] + 1)
    return float((rx @ ry) / math.sqrt((rx @ rx) * (ry @ ry)))
