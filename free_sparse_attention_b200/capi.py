"""Thin Python binding of libscope.so (the C ABI in include/scope.h).

Argument marshalling only: every step of the SCOPE path runs in the library's CUDA
kernels.  PyTorch provides device memory and the current stream.  If the library is
missing or cannot be loaded, every call raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

from .workloads import Workload

HERE = os.path.dirname(os.path.abspath(__file__))
# SCOPE_LIB_PATH selects another build of the library (the debug build's tests use it)
LIB_PATH = os.environ.get("SCOPE_LIB_PATH") or os.path.join(HERE, "libscope.so")

SCOPE_F32, SCOPE_BF16 = 0, 1
STATUS = {0: "SCOPE_OK", 1: "SCOPE_ERR_INVALID_ARGUMENT", 2: "SCOPE_ERR_UNSUPPORTED",
          3: "SCOPE_ERR_WORKSPACE_TOO_SMALL", 4: "SCOPE_ERR_CUDA", 5: "SCOPE_ERR_DEVICE_CHECK",
          6: "SCOPE_ERR_TIMEOUT"}
DEV_BAD_INIT_INDEX, DEV_SELECT_TIE, DEV_BAD_ASSIGN = 0x1, 0x2, 0x4

EXPORTS = ("scope_workspace_bytes", "scope_cluster_queries", "scope_cluster_keys",
           "scope_build_lut_and_select", "scope_sparse_attention", "scope_forward",
           "scope_status_string", "scope_get_device_status", "scope_get_selection_stats",
           "scope_build_lut_and_select_noalloc",
           "scope_selection_recall", "scope_permute_channels", "scope_dense_attention",
           "scope_rope3d", "scope_layer_is_dense", "scope_attention_layer",
           "scope_rank_correlation_scratch_bytes", "scope_rank_correlation", "scope_check_wait_timeout",
           "scope_tc_accumulation_probe")


class ScopeError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} returned {STATUS.get(code, code)}")
        self.code = code


SCOPE_KHEAD_ONLINE = 0   # Eqs. 9-10: clusters topped up to k_head
SCOPE_KHEAD_OFF = 1      # ablation: r_c = b_c
SCOPE_KEYS_SUBSPACES = 0  # the method: T / H / W key subspaces
SCOPE_KEYS_FULL = 1       # ablation: one full-d key clustering (cluster-level proxy)


class Params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int),
                ("Hg", ctypes.c_int), ("Wg", ctypes.c_int), ("d", ctypes.c_int),
                ("d_t", ctypes.c_int), ("d_h", ctypes.c_int), ("d_w", ctypes.c_int),
                ("Cq", ctypes.c_int), ("Cm", ctypes.c_int), ("iters", ctypes.c_int),
                ("rho", ctypes.c_double), ("alpha", ctypes.c_double), ("dtype", ctypes.c_int),
                ("khead_mode", ctypes.c_int), ("key_clustering", ctypes.c_int)]

    @classmethod
    def from_workload(cls, w: Workload, **over) -> "Params":
        kw = dict(B=w.B, H=w.H, T=w.T, Hg=w.Hg, Wg=w.Wg, d=w.d, d_t=w.d_t, d_h=w.d_h,
                  d_w=w.d_w, Cq=w.Cq, Cm=w.Cm, iters=w.iters, rho=w.rho, alpha=w.alpha,
                  dtype=SCOPE_BF16 if w.dtype == "bf16" else SCOPE_F32)
        kw.update(over)
        return cls(**kw)

    @property
    def N(self) -> int:
        return self.T * self.Hg * self.Wg

    @property
    def nw(self) -> int:
        return (self.N + 31) // 32


class Schedule(ctypes.Structure):
    """scope_layer_schedule: the layer's place in the sampling loop and the dense-prefix
    schedule (dense when layer < dense_layers or step < dense_steps)."""
    _fields_ = [("layer", ctypes.c_int), ("step", ctypes.c_int), ("dense_layers", ctypes.c_int),
                ("dense_steps", ctypes.c_int), ("rope", ctypes.c_int), ("rope_base", ctypes.c_double)]


class Intermediates(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("q_centroids", "q_assign", "q_sizes", "k_centroids", "k_codes", "topp_counts",
                 "base_counts", "k_head", "final_counts", "sel_mask")] + \
               [("stage_events", ctypes.c_void_p * 5)]


_lib = None


def lib() -> ctypes.CDLL:
    """Loads libscope.so (raises if it is missing: there is no CPU fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with free_sparse_attention_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        P, vp, sz, i = ctypes.POINTER(Params), ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        L.scope_workspace_bytes.restype = sz
        L.scope_workspace_bytes.argtypes = [P]
        L.scope_cluster_queries.restype = i
        L.scope_cluster_queries.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.scope_cluster_keys.restype = i
        L.scope_cluster_keys.argtypes = [P, vp, vp, vp, vp, vp, vp, sz, vp]
        L.scope_build_lut_and_select.restype = i
        L.scope_build_lut_and_select.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.scope_sparse_attention.restype = i
        L.scope_sparse_attention.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.scope_forward.restype = i
        L.scope_forward.argtypes = [P, vp, vp, vp, vp, vp, vp, ctypes.POINTER(Intermediates),
                                    vp, sz, vp]
        L.scope_build_lut_and_select_noalloc.restype = i
        L.scope_build_lut_and_select_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.scope_selection_recall.restype = i
        L.scope_selection_recall.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, i, ctypes.c_double,
                                             vp, vp, vp, sz, vp]
        L.scope_rank_correlation_scratch_bytes.restype = sz
        L.scope_rank_correlation_scratch_bytes.argtypes = [P, i]
        L.scope_rank_correlation.restype = i
        L.scope_rank_correlation.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, i, vp, vp, sz, vp]
        L.scope_permute_channels.restype = i
        L.scope_permute_channels.argtypes = [P, vp, vp, vp, vp]
        L.scope_dense_attention.restype = i
        L.scope_dense_attention.argtypes = [P, vp, vp, vp, vp, vp, sz, vp]
        L.scope_rope3d.restype = i
        L.scope_rope3d.argtypes = [P, ctypes.c_double, vp, vp, vp, vp, vp]
        S = ctypes.POINTER(Schedule)
        L.scope_layer_is_dense.restype = i
        L.scope_layer_is_dense.argtypes = [S]
        L.scope_attention_layer.restype = i
        L.scope_attention_layer.argtypes = [P, S, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.scope_status_string.restype = ctypes.c_char_p
        L.scope_status_string.argtypes = [i]
        L.scope_get_device_status.restype = i
        L.scope_get_device_status.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_int32)]
        L.scope_get_selection_stats.restype = i
        L.scope_get_selection_stats.argtypes = [ctypes.POINTER(Params), vp, vp, ctypes.POINTER(ctypes.c_int32)]
        L.scope_check_wait_timeout.restype = i
        L.scope_check_wait_timeout.argtypes = [P, ctypes.c_uint64, vp, sz, vp]
        L.scope_tc_accumulation_probe.restype = i
        L.scope_tc_accumulation_probe.argtypes = [vp, vp, i, i, vp, vp]
        _lib = L
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn, code):
    if code != 0:
        raise ScopeError(fn, code)


def torch_dtype(p: Params):
    return torch.bfloat16 if p.dtype == SCOPE_BF16 else torch.float32


def workspace_bytes(p: Params) -> int:
    return int(lib().scope_workspace_bytes(ctypes.byref(p)))


def alloc_workspace(p: Params, device="cuda") -> torch.Tensor:
    n = workspace_bytes(p)
    if n == 0:
        raise ScopeError("scope_workspace_bytes", 1)
    return torch.empty(n, dtype=torch.uint8, device=device)


def cluster_queries(p, Q, init_idx=None, init_cent=None, ws=None, stream=None):
    dev = Q.device
    ws = alloc_workspace(p, dev) if ws is None else ws
    qc = torch.empty((p.B, p.H, p.Cq, p.d), dtype=torch.float64, device=dev)
    qa = torch.empty((p.B, p.H, p.N), dtype=torch.uint16, device=dev)
    qs = torch.empty((p.B, p.H, p.Cq), dtype=torch.int32, device=dev)
    _check("scope_cluster_queries", lib().scope_cluster_queries(
        ctypes.byref(p), _ptr(Q), _ptr(init_idx), _ptr(init_cent), _ptr(qc), _ptr(qa), _ptr(qs),
        _ptr(ws), ws.numel(), _stream(stream)))
    return qc, qa, qs


def cluster_keys(p, K, init_idx=None, init_cent=None, ws=None, stream=None):
    dev = K.device
    ws = alloc_workspace(p, dev) if ws is None else ws
    kc = torch.empty((p.B, p.H, p.Cm, p.d), dtype=torch.float64, device=dev)
    kk = torch.empty((p.B, p.H, 3, p.N), dtype=torch.uint16, device=dev)
    _check("scope_cluster_keys", lib().scope_cluster_keys(
        ctypes.byref(p), _ptr(K), _ptr(init_idx), _ptr(init_cent), _ptr(kc), _ptr(kk), _ptr(ws),
        ws.numel(), _stream(stream)))
    return kc, kk


def build_lut_and_select(p, q_centroids, q_sizes, k_centroids, k_codes, ws=None, stream=None):
    dev = q_centroids.device
    ws = alloc_workspace(p, dev) if ws is None else ws
    shp = (p.B, p.H, p.Cq)
    tp = torch.empty(shp, dtype=torch.int32, device=dev)
    bc = torch.empty(shp, dtype=torch.int32, device=dev)
    fc = torch.empty(shp, dtype=torch.int32, device=dev)
    kh = torch.empty((p.B, p.H), dtype=torch.int32, device=dev)
    mk = torch.empty((p.B, p.H, p.Cq, p.nw), dtype=torch.int32, device=dev)
    _check("scope_build_lut_and_select", lib().scope_build_lut_and_select(
        ctypes.byref(p), _ptr(q_centroids), _ptr(q_sizes), _ptr(k_centroids), _ptr(k_codes),
        _ptr(tp), _ptr(bc), _ptr(kh), _ptr(fc), _ptr(mk), _ptr(ws), ws.numel(), _stream(stream)))
    return {"topp_counts": tp, "base_counts": bc, "k_head": kh, "final_counts": fc, "sel_mask": mk}


def build_lut_and_select_noalloc(p, q_centroids, q_sizes, k_centroids, k_codes, stream=None):
    """scope_build_lut_and_select without a workspace: for callers that cannot allocate
    device memory at run time.  The library keeps the scratch in a fixed device array
    shared by all calls, so calls must not overlap on the GPU (the output tensors below
    are the caller's; a caller that cannot allocate passes its own preallocated ones
    through the C ABI directly)."""
    dev = q_centroids.device
    shp = (p.B, p.H, p.Cq)
    tp = torch.empty(shp, dtype=torch.int32, device=dev)
    bc = torch.empty(shp, dtype=torch.int32, device=dev)
    fc = torch.empty(shp, dtype=torch.int32, device=dev)
    kh = torch.empty((p.B, p.H), dtype=torch.int32, device=dev)
    mk = torch.empty((p.B, p.H, p.Cq, p.nw), dtype=torch.int32, device=dev)
    _check("scope_build_lut_and_select_noalloc", lib().scope_build_lut_and_select_noalloc(
        ctypes.byref(p), _ptr(q_centroids), _ptr(q_sizes), _ptr(k_centroids), _ptr(k_codes),
        _ptr(tp), _ptr(bc), _ptr(kh), _ptr(fc), _ptr(mk), _stream(stream)))
    return {"topp_counts": tp, "base_counts": bc, "k_head": kh, "final_counts": fc, "sel_mask": mk}


def sparse_attention(p, Q, K, V, q_assign, sel_mask, final_counts, ws=None, out=None, stream=None):
    dev = Q.device
    ws = alloc_workspace(p, dev) if ws is None else ws
    O = torch.empty_like(Q) if out is None else out
    _check("scope_sparse_attention", lib().scope_sparse_attention(
        ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(q_assign), _ptr(sel_mask),
        _ptr(final_counts), _ptr(O), _ptr(ws), ws.numel(), _stream(stream)))
    return O


def forward(p, Q, K, V, q_init_idx, k_init_idx, ws=None, out=None, intermediates=False,
            stage_events=None, stream=None):
    """The whole layer.  With intermediates=True also returns every stage's outputs.

    stage_events: optional list of 5 recorded torch.cuda.Event (timing enabled) that
    the library records at the stage boundaries (see scope_intermediates)."""
    dev = Q.device
    ws = alloc_workspace(p, dev) if ws is None else ws
    O = torch.empty_like(Q) if out is None else out
    inter = None
    tensors = {}
    if stage_events is not None:
        inter = Intermediates()
        for k, ev in enumerate(stage_events):
            inter.stage_events[k] = ev.cuda_event
    if intermediates:
        shp = (p.B, p.H)
        tensors = {
            "q_centroids": torch.empty(shp + (p.Cq, p.d), dtype=torch.float64, device=dev),
            "q_assign": torch.empty(shp + (p.N,), dtype=torch.uint16, device=dev),
            "q_sizes": torch.empty(shp + (p.Cq,), dtype=torch.int32, device=dev),
            "k_centroids": torch.empty(shp + (p.Cm, p.d), dtype=torch.float64, device=dev),
            "k_codes": torch.empty(shp + (3, p.N), dtype=torch.uint16, device=dev),
            "topp_counts": torch.empty(shp + (p.Cq,), dtype=torch.int32, device=dev),
            "base_counts": torch.empty(shp + (p.Cq,), dtype=torch.int32, device=dev),
            "k_head": torch.empty(shp, dtype=torch.int32, device=dev),
            "final_counts": torch.empty(shp + (p.Cq,), dtype=torch.int32, device=dev),
            "sel_mask": torch.empty(shp + (p.Cq, p.nw), dtype=torch.int32, device=dev),
        }
        inter = Intermediates() if inter is None else inter
        for k, v in tensors.items():
            setattr(inter, k, v.data_ptr())
    _check("scope_forward", lib().scope_forward(
        ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(q_init_idx), _ptr(k_init_idx), _ptr(O),
        ctypes.byref(inter) if inter is not None else None, _ptr(ws), ws.numel(), _stream(stream)))
    if intermediates:
        return O, tensors
    return O


def selection_recall(p, Q, K, q_assign, q_centroids, k_centroids, k_codes, sel_mask, samples, frac,
                     scratch=None, stream=None):
    """Proxy-ranking fidelity for the sampled queries (int64 indices (b*H + h)*N + i):
    returns (recall_sel, recall_proxy), float64 [n_samples] each."""
    dev = Q.device
    n = samples.numel()
    rs = torch.empty(n, dtype=torch.float64, device=dev)
    rp = torch.empty(n, dtype=torch.float64, device=dev)
    if scratch is None:
        scratch = torch.empty(16 * p.N * min(max(n, 1), 148), dtype=torch.uint8, device=dev)
    _check("scope_selection_recall", lib().scope_selection_recall(
        ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(q_assign), _ptr(q_centroids), _ptr(k_centroids),
        _ptr(k_codes), _ptr(sel_mask), _ptr(samples), n, float(frac), _ptr(rs), _ptr(rp),
        _ptr(scratch), scratch.numel(), _stream(stream)))
    return rs, rp


def rank_correlation(p, Q, K, q_assign, q_centroids, k_centroids, k_codes, samples, stream=None):
    """Spearman's rho between each sampled query's exact logits and its cluster's Eq. 6
    proxy logits over all keys (int64 samples (b*H + h)*N + i): float64 [n_samples]."""
    n = samples.numel()
    out = torch.empty(n, dtype=torch.float64, device=Q.device)
    if n == 0:
        return out
    need = int(lib().scope_rank_correlation_scratch_bytes(ctypes.byref(p), n))
    if need == 0:
        raise ScopeError("scope_rank_correlation_scratch_bytes", 2)
    scratch = torch.empty(need, dtype=torch.uint8, device=Q.device)
    _check("scope_rank_correlation", lib().scope_rank_correlation(
        ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(q_assign), _ptr(q_centroids), _ptr(k_centroids), _ptr(k_codes),
        _ptr(samples), n, _ptr(out), _ptr(scratch), scratch.numel(), _stream(stream)))
    return out


def permute_channels(p, X, perm, out=None, stream=None):
    """Y[..., e] = X[..., perm[e]] (perm: int32 [d] on the device)."""
    Y = torch.empty_like(X) if out is None else out
    _check("scope_permute_channels", lib().scope_permute_channels(
        ctypes.byref(p), _ptr(X), _ptr(perm), _ptr(Y), _stream(stream)))
    return Y


def dense_attention(p, Q, K, V, ws=None, out=None, stream=None):
    """Softmax attention of every query over all N keys (the schedule's dense branch)."""
    ws = alloc_workspace(p, Q.device) if ws is None else ws
    O = torch.empty_like(Q) if out is None else out
    _check("scope_dense_attention", lib().scope_dense_attention(
        ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(ws), ws.numel(), _stream(stream)))
    return O


def rope3d(p, Q, K=None, base=10000.0, out_q=None, out_k=None, stream=None):
    """3D RoPE of pre-RoPE Q (and K); out_q / out_k may be Q / K (in place).
    Returns (Qr, Kr) (Kr is None when K is None)."""
    Qr = torch.empty_like(Q) if out_q is None else out_q
    Kr = None if K is None else (torch.empty_like(K) if out_k is None else out_k)
    _check("scope_rope3d", lib().scope_rope3d(
        ctypes.byref(p), float(base), _ptr(Q), _ptr(K), _ptr(Qr), _ptr(Kr), _stream(stream)))
    return Qr, Kr


def layer_is_dense(sched: Schedule) -> bool:
    """The schedule's decision, taken by the library on the host (no device needed)."""
    r = int(lib().scope_layer_is_dense(ctypes.byref(sched)))
    if r < 0:
        raise ScopeError("scope_layer_is_dense", 1)
    return bool(r)


def attention_layer(p, sched: Schedule, Q, K, V, q_init_idx=None, k_init_idx=None, ws=None, out=None,
                    out_q=None, out_k=None, stream=None):
    """One layer under the dense-prefix schedule ([RoPE] then dense attention or SCOPE).
    With sched.rope, the rotated Q and K go to out_q / out_k (new tensors when None)."""
    ws = alloc_workspace(p, Q.device) if ws is None else ws
    O = torch.empty_like(Q) if out is None else out
    Qr = Kr = None
    if sched.rope:
        Qr = torch.empty_like(Q) if out_q is None else out_q
        Kr = torch.empty_like(K) if out_k is None else out_k
    _check("scope_attention_layer", lib().scope_attention_layer(
        ctypes.byref(p), ctypes.byref(sched), _ptr(Q), _ptr(K), _ptr(V), _ptr(q_init_idx), _ptr(k_init_idx),
        _ptr(O), _ptr(Qr), _ptr(Kr), _ptr(ws), ws.numel(), _stream(stream)))
    return O


def check_wait_timeout(p, wait_limit_ns, ws=None, stream=None):
    """Runs the attention kernel with its scheduler held so every first wait gives up after
    wait_limit_ns (the device-side timeout path); returns the workspace used."""
    ws = alloc_workspace(p) if ws is None else ws
    _check("scope_check_wait_timeout", lib().scope_check_wait_timeout(
        ctypes.byref(p), int(wait_limit_ns), _ptr(ws), ws.numel(), _stream(stream)))
    return ws


def tc_accumulation_probe(A, B, stream=None):
    """The tensor core's fp32 result of A @ B^T (A [128, K], B [N, K] bf16 on the device) as
    one chain of K/16 tcgen05.mma steps."""
    K, N = A.shape[1], B.shape[0]
    D = torch.empty((128, N), dtype=torch.float32, device=A.device)
    _check("scope_tc_accumulation_probe", lib().scope_tc_accumulation_probe(
        _ptr(A), _ptr(B), int(K), int(N), _ptr(D), _stream(stream)))
    return D


def device_status_code(ws, stream=None):
    """(return code of scope_get_device_status, status word)."""
    out = ctypes.c_int32(0)
    code = lib().scope_get_device_status(_ptr(ws), _stream(stream), ctypes.byref(out))
    return int(code), int(out.value)


def get_selection_stats(p, ws, stream=None) -> dict:
    """Top-p decisions of the last selection on `ws` and how many lay within 1e-6 / 3e-7 of a
    tie (the margin the binary64 reference logs; scope_get_selection_stats)."""
    out = (ctypes.c_int32 * 4)()
    _check("scope_get_selection_stats", lib().scope_get_selection_stats(ctypes.byref(p), _ptr(ws), _stream(stream), out))
    return {"decisions": int(out[0]), "margin_below_1e-6": int(out[1]), "margin_below_3e-7": int(out[2])}


def get_device_status(ws, stream=None) -> int:
    out = ctypes.c_int32(0)
    code = lib().scope_get_device_status(_ptr(ws), _stream(stream), ctypes.byref(out))
    if code not in (0, 5, 6):
        raise ScopeError("scope_get_device_status", code)
    return int(out.value)
