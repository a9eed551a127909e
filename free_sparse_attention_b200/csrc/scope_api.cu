// C ABI of the SCOPE hot path: argument validation, workspace carving and the launch
// sequences of the five entry points declared in include/scope.h.
#include "common.cuh"

#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>

using namespace scope;

namespace {

constexpr size_t kAlign = 256;

// An NVTX range over a scope (NVTX 3 is header-only and costs a load and a branch unless a
// profiler has injected itself): the host side of every entry point and of the layer's three
// stages, so that a timeline shows which launches belong to which stage.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

size_t align_up(size_t x)
{
    return (x + kAlign - 1) / kAlign * kAlign;
}

scope_status validate(const scope_params *p)
{
    if (!p) return SCOPE_ERR_INVALID_ARGUMENT;
    if (p->B < 1 || p->H < 1 || p->T < 1 || p->Hg < 1 || p->Wg < 1) return SCOPE_ERR_INVALID_ARGUMENT;
    const long long N = (long long)p->T * p->Hg * p->Wg;
    if (N > (1ll << 22)) return SCOPE_ERR_UNSUPPORTED;
    const long long BH = (long long)p->B * p->H;
    if (BH > 16383 || BH * N >= (1ll << 31)) return SCOPE_ERR_UNSUPPORTED;
    if (p->d_t < 1 || p->d_h < 1 || p->d_w < 1 || p->d_t + p->d_h + p->d_w != p->d)
        return SCOPE_ERR_INVALID_ARGUMENT;
    if (p->d != 64 && p->d != 128) return SCOPE_ERR_UNSUPPORTED;
    if (p->Cq < 1 || p->Cm < 1 || p->Cq > N || p->Cm > N) return SCOPE_ERR_INVALID_ARGUMENT;
    if (p->Cq > kMaxC || p->Cm > kMaxC) return SCOPE_ERR_UNSUPPORTED;
    if (p->iters < 1 || p->iters > 64) return SCOPE_ERR_INVALID_ARGUMENT;
    if (!(p->rho > 0.0 && p->rho <= 1.0)) return SCOPE_ERR_INVALID_ARGUMENT;
    if (!(p->alpha >= 0.0 && p->alpha <= 1.0)) return SCOPE_ERR_INVALID_ARGUMENT;
    if (p->khead_mode != SCOPE_KHEAD_ONLINE && p->khead_mode != SCOPE_KHEAD_OFF) return SCOPE_ERR_INVALID_ARGUMENT;
    if (p->key_clustering != SCOPE_KEYS_SUBSPACES && p->key_clustering != SCOPE_KEYS_FULL)
        return SCOPE_ERR_INVALID_ARGUMENT;
    if (p->dtype != SCOPE_F32 && p->dtype != SCOPE_BF16) return SCOPE_ERR_INVALID_ARGUMENT;
    return SCOPE_OK;
}

bool aligned(const void *ptr)
{
    return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0;
}

bool ok_ptr(const void *ptr)
{
    return ptr && aligned(ptr);
}

bool ok_opt(const void *ptr)
{
    return !ptr || aligned(ptr);
}

struct Dims {
    long long BH, N, nw, Cs, P, nchunk;
    int d;
};

Dims dims_of(const scope_params &p)
{
    Dims D;
    D.BH = (long long)p.B * p.H;
    D.N = (long long)p.T * p.Hg * p.Wg;
    D.nw = (D.N + 31) / 32;
    D.Cs = std::max(p.Cq, p.Cm);
    D.P = D.BH * 4;
    D.nchunk = (D.N + kSortChunk - 1) / kSortChunk;
    D.d = p.d;
    return D;
}

template <typename T>
T *at(void *ws, size_t off)
{
    return reinterpret_cast<T *>(static_cast<char *>(ws) + off);
}

KmArgs km_base(const scope_params &p, const WsLayout &L, void *ws)
{
    const Dims D = dims_of(p);
    KmArgs a{};
    a.BH = (int)D.BH;
    a.N = (int)D.N;
    a.d = p.d;
    a.is_bf16 = p.dtype == SCOPE_BF16;
    a.cent32 = at<float>(ws, L.cent32);
    a.cent64T = at<double>(ws, L.cent64T);
    a.cnorm = at<float>(ws, L.cnorm);
    a.cnrm2 = at<float>(ws, L.cnrm2);
    a.cslack = at<float>(ws, L.cslack);
    a.perm = at<int32_t>(ws, L.perm);
    a.off = at<int32_t>(ws, L.off);
    a.chunk_hist = at<int32_t>(ws, L.chunk_hist);
    a.cent_bf = at<__nv_bfloat16>(ws, L.cent_bf);
    a.cn2p = at<float>(ws, L.cn2p);
    a.xnorm = at<float>(ws, L.xnorm);
    a.unsure_list = at<int32_t>(ws, L.unsure_list);
    a.unsure_count = at<int32_t>(ws, L.unsure_count);
    a.nchunk = (int)D.nchunk;
    a.status = at<int32_t>(ws, L.status);
    return a;
}

RoleDesc query_role(const scope_params &p, const void *Q, double *cent, uint16_t *assign,
                    int32_t *sizes, const int32_t *init_idx, const double *init_cent)
{
    const long long N = (long long)p.T * p.Hg * p.Wg;
    RoleDesc r{};
    r.X = Q;
    r.ch0 = 0;
    r.dm = p.d;
    r.C = p.Cq;
    r.cent = cent;
    r.assign = assign;
    r.assign_bh = N;
    r.sizes = sizes;
    r.sizes_bh = p.Cq;
    r.init_idx = init_idx;
    r.init_bh = p.Cq;
    r.init_cent = init_cent;
    return r;
}

// Number of key k-means problems per head: three channel ranges, or one over all d.
int key_roles(const scope_params &p)
{
    return p.key_clustering == SCOPE_KEYS_FULL ? 1 : 3;
}

// Channel range m of the key clustering: (start, width).
void key_range(const scope_params &p, int m, int &ch0, int &dm)
{
    if (p.key_clustering == SCOPE_KEYS_FULL) {
        ch0 = 0;
        dm = p.d;
        return;
    }
    const int bnd[4] = {0, p.d_t, p.d_t + p.d_h, p.d};
    ch0 = bnd[m];
    dm = bnd[m + 1] - bnd[m];
}

RoleDesc key_role(const scope_params &p, int m, const void *K, double *cent, uint16_t *codes,
                  int32_t *sizes3, const int32_t *init_idx, const double *init_cent)
{
    const long long N = (long long)p.T * p.Hg * p.Wg;
    RoleDesc r{};
    r.X = K;
    key_range(p, m, r.ch0, r.dm);
    r.C = p.Cm;
    r.cent = cent;
    r.assign = codes + m * N;
    r.assign_bh = 3 * N;
    r.sizes = sizes3 + (size_t)m * p.Cm;
    r.sizes_bh = 3ll * p.Cm;
    r.init_idx = init_idx ? init_idx + (size_t)m * p.Cm : nullptr;
    r.init_bh = 3ll * p.Cm;
    r.init_cent = init_cent;
    return r;
}

// With one full-d key clustering, code rows 1 and 2 of every head are zero.
cudaError_t zero_unused_codes(const scope_params &p, uint16_t *codes, cudaStream_t s)
{
    if (p.key_clustering != SCOPE_KEYS_FULL) return cudaSuccess;
    const size_t N = (size_t)p.T * p.Hg * p.Wg, BH = (size_t)p.B * p.H;
    return cudaMemset2DAsync(codes + N, 3 * N * sizeof(uint16_t), 0, 2 * N * sizeof(uint16_t), BH, s);
}

// Subspace split the selection and the fidelity kernels read the codes with.
void code_split(const scope_params &p, int &dt, int &dh, int &dw)
{
    if (p.key_clustering == SCOPE_KEYS_FULL) {
        dt = p.d;
        dh = dw = 0;
    } else {
        dt = p.d_t;
        dh = p.d_h;
        dw = p.d_w;
    }
}

scope_status cuda_status(cudaError_t e)
{
    return e == cudaSuccess ? SCOPE_OK : SCOPE_ERR_CUDA;
}

scope_status begin(const scope_params *p, void *ws, size_t ws_bytes, WsLayout &L, cudaStream_t s)
{
    scope_status st = validate(p);
    if (st != SCOPE_OK) return st;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1))) return SCOPE_ERR_INVALID_ARGUMENT;
    L = ws_layout(*p);
    if (ws_bytes < L.total) return SCOPE_ERR_WORKSPACE_TOO_SMALL;
    return SCOPE_OK;
}

scope_status clear_status(void *ws, const WsLayout &L, cudaStream_t s)
{
    return cuda_status(cudaMemsetAsync(at<char>(ws, L.status), 0, sizeof(int32_t), s));
}

SelArgs sel_args(const scope_params &p, const WsLayout &L, void *ws, const double *qc,
                 const int32_t *qs, const double *kc, const uint16_t *codes, int32_t *topp,
                 int32_t *base, int32_t *khead, int32_t *fin, uint32_t *mask)
{
    const Dims D = dims_of(p);
    SelArgs a{};
    a.qcent = qc;
    a.qsizes = qs;
    a.kcent = kc;
    a.codes = codes;
    a.topp = topp;
    a.base = base;
    a.khead = khead;
    a.final_cnt = fin;
    a.mask = mask;
    a.state = at<double>(ws, L.sel_state);
    a.hist = at<int32_t>(ws, L.sel_hist);
    a.bins = at<uint16_t>(ws, L.key_lists);
    a.bins_stride = (D.N + 7) / 8 * 8;
    a.lut = at<double>(ws, L.sel_lut);
    a.stats = at<int32_t>(ws, L.sel_stats);
    a.BH = (int)D.BH;
    a.N = (int)D.N;
    a.d = p.d;
    code_split(p, a.dt, a.dh, a.dw);
    a.Cq = p.Cq;
    a.Cm = p.Cm;
    a.nw = (int)D.nw;
    a.rho = p.rho;
    a.inv_sqrt_d = 1.0 / std::sqrt((double)p.d);
    double kf = std::ceil(p.alpha * (double)D.N);
    a.kfix = kf < 0 ? 0 : (kf > (double)D.N ? (int)D.N : (int)kf);
    a.khead_mode = p.khead_mode;
    a.status = at<int32_t>(ws, L.status);
    return a;
}

AttnArgs attn_args(const scope_params &p, const WsLayout &L, void *ws, const void *Q,
                   const void *K, const void *V, void *O, const int32_t *perm, long long perm_bh,
                   const int32_t *off, long long off_bh, const uint32_t *mask,
                   const int32_t *fin)
{
    const Dims D = dims_of(p);
    AttnArgs a{};
    a.Q = Q;
    a.K = K;
    a.V = V;
    a.O = O;
    a.perm = perm;
    a.perm_bh = perm_bh;
    a.off = off;
    a.off_bh = off_bh;
    a.mask = mask;
    a.final_cnt = fin;
    a.items = at<int4>(ws, L.work_items);
    a.lists = at<int32_t>(ws, L.key_lists);
    a.list_stride = (D.N + 3) / 4 * 4;
    a.counter = at<int32_t>(ws, L.counters);
    a.BH = (int)D.BH;
    a.N = (int)D.N;
    a.d = p.d;
    a.Cq = p.Cq;
    a.nw = (int)D.nw;
    a.is_bf16 = p.dtype == SCOPE_BF16;
    a.use_tc = a.is_bf16;
    a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)p.d));
    a.status = at<int32_t>(ws, L.status);
    int dev = 0;
    cudaGetDevice(&dev);
    a.num_sms = 148;
    cudaDeviceGetAttribute(&a.num_sms, cudaDevAttrMultiProcessorCount, dev);
    a.wait_ns = kTcWaitDefaultNs;
    a.hold_items = 0;
    return a;
}

}  // namespace

namespace scope {

WsLayout ws_layout(const scope_params &p)
{
    const Dims D = dims_of(p);
    WsLayout L{};
    size_t o = 0;
    auto take = [&](size_t bytes) {
        size_t r = o;
        o += align_up(bytes);
        return r;
    };
    L.status = take(sizeof(int32_t));
    L.counters = take(4 * sizeof(int32_t));
    L.cent32 = take(sizeof(float) * D.P * D.d * D.Cs);
    L.cent64T = take(sizeof(double) * D.P * D.d * D.Cs);
    L.cnorm = take(sizeof(float) * D.P * D.Cs);
    L.cnrm2 = take(sizeof(float) * D.P * D.Cs);
    L.cslack = take(sizeof(float) * D.P * D.Cs);
    L.perm = take(sizeof(int32_t) * D.P * D.N);
    L.off = take(sizeof(int32_t) * D.P * (D.Cs + 1));
    L.chunk_hist = take(sizeof(int32_t) * D.P * D.nchunk * D.Cs);
    const long long Cpad = (D.Cs + 15) / 16 * 16;
    L.cent_bf = take(sizeof(__nv_bfloat16) * D.P * 2 * Cpad * D.d);
    L.cn2p = take(sizeof(float) * D.P * (Cpad + 4));
    L.xnorm = take(sizeof(float) * D.P * D.N);
    L.unsure_list = take(sizeof(int32_t) * D.P * D.N);
    L.unsure_count = take(4 * sizeof(int32_t));
    L.q_cent = take(sizeof(double) * D.BH * p.Cq * p.d);
    L.q_assign = take(sizeof(uint16_t) * D.BH * D.N);
    L.q_sizes = take(sizeof(int32_t) * D.BH * p.Cq);
    L.k_cent = take(sizeof(double) * D.BH * p.Cm * p.d);
    L.k_codes = take(sizeof(uint16_t) * D.BH * 3 * D.N);
    L.k_sizes = take(sizeof(int32_t) * D.BH * 3 * p.Cm);
    L.topp = take(sizeof(int32_t) * D.BH * p.Cq);
    L.base = take(sizeof(int32_t) * D.BH * p.Cq);
    L.khead = take(sizeof(int32_t) * D.BH);
    L.final_cnt = take(sizeof(int32_t) * D.BH * p.Cq);
    L.mask = take(sizeof(uint32_t) * D.BH * p.Cq * D.nw);
    L.sel_state = take(sizeof(double) * 8 * D.BH * p.Cq);
    L.sel_hist = take(sizeof(int32_t) * kSelBins * D.BH * p.Cq);
    L.sel_stats = take(4 * sizeof(int32_t));
    L.sel_lut = take(sizeof(double) * 3 * p.Cm * D.BH * p.Cq);
    L.work_items = take(sizeof(int4) * D.BH * ((D.N + kAttnTile - 1) / kAttnTile + p.Cq));
    L.key_lists = take(sizeof(int32_t) * D.BH * p.Cq * ((D.N + 3) / 4 * 4));
    L.total = o;
    return L;
}

}  // namespace scope

extern "C" {

size_t scope_workspace_bytes(const scope_params *p)
{
    if (validate(p) != SCOPE_OK) return 0;
    return ws_layout(*p).total;
}

const char *scope_status_string(scope_status s)
{
    switch (s) {
    case SCOPE_OK: return "SCOPE_OK";
    case SCOPE_ERR_INVALID_ARGUMENT: return "SCOPE_ERR_INVALID_ARGUMENT";
    case SCOPE_ERR_UNSUPPORTED: return "SCOPE_ERR_UNSUPPORTED";
    case SCOPE_ERR_WORKSPACE_TOO_SMALL: return "SCOPE_ERR_WORKSPACE_TOO_SMALL";
    case SCOPE_ERR_CUDA: return "SCOPE_ERR_CUDA";
    case SCOPE_ERR_DEVICE_CHECK: return "SCOPE_ERR_DEVICE_CHECK";
    case SCOPE_ERR_TIMEOUT: return "SCOPE_ERR_TIMEOUT";
    }
    return "SCOPE_ERR_UNKNOWN";
}

scope_status scope_get_device_status(const void *ws, void *stream, int32_t *out)
{
    if (!ws || !out) return SCOPE_ERR_INVALID_ARGUMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return SCOPE_ERR_CUDA;
    *out = v;
    if (v & SCOPE_DEV_TIMEOUT) return SCOPE_ERR_TIMEOUT;
    return v ? SCOPE_ERR_DEVICE_CHECK : SCOPE_OK;
}

scope_status scope_get_selection_stats(const scope_params *p, const void *ws, void *stream, int32_t *out)
{
    if (!ws || !out || validate(p) != SCOPE_OK) return SCOPE_ERR_INVALID_ARGUMENT;
    const WsLayout L = ws_layout(*p);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t v[4] = {0, 0, 0, 0};
    cudaError_t e = cudaMemcpyAsync(v, static_cast<const char *>(ws) + L.sel_stats, sizeof(v),
                                    cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return SCOPE_ERR_CUDA;
    for (int k = 0; k < 4; ++k) out[k] = v[k];
    return SCOPE_OK;
}

scope_status scope_cluster_queries(const scope_params *p, const void *Q, const int32_t *init_idx,
                                   const double *init_cent, double *q_centroids,
                                   uint16_t *q_assign, int32_t *q_sizes, void *ws,
                                   size_t ws_bytes, void *stream)
{
    NvtxRange nvtx("scope_cluster_queries");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    WsLayout L;
    scope_status st = begin(p, ws, ws_bytes, L, s);
    if (st != SCOPE_OK) return st;
    if (!ok_ptr(Q) || !ok_ptr(q_centroids) || !ok_ptr(q_assign) || !ok_ptr(q_sizes) ||
        !ok_opt(init_idx) || !ok_opt(init_cent) || (!init_idx && !init_cent))
        return SCOPE_ERR_INVALID_ARGUMENT;
    if ((st = clear_status(ws, L, s)) != SCOPE_OK) return st;
    KmArgs a = km_base(*p, L, ws);
    a.role0 = 0;
    a.nroles = 1;
    a.role[0] = query_role(*p, Q, q_centroids, q_assign, q_sizes, init_idx, init_cent);
    a.Cs = p->Cq;
    a.ds = p->d;
    return cuda_status(km_run(a, p->iters, s));
}

scope_status scope_cluster_keys(const scope_params *p, const void *K, const int32_t *init_idx,
                                const double *init_cent, double *k_centroids, uint16_t *k_codes,
                                void *ws, size_t ws_bytes, void *stream)
{
    NvtxRange nvtx("scope_cluster_keys");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    WsLayout L;
    scope_status st = begin(p, ws, ws_bytes, L, s);
    if (st != SCOPE_OK) return st;
    if (!ok_ptr(K) || !ok_ptr(k_centroids) || !ok_ptr(k_codes) || !ok_opt(init_idx) ||
        !ok_opt(init_cent) || (!init_idx && !init_cent))
        return SCOPE_ERR_INVALID_ARGUMENT;
    if ((st = clear_status(ws, L, s)) != SCOPE_OK) return st;
    KmArgs a = km_base(*p, L, ws);
    a.role0 = 1;
    a.nroles = key_roles(*p);
    for (int m = 0; m < a.nroles; ++m)
        a.role[1 + m] = key_role(*p, m, K, k_centroids, k_codes, at<int32_t>(ws, L.k_sizes),
                                 init_idx, init_cent);
    a.Cs = p->Cm;
    a.ds = p->key_clustering == SCOPE_KEYS_FULL ? p->d : std::max(p->d_t, std::max(p->d_h, p->d_w));
    cudaError_t e = km_run(a, p->iters, s);
    if (e == cudaSuccess) e = zero_unused_codes(*p, k_codes, s);
    return cuda_status(e);
}

scope_status scope_build_lut_and_select(const scope_params *p, const double *q_centroids,
                                        const int32_t *q_sizes, const double *k_centroids,
                                        const uint16_t *k_codes, int32_t *topp_counts,
                                        int32_t *base_counts, int32_t *k_head,
                                        int32_t *final_counts, uint32_t *sel_mask, void *ws,
                                        size_t ws_bytes, void *stream)
{
    NvtxRange nvtx("scope_build_lut_and_select");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    WsLayout L;
    scope_status st = begin(p, ws, ws_bytes, L, s);
    if (st != SCOPE_OK) return st;
    if (!ok_ptr(q_centroids) || !ok_ptr(q_sizes) || !ok_ptr(k_centroids) || !ok_ptr(k_codes) ||
        !ok_opt(topp_counts) || !ok_ptr(base_counts) || !ok_ptr(k_head) ||
        !ok_ptr(final_counts) || !ok_ptr(sel_mask))
        return SCOPE_ERR_INVALID_ARGUMENT;
    if ((st = clear_status(ws, L, s)) != SCOPE_OK) return st;
    SelArgs a = sel_args(*p, L, ws, q_centroids, q_sizes, k_centroids, k_codes, topp_counts,
                         base_counts, k_head, final_counts, sel_mask);
    return cuda_status(select_run(a, s));
}

namespace {

// Groups the queries by cluster (stable counting sort of q_assign) and runs the attention
// kernel; arguments already validated, status word already cleared.
scope_status attention_impl(const scope_params &p, const WsLayout &L, void *ws, const void *Q, const void *K,
                            const void *V, const uint16_t *q_assign, const uint32_t *sel_mask,
                            const int32_t *final_counts, void *O, cudaStream_t s)
{
    KmArgs a = km_base(p, L, ws);
    a.role0 = 0;
    a.nroles = 1;
    a.role[0] = query_role(p, Q, nullptr, const_cast<uint16_t *>(q_assign), at<int32_t>(ws, L.q_sizes), nullptr,
                           nullptr);
    a.Cs = p.Cq;
    a.ds = p.d;
    cudaError_t e = sort_by_cluster(a, s);
    if (e != cudaSuccess) return SCOPE_ERR_CUDA;
    const Dims D = dims_of(p);
    AttnArgs t = attn_args(p, L, ws, Q, K, V, O, a.perm, D.N, a.off, p.Cq + 1, sel_mask, final_counts);
    return cuda_status(attention_run(t, s));
}

// Dense attention: the layout of the one-cluster problem inside the caller's workspace
// (never larger than the layout of `p` itself).
scope_status dense_impl(const scope_params &p, void *ws, size_t ws_bytes, const void *Q, const void *K,
                        const void *V, void *O, cudaStream_t s)
{
    scope_params p1 = p;
    p1.Cq = 1;
    const WsLayout L = ws_layout(p1);
    if (ws_bytes < L.total) return SCOPE_ERR_WORKSPACE_TOO_SMALL;
    const Dims D = dims_of(p1);
    uint16_t *qa = at<uint16_t>(ws, L.q_assign);
    uint32_t *mk = at<uint32_t>(ws, L.mask);
    int32_t *fc = at<int32_t>(ws, L.final_cnt);
    scope_status st = clear_status(ws, L, s);
    if (st != SCOPE_OK) return st;
    if (attention_dense_setup(qa, mk, fc, D.BH, D.N, D.nw, s) != cudaSuccess) return SCOPE_ERR_CUDA;
    return attention_impl(p1, L, ws, Q, K, V, qa, mk, fc, O, s);
}

scope_status validate_rope(const scope_params &p, double base)
{
    if ((p.d_t & 1) || (p.d_h & 1) || (p.d_w & 1)) return SCOPE_ERR_INVALID_ARGUMENT;
    if (!(base > 0.0) || !std::isfinite(base)) return SCOPE_ERR_INVALID_ARGUMENT;
    if (rope_table_bytes(p.T, p.Hg, p.Wg, p.d_t, p.d_h, p.d_w) > kRopeMaxTableBytes) return SCOPE_ERR_UNSUPPORTED;
    return SCOPE_OK;
}

scope_status rope_impl(const scope_params &p, double base, const void *Q, const void *K, void *Qr, void *Kr,
                       cudaStream_t s)
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return SCOPE_ERR_CUDA;
    const Dims D = dims_of(p);
    RopeArgs a{};
    a.X[0] = Q;
    a.Y[0] = Qr;
    a.X[1] = K;
    a.Y[1] = Kr;
    a.n_tensors = K ? 2 : 1;
    a.rows = D.BH * D.N;
    a.N = (int)D.N;
    a.T = p.T;
    a.Hg = p.Hg;
    a.Wg = p.Wg;
    a.d = p.d;
    a.dt = p.d_t;
    a.dh = p.d_h;
    a.dw = p.d_w;
    a.base = base;
    a.is_bf16 = p.dtype == SCOPE_BF16;
    return cuda_status(rope3d_run(a, sms, s));
}

bool schedule_ok(const scope_layer_schedule *sc)
{
    return sc && sc->layer >= 0 && sc->step >= 0 && sc->dense_layers >= 0 && sc->dense_steps >= 0;
}

}  // namespace

scope_status scope_sparse_attention(const scope_params *p, const void *Q, const void *K,
                                    const void *V, const uint16_t *q_assign,
                                    const uint32_t *sel_mask, const int32_t *final_counts,
                                    void *O, void *ws, size_t ws_bytes, void *stream)
{
    NvtxRange nvtx("scope_sparse_attention");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    WsLayout L;
    scope_status st = begin(p, ws, ws_bytes, L, s);
    if (st != SCOPE_OK) return st;
    if (!ok_ptr(Q) || !ok_ptr(K) || !ok_ptr(V) || !ok_ptr(q_assign) || !ok_ptr(sel_mask) ||
        !ok_ptr(final_counts) || !ok_ptr(O))
        return SCOPE_ERR_INVALID_ARGUMENT;
    if ((st = clear_status(ws, L, s)) != SCOPE_OK) return st;
    return attention_impl(*p, L, ws, Q, K, V, q_assign, sel_mask, final_counts, O, s);
}

scope_status scope_dense_attention(const scope_params *p, const void *Q, const void *K, const void *V, void *O,
                                   void *ws, size_t ws_bytes, void *stream)
{
    NvtxRange nvtx("scope_dense_attention");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    WsLayout L;
    scope_status st = begin(p, ws, ws_bytes, L, s);
    if (st != SCOPE_OK) return st;
    if (!ok_ptr(Q) || !ok_ptr(K) || !ok_ptr(V) || !ok_ptr(O)) return SCOPE_ERR_INVALID_ARGUMENT;
    return dense_impl(*p, ws, ws_bytes, Q, K, V, O, s);
}

scope_status scope_rope3d(const scope_params *p, double base, const void *Q, const void *K, void *Qr, void *Kr,
                          void *stream)
{
    NvtxRange nvtx("scope_rope3d");
    scope_status st = validate(p);
    if (st != SCOPE_OK) return st;
    if ((st = validate_rope(*p, base)) != SCOPE_OK) return st;
    if (!ok_ptr(Q) || !ok_ptr(Qr) || !ok_opt(K) || !ok_opt(Kr) || (!K) != (!Kr)) return SCOPE_ERR_INVALID_ARGUMENT;
    return rope_impl(*p, base, Q, K, Qr, Kr, static_cast<cudaStream_t>(stream));
}

int scope_layer_is_dense(const scope_layer_schedule *sc)
{
    if (!schedule_ok(sc)) return -1;
    return (sc->layer < sc->dense_layers || sc->step < sc->dense_steps) ? 1 : 0;
}

scope_status scope_attention_layer(const scope_params *p, const scope_layer_schedule *sc, const void *Q,
                                   const void *K, const void *V, const int32_t *q_init_idx,
                                   const int32_t *k_init_idx, void *O, void *Qr, void *Kr, void *ws,
                                   size_t ws_bytes, void *stream)
{
    NvtxRange nvtx("scope_attention_layer");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    WsLayout L;
    scope_status st = begin(p, ws, ws_bytes, L, s);
    if (st != SCOPE_OK) return st;
    if (!schedule_ok(sc) || !ok_ptr(Q) || !ok_ptr(K) || !ok_ptr(V) || !ok_ptr(O)) return SCOPE_ERR_INVALID_ARGUMENT;
    const bool dense = scope_layer_is_dense(sc) == 1;
    if (!dense && (!ok_ptr(q_init_idx) || !ok_ptr(k_init_idx))) return SCOPE_ERR_INVALID_ARGUMENT;
    if (sc->rope) {
        if ((st = validate_rope(*p, sc->rope_base)) != SCOPE_OK) return st;
        if (!ok_ptr(Qr) || !ok_ptr(Kr)) return SCOPE_ERR_INVALID_ARGUMENT;
        if ((st = rope_impl(*p, sc->rope_base, Q, K, Qr, Kr, s)) != SCOPE_OK) return st;
        Q = Qr;
        K = Kr;
    }
    if (dense) return dense_impl(*p, ws, ws_bytes, Q, K, V, O, s);
    return scope_forward(p, Q, K, V, q_init_idx, k_init_idx, O, nullptr, ws, ws_bytes, stream);
}

scope_status scope_selection_recall(const scope_params *p, const void *Q, const void *K,
                                    const uint16_t *q_assign, const double *q_centroids,
                                    const double *k_centroids, const uint16_t *k_codes,
                                    const uint32_t *sel_mask, const int64_t *samples, int n_samples,
                                    double frac, double *recall_sel, double *recall_proxy,
                                    void *scratch, size_t scratch_bytes, void *stream)
{
    NvtxRange nvtx("scope_selection_recall");
    scope_status st = validate(p);
    if (st != SCOPE_OK) return st;
    if (!ok_ptr(Q) || !ok_ptr(K) || !ok_ptr(q_assign) || !ok_ptr(q_centroids) || !ok_ptr(k_centroids) ||
        !ok_ptr(k_codes) || !ok_ptr(sel_mask) || n_samples < 0 || (n_samples > 0 && !ok_ptr(samples)) ||
        (n_samples > 0 && (!ok_ptr(recall_sel) || !ok_ptr(recall_proxy))) || !ok_ptr(scratch) ||
        !(frac > 0.0 && frac <= 1.0))
        return SCOPE_ERR_INVALID_ARGUMENT;
    if (p->Cm > kMaxFidCm) return SCOPE_ERR_UNSUPPORTED;
    const Dims D = dims_of(*p);
    const size_t per = (size_t)16 * (size_t)D.N;
    if (scratch_bytes < per) return SCOPE_ERR_WORKSPACE_TOO_SMALL;
    if (n_samples == 0) return SCOPE_OK;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return SCOPE_ERR_CUDA;
    FidArgs a{};
    a.Q = Q;
    a.K = K;
    a.q_assign = q_assign;
    a.qcent = q_centroids;
    a.kcent = k_centroids;
    a.codes = k_codes;
    a.mask = sel_mask;
    a.samples = reinterpret_cast<const long long *>(samples);
    a.n_samples = n_samples;
    a.total = D.BH * D.N;
    a.recall_sel = recall_sel;
    a.recall_proxy = recall_proxy;
    a.scratch = static_cast<double *>(scratch);
    const size_t fit = scratch_bytes / per;
    a.blocks = (int)(fit < (size_t)sms ? fit : (size_t)sms);
    a.N = (int)D.N;
    a.d = p->d;
    code_split(*p, a.dt, a.dh, a.dw);
    a.Cq = p->Cq;
    a.Cm = p->Cm;
    a.nw = (int)D.nw;
    a.is_bf16 = p->dtype == SCOPE_BF16;
    a.inv_sqrt_d = 1.0 / std::sqrt((double)p->d);
    const double kk = std::ceil(frac * (double)D.N);
    a.k = kk < 1.0 ? 1 : (kk > (double)D.N ? D.N : (long long)kk);
    return cuda_status(fidelity_run(a, static_cast<cudaStream_t>(stream)));
}

size_t scope_rank_correlation_scratch_bytes(const scope_params *p, int n_samples)
{
    if (validate(p) != SCOPE_OK || n_samples < 1) return 0;
    const long long N = (long long)p->T * p->Hg * p->Wg;
    if (2ll * n_samples * N >= (1ll << 31)) return 0;
    return rank_corr_scratch_bytes((int)N, n_samples);
}

scope_status scope_rank_correlation(const scope_params *p, const void *Q, const void *K, const uint16_t *q_assign,
                                    const double *q_centroids, const double *k_centroids, const uint16_t *k_codes,
                                    const int64_t *samples, int n_samples, double *spearman, void *scratch,
                                    size_t scratch_bytes, void *stream)
{
    NvtxRange nvtx("scope_rank_correlation");
    scope_status st = validate(p);
    if (st != SCOPE_OK) return st;
    if (!ok_ptr(Q) || !ok_ptr(K) || !ok_ptr(q_assign) || !ok_ptr(q_centroids) || !ok_ptr(k_centroids) ||
        !ok_ptr(k_codes) || n_samples < 0 || (n_samples > 0 && (!ok_ptr(samples) || !ok_ptr(spearman))) ||
        !ok_ptr(scratch))
        return SCOPE_ERR_INVALID_ARGUMENT;
    if (p->Cm > kMaxFidCm) return SCOPE_ERR_UNSUPPORTED;
    if (n_samples == 0) return SCOPE_OK;
    const Dims D = dims_of(*p);
    if (2ll * n_samples * D.N >= (1ll << 31)) return SCOPE_ERR_UNSUPPORTED;
    const size_t need = scope_rank_correlation_scratch_bytes(p, n_samples);
    if (need == 0) return SCOPE_ERR_CUDA;
    if (scratch_bytes < need) return SCOPE_ERR_WORKSPACE_TOO_SMALL;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return SCOPE_ERR_CUDA;
    FidArgs a{};
    a.Q = Q;
    a.K = K;
    a.q_assign = q_assign;
    a.qcent = q_centroids;
    a.kcent = k_centroids;
    a.codes = k_codes;
    a.samples = reinterpret_cast<const long long *>(samples);
    a.n_samples = n_samples;
    a.total = D.BH * D.N;
    a.N = (int)D.N;
    a.d = p->d;
    code_split(*p, a.dt, a.dh, a.dw);
    a.Cq = p->Cq;
    a.Cm = p->Cm;
    a.nw = (int)D.nw;
    a.is_bf16 = p->dtype == SCOPE_BF16;
    a.inv_sqrt_d = 1.0 / std::sqrt((double)p->d);
    return cuda_status(rank_corr_run(a, spearman, scratch, sms, static_cast<cudaStream_t>(stream)));
}

scope_status scope_permute_channels(const scope_params *p, const void *X, const int32_t *perm, void *Y,
                                    void *stream)
{
    NvtxRange nvtx("scope_permute_channels");
    scope_status st = validate(p);
    if (st != SCOPE_OK) return st;
    if (!ok_ptr(X) || !ok_ptr(perm) || !ok_ptr(Y) || X == Y) return SCOPE_ERR_INVALID_ARGUMENT;
    const Dims D = dims_of(*p);
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return SCOPE_ERR_CUDA;
    return cuda_status(permute_channels_run(X, perm, Y, D.BH * D.N, p->d, p->dtype == SCOPE_BF16, sms,
                                            static_cast<cudaStream_t>(stream)));
}

scope_status scope_check_wait_timeout(const scope_params *p, uint64_t wait_limit_ns, void *ws, size_t ws_bytes,
                                      void *stream)
{
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    WsLayout L;
    scope_status st = begin(p, ws, ws_bytes, L, s);
    if (st != SCOPE_OK) return st;
    if (p->dtype != SCOPE_BF16) return SCOPE_ERR_UNSUPPORTED;
    if (wait_limit_ns < 1 || wait_limit_ns > 10000000000ull) return SCOPE_ERR_INVALID_ARGUMENT;
    if ((st = clear_status(ws, L, s)) != SCOPE_OK) return st;
    if (cudaMemsetAsync(at<char>(ws, L.counters), 0, 4 * sizeof(int32_t), s) != cudaSuccess) return SCOPE_ERR_CUDA;
    // no tensor is read: the held scheduler never hands out an item
    AttnArgs t = attn_args(*p, L, ws, nullptr, nullptr, nullptr, nullptr, nullptr, 0, nullptr, 0, nullptr, nullptr);
    t.wait_ns = wait_limit_ns;
    t.hold_items = 1;
    return cuda_status(attention_kernel(t, s));
}

scope_status scope_forward(const scope_params *p, const void *Q, const void *K, const void *V,
                           const int32_t *q_init_idx, const int32_t *k_init_idx, void *O,
                           const scope_intermediates *inter, void *ws, size_t ws_bytes,
                           void *stream)
{
    NvtxRange nvtx("scope_forward");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    WsLayout L;
    scope_status st = begin(p, ws, ws_bytes, L, s);
    if (st != SCOPE_OK) return st;
    if (!ok_ptr(Q) || !ok_ptr(K) || !ok_ptr(V) || !ok_ptr(q_init_idx) || !ok_ptr(k_init_idx) ||
        !ok_ptr(O))
        return SCOPE_ERR_INVALID_ARGUMENT;
    scope_intermediates I{};
    if (inter) I = *inter;
    const void *all[] = {I.q_centroids, I.q_assign, I.q_sizes, I.k_centroids, I.k_codes,
                         I.topp_counts, I.base_counts, I.k_head, I.final_counts, I.sel_mask};
    for (const void *ptr : all)
        if (!ok_opt(ptr)) return SCOPE_ERR_INVALID_ARGUMENT;
    double *qc = I.q_centroids ? I.q_centroids : at<double>(ws, L.q_cent);
    uint16_t *qa = I.q_assign ? I.q_assign : at<uint16_t>(ws, L.q_assign);
    int32_t *qs = I.q_sizes ? I.q_sizes : at<int32_t>(ws, L.q_sizes);
    double *kc = I.k_centroids ? I.k_centroids : at<double>(ws, L.k_cent);
    uint16_t *kk = I.k_codes ? I.k_codes : at<uint16_t>(ws, L.k_codes);
    int32_t *tp = I.topp_counts ? I.topp_counts : at<int32_t>(ws, L.topp);
    int32_t *bc = I.base_counts ? I.base_counts : at<int32_t>(ws, L.base);
    int32_t *kh = I.k_head ? I.k_head : at<int32_t>(ws, L.khead);
    int32_t *fc = I.final_counts ? I.final_counts : at<int32_t>(ws, L.final_cnt);
    uint32_t *mk = I.sel_mask ? I.sel_mask : at<uint32_t>(ws, L.mask);
    if ((st = clear_status(ws, L, s)) != SCOPE_OK) return st;
    auto mark = [&](int k) {
        return I.stage_events[k] ? cudaEventRecord(static_cast<cudaEvent_t>(I.stage_events[k]), s)
                                 : cudaSuccess;
    };
    if (mark(0) != cudaSuccess) return SCOPE_ERR_CUDA;

    // stage 1: query clustering and the three key-subspace clusterings, one launch set
    nvtxRangePushA("scope/clustering");
    KmArgs a = km_base(*p, L, ws);
    a.role0 = 0;
    a.nroles = 1 + key_roles(*p);
    a.role[0] = query_role(*p, Q, qc, qa, qs, q_init_idx, nullptr);
    for (int m = 0; m + 1 < a.nroles; ++m)
        a.role[1 + m] = key_role(*p, m, K, kc, kk, at<int32_t>(ws, L.k_sizes), k_init_idx, nullptr);
    a.Cs = std::max(p->Cq, p->Cm);
    a.ds = p->d;
    cudaError_t e = km_run(a, p->iters, s);
    if (e == cudaSuccess) e = zero_unused_codes(*p, kk, s);
    nvtxRangePop();
    if (e != cudaSuccess || mark(1) != cudaSuccess) return SCOPE_ERR_CUDA;

    // stage 2: LUT, proxy logits, Top-p, k_head, top-up, masks
    SelArgs sa = sel_args(*p, L, ws, qc, qs, kc, kk, tp, bc, kh, fc, mk);
    nvtxRangePushA("scope/selection");
    e = select_run(sa, s);
    nvtxRangePop();
    if (e != cudaSuccess || mark(2) != cudaSuccess) return SCOPE_ERR_CUDA;

    // stage 3: attention; the last clustering iteration already grouped the queries
    const Dims D = dims_of(*p);
    AttnArgs t = attn_args(*p, L, ws, Q, K, V, O, a.perm, a.nroles * D.N, a.off, a.nroles * (a.Cs + 1), mk, fc);
    nvtxRangePushA("scope/attention");
    e = attention_items(t, s);
    const bool marked = e == cudaSuccess && mark(3) == cudaSuccess;
    if (marked) e = attention_kernel(t, s);
    nvtxRangePop();
    if (!marked || e != cudaSuccess || mark(4) != cudaSuccess) return SCOPE_ERR_CUDA;
    return SCOPE_OK;
}

}  // extern "C"
