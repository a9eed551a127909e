// scope_build_lut_and_select_noalloc: the selection stage without a caller workspace.
//
// Some callers cannot call cudaMalloc: a host application that owns every device
// allocation through its own pool and does not let libraries allocate, or a
// latency-critical loop in which cudaMalloc / cudaFree (which may synchronise the
// device) are not allowed.  For them this entry point runs the same selection
// kernels as scope_build_lut_and_select, with its scratch (a status word and 64 bytes
// of state per (b, h, query cluster) unit) in a fixed device array of this library
// instead of a caller workspace.  It allocates nothing.
//
// The array is shared by every call and keeps the last call's contents: the status
// word is cleared at the start of each call (the per-unit state is written before it
// is read), and calls whose work overlaps on the GPU race on it.
#include "common.cuh"

#include <cmath>

namespace scope {

namespace {

constexpr size_t kNoAllocStatusBytes = 256;
constexpr size_t kNoAllocStateBytes = (size_t)SCOPE_NOALLOC_MAX_UNITS * 8 * sizeof(double);

// Every GPU that loads the library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_select_scratch[kNoAllocStatusBytes + kNoAllocStateBytes];

// Device address of g_select_scratch on the current device, looked up on every call (host
// code must not use the symbol itself as a device address).  The lookup allocates nothing
// and enqueues nothing; not caching it keeps the address right after a device reset, which
// gives the array a new address in the new context.
cudaError_t scratch_address(void **out)
{
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_select_scratch);
    if (e != cudaSuccess) return e;
    *out = p;
    return cudaSuccess;
}

bool aligned16(const void *p)
{
    return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

}  // namespace

}  // namespace scope

extern "C" scope_status scope_build_lut_and_select_noalloc(
    const scope_params *p, const double *q_centroids, const int32_t *q_sizes,
    const double *k_centroids, const uint16_t *k_codes, int32_t *topp_counts, int32_t *base_counts,
    int32_t *k_head, int32_t *final_counts, uint32_t *sel_mask, void *stream)
{
    using namespace scope;
    if (scope_workspace_bytes(p) == 0) return SCOPE_ERR_INVALID_ARGUMENT;   // invalid params
    const long long BH = (long long)p->B * p->H;
    if (BH * p->Cq > SCOPE_NOALLOC_MAX_UNITS) return SCOPE_ERR_UNSUPPORTED;
    if (!aligned16(q_centroids) || !aligned16(q_sizes) || !aligned16(k_centroids) ||
        !aligned16(k_codes) || (topp_counts && !aligned16(topp_counts)) || !aligned16(base_counts) ||
        !aligned16(k_head) || !aligned16(final_counts) || !aligned16(sel_mask))
        return SCOPE_ERR_INVALID_ARGUMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    void *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return SCOPE_ERR_CUDA;
    int32_t *status = static_cast<int32_t *>(scratch);
    if (cudaMemsetAsync(status, 0, sizeof(int32_t), s) != cudaSuccess) return SCOPE_ERR_CUDA;

    const long long N = (long long)p->T * p->Hg * p->Wg;
    SelArgs a{};
    a.qcent = q_centroids;
    a.qsizes = q_sizes;
    a.kcent = k_centroids;
    a.codes = k_codes;
    a.topp = topp_counts;
    a.base = base_counts;
    a.khead = k_head;
    a.final_cnt = final_counts;
    a.mask = sel_mask;
    a.state = reinterpret_cast<double *>(static_cast<unsigned char *>(scratch) + kNoAllocStatusBytes);
    a.BH = (int)BH;
    a.N = (int)N;
    a.d = p->d;
    const bool full = p->key_clustering == SCOPE_KEYS_FULL;   // one subspace of all d channels
    a.dt = full ? p->d : p->d_t;
    a.dh = full ? 0 : p->d_h;
    a.dw = full ? 0 : p->d_w;
    a.Cq = p->Cq;
    a.Cm = p->Cm;
    a.nw = (int)((N + 31) / 32);
    a.rho = p->rho;
    a.inv_sqrt_d = 1.0 / std::sqrt((double)p->d);
    const double kf = std::ceil(p->alpha * (double)N);
    a.kfix = kf < 0 ? 0 : (kf > (double)N ? (int)N : (int)kf);
    a.khead_mode = p->khead_mode;
    a.status = status;
    return select_run(a, s) == cudaSuccess ? SCOPE_OK : SCOPE_ERR_CUDA;
}
