// Internal declarations shared by the SCOPE CUDA sources (not part of the C ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/scope.h"

namespace scope {

constexpr int kMaxC = 2048;         // max centroids per problem (LUT and histogram sizes)
constexpr int kSortChunk = 512;     // tokens per warp in the stable counting sort
constexpr int kAttnTile = 256;      // queries per attention work item (two 128-row tiles)
constexpr unsigned long long kTcWaitDefaultNs = 4000000000ull;   // pipeline wait limit (4 s)

// ---------------------------------------------------------------------------------
// Clustering problems.  Role 0 = queries (all d channels, C = Cq); roles 1..3 = the
// key subspaces T, H, W (their channel range, C = Cm).  A launch covers a contiguous
// range of roles for every (b, h): problem index p = bh * nroles + (role - role0).
struct RoleDesc {
    const void *X;        // [BH, N, d] input (Q or K)
    int ch0, dm, C;       // channel range and centroid count
    double *cent;         // fp64 centroids, element (bh, c, i) at cent[bh*C*d + c*d + i]
    uint16_t *assign;     // assignments, element (bh, j) at assign[bh*assign_bh + j]
    long long assign_bh;  // bh stride of assign
    int32_t *sizes;       // member counts, (bh, c) at sizes[bh*sizes_bh + c]
    long long sizes_bh;
    const int32_t *init_idx;   // initial centroid rows, (bh, c) at init_idx[bh*init_bh + c]
    long long init_bh;
    const double *init_cent;   // or initial centroids, same layout as cent
};

struct KmArgs {
    RoleDesc role[4];
    int role0, nroles;
    int BH, N, d;
    int is_bf16;
    // per-problem scratch (problem p = bh*nroles + r)
    float *cent32;        // [P, ds, Cs] fp32 centroids, transposed
    double *cent64T;      // [P, ds, Cs] binary64 centroids, transposed (exact re-decisions)
    float *cnorm;         // [P, Cs]  ||mu32_c|| rounded up
    float *cnrm2;         // [P, Cs]  ||mu_c||^2 rounded to fp32
    float *cslack;        // [P, Cs]  2^-22 ||mu_c||^2 rounded up (error-bound term)
    int Cs, ds;           // strides: max C and max dm over the launched roles
    int32_t *perm;        // [P, N] members sorted by cluster, token order inside
    int32_t *off;         // [P, Cs+1] segment offsets into perm
    int32_t *chunk_hist;  // [P, nchunk, Cs] per-chunk counts -> prefix
    int nchunk;
    int32_t *status;      // device status word
    // tensor-core assignment (bf16 inputs): packed centroid operands, Cpad = Cs rounded up to 16
    __nv_bfloat16 *cent_bf;   // [P, 2 (hi, lo), Cpad, d] bf16 split of the centroids
    float *cn2p;              // [P, Cpad + 4] |mu|^2 (+inf padding), max |mu|, max slack
    float *xnorm;             // [P, N] |x| over the role's channels, rounded up (per run)
    // tokens whose assignment the fast kernels could not certify, one list per launched
    // role r: entries bh * N + j at unsure_list[r * BH * N ...], count unsure_count[r]
    int32_t *unsure_list;     // [4, BH * N]
    int32_t *unsure_count;    // [4], cleared before every assignment launch
};

// Workspace layout (byte offsets); computed identically by every entry point.  The selection
// stage keeps its per-key bins in the key-list region, which only the attention stage
// writes afterwards (2 bytes per key and unit fit in the 4 of a list entry).
struct WsLayout {
    size_t status, counters;
    size_t cent32, cent64T, cnorm, cnrm2, cslack, perm, off, chunk_hist, cent_bf, cn2p, xnorm, unsure_list,
        unsure_count;
    size_t q_cent, q_assign, q_sizes, k_cent, k_codes, k_sizes;
    size_t topp, base, khead, final_cnt, mask, sel_state, sel_hist, sel_stats, sel_lut;
    size_t q_perm, q_off, q_hist, work_items, attn_counter, key_lists;
    size_t total;
};

WsLayout ws_layout(const scope_params &p);

// Launchers (enqueue only; return cudaGetLastError()).
cudaError_t km_run(KmArgs a, int iters, cudaStream_t s);
cudaError_t sort_by_cluster(KmArgs a, cudaStream_t s);  // stable counting sort, all problems
bool km_assign_tc_supported(const KmArgs &a);            // bf16 and the operands fit on chip
cudaError_t km_pack(const KmArgs &a, cudaStream_t s);     // centroids -> cent_bf, cn2p
cudaError_t km_norms(const KmArgs &a, cudaStream_t s);    // token norms -> xnorm (once per run)
cudaError_t km_assign_tc(const KmArgs &a, int num_sms, cudaStream_t s);

struct SelArgs {
    const double *qcent;      // [BH, Cq, d]
    const int32_t *qsizes;    // [BH, Cq]
    const double *kcent;      // [BH, Cm, d]
    const uint16_t *codes;    // [BH, 3, N]
    int32_t *topp, *base, *khead, *final_cnt;
    uint32_t *mask;           // [BH, Cq, nw]
    double *state;            // [BH*Cq, 8] per-unit selection state
    int32_t *hist;            // [BH*Cq, 2048] level-0 key counts of the Top-p pass (or NULL)
    uint16_t *bins;           // [BH*Cq, bins_stride] each key's level-0 bin (or NULL)
    long long bins_stride;    // N rounded up to a multiple of 8
    double *lut;              // [BH*Cq, 3*Cm] the Top-p kernel's tables (or NULL)
    int32_t *stats;           // [4] Top-p decisions: made, with margin < 1e-6, < 3e-7 (or NULL)
    int BH, N, d, dt, dh, dw, Cq, Cm, nw;
    double rho, inv_sqrt_d;
    int kfix;
    int khead_mode;           // SCOPE_KHEAD_ONLINE: r_c = max(b_c, k_head); SCOPE_KHEAD_OFF: r_c = b_c
    int32_t *status;
};
cudaError_t select_run(const SelArgs &a, cudaStream_t s);

struct AttnArgs {
    const void *Q, *K, *V;
    void *O;
    const int32_t *perm;      // queries sorted by cluster, (bh, m) at perm[bh*perm_bh + m]
    const int32_t *off;       // cluster offsets into perm, (bh, c) at off[bh*off_bh + c]
    long long perm_bh, off_bh;
    const uint32_t *mask;     // [BH, Cq, nw]
    const int32_t *final_cnt; // [BH, Cq]
    int4 *items;              // work list (bh, c, q0, nq)
    int32_t *lists;           // selected key indices of unit u at lists[u*list_stride ...], ascending
    long long list_stride;    // N rounded up to a multiple of 4
    int32_t *counter;         // [2]: item count, dynamic scheduler
    int BH, N, d, Cq, nw, is_bf16;
    int use_tc;               // bf16 on the tensor cores (else CUDA cores)
    float scale_log2;         // log2(e)/sqrt(d)
    int32_t *status;
    int num_sms;
    unsigned long long wait_ns;   // limit of every pipeline wait of the tensor-core kernel
    int hold_items;           // nonzero: the kernel's scheduler publishes no item (timeout check)
};
cudaError_t attention_run(const AttnArgs &a, cudaStream_t s);     // items + kernel
cudaError_t attention_items(const AttnArgs &a, cudaStream_t s);   // work list only
cudaError_t attention_kernel(const AttnArgs &a, cudaStream_t s);  // kernel only
cudaError_t attention_simt_run(const AttnArgs &a, cudaStream_t s);

constexpr int kMaxFidCm = 1024;     // key centroids per subspace the fidelity kernel accepts
struct FidArgs {
    const void *Q, *K;
    const uint16_t *q_assign;   // [BH, N]
    const double *qcent;        // [BH, Cq, d]
    const double *kcent;        // [BH, Cm, d]
    const uint16_t *codes;      // [BH, 3, N]
    const uint32_t *mask;       // [BH, Cq, nw]
    const long long *samples;   // global query indices bh * N + i
    int n_samples;
    long long total;            // BH * N (samples outside [0, total) give NaN)
    double *recall_sel, *recall_proxy;
    double *scratch;            // [blocks, 2, N]
    int blocks;
    int N, d, dt, dh, dw, Cq, Cm, nw, is_bf16;
    double inv_sqrt_d;
    long long k;                // ceil(frac * N)
};
cudaError_t fidelity_run(const FidArgs &a, cudaStream_t s);
// Spearman's rho of each sample's exact logits with its proxy logits (rankcorr.cu).
size_t rank_corr_scratch_bytes(int N, int n_samples);
cudaError_t rank_corr_run(const FidArgs &a, double *spearman, void *scratch, int num_sms, cudaStream_t s);
// Divisor for x / d by multiply and shift (rope.cu).
struct FastDiv {
    unsigned m, l;
};
// 3D RoPE of up to two [rows, d] tensors (rope.cu).
struct RopeArgs {
    const void *X[2];
    void *Y[2];
    int n_tensors;
    long long rows;   // B*H*N
    int N, T, Hg, Wg;
    int d, dt, dh, dw;
    double base;
    int is_bf16;
    FastDiv div_N, div_HW, div_Wg;   // filled by rope3d_run
};
constexpr size_t kRopeMaxTableBytes = 192 * 1024;   // shared-memory cos/sin table limit
size_t rope_table_bytes(int T, int Hg, int Wg, int dt, int dh, int dw);
cudaError_t rope3d_run(const RopeArgs &a, int num_sms, cudaStream_t s);
// Dense attention as the sparse kernel's special case: one query cluster that selects
// every key (attention.cu).
cudaError_t attention_dense_setup(uint16_t *q_assign, uint32_t *mask, int32_t *final_counts, long long BH,
                                  long long N, long long nw, cudaStream_t s);
cudaError_t permute_channels_run(const void *X, const int32_t *perm, void *Y, long long rows, int d,
                                 int is_bf16, int num_sms, cudaStream_t s);
size_t select_smem_bytes(int Cm, int d);
constexpr int kSelBins = 2048;      // histogram bins of the selection passes

// ---------------------------------------------------------------------------------
__device__ __forceinline__ float load_x(const void *X, long long idx, int is_bf16)
{
    if (is_bf16)
        return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(X)[idx]);
    return reinterpret_cast<const float *>(X)[idx];
}

__device__ __forceinline__ void set_status(int32_t *status, int bits)
{
    if (status) atomicOr(status, bits);
}

// Debug builds (-DSCOPE_DEBUG): the internal indices the kernels derive (token rows taken from
// permutations and key lists, cluster indices about to be stored) are checked before use; an
// index outside [0, n) sets SCOPE_DEV_DEBUG_CHECK and is replaced by 0, so the access stays in
// bounds and the kernel carries on.  Release builds compile the check away.
#ifdef SCOPE_DEBUG
__device__ __forceinline__ long long debug_index(long long i, long long n, int32_t *status)
{
    if (i < 0 || i >= n) {
        set_status(status, SCOPE_DEV_DEBUG_CHECK);
        return 0;
    }
    return i;
}
#define SCOPE_DCHECK(i, n, status) ((int)::scope::debug_index((i), (n), (status)))
#else
#define SCOPE_DCHECK(i, n, status) (i)
#endif

// Appends `value` for every lane with `take` to list[*count ...] with one atomic per
// warp.  All 32 lanes of the warp must call it.
__device__ __forceinline__ void warp_append(bool take, int32_t value, int32_t *list, int32_t *count)
{
    const unsigned m = __ballot_sync(0xffffffffu, take);
    if (!m) return;
    const int lane = threadIdx.x & 31, leader = __ffs(m) - 1;
    int base = 0;
    if (lane == leader) base = atomicAdd(count, __popc(m));
    base = __shfl_sync(0xffffffffu, base, leader);
    if (take) list[base + __popc(m & ((1u << lane) - 1u))] = value;
}

}  // namespace scope
