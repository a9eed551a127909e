// Sparse attention over each query cluster's selected original keys and values
// (SCOPE, arXiv 2608.12780, abstract: the attention runs over the original keys and values
// each cluster selected, not over centroids; review page, forward_implications[1]).
//
//   O_i = sum_{j in S_c} softmax_j(q_i . k_j / sqrt d) v_j,   c = cluster of query i.
//
// This file holds the work-list builder shared by the attention kernels and the
// CUDA-core kernel used for fp32 inputs (one warp per query, fp32 online softmax).
// bf16 inputs run on the tensor-core kernel in attention_tc.cu.
#include "common.cuh"

namespace scope {

cudaError_t attention_tc_run(const AttnArgs &a, cudaStream_t s);

namespace {

// Work list: one item per kAttnTile queries of one (bh, cluster), head-major.
// Single block; counter[0] = number of items, counter[1] = 0 (scheduler).
__global__ void __launch_bounds__(1024) attn_items_kernel(AttnArgs a)
{
    __shared__ int wsum[32];
    __shared__ int carry;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int total = a.BH * a.Cq;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < total; base += 1024) {
        const int u = base + tid;
        int nq = 0, q0 = 0, bh = 0, c = 0;
        if (u < total) {
            bh = u / a.Cq;
            c = u - bh * a.Cq;
            const int32_t *off = a.off + (size_t)bh * a.off_bh;
            q0 = off[c];
            nq = off[c + 1] - q0;
            if (a.final_cnt[u] <= 0) nq = 0;   // nothing selected: output written as zeros below
        }
        const int tiles = (nq + kAttnTile - 1) / kAttnTile;
        int v = tiles;
        for (int o = 1; o < 32; o <<= 1) {
            int n = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += n;
        }
        if (lane == 31) wsum[w] = v;
        __syncthreads();
        if (w == 0) {
            int s = wsum[lane];
            for (int o = 1; o < 32; o <<= 1) {
                int n = __shfl_up_sync(0xffffffffu, s, o);
                if (lane >= o) s += n;
            }
            wsum[lane] = s;
        }
        __syncthreads();
        int pos = carry + v - tiles + (w ? wsum[w - 1] : 0);
        for (int t = 0; t < tiles; ++t) {
            const int qs = q0 + t * kAttnTile;
            a.items[pos + t] = make_int4(bh, c, qs, min(kAttnTile, q0 + nq - qs));
        }
        __syncthreads();
        if (tid == 0) carry += wsum[31];
        __syncthreads();
    }
    if (tid == 0) {
        a.counter[0] = carry;
        a.counter[1] = 0;
    }
}

// Expands the selection bitmask of every (bh, cluster) that has queries into its
// ascending list of selected key indices (the gather order of the attention kernel).
// grid = BH*Cq units, 256 threads.  Per chunk of 256 mask words: one word per thread,
// a block prefix sum of the popcounts, then each warp writes its 32 words one word at
// a time with lane l handling bit l, so consecutive selected keys go to consecutive
// addresses (coalesced stores).
__global__ void __launch_bounds__(256) attn_lists_kernel(AttnArgs a)
{
    __shared__ int wsum[8];
    const int u = blockIdx.x, tid = threadIdx.x, lane = tid & 31, w8 = tid >> 5;
    const int bh = u / a.Cq, c = u - bh * a.Cq;
    const int32_t *off = a.off + (size_t)bh * a.off_bh;
    if (off[c + 1] == off[c] || a.final_cnt[u] <= 0) return;
    const uint32_t *row = a.mask + (size_t)u * a.nw;
    int32_t *out = a.lists + (size_t)u * a.list_stride;
    const uint32_t below = (1u << lane) - 1u;
    int base = 0;
    for (int w0 = 0; w0 < a.nw; w0 += 256) {
        const int w = w0 + tid;
        uint32_t bits = 0;
        if (w < a.nw) {
            bits = row[w];
            if (w == a.nw - 1 && (a.N & 31)) bits &= (1u << (a.N & 31)) - 1u;
        }
        const int pc = __popc(bits);
        int incl = pc;
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        if (lane == 31) wsum[w8] = incl;
        __syncthreads();
        int before = 0, total = 0;
        for (int k = 0; k < 8; ++k) {
            before += k < w8 ? wsum[k] : 0;
            total += wsum[k];
        }
        const int excl = base + before + incl - pc;   // list position of this word's first key
        const int wbase = (w0 + w8 * 32) * 32;        // key index of bit 0 of the warp's word 0
#pragma unroll 4
        for (int k = 0; k < 32; ++k) {
            const uint32_t bk = __shfl_sync(0xffffffffu, bits, k);
            const int pk = __shfl_sync(0xffffffffu, excl, k);
            if ((bk >> lane) & 1u) out[pk + __popc(bk & below)] = wbase + k * 32 + lane;
        }
        base += total;
        __syncthreads();
    }
}

// Queries of clusters that select no key get zeros.
__global__ void attn_zero_empty_kernel(AttnArgs a)
{
    const int u = blockIdx.x;
    const int bh = u / a.Cq, c = u - bh * a.Cq;
    if (a.final_cnt[u] > 0) return;
    const int32_t *off = a.off + (size_t)bh * a.off_bh;
    const int32_t *perm = a.perm + (size_t)bh * a.perm_bh;
    for (int m = off[c]; m < off[c + 1]; ++m) {
        const long long row = ((long long)bh * a.N + perm[m]) * a.d;
        for (int e = threadIdx.x; e < a.d; e += blockDim.x) {
            if (a.is_bf16)
                reinterpret_cast<__nv_bfloat16 *>(a.O)[row + e] = __float2bfloat16(0.f);
            else
                reinterpret_cast<float *>(a.O)[row + e] = 0.f;
        }
    }
}

// One warp per query; lane l owns channels l, l+32, ... (d/32 of them).
template <int D>
__global__ void __launch_bounds__(256) attn_simt_kernel(AttnArgs a)
{
    constexpr int PER = D / 32;
    const int lane = threadIdx.x & 31;
    const long long gw = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const long long total = (long long)a.BH * a.N;
    if (gw >= total) return;
    const int bh = (int)(gw / a.N);
    const int m = (int)(gw - (long long)bh * a.N);   // position in the cluster-sorted order
    const int i = a.perm[(size_t)bh * a.perm_bh + m];
    // cluster of query i: locate m in the offsets (binary search)
    const int32_t *off = a.off + (size_t)bh * a.off_bh;
    int lo = 0, hi = a.Cq;   // off[lo] <= m < off[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (off[mid] <= m) lo = mid; else hi = mid;
    }
    const int c = lo;
    if (a.final_cnt[(size_t)bh * a.Cq + c] <= 0) return;
    const uint32_t *row = a.mask + ((size_t)bh * a.Cq + c) * a.nw;
    const long long qrow = ((long long)bh * a.N + i) * D;
    float q[PER], o[PER];
#pragma unroll
    for (int k = 0; k < PER; ++k) {
        q[k] = load_x(a.Q, qrow + lane + 32 * k, a.is_bf16);
        o[k] = 0.f;
    }
    float mx = -INFINITY, l = 0.f;
    for (int w = 0; w < a.nw; ++w) {
        unsigned bits = row[w];
        if (w == a.nw - 1 && (a.N & 31)) bits &= (1u << (a.N & 31)) - 1u;   // keys >= N
        while (bits) {
            const int j = w * 32 + __ffs(bits) - 1;
            bits &= bits - 1;
            const long long krow = ((long long)bh * a.N + j) * D;
            float part = 0.f;
#pragma unroll
            for (int k = 0; k < PER; ++k) part = fmaf(q[k], load_x(a.K, krow + lane + 32 * k, a.is_bf16), part);
            for (int s = 16; s; s >>= 1) part += __shfl_xor_sync(0xffffffffu, part, s);
            const float t = part * a.scale_log2;
            const float mn = fmaxf(mx, t);
            const float corr = exp2f(mx - mn);
            const float p = exp2f(t - mn);
            l = l * corr + p;
#pragma unroll
            for (int k = 0; k < PER; ++k)
                o[k] = fmaf(p, load_x(a.V, krow + lane + 32 * k, a.is_bf16), o[k] * corr);
            mx = mn;
        }
    }
    const float inv = 1.f / l;
#pragma unroll
    for (int k = 0; k < PER; ++k) {
        const long long idx = qrow + lane + 32 * k;
        if (a.is_bf16)
            reinterpret_cast<__nv_bfloat16 *>(a.O)[idx] = __float2bfloat16(o[k] * inv);
        else
            reinterpret_cast<float *>(a.O)[idx] = o[k] * inv;
    }
}

}  // namespace

cudaError_t attention_items(const AttnArgs &a, cudaStream_t s)
{
    attn_items_kernel<<<1, 1024, 0, s>>>(a);
    attn_zero_empty_kernel<<<a.BH * a.Cq, 128, 0, s>>>(a);
    if (a.is_bf16 && a.use_tc) attn_lists_kernel<<<a.BH * a.Cq, 256, 0, s>>>(a);
    return cudaGetLastError();
}

namespace {

__global__ void dense_counts_kernel(int32_t *final_counts, long long BH, int N)
{
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < BH; i += (long long)gridDim.x * blockDim.x)
        final_counts[i] = N;
}

}  // namespace

// Dense attention as one query cluster selecting every key: q_assign = 0, every mask bit
// set (bits past N are ignored by the list kernel), r_0 = N.
cudaError_t attention_dense_setup(uint16_t *q_assign, uint32_t *mask, int32_t *final_counts, long long BH,
                                  long long N, long long nw, cudaStream_t s)
{
    cudaError_t e = cudaMemsetAsync(q_assign, 0, sizeof(uint16_t) * (size_t)(BH * N), s);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(mask, 0xFF, sizeof(uint32_t) * (size_t)(BH * nw), s);
    if (e != cudaSuccess) return e;
    dense_counts_kernel<<<(unsigned)((BH + 255) / 256), 256, 0, s>>>(final_counts, BH, (int)N);
    return cudaGetLastError();
}

cudaError_t attention_simt_run(const AttnArgs &a, cudaStream_t s)
{
    const long long warps = (long long)a.BH * a.N;
    const unsigned grid = (unsigned)((warps + 7) / 8);
    if (a.d == 64)
        attn_simt_kernel<64><<<grid, 256, 0, s>>>(a);
    else
        attn_simt_kernel<128><<<grid, 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t attention_kernel(const AttnArgs &a, cudaStream_t s)
{
    if (a.is_bf16 && a.use_tc) return attention_tc_run(a, s);
    return attention_simt_run(a, s);
}

cudaError_t attention_run(const AttnArgs &a, cudaStream_t s)
{
    cudaError_t e = attention_items(a, s);
    if (e != cudaSuccess) return e;
    return attention_kernel(a, s);
}

}  // namespace scope
