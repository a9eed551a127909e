// Rank correlation of the Eq. 6 proxy logits with the exact logits (review page: the test the
// skeptic asks for, how well the proxy ranking of the keys follows the true one).
//
// For each sampled query i of head (b, h) in cluster c: Spearman's rho over all N keys, the
// Pearson correlation of the two vectors of average ranks (tied values share the mean of
// their 1-based ranks), x = the exact logits q_i . k_j, y = the proxy logits s~_{c,j}.
//   1. rc_values_kernel   one block per sample writes x and y (binary64, the same code as the
//                         recall kernel) as two segments of sort keys, with key indices
//   2. CUB segmented radix sort of the 2 S segments (ascending, keys with their indices)
//   3. rc_ranks_kernel    one block per segment gives every run of equal keys its mean rank
//   4. rc_pearson_kernel  one block per sample: sums of products of centred ranks (binary64)
#include "fid_common.cuh"

#include <cub/device/device_segmented_radix_sort.cuh>

namespace scope {

namespace {

constexpr int kRcThreads = 512;

__global__ void __launch_bounds__(kRcThreads) rc_values_kernel(FidArgs a, double *keys, int32_t *vals, int32_t *bad)
{
    __shared__ double qs[128];
    __shared__ double lut[3 * kMaxFidCm];
    for (int si = blockIdx.x; si < a.n_samples; si += gridDim.x) {
        const long long g = a.samples[si];
        double *x = keys + (size_t)2 * si * a.N, *y = x + a.N;
        int32_t *v = vals + (size_t)2 * si * a.N;
        const bool ok = g >= 0 && g < a.total;
        if (threadIdx.x == 0) bad[si] = ok ? 0 : 1;
        if (ok) {
            sample_logits<kRcThreads>(a, g, x, y, qs, lut);
        } else {
            for (int j = threadIdx.x; j < a.N; j += kRcThreads) x[j] = y[j] = 0.0;
        }
        for (int j = threadIdx.x; j < a.N; j += kRcThreads) v[j] = v[a.N + j] = j;
        __syncthreads();
    }
}

__global__ void rc_offsets_kernel(int32_t *off, int nseg, int N)
{
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i <= nseg; i += gridDim.x * blockDim.x) off[i] = i * N;
}

// Mean 1-based rank of every run of equal keys in one sorted segment, scattered back to the
// keys' original positions.  A thread that starts a run walks it.
__global__ void __launch_bounds__(kRcThreads) rc_ranks_kernel(const double *skeys, const int32_t *svals, double *ranks,
                                                              int N)
{
    const size_t base = (size_t)blockIdx.x * N;
    const double *k = skeys + base;
    const int32_t *v = svals + base;
    double *r = ranks + base;
    for (int p = threadIdx.x; p < N; p += kRcThreads) {
        if (p > 0 && k[p] == k[p - 1]) continue;   // not the start of a run
        int hi = p + 1;
        while (hi < N && k[hi] == k[p]) ++hi;
        const double mean = 0.5 * (double)(p + 1 + hi);   // mean of ranks p+1 .. hi
        for (int q = p; q < hi; ++q) r[min(max(v[q], 0), N - 1)] = mean;
    }
}

__global__ void __launch_bounds__(kRcThreads) rc_pearson_kernel(const double *ranks, const int32_t *bad, int N,
                                                                double *out, int n_samples)
{
    __shared__ double red[3][kRcThreads / 32];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    for (int si = blockIdx.x; si < n_samples; si += gridDim.x) {
        const double *rx = ranks + (size_t)2 * si * N, *ry = rx + N;
        const double mu = 0.5 * ((double)N + 1.0);
        double sxy = 0.0, sxx = 0.0, syy = 0.0;
        for (int j = threadIdx.x; j < N; j += kRcThreads) {
            const double dx = rx[j] - mu, dy = ry[j] - mu;
            sxy = fma(dx, dy, sxy);
            sxx = fma(dx, dx, sxx);
            syy = fma(dy, dy, syy);
        }
        for (int o = 16; o; o >>= 1) {
            sxy += __shfl_xor_sync(0xffffffffu, sxy, o);
            sxx += __shfl_xor_sync(0xffffffffu, sxx, o);
            syy += __shfl_xor_sync(0xffffffffu, syy, o);
        }
        if (lane == 0) {
            red[0][w] = sxy;
            red[1][w] = sxx;
            red[2][w] = syy;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            double a = 0.0, b = 0.0, c = 0.0;
            for (int q = 0; q < kRcThreads / 32; ++q) {
                a += red[0][q];
                b += red[1][q];
                c += red[2][q];
            }
            const double den = sqrt(b * c);
            out[si] = (bad[si] || !(den > 0.0)) ? __longlong_as_double(0x7ff8000000000000ll) : a / den;
        }
        __syncthreads();
    }
}

struct RcLayout {
    size_t keys, keys_out, vals, vals_out, ranks, off, bad, temp, temp_bytes, total;
};

size_t align256(size_t x)
{
    return (x + 255) / 256 * 256;
}

RcLayout rc_layout(int N, int S)
{
    RcLayout L{};
    const size_t items = (size_t)2 * S * N;
    size_t temp = 0;
    cub::DeviceSegmentedRadixSort::SortPairs(nullptr, temp, (const double *)nullptr, (double *)nullptr,
                                             (const int32_t *)nullptr, (int32_t *)nullptr, (int)items, 2 * S,
                                             (const int32_t *)nullptr, (const int32_t *)nullptr + 1);
    size_t o = 0;
    L.keys = o;
    o = align256(o + items * 8);
    L.keys_out = o;
    o = align256(o + items * 8);
    L.vals = o;
    o = align256(o + items * 4);
    L.vals_out = o;
    o = align256(o + items * 4);
    L.ranks = o;
    o = align256(o + items * 8);
    L.off = o;
    o = align256(o + (size_t)(2 * S + 1) * 4);
    L.bad = o;
    o = align256(o + (size_t)S * 4);
    L.temp = o;
    L.temp_bytes = temp;
    L.total = align256(o + temp);
    return L;
}

}  // namespace

size_t rank_corr_scratch_bytes(int N, int n_samples)
{
    return rc_layout(N, n_samples).total;
}

cudaError_t rank_corr_run(const FidArgs &a, double *spearman, void *scratch, int num_sms, cudaStream_t s)
{
    const int S = a.n_samples, N = a.N;
    const RcLayout L = rc_layout(N, S);
    char *base = static_cast<char *>(scratch);
    double *keys = reinterpret_cast<double *>(base + L.keys), *keys_out = reinterpret_cast<double *>(base + L.keys_out);
    int32_t *vals = reinterpret_cast<int32_t *>(base + L.vals), *vals_out = reinterpret_cast<int32_t *>(base + L.vals_out);
    double *ranks = reinterpret_cast<double *>(base + L.ranks);
    int32_t *off = reinterpret_cast<int32_t *>(base + L.off), *bad = reinterpret_cast<int32_t *>(base + L.bad);
    const int grid = S < num_sms ? S : num_sms;
    rc_values_kernel<<<grid, kRcThreads, 0, s>>>(a, keys, vals, bad);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    rc_offsets_kernel<<<(2 * S + 256) / 256, 256, 0, s>>>(off, 2 * S, N);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    size_t temp = L.temp_bytes;
    e = cub::DeviceSegmentedRadixSort::SortPairs(base + L.temp, temp, keys, keys_out, vals, vals_out, 2 * S * N, 2 * S,
                                                 off, off + 1, 0, 64, s);
    if (e != cudaSuccess) return e;
    rc_ranks_kernel<<<2 * S, kRcThreads, 0, s>>>(keys_out, vals_out, ranks, N);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    rc_pearson_kernel<<<grid, kRcThreads, 0, s>>>(ranks, bad, N, spearman, S);
    return cudaGetLastError();
}

}  // namespace scope
