// Proxy-ranking fidelity of SCOPE's selection (review page: the falsifier and the
// skeptic's concrete test ask how many of a query's truly dominant keys the
// centroid-product proxy of Eq. 6 and the selected set retain).
//
// For a sampled query i of head (b, h) in query cluster c:
//   l_j  = q_i . k_j                        (binary64; bf16 or fp32 inputs, products exact)
//   T    = the ceil(frac N) keys with the largest l_j, ties to the lower index
//   P    = the ceil(frac N) keys with the largest proxy logit s~_{c,j} (Eq. 6, the
//          selection's binary64 formula and order), ties to the lower index
//   recall_sel   = |T n S_c| / |T|          (S_c from the selection mask)
//   recall_proxy = |T n P| / |T|
// One block per sample (grid-stride over the samples), 512 threads.  The block writes the
// logits and proxy logits to its own slice of the workspace, finds each k-th largest
// value with a radix select on order-preserving 64-bit keys (8 passes of 8 bits), then
// counts the intersections in one pass in key order (ties resolved by a block prefix
// count, so the sets are exactly the index-ordered ones).
#include "common.cuh"
#include "fid_common.cuh"

#include <cfloat>

namespace scope {

namespace {

constexpr int kFidThreads = 512;

// Order-preserving map of a binary64 value to an unsigned 64-bit key (larger value,
// larger key; -0 and +0 map to adjacent keys, NaN does not occur here).
__device__ __forceinline__ unsigned long long okey(double v)
{
    const unsigned long long b = (unsigned long long)__double_as_longlong(v);
    return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

// The key of the k-th largest value among vals[0..n) (k >= 1) by an MSB-first radix
// select; *above = the number of values with a strictly larger key.
__device__ unsigned long long kth_largest(const double *vals, int n, long long k, int *hist, long long *above)
{
    unsigned long long prefix = 0, mask = 0;
    long long need = k;   // rank to find among the values matching the prefix so far
    long long gt = 0;     // values with larger keys (decided in earlier passes)
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int b = threadIdx.x; b < 256; b += kFidThreads) hist[b] = 0;
        __syncthreads();
        for (int j = threadIdx.x; j < n; j += kFidThreads) {
            const unsigned long long key = okey(vals[j]);
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 0xFF], 1);
        }
        __syncthreads();
        // descending digit order: the digit where the cumulative count reaches `need`
        __shared__ int dsel;
        __shared__ long long dbefore;
        if (threadIdx.x == 0) {
            long long run = 0;
            int d = 0;
            for (d = 255; d >= 0; --d) {
                if (run + hist[d] >= need) break;
                run += hist[d];
            }
            dsel = d < 0 ? 0 : d;
            dbefore = run;
        }
        __syncthreads();
        prefix |= (unsigned long long)dsel << shift;
        mask |= 0xFFull << shift;
        gt += dbefore;
        need -= dbefore;
        __syncthreads();
    }
    *above = gt;
    return prefix;
}

// Membership of key j in a top-k set given its threshold key `thr`, the count `gt` of
// strictly larger keys and the number of ties seen before j (in key order).
__device__ __forceinline__ bool in_top(unsigned long long key, unsigned long long thr, long long gt,
                                       long long ties_before, long long k)
{
    return key > thr || (key == thr && gt + ties_before < k);
}

__global__ void __launch_bounds__(kFidThreads) fidelity_kernel(FidArgs a)
{
    __shared__ double qs[128];
    __shared__ double lut[3 * kMaxFidCm];
    __shared__ int hist[256];
    __shared__ long long wsum[2][kFidThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    double *logit = a.scratch + (size_t)blockIdx.x * 2 * a.N;
    double *proxy = logit + a.N;
    const long long k = a.k;
    for (int si = blockIdx.x; si < a.n_samples; si += gridDim.x) {
        const long long g = a.samples[si];
        if (g < 0 || g >= a.total) {   // not a query of this layer
            if (tid == 0) a.recall_sel[si] = a.recall_proxy[si] = __longlong_as_double(0x7ff8000000000000ll);
            continue;
        }
        const int bh = (int)(g / a.N);
        const int c = min((int)a.q_assign[g], a.Cq - 1);
        sample_logits<kFidThreads>(a, g, logit, proxy, qs, lut);
        long long gt_l, gt_p;
        const unsigned long long thr_l = kth_largest(logit, a.N, k, hist, &gt_l);
        const unsigned long long thr_p = kth_largest(proxy, a.N, k, hist, &gt_p);
        // one pass in key order: ties counted by a block prefix over each chunk
        const uint32_t *mrow = a.mask + ((size_t)bh * a.Cq + c) * a.nw;
        long long tl = 0, tp = 0;     // ties seen before the chunk
        long long n_sel = 0, n_prx = 0;
        for (int base = 0; base < a.N; base += kFidThreads) {
            const int j = base + tid;
            unsigned long long kl = 0, kp = 0;
            int el = 0, ep = 0;
            if (j < a.N) {
                kl = okey(logit[j]);
                kp = okey(proxy[j]);
                el = kl == thr_l;
                ep = kp == thr_p;
            }
            // exclusive block scan of the tie flags
            int il = el, ip = ep;
            for (int o = 1; o < 32; o <<= 1) {
                const int x1 = __shfl_up_sync(0xffffffffu, il, o), x2 = __shfl_up_sync(0xffffffffu, ip, o);
                if (lane >= o) {
                    il += x1;
                    ip += x2;
                }
            }
            if (lane == 31) {
                wsum[0][w] = il;
                wsum[1][w] = ip;
            }
            __syncthreads();
            long long bl = 0, bp = 0, sl = 0, sp = 0;
            for (int q = 0; q < kFidThreads / 32; ++q) {
                if (q < w) {
                    bl += wsum[0][q];
                    bp += wsum[1][q];
                }
                sl += wsum[0][q];
                sp += wsum[1][q];
            }
            bool inT = false, inP = false, inS = false;
            if (j < a.N) {
                inT = in_top(kl, thr_l, gt_l, tl + bl + il - el, k);
                inP = in_top(kp, thr_p, gt_p, tp + bp + ip - ep, k);
                inS = (mrow[j >> 5] >> (j & 31)) & 1u;
            }
            n_sel += (inT && inS) ? 1 : 0;
            n_prx += (inT && inP) ? 1 : 0;
            tl += sl;
            tp += sp;
            __syncthreads();
        }
        // block sums of the two counts
        for (int o = 16; o; o >>= 1) {
            n_sel += __shfl_xor_sync(0xffffffffu, n_sel, o);
            n_prx += __shfl_xor_sync(0xffffffffu, n_prx, o);
        }
        if (lane == 0) {
            wsum[0][w] = n_sel;
            wsum[1][w] = n_prx;
        }
        __syncthreads();
        if (tid == 0) {
            long long s0 = 0, s1 = 0;
            for (int q = 0; q < kFidThreads / 32; ++q) {
                s0 += wsum[0][q];
                s1 += wsum[1][q];
            }
            a.recall_sel[si] = (double)s0 / (double)k;
            a.recall_proxy[si] = (double)s1 / (double)k;
        }
        __syncthreads();
    }
}

}  // namespace

cudaError_t fidelity_run(const FidArgs &a, cudaStream_t s)
{
    int grid = a.blocks;
    if (grid > a.n_samples) grid = a.n_samples;
    if (grid < 1) return cudaSuccess;
    fidelity_kernel<<<grid, kFidThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace scope
