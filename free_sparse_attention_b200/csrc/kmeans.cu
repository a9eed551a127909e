// Lloyd k-means for SCOPE's query clustering and key-subspace clustering.
//
// SCOPE (arXiv 2608.12780) clusters post-RoPE queries (Cq centroids) and, per 3D-RoPE
// subspace, post-RoPE keys (Cm centroids each) with k-means minimising the Euclidean
// reconstruction error (review page, load_bearing_attack: Eq. 3).  One iteration:
// every token goes to its nearest centroid (lowest index on a tie), then every
// non-empty centroid moves to the mean of its members.
//
// Design (B200): the assignment is a [tokens x dm] x [dm x C] contraction followed by
// an argmin.  For bf16 inputs it runs on the tensor cores (kmeans_tc.cu, whose error
// bound rests on a measured model of the tensor core's accumulation); otherwise
// (fp32 inputs, or centroid sets too large for shared memory) on the fp32 FMA pipes
// with centroids staged in shared memory (km_assign_fast_kernel below), where each
// distance carries an error bound proven from IEEE binary32 arithmetic.  A token whose
// best and runner-up cannot be told apart under its bound is re-decided in binary64
// with the channels summed in order (one rounding per operation).  Hence the assignment
// equals a binary64 evaluation of the definition exactly.  The update sums each centroid's
// members in increasing token order in binary64: a stable counting sort by cluster
// gives every (centroid, channel) pair its member list, so the sum is sequential and
// the means are bit-identical to an in-order binary64 evaluation.
#include "common.cuh"

#include <cfloat>

namespace scope {

namespace {

constexpr int kTok = 128;     // tokens per CTA in the fast assignment
constexpr int kCC = 64;       // centroids per shared-memory chunk
constexpr int kAssignThreads = 256;
constexpr uint16_t kUnsure = 0xFFFF;

__device__ __forceinline__ const RoleDesc &role_of(const KmArgs &a, int p, int &bh, int &r)
{
    r = p % a.nroles;
    bh = p / a.nroles;
    return a.role[a.role0 + r];
}

// fp32 and binary64 transposed copies, norms and the error-bound term of one centroid
// row (cent64 has dm values, all written before the caller's barrier).  Thread i
// handles channel i.
__device__ void finalize_row(const KmArgs &a, int p, int c, const double *cent64, int dm, int i)
{
    float *cent32T = a.cent32 + (size_t)p * a.Cs * a.ds;
    cent32T[(size_t)i * a.Cs + c] = __double2float_rn(cent64[i]);
    a.cent64T[(size_t)p * a.Cs * a.ds + (size_t)i * a.Cs + c] = cent64[i];
    if (i == 0) {
        double n2 = 0.0, n32 = 0.0;
        for (int k = 0; k < dm; ++k) {
            double m = cent64[k];
            double m32 = (double)__double2float_rn(m);
            n2 += m * m;
            n32 += m32 * m32;
        }
        a.cnrm2[(size_t)p * a.Cs + c] = __double2float_rn(n2);
        a.cnorm[(size_t)p * a.Cs + c] = __double2float_ru(sqrt(n32));
        a.cslack[(size_t)p * a.Cs + c] = __double2float_ru(ldexp(n2, -22));
    }
}

// ------------------------------------------------------------------------- init
// grid (ceil(Cs/G), P), block 128: a group of dm threads per centroid.
__global__ void __launch_bounds__(128) km_init_kernel(KmArgs a)
{
    int bh, r;
    const int p = blockIdx.y;
    const RoleDesc &R = role_of(a, p, bh, r);
    const int dm = R.dm, G = max(1, 128 / dm);
    const int g = threadIdx.x / dm, i = threadIdx.x % dm;
    const int c = blockIdx.x * G + g;
    const bool active = g < G && c < R.C;
    double *cent = R.cent + ((size_t)bh * R.C + c) * a.d + R.ch0;
    if (active) {
        if (R.init_idx) {
            int row = R.init_idx[(size_t)bh * R.init_bh + c];
            if (row < 0 || row >= a.N) {
                if (i == 0) set_status(a.status, SCOPE_DEV_BAD_INIT_INDEX);
                row = 0;
            }
            cent[i] = (double)load_x(R.X, ((long long)bh * a.N + row) * a.d + R.ch0 + i, a.is_bf16);
        } else {
            cent[i] = R.init_cent[((size_t)bh * R.C + c) * a.d + R.ch0 + i];
        }
    }
    __syncthreads();
    if (active) finalize_row(a, p, c, cent, dm, i);
}

// ------------------------------------------------------------------------- fast assignment
// grid (ceil(N/kTok), P), block 256.  Thread (ty, tx): tokens ty*8..+8, chunk
// centroids tx*4..+4.  For every pair the fp32 score A = |mu|^2 - 2 x.mu approximates
// S = |mu|^2 - 2 x.mu (exact, binary64 mu) within
//     E = 2^-22 ((dm+3) |x| |mu| + |mu|^2) + 2^-40 |x|^2,
// twice the first-order bound of the three roundings (mu to fp32, the fp32 dot
// product, the final subtraction) plus the binary64 rounding of the reference sum.
// With L = A - E and U = A + E, the token's winner is certain when the second-smallest
// L exceeds the smallest U; otherwise the token is marked for the exact path.
__global__ void __launch_bounds__(kAssignThreads) km_assign_fast_kernel(KmArgs a)
{
    int bh, r;
    const int p = blockIdx.y;
    const RoleDesc &R = role_of(a, p, bh, r);
    const int dm = R.dm, C = R.C;
    const int j0 = blockIdx.x * kTok;
    if (j0 >= a.N) return;
    extern __shared__ __align__(16) float sm[];
    float *Xs = sm;                     // [dm][kTok]
    float *Ms = Xs + dm * kTok;         // [dm][kCC]
    float *Mn2 = Ms + dm * kCC;         // [kCC]
    float *Mnorm = Mn2 + kCC;           // [kCC]
    float *Mslack = Mnorm + kCC;        // [kCC]
    float *Xn = Mslack + kCC;           // [kTok]

    const int tid = threadIdx.x;
    for (int idx = tid; idx < kTok * dm; idx += kAssignThreads) {
        int t = idx / dm, i = idx - t * dm;
        int j = j0 + t;
        float v = 0.f;
        if (j < a.N) v = load_x(R.X, ((long long)bh * a.N + j) * a.d + R.ch0 + i, a.is_bf16);
        Xs[i * kTok + t] = v;
    }
    __syncthreads();
    if (tid < kTok) {
        float s = 0.f;
        for (int i = 0; i < dm; ++i) s = fmaf(Xs[i * kTok + tid], Xs[i * kTok + tid], s);
        Xn[tid] = sqrtf(s) * (1.0f + 0x1p-12f);
    }
    const int ty = tid >> 4, tx = tid & 15;
    float xk[8], e0[8], minL[8], min2L[8], minU[8];
    int idxL[8];
    __syncthreads();
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        float xn = Xn[ty * 8 + t];
        xk[t] = 0x1p-22f * (float)(dm + 3) * xn;
        e0[t] = 0x1p-40f * xn * xn;
        minL[t] = FLT_MAX;
        min2L[t] = FLT_MAX;
        minU[t] = FLT_MAX;
        idxL[t] = 0;
    }
    const float *cent32T = a.cent32 + (size_t)p * a.Cs * a.ds;
    const float *cn2 = a.cnrm2 + (size_t)p * a.Cs;
    const float *cnm = a.cnorm + (size_t)p * a.Cs;
    const float *csl = a.cslack + (size_t)p * a.Cs;

    for (int c0 = 0; c0 < C; c0 += kCC) {
        __syncthreads();
        for (int idx = tid; idx < dm * kCC; idx += kAssignThreads) {
            int i = idx / kCC, cc = idx - i * kCC;
            Ms[idx] = (c0 + cc < C) ? cent32T[(size_t)i * a.Cs + c0 + cc] : 0.f;
        }
        if (tid < kCC) {
            bool ok = c0 + tid < C;
            Mn2[tid] = ok ? cn2[c0 + tid] : INFINITY;
            Mnorm[tid] = ok ? cnm[c0 + tid] : 0.f;
            Mslack[tid] = ok ? csl[c0 + tid] : 0.f;
        }
        __syncthreads();
        float acc[8][4];
#pragma unroll
        for (int t = 0; t < 8; ++t)
#pragma unroll
            for (int b = 0; b < 4; ++b) acc[t][b] = 0.f;
#pragma unroll 4
        for (int i = 0; i < dm; ++i) {
            const float4 xa = *reinterpret_cast<const float4 *>(Xs + i * kTok + ty * 8);
            const float4 xb = *reinterpret_cast<const float4 *>(Xs + i * kTok + ty * 8 + 4);
            const float4 m = *reinterpret_cast<const float4 *>(Ms + i * kCC + tx * 4);
            const float xv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
            const float mv[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
            for (int t = 0; t < 8; ++t)
#pragma unroll
                for (int b = 0; b < 4; ++b) acc[t][b] = fmaf(xv[t], mv[b], acc[t][b]);
        }
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int cc = tx * 4 + b;
            const float n2 = Mn2[cc], nm = Mnorm[cc], sl = Mslack[cc];
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                float A = fmaf(-2.f, acc[t][b], n2);
                float E = fmaf(xk[t], nm, sl + e0[t]);
                float L = A - E, U = A + E;
                if (L < minL[t]) {
                    min2L[t] = minL[t];
                    minL[t] = L;
                    idxL[t] = c0 + cc;
                } else if (L < min2L[t]) {
                    min2L[t] = L;
                }
                minU[t] = fminf(minU[t], U);
            }
        }
    }
    // merge the 16 partial states of each token (lanes sharing ty)
#pragma unroll
    for (int t = 0; t < 8; ++t) {
#pragma unroll
        for (int off = 1; off < 16; off <<= 1) {
            float oL = __shfl_xor_sync(0xffffffffu, minL[t], off);
            float o2 = __shfl_xor_sync(0xffffffffu, min2L[t], off);
            float oU = __shfl_xor_sync(0xffffffffu, minU[t], off);
            int oi = __shfl_xor_sync(0xffffffffu, idxL[t], off);
            if (oL < minL[t] || (oL == minL[t] && oi < idxL[t])) {
                min2L[t] = fminf(o2, minL[t]);
                minL[t] = oL;
                idxL[t] = oi;
            } else {
                min2L[t] = fminf(min2L[t], oL);
            }
            minU[t] = fminf(minU[t], oU);
        }
    }
    // lane tx writes token ty*8 + tx for tx < 8; undecided tokens go to the exact list
    bool unsure = false;
    int32_t entry = 0;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        if (tx == t) {
            int j = j0 + ty * 8 + t;
            if (j < a.N) {
                bool sure = min2L[t] > minU[t];
                R.assign[(size_t)bh * R.assign_bh + j] = sure ? (uint16_t)SCOPE_DCHECK(idxL[t], R.C, a.status) : kUnsure;
                unsure = !sure;
                entry = bh * a.N + j;
            }
        }
    }
    warp_append(unsure, entry, a.unsure_list + (size_t)r * a.BH * a.N, a.unsure_count + r);
}

// ------------------------------------------------------------------------- exact assignment
// One warp per listed unsure token (grid-stride over the list the fast kernels filled);
// the token is re-decided in binary64 against all centroids.  The token's channels go
// to shared memory; lane l takes centroids l, l+32, ... two at a time, reading the
// channel-major binary64 copy (consecutive lanes, consecutive centroids), and sums the
// squared differences in channel order with one rounding per operation, as the
// definition is evaluated.
constexpr int kExactWarps = 8;

__global__ void __launch_bounds__(kExactWarps * 32) km_assign_exact_kernel(KmArgs a)
{
    __shared__ double xs[kExactWarps][128];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    int cnt[4], total = 0;
    for (int r = 0; r < a.nroles; ++r) total += (cnt[r] = a.unsure_count[r]);
    for (int g = blockIdx.x * kExactWarps + wib; g < total; g += gridDim.x * kExactWarps) {
        int r = 0, k = g;
        while (k >= cnt[r]) k -= cnt[r++];
        const int entry = a.unsure_list[(size_t)r * a.BH * a.N + k];
        const int bh = entry / a.N, jj = entry - bh * a.N;
        const int p = bh * a.nroles + r;
        const RoleDesc &R = a.role[a.role0 + r];
        const double *muT = a.cent64T + (size_t)p * a.Cs * a.ds;
        const long long xrow = ((long long)bh * a.N + jj) * a.d + R.ch0;
        __syncwarp();
        for (int i = lane; i < R.dm; i += 32) xs[wib][i] = (double)load_x(R.X, xrow + i, a.is_bf16);
        __syncwarp();
        // lane takes centroids lane, lane + 32, ... in ascending order, four at a time (four
        // independent binary64 sums, each over the channels in order)
        double best = INFINITY;
        int bi = 0x7fffffff;
        constexpr int kChains = 4;
        for (int c = lane; c < R.C; c += 32 * kChains) {
            int cc[kChains];
            double dd[kChains];
#pragma unroll
            for (int k = 0; k < kChains; ++k) {
                cc[k] = min(c + 32 * k, R.C - 1);
                dd[k] = 0.0;
            }
            for (int i = 0; i < R.dm; ++i) {
                const double x = xs[wib][i];
                const double *mrow = muT + (size_t)i * a.Cs;
#pragma unroll
                for (int k = 0; k < kChains; ++k) {
                    const double e = __dsub_rn(x, mrow[cc[k]]);
                    dd[k] = __dadd_rn(dd[k], __dmul_rn(e, e));
                }
            }
#pragma unroll
            for (int k = 0; k < kChains; ++k) {
                if (c + 32 * k < R.C && dd[k] < best) {
                    best = dd[k];
                    bi = c + 32 * k;
                }
            }
        }
        for (int off = 16; off; off >>= 1) {
            double ob = __shfl_xor_sync(0xffffffffu, best, off);
            int oi = __shfl_xor_sync(0xffffffffu, bi, off);
            if (ob < best || (ob == best && oi < bi)) {
                best = ob;
                bi = oi;
            }
        }
        if (lane == 0) R.assign[(size_t)bh * R.assign_bh + jj] = (uint16_t)bi;
    }
}

// ------------------------------------------------------------------------- counting sort
// Chunk histogram: one warp per chunk of kSortChunk tokens, block of 4 warps.
__global__ void __launch_bounds__(128) sort_hist_kernel(KmArgs a)
{
    extern __shared__ int hs[];
    const int w = threadIdx.x / 32, lane = threadIdx.x & 31;
    const int k = blockIdx.x * 4 + w;
    const int p = blockIdx.y;
    int bh, r;
    const RoleDesc &R = role_of(a, p, bh, r);
    if (k >= a.nchunk) return;
    int *h = hs + w * a.Cs;
    for (int c = lane; c < R.C; c += 32) h[c] = 0;
    __syncwarp();
    const uint16_t *asg = R.assign + (size_t)bh * R.assign_bh;
    const int jend = min(a.N, (k + 1) * kSortChunk);
    for (int j = k * kSortChunk + lane; j < jend; j += 32) {
        int z = asg[j];
        if (z >= R.C) {   // only a caller-supplied assignment can be out of range
            set_status(a.status, SCOPE_DEV_BAD_ASSIGN);
            z = R.C - 1;
        }
        atomicAdd(&h[z], 1);
    }
    __syncwarp();
    int32_t *out = a.chunk_hist + ((size_t)p * a.nchunk + k) * a.Cs;
    for (int c = lane; c < R.C; c += 32) out[c] = h[c];
}

// Per problem: prefix over chunks for every cluster, sizes, and cluster offsets.
constexpr int kScanBatch = 16;

__global__ void __launch_bounds__(1024) sort_scan_kernel(KmArgs a)
{
    __shared__ int wsum[32];
    const int p = blockIdx.x;
    int bh, r;
    const RoleDesc &R = role_of(a, p, bh, r);
    const int C = R.C;
    const int per = (C + 1023) / 1024;
    int loc[4];  // C <= 4096
    int tot = 0;
    for (int q = 0; q < per; ++q) {
        int c = threadIdx.x * per + q;
        int run = 0;
        if (c < C) {
            // the column's chunk counts are read kScanBatch at a time (independent loads in
            // flight), then replaced by their exclusive prefix
            int32_t *col = a.chunk_hist + (size_t)p * a.nchunk * a.Cs + c;
            int k = 0;
            for (; k + kScanBatch <= a.nchunk; k += kScanBatch) {
                int h[kScanBatch];
#pragma unroll
                for (int q = 0; q < kScanBatch; ++q) h[q] = col[(size_t)(k + q) * a.Cs];
#pragma unroll
                for (int q = 0; q < kScanBatch; ++q) {
                    col[(size_t)(k + q) * a.Cs] = run;
                    run += h[q];
                }
            }
            for (; k < a.nchunk; ++k) {
                const int h = col[(size_t)k * a.Cs];
                col[(size_t)k * a.Cs] = run;
                run += h;
            }
            R.sizes[(size_t)bh * R.sizes_bh + c] = run;
        }
        loc[q] = run;
        tot += run;
    }
    // exclusive block scan of tot
    const int lane = threadIdx.x & 31, wid = threadIdx.x / 32;
    int v = tot;
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) wsum[wid] = v;
    __syncthreads();
    if (wid == 0) {
        int s = wsum[lane];
        for (int o = 1; o < 32; o <<= 1) {
            int n = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += n;
        }
        wsum[lane] = s;
    }
    __syncthreads();
    int excl = v - tot + (wid ? wsum[wid - 1] : 0);
    int32_t *off = a.off + (size_t)p * (a.Cs + 1);
    for (int q = 0; q < per; ++q) {
        int c = threadIdx.x * per + q;
        if (c < C) off[c] = excl;
        excl += loc[q];
    }
    if (threadIdx.x == 0) off[C] = a.N;
}

// Stable scatter: warp k walks its chunk in token order, 32 tokens at a time.
__global__ void __launch_bounds__(128) sort_scatter_kernel(KmArgs a)
{
    extern __shared__ int cs[];
    const int w = threadIdx.x / 32, lane = threadIdx.x & 31;
    const int k = blockIdx.x * 4 + w;
    const int p = blockIdx.y;
    int bh, r;
    const RoleDesc &R = role_of(a, p, bh, r);
    if (k >= a.nchunk) return;
    int *cnt = cs + w * a.Cs;
    const int32_t *off = a.off + (size_t)p * (a.Cs + 1);
    const int32_t *pre = a.chunk_hist + ((size_t)p * a.nchunk + k) * a.Cs;
    for (int c = lane; c < R.C; c += 32) cnt[c] = off[c] + pre[c];
    __syncwarp();
    const uint16_t *asg = R.assign + (size_t)bh * R.assign_bh;
    int32_t *perm = a.perm + (size_t)p * a.N;
    const int jend = min(a.N, (k + 1) * kSortChunk);
    for (int jb = k * kSortChunk; jb < jend; jb += 32) {
        const int j = jb + lane;
        const int z = j < jend ? min((int)asg[j], R.C - 1) : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, z);
        const int leader = __ffs(peers) - 1;
        const int rank = __popc(peers & ((1u << lane) - 1u));
        int base = (lane == leader && z >= 0) ? cnt[z] : 0;
        base = __shfl_sync(0xffffffffu, base, leader);
        if (z >= 0) perm[SCOPE_DCHECK(base + rank, a.N, a.status)] = j;
        __syncwarp();
        if (lane == leader && z >= 0) cnt[z] = base + __popc(peers);
        __syncwarp();
    }
}

// ------------------------------------------------------------------------- update
// grid (Cs, P), block kUpdThreads: one centroid per block.  Thread (s, g) sums channels
// CH*g .. CH*g+CH-1 over segment s of the member list (members in token order, the list
// split into S = kUpdThreads / (dm / CH) contiguous segments) in binary64, and records
// the smallest ulp among its nonzero values and the sum of magnitudes.  Every input
// value is an integer multiple of the smallest ulp u, so every partial sum in any order
// is too; when the sum of magnitudes stays below 2^52 u (a factor 2 of margin under
// 2^53 u), every partial sum is exactly representable and the segment sums add up (in
// segment order) to exactly the in-order binary64 sum.  Otherwise, or for subnormal
// inputs, that channel is summed again sequentially.  The mean is the sum divided by the
// member count (one rounding).  bf16 inputs whose channel range starts and ends on an
// even channel are read two channels (4 bytes) per load.
constexpr int kUpdThreads = 256;
constexpr int kUpdUnroll = 16;

// Value and ulp exponent of one input element (bf16: 8 significant bits, fp32: 24); a
// subnormal gives INT_MIN (no usable bound), 0 gives INT_MAX (no ulp).
__device__ __forceinline__ void elem_bf16(uint32_t b16, double &x, int &e)
{
    x = (double)__uint_as_float(b16 << 16);
    const int be = (b16 >> 7) & 0xFF;
    e = (b16 & 0x7FFF) == 0 ? 0x7fffffff : (be == 0 ? (int)0x80000000 : be - 127 - 7);
}

__device__ __forceinline__ void elem_f32(uint32_t b32, double &x, int &e)
{
    x = (double)__uint_as_float(b32);
    const int be = (b32 >> 23) & 0xFF;
    e = (b32 & 0x7FFFFFFF) == 0 ? 0x7fffffff : (be == 0 ? (int)0x80000000 : be - 127 - 23);
}

template <int CH>
__global__ void __launch_bounds__(kUpdThreads) km_update_kernel(KmArgs a)
{
    __shared__ double psum[kUpdThreads * CH], pabs[kUpdThreads * CH];
    __shared__ int pexp[kUpdThreads * CH];
    int bh, r;
    const int p = blockIdx.y, c = blockIdx.x;
    const RoleDesc &R = role_of(a, p, bh, r);
    const int dm = R.dm, dmc = dm / CH, S = kUpdThreads / dmc;
    const int s = threadIdx.x / dmc, g = threadIdx.x - s * dmc;
    const bool active = c < R.C;
    const int32_t *off = a.off + (size_t)p * (a.Cs + 1);
    const int32_t *perm = a.perm + (size_t)p * a.N;
    const int beg = active ? off[c] : 0, end = active ? off[c + 1] : 0, n = end - beg;
    double *cent = R.cent + ((size_t)bh * R.C + (active ? c : 0)) * a.d + R.ch0;
    const long long base = (long long)bh * a.N * a.d + R.ch0 + CH * g;   // element index
    if (s < S && n > 0) {
        const int m0 = beg + (int)((long long)n * s / S), m1 = beg + (int)((long long)n * (s + 1) / S);
        double acc[CH], mag[CH];
        int emin[CH];
#pragma unroll
        for (int h = 0; h < CH; ++h) {
            acc[h] = 0.0;
            mag[h] = 0.0;
            emin[h] = 0x7fffffff;
        }
        auto take = [&](uint32_t bits) {
#pragma unroll
            for (int h = 0; h < CH; ++h) {
                double x;
                int e;
                if (CH == 2)
                    elem_bf16(h ? bits >> 16 : bits & 0xFFFFu, x, e);
                else if (a.is_bf16)
                    elem_bf16(bits, x, e);
                else
                    elem_f32(bits, x, e);
                acc[h] = __dadd_rn(acc[h], x);
                mag[h] = __dadd_rn(mag[h], fabs(x));
                emin[h] = min(emin[h], e);
            }
        };
        auto load = [&](int tok) -> uint32_t {
            const long long e = base + (long long)tok * a.d;
            if (CH == 2) return *reinterpret_cast<const uint32_t *>(reinterpret_cast<const uint16_t *>(R.X) + e);
            if (a.is_bf16) return reinterpret_cast<const uint16_t *>(R.X)[e];
            return reinterpret_cast<const uint32_t *>(R.X)[e];
        };
        int m = m0;
        for (; m + kUpdUnroll <= m1; m += kUpdUnroll) {
            int tok[kUpdUnroll];
#pragma unroll
            for (int q = 0; q < kUpdUnroll; ++q) tok[q] = SCOPE_DCHECK(perm[m + q], a.N, a.status);
            uint32_t bits[kUpdUnroll];
#pragma unroll
            for (int q = 0; q < kUpdUnroll; ++q) bits[q] = load(tok[q]);
#pragma unroll
            for (int q = 0; q < kUpdUnroll; ++q) take(bits[q]);
        }
        for (; m < m1; ++m) take(load(SCOPE_DCHECK(perm[m], a.N, a.status)));
#pragma unroll
        for (int h = 0; h < CH; ++h) {
            psum[threadIdx.x * CH + h] = acc[h];
            pabs[threadIdx.x * CH + h] = mag[h];
            pexp[threadIdx.x * CH + h] = emin[h];
        }
    }
    __syncthreads();
    if (s == 0 && active && n > 0) {
#pragma unroll
        for (int h = 0; h < CH; ++h) {
            double sum = 0.0, mag = 0.0;
            int emin = 0x7fffffff;
            for (int q = 0; q < S; ++q) {
                const int t = (q * dmc + g) * CH + h;
                sum = __dadd_rn(sum, psum[t]);
                mag = __dadd_rn(mag, pabs[t]);
                emin = min(emin, pexp[t]);
            }
            const bool exact = emin == 0x7fffffff ||
                               (emin != (int)0x80000000 && emin > -1000 && mag <= ldexp(1.0, 52 + emin));
            if (!exact) {
                sum = 0.0;
                for (int m = beg; m < end; ++m)
                    sum = __dadd_rn(sum, (double)load_x(R.X, base + h + (long long)perm[m] * a.d, a.is_bf16));
            }
            cent[CH * g + h] = __ddiv_rn(sum, (double)n);
        }
    }
    __syncthreads();
    if (threadIdx.x < dm && active) finalize_row(a, p, c, cent, dm, threadIdx.x);
}

int max_blocks_for_groups(const KmArgs &a)
{
    int mx = 1;
    for (int r = 0; r < a.nroles; ++r) {
        const RoleDesc &R = a.role[a.role0 + r];
        int G = R.dm >= 128 ? 1 : 128 / R.dm;
        mx = max(mx, (R.C + G - 1) / G);
    }
    return mx;
}

}  // namespace

cudaError_t sort_by_cluster(KmArgs a, cudaStream_t s)
{
    const int P = a.BH * a.nroles;
    const size_t hsm = (size_t)4 * a.Cs * sizeof(int);
    dim3 gh((a.nchunk + 3) / 4, P);
    sort_hist_kernel<<<gh, 128, hsm, s>>>(a);
    sort_scan_kernel<<<P, 1024, 0, s>>>(a);
    sort_scatter_kernel<<<gh, 128, hsm, s>>>(a);
    return cudaGetLastError();
}

cudaError_t km_run(KmArgs a, int iters, cudaStream_t s)
{
    static bool attr_done = false;
    const int P = a.BH * a.nroles;
    const size_t fsm = ((size_t)a.ds * (kTok + kCC) + 3 * kCC + kTok) * sizeof(float);
    if (!attr_done) {
        cudaFuncSetAttribute(km_assign_fast_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(((size_t)128 * (kTok + kCC) + 3 * kCC + kTok) * sizeof(float)));
        cudaFuncSetAttribute(sort_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             4 * kMaxC * (int)sizeof(int));
        cudaFuncSetAttribute(sort_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             4 * kMaxC * (int)sizeof(int));
        attr_done = true;
    }
    const int gb = max_blocks_for_groups(a);
    km_init_kernel<<<dim3(gb, P), 128, 0, s>>>(a);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // bf16 inputs whose centroid operands fit in shared memory take the tensor-core
    // assignment (kmeans_tc.cu); both paths certify their winners the same way and leave
    // the undecided tokens to the binary64 kernel.
    const bool tc = km_assign_tc_supported(a);
    // two channels per 4-byte load when every launched channel range is even-aligned
    bool upd2 = a.is_bf16 != 0;
    for (int r = 0; r < a.nroles; ++r)
        upd2 = upd2 && (a.role[a.role0 + r].ch0 % 2 == 0) && (a.role[a.role0 + r].dm % 2 == 0);
    if (tc) {
        cudaError_t e = km_norms(a, s);
        if (e != cudaSuccess) return e;
    }
    for (int it = 0; it < iters; ++it) {
        if (cudaMemsetAsync(a.unsure_count, 0, 4 * sizeof(int32_t), s) != cudaSuccess) return cudaGetLastError();
        if (tc) {
            cudaError_t e = km_pack(a, s);
            if (e == cudaSuccess) e = km_assign_tc(a, sms, s);
            if (e != cudaSuccess) return e;
        } else {
            km_assign_fast_kernel<<<dim3((a.N + kTok - 1) / kTok, P), kAssignThreads, fsm, s>>>(a);
        }
        km_assign_exact_kernel<<<sms * 4, kExactWarps * 32, 0, s>>>(a);
        cudaError_t e = sort_by_cluster(a, s);
        if (e != cudaSuccess) return e;
        if (upd2)
            km_update_kernel<2><<<dim3(a.Cs, P), kUpdThreads, 0, s>>>(a);
        else
            km_update_kernel<1><<<dim3(a.Cs, P), kUpdThreads, 0, s>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace scope
