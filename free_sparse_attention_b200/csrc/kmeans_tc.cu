// k-means assignment on the Blackwell tensor cores (tcgen05, sm_100a), bf16 inputs.
//
// The assignment step of Lloyd's k-means (SCOPE's query clustering and the per-subspace
// key clustering, review page, load_bearing_attack: Eq. 3) picks, for every token x,
// the centroid c minimising |x - mu_c|^2, i.e. minimising S_c = |mu_c|^2 - 2 x.mu_c.
// x.mu_c for a tile of 128 tokens against every centroid is a dense [128 x K] x [K x C]
// product, so it runs as tcgen05 MMAs with the fp32 accumulator in TMEM:
//   * x is bf16 already (the layer's Q or K), loaded by TMA straight into the 128-byte
//     swizzled K-major layout.  A subspace uses the 16-channel-aligned window around its
//     channel range; the centroid matrix is zero outside the range, so channels of other
//     subspaces contribute exactly nothing.
//   * each binary64 centroid is split as mu = hi + lo + r with hi = bf16(mu),
//     lo = bf16(mu - hi), |r| <= 2^-16 |mu| (the largest |r| of the centroid set enters
//     the bound); both halves accumulate into one TMEM accumulator (x.hi + x.lo),
//     products being exact in fp32.
//   * the epilogue (one thread per token = TMEM lane) keeps the smallest and the
//     second-smallest fp32 score and the winner.  The winner is accepted when the gap
//     exceeds twice a bound on |score - S_c| (the bf16 split remainder, the fp32
//     accumulation inside the tensor core, the rounding of |mu|^2 and of the score, and
//     the binary64 rounding of the reference); otherwise the token is marked unsure and
//     the binary64 kernel of kmeans.cu re-decides it exactly.  Every term of the bound is
//     proven except the accumulation term, which rests on a model of the tensor core's
//     addition (below) that NVIDIA does not document for tcgen05; a GPU test measures the
//     hardware against it (tests/test_gpu_tc_accumulation.py).  Under that model the
//     assignment equals the binary64 evaluation of the definition, as on the CUDA-core
//     path.
//
// Per CTA (persistent, one per SM, a contiguous range of (problem, 128-token tile) units):
//   warp 0     TMA producer: the problem's centroid matrix (hi, lo) and |mu|^2 row once
//              per problem, the token tile into a 2-deep ring
//   warp 1     TMEM allocation and MMA issue (one thread)
//   warps 2-9  epilogue, two warpgroups splitting every chunk's columns: TMEM loads,
//              running minima, certification against the token norms that
//              km_norms_kernel computes once per clustering run
// The centroids are split in chunks of at most 256 columns, double-buffered in TMEM
// (2 x 256 columns), so the epilogue of one chunk overlaps the MMAs of the next.
// Every mbarrier wait gives up after ~4 s, sets a status bit and lets the CTA drain.
#include "tc_common.cuh"

#include <cfloat>

namespace scope {

namespace {

constexpr int kTile = 128;             // tokens per unit (TMEM lanes)
#ifndef SCOPE_KM_EPI_WG
#define SCOPE_KM_EPI_WG 2
#endif
constexpr int kEpiWG = SCOPE_KM_EPI_WG;  // epilogue warpgroups
constexpr int kThreadsTc = 64 + 128 * kEpiWG;   // producer warp, MMA warp, epilogue
constexpr int kChunkMax = 256;         // centroid columns per TMEM buffer
constexpr uint32_t kTmemColsTc = 512;  // two accumulator buffers
constexpr uint16_t kUnsureTc = 0xFFFF;
constexpr int kBoxRows = 16;           // centroid rows per TMA box
constexpr int kSmemLimit = 232448;

struct __align__(8) TcBars {
    uint64_t b_full, b_empty;
    uint64_t x_full[2], x_empty[2];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t mg_full[2], mg_empty[2];   // epilogue warpgroup 1 -> 0 hand-off slots
    uint64_t drain;
};

// Channel window of a role: [ws, ws + 16*ks), ks 16-channel MMA steps in nbox 64-channel boxes.
struct Window {
    int ws, ks, nbox;
};

__host__ __device__ inline Window window_of(int ch0, int dm)
{
    Window w;
    w.ws = ch0 & ~15;
    const int we = (ch0 + dm + 15) & ~15;
    w.ks = (we - w.ws) / 16;
    w.nbox = (we - w.ws + 63) / 64;
    return w;
}

// Per role: C padded to 16 (Cr), split into nch chunks of at most 256 columns.
struct Chunks {
    int Cr, nch, chunk0;   // chunk0 = size of every chunk but the last (a multiple of 16)
};

__host__ __device__ inline Chunks chunks_of(int C)
{
    Chunks k;
    k.Cr = (C + 15) & ~15;
    k.nch = (k.Cr + kChunkMax - 1) / kChunkMax;
    k.chunk0 = ((k.Cr + k.nch - 1) / k.nch + 15) & ~15;
    return k;
}

struct TcLayout {
    int Cpad;               // row stride of the packed centroid arrays (all roles)
    int nbox_max, cr_max;
    size_t b_bytes, x_stage, n2_off, merge_off, bars_off, total;
};

TcLayout tc_layout(const KmArgs &a)
{
    TcLayout L{};
    L.Cpad = (a.Cs + 15) & ~15;
    size_t bmax = 0;
    int nbm = 1, crm = 16;
    for (int r = 0; r < a.nroles; ++r) {
        const RoleDesc &R = a.role[a.role0 + r];
        const Window w = window_of(R.ch0, R.dm);
        const Chunks k = chunks_of(R.C);
        nbm = w.nbox > nbm ? w.nbox : nbm;
        crm = k.Cr > crm ? k.Cr : crm;
        const size_t b = (size_t)2 * w.nbox * k.Cr * 128;
        bmax = b > bmax ? b : bmax;
    }
    L.nbox_max = nbm;
    L.cr_max = crm;
    L.b_bytes = bmax;
    L.x_stage = (size_t)nbm * kTile * 128;
    L.n2_off = L.b_bytes + 2 * L.x_stage;
    L.merge_off = (L.n2_off + (size_t)(crm + 4) * 4 + 15) & ~size_t(15);
    L.bars_off = L.merge_off + (size_t)(kEpiWG - 1) * 2 * 3 * kTile * 4;   // [wg-1][slot][m1, m2, ix][128]
    L.total = L.bars_off + sizeof(TcBars) + 16 + 1024;
    return L;
}

struct TcParams {
    int TT;                 // token tiles per problem
    int Cpad;               // row stride of cent_bf / cn2p
    long long n_units;      // problems x TT
    unsigned x_off, x_stage, n2_off, merge_off, bars_off;   // shared-memory offsets
};

// A bounded wait without the abort check, for draining copies and MMAs already issued.
__device__ __forceinline__ void drain_wait(uint64_t *b, uint32_t parity)
{
    const unsigned long long t0 = global_ns();
    while (!bar_test(b, parity) && global_ns() - t0 < kTcWaitNs) __nanosleep(64);
}

// Bound on |score - S_c| for a token of norm |x| <= xn, with M = max |mu_c|,
// Rm = max |mu_c - hi_c - lo_c| and ks MMA steps per half (|hi| <= (1 + 2^-8) |mu|,
// |lo| <= 2^-8 (1 + 2^-8) |mu|):
//   2 |x.r_c|                      <= 2 xn Rm               (Cauchy-Schwarz)
//   2 x fp32 accumulation error     <= 2 x 18 2^-23 x (sum over steps of the largest
//                                      magnitude the step holds); the ks lo steps run
//                                      first and hold at most sum |x_i lo_i| <= 2^-8 (1 + 2^-8)
//                                      xn M each, the ks hi steps at most sum |x_i lo_i| +
//                                      sum |x_i hi_i| <= (1 + 2^-7 + 2^-16) xn M each, so
//                                   <= 9 ks 2^-21 (1 + 2^-7 + 2^-8 + 2^-15) xn M
//                                   <= 9 ks 2^-21 1.012 xn M
//   rounding of the score           <= 2^-21 xn M  (+ the |mu|^2 part, in the slack)
//   |mu|^2 to fp32, reference sum   <= slack_max + 2^-40 xn^2
// Accumulation model (Fasi, Higham, Mikaitis, Pranesh, "Numerical behavior of NVIDIA
// tensor cores", PeerJ Comput. Sci. 7:e330, 2021, for earlier generations): the products
// of a step are exact, the step adds them and the accumulator after aligning every term
// to the largest one and truncating, then normalises.  Each of the 17 terms then loses
// less than one unit in the last place of the largest term, and the normalisation one
// more: 18 units of 2^-23 of that magnitude per step, which the running sum of |x_i mu_i|
// bounds.  The model is not documented for tcgen05; the accumulation test measures the
// hardware against this allowance on random, wide-exponent, cancelling and swamping
// operands.
__device__ __forceinline__ float bound_E(int ks, float xn, float M, float Rm, float slack)
{
    const float coef = (9.f * (float)ks * 1.012f + 1.f) * 0x1p-21f;
    return fmaf(xn, fmaf(coef, M, 2.f * Rm), fmaf(0x1p-40f * xn, xn, slack));
}

__device__ __forceinline__ float fmin3f(float a, float b, float c)
{
    float d;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Scores of centroids i and i+1 from their products v0, v1 and norms n0, n1, folded into a
// running (smallest m1, second smallest m2, index of the smallest mi).  The second smallest
// of {m1, m2} and {lo, hi} is min(m2, hi, max(m1, lo)); on equal scores the index of the
// pair's first element is kept (ties are never certified: they are re-decided exactly).
__device__ __forceinline__ void pair_update(float v0, float v1, float n0, float n1, int i, float &m1, float &m2,
                                            int &mi)
{
    const float2 A = f2unpack(f2fma(f2pack(-2.f, -2.f), f2pack(v0, v1), f2pack(n0, n1)));
    const float lo = fminf(A.x, A.y), hi = fmaxf(A.x, A.y);
    const int li = A.y < A.x ? i + 1 : i;
    m2 = fmin3f(m2, hi, fmaxf(m1, lo));
    mi = lo < m1 ? li : mi;
    m1 = fminf(m1, lo);
}

__device__ __forceinline__ void bulk_copy(uint32_t dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// ------------------------------------------------------------------------- pack
// grid (P, kPackSplit), block 256: block (p, y) handles the centroid rows c = y mod kPackSplit
// of problem p: the bf16 hi / lo split of every row over all d channels (zero outside the
// role's channel range and for padded rows), |mu|^2 in fp32 with +inf for padded rows, and
// (one warp per row) the block's largest |mu|^2, split remainder and slack term, folded into
// the problem's maxima with integer atomicMax on the non-negative float bits (the launcher
// zeroes them first): max |mu| (rounded up), the largest slack term, max |mu - hi - lo|.
constexpr int kPackSplit = 8;

__global__ void __launch_bounds__(256) km_pack_kernel(KmArgs a, int Cpad)
{
    const int p = blockIdx.x, part = blockIdx.y;
    const int r = p % a.nroles, bh = p / a.nroles;
    const RoleDesc &R = a.role[a.role0 + r];
    __nv_bfloat16 *hi = a.cent_bf + (size_t)p * 2 * Cpad * a.d;
    __nv_bfloat16 *lo = hi + (size_t)Cpad * a.d;
    const int rows = (Cpad - part + kPackSplit - 1) / kPackSplit;
    for (int k = threadIdx.x; k < rows * a.d; k += blockDim.x) {
        const int c = part + (k / a.d) * kPackSplit, i = k % a.d;
        float h = 0.f, l = 0.f;
        if (c < R.C && i >= R.ch0 && i < R.ch0 + R.dm) {
            const double m = R.cent[((size_t)bh * R.C + c) * a.d + i];
            const __nv_bfloat16 hb = __double2bfloat16(m);
            const double rem = m - (double)__bfloat162float(hb);   // exact in binary64
            h = __bfloat162float(hb);
            l = __bfloat162float(__double2bfloat16(rem));
        }
        hi[(size_t)c * a.d + i] = __float2bfloat16(h);
        lo[(size_t)c * a.d + i] = __float2bfloat16(l);
    }
    float *n2 = a.cn2p + (size_t)p * (Cpad + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    double mx = 0.0, mr = 0.0;
    float msl = 0.f;
    for (int c = part + warp * kPackSplit; c < Cpad; c += 8 * kPackSplit) {
        if (c < R.C) {
            const double *mu = R.cent + ((size_t)bh * R.C + c) * a.d + R.ch0;
            double s = 0.0, rr = 0.0;
            for (int i = lane; i < R.dm; i += 32) {
                const double m = mu[i];
                const double h = (double)__bfloat162float(__double2bfloat16(m));
                const double rem = m - h;
                const double res = rem - (double)__bfloat162float(__double2bfloat16(rem));  // exact
                s += m * m;
                rr += res * res;
            }
            for (int o = 16; o; o >>= 1) {
                s += __shfl_xor_sync(0xffffffffu, s, o);
                rr += __shfl_xor_sync(0xffffffffu, rr, o);
            }
            mx = fmax(mx, s);
            mr = fmax(mr, rr);
            if (lane == 0) {
                n2[c] = a.cnrm2[(size_t)p * a.Cs + c];
                msl = fmaxf(msl, a.cslack[(size_t)p * a.Cs + c]);
            }
        } else if (lane == 0) {
            n2[c] = INFINITY;
        }
    }
    __shared__ double smx[8], smr[8];
    __shared__ float ssl[8];
    if (lane == 0) {
        smx[warp] = mx;
        smr[warp] = mr;
        ssl[warp] = msl;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < 8; ++w) {
            mx = fmax(mx, smx[w]);
            mr = fmax(mr, smr[w]);
            msl = fmaxf(msl, ssl[w]);
        }
        // square roots of binary64 sums of squares (each within ~1e-14 of the exact
        // value), rounded up with a margin: max |mu_c| and max |mu_c - hi_c - lo_c|
        int *n2i = reinterpret_cast<int *>(n2);
        atomicMax(n2i + Cpad, __float_as_int(__double2float_ru(sqrt(mx) * (1.0 + 0x1p-20))));
        atomicMax(n2i + Cpad + 1, __float_as_int(msl));
        atomicMax(n2i + Cpad + 2, __float_as_int(__double2float_ru(sqrt(mr) * (1.0 + 0x1p-20))));
    }
}

// ------------------------------------------------------------------------- token norms
// grid (ceil(N / 256), P), block 256: thread j of problem p computes |x_j| over the role's
// channels, summing x_i^2 in fp32 with one fma per channel in channel order, and stores
// sqrt(sum) (1 + 2^-12): an upper bound of the binary64 norm (the fp32 sum of dm squares is
// within dm 2^-24 of it, the square root within 2^-24).  The inputs do not change between
// Lloyd iterations, so this runs once per clustering run.
__global__ void __launch_bounds__(256) km_norms_kernel(KmArgs a)
{
    const int p = blockIdx.y, j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= a.N) return;
    const int bh = p / a.nroles;
    const RoleDesc &R = a.role[a.role0 + p % a.nroles];
    const uint4 *row = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(R.X) +
                                                       ((size_t)bh * a.N + j) * a.d);
    const int lo_c = R.ch0, hi_c = R.ch0 + R.dm;
    float ss = 0.f;
    for (int q8 = lo_c >> 3; q8 <= (hi_c - 1) >> 3; ++q8) {
        const uint4 v = row[q8];
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int c = q8 * 8 + q;
            const float x = __uint_as_float((q & 1) ? (wv[q >> 1] & 0xFFFF0000u) : (wv[q >> 1] << 16));
            if (c >= lo_c && c < hi_c) ss = fmaf(x, x, ss);
        }
    }
    a.xnorm[(size_t)p * a.N + j] = sqrtf(ss) * (1.0f + 0x1p-12f);
}

// ------------------------------------------------------------------------- assignment
// The 2 KS products of one chunk: x . lo over the KS 16-channel steps, then x . hi (the order
// bound_E assumes), into one TMEM accumulator.  The step offsets are compile-time constants
// added to the low word of the descriptors (the start address field; no carry out of it for
// shared-memory addresses), so the issuing thread spends a few instructions per product.
// bstride16 = the centroid box stride (Cr rows of 128 bytes) in 16-byte units.
template <int KS>
__device__ __forceinline__ void issue_chunk_ks(uint32_t dst, uint64_t ad, uint64_t bd_lo, uint64_t bd_hi,
                                               uint32_t bstride16, uint32_t idesc)
{
    const uint32_t ahi = (uint32_t)(ad >> 32), alo = (uint32_t)ad;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint64_t bd = h == 0 ? bd_lo : bd_hi;
        const uint32_t bhi = (uint32_t)(bd >> 32), blo = (uint32_t)bd;
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            const uint32_t oa = (uint32_t)(((kk >> 2) * (kTile * 128) + (kk & 3) * 32) >> 4);
            const uint32_t ob = (uint32_t)(kk >> 2) * bstride16 + (uint32_t)((kk & 3) * 2);
            mma_bf16(dst, ((uint64_t)ahi << 32) | (alo + oa), ((uint64_t)bhi << 32) | (blo + ob), idesc,
                     (h | kk) != 0 ? 1u : 0u);
        }
    }
}

__device__ __forceinline__ void issue_chunk(int ks, uint32_t dst, uint64_t ad, uint64_t bd_lo, uint64_t bd_hi,
                                            uint32_t bstride16, uint32_t idesc)
{
    switch (ks) {
    case 1: issue_chunk_ks<1>(dst, ad, bd_lo, bd_hi, bstride16, idesc); break;
    case 2: issue_chunk_ks<2>(dst, ad, bd_lo, bd_hi, bstride16, idesc); break;
    case 3: issue_chunk_ks<3>(dst, ad, bd_lo, bd_hi, bstride16, idesc); break;
    case 4: issue_chunk_ks<4>(dst, ad, bd_lo, bd_hi, bstride16, idesc); break;
    case 5: issue_chunk_ks<5>(dst, ad, bd_lo, bd_hi, bstride16, idesc); break;
    case 6: issue_chunk_ks<6>(dst, ad, bd_lo, bd_hi, bstride16, idesc); break;
    case 7: issue_chunk_ks<7>(dst, ad, bd_lo, bd_hi, bstride16, idesc); break;
    default: issue_chunk_ks<8>(dst, ad, bd_lo, bd_hi, bstride16, idesc); break;
    }
}

__global__ void __launch_bounds__(kThreadsTc, 1)
    km_assign_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmB, KmArgs a, TcParams t)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    TcBars *bars = reinterpret_cast<TcBars *>(sm + t.bars_off);
    int *misc = reinterpret_cast<int *>(sm + t.bars_off + sizeof(TcBars));
    volatile int *abort_flag = misc;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t sbase = smem_u32(sm);
    const long long ub = t.n_units * blockIdx.x / gridDim.x;
    const long long ue = t.n_units * (blockIdx.x + 1) / gridDim.x;

    if (threadIdx.x == 0) {
        misc[0] = 0;
        bar_init(&bars->b_full, 1);
        bar_init(&bars->b_empty, 1 + 4 * kEpiWG);
        for (int s = 0; s < 2; ++s) {
            bar_init(&bars->x_full[s], 1);
            bar_init(&bars->x_empty[s], 1);
            bar_init(&bars->acc_full[s], 1);
            bar_init(&bars->acc_empty[s], 4 * kEpiWG);
            bar_init(&bars->mg_full[s], 4 * (kEpiWG - 1));
            bar_init(&bars->mg_empty[s], 4);
        }
        bar_init(&bars->drain, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(kTmemColsTc)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int cur_p = -1;
            uint32_t nb = 0, xi = 0;
            for (long long u = ub; u < ue && !*abort_flag; ++u) {
                const int p = (int)(u / t.TT), tile = (int)(u % t.TT);
                const int ra = a.role0 + p % a.nroles, bh = p / a.nroles;
                const RoleDesc &R = a.role[ra];
                const Window w = window_of(R.ch0, R.dm);
                if (p != cur_p) {
                    const Chunks k = chunks_of(R.C);
                    if (nb > 0 && !bar_wait(&bars->b_empty, (nb - 1) & 1, abort_flag, a.status)) break;
                    bar_expect_tx(&bars->b_full, 2u * w.nbox * k.Cr * 128 + (uint32_t)(k.Cr + 4) * 4);
                    for (int sp = 0; sp < 2; ++sp)
                        for (int b = 0; b < w.nbox; ++b)
                            for (int c0 = 0; c0 < k.Cr; c0 += kBoxRows)
                                tma_tile2d(sbase + ((sp * w.nbox + b) * k.Cr + c0) * 128, &tmB, w.ws + 64 * b,
                                           (p * 2 + sp) * t.Cpad + c0, &bars->b_full);
                    const float *n2g = a.cn2p + (size_t)p * (t.Cpad + 4);
                    bulk_copy(sbase + t.n2_off, n2g, (uint32_t)k.Cr * 4, &bars->b_full);
                    bulk_copy(sbase + t.n2_off + k.Cr * 4, n2g + t.Cpad, 16, &bars->b_full);
                    cur_p = p;
                    ++nb;
                }
                const int s = xi & 1;
                if (!bar_wait(&bars->x_empty[s], ((xi >> 1) & 1) ^ 1, abort_flag, a.status)) break;
                bar_expect_tx(&bars->x_full[s], (uint32_t)w.nbox * kTile * 128);
                const CUtensorMap *tm = ra == 0 ? &tmQ : &tmK;
                for (int b = 0; b < w.nbox; ++b)
                    tma_tile2d(sbase + t.x_off + s * t.x_stage + b * (kTile * 128), tm, w.ws + 64 * b,
                               bh * a.N + tile * kTile, &bars->x_full[s]);
                ++xi;
            }
            // copies still in flight complete before the CTA exits
            if (nb > 0) drain_wait(&bars->b_full, (nb - 1) & 1);
            for (uint32_t k = xi > 2 ? xi - 2 : 0; k < xi; ++k) drain_wait(&bars->x_full[k & 1], (k >> 1) & 1);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issue
        if (lane == 0) {
            int cur_p = -1;
            uint32_t nb = 0, xi = 0, g = 0;
            // the unit's (problem, tile) advance incrementally; role constants change per problem
            int p = (int)(ub / t.TT), tile = (int)(ub % t.TT);
            int ks = 1, nbox = 1, nch = 1, chunk0 = 16, Cr = 16;
            for (long long u = ub; u < ue && !*abort_flag; ++u) {
                if (p != cur_p) {
                    const RoleDesc &R = a.role[a.role0 + p % a.nroles];
                    const Window w = window_of(R.ch0, R.dm);
                    const Chunks k = chunks_of(R.C);
                    ks = w.ks;
                    nbox = w.nbox;
                    nch = k.nch;
                    chunk0 = k.chunk0;
                    Cr = k.Cr;
                    if (!bar_wait(&bars->b_full, nb & 1, abort_flag, a.status)) break;
                    ++nb;
                    cur_p = p;
                }
                const int s = xi & 1;
                if (!bar_wait(&bars->x_full[s], (xi >> 1) & 1, abort_flag, a.status)) break;
                tc_fence_after();
                const uint64_t ad0 = sw128_desc(sbase + t.x_off + s * t.x_stage, 16, 1024);
                bool ok = true;
                for (int ch = 0; ch < nch; ++ch) {
                    const int n0 = ch * chunk0, nc = min(chunk0, Cr - n0);
                    const int buf = g & 1;
                    if (!bar_wait(&bars->acc_empty[buf], ((g >> 1) & 1) ^ 1, abort_flag, a.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    issue_chunk(ks, tmem + buf * kChunkMax, ad0, sw128_desc(sbase + (nbox * Cr + n0) * 128, 16, 1024),
                                sw128_desc(sbase + n0 * 128, 16, 1024), (uint32_t)(Cr * 128) >> 4,
                                f16_idesc(kTile, nc, false));
                    mma_commit(&bars->acc_full[buf]);
                    ++g;
                }
                if (!ok) break;
                mma_commit(&bars->x_empty[s]);
                ++xi;
                if (++tile == t.TT) {
                    tile = 0;
                    ++p;
                }
                // the CTA's last unit of this problem releases the centroids
                if (u + 1 == ue || tile == 0) mma_commit(&bars->b_empty);
            }
            // every issued MMA completes before TMEM is freed
            mma_commit(&bars->drain);
            drain_wait(&bars->drain, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue (warps 2-)
        // kEpiWG warpgroups share every chunk: warpgroup e takes the 16-column groups
        // g = e, e + kEpiWG, ... (two at a time, one TMEM wait per pair, one running minimum
        // pair per group slot so consecutive columns do not form one dependency chain).
        // Warpgroups 1.. hand their (min, second min, winner) per token to warpgroup 0
        // through a double-buffered slot; warpgroup 0 merges, certifies (with the token's
        // norm, computed once per run by km_norms_kernel) and writes the assignment.
        const int e = (warp - 2) >> 2;                 // epilogue warpgroup
        const int q4 = warp & 3;                       // TMEM lane quarter of this warp
        const int row = q4 * 32 + lane;                // token row of the tile = TMEM lane
        const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
        const float *n2s = reinterpret_cast<const float *>(sm + t.n2_off);
        float *mg = reinterpret_cast<float *>(sm + t.merge_off);   // [kEpiWG-1][2][3][128]
        int cur_p = -1;
        uint32_t nb = 0, g = 0;
        float maxnm = 0.f, maxsl = 0.f, maxres = 0.f;
        // the unit's (problem, tile) advance incrementally; role constants change per problem
        int p = (int)(ub / t.TT), tile = (int)(ub % t.TT);
        int bh = 0, r = 0, ks = 1;
#ifdef SCOPE_DEBUG
        int Cn = 1;   // the centroid count, the bound of the debug build's index check
#endif
        Chunks k{16, 1, 16};
        uint16_t *assign = nullptr;
        long long assign_bh = 0;
        for (long long u = ub; u < ue; ++u, (++tile == t.TT ? (tile = 0, ++p) : 0)) {
            if (warp_aborted(abort_flag)) break;
            if (p != cur_p) {
                bh = p / a.nroles;
                r = p % a.nroles;
                const RoleDesc &R = a.role[a.role0 + r];
                ks = window_of(R.ch0, R.dm).ks;
                k = chunks_of(R.C);
#ifdef SCOPE_DEBUG
                Cn = R.C;
#endif
                assign = R.assign;
                assign_bh = R.assign_bh;
                if (!warp_wait(&bars->b_full, nb & 1, abort_flag, a.status)) break;
                ++nb;
                cur_p = p;
                maxnm = n2s[k.Cr];
                maxsl = n2s[k.Cr + 1];
                maxres = n2s[k.Cr + 2];
            }
            const int j = tile * kTile + row;
            // |x| of this token over the role's channels (computed once per run)
            float xn = 0.f;
            if (e == 0 && j < a.N) xn = a.xnorm[(size_t)p * a.N + j];
            // running (min, second min, winner) for the two group slots of this thread
            float a1 = INFINITY, a2 = INFINITY, b1 = INFINITY, b2 = INFINITY;
            int ai = 0, bi = 0;
            bool ok = true;
            for (int ch = 0; ch < k.nch; ++ch) {
                const int n0 = ch * k.chunk0, nc = min(k.chunk0, k.Cr - n0);
                const int ng = nc >> 4;                // 16-column groups in this chunk
                const int buf = g & 1;
                if (!warp_wait(&bars->acc_full[buf], (g >> 1) & 1, abort_flag, a.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int gi = e; gi < ng; gi += 2 * kEpiWG) {
                    const bool two = gi + kEpiWG < ng;
                    float v[32];
                    const uint32_t ta = tmem + lane_base + buf * kChunkMax + gi * 16;
                    tmem_ld16(ta, v);
                    if (two) tmem_ld16(ta + 16 * kEpiWG, v + 16);
                    tmem_wait_ld();
                    const int c0 = n0 + gi * 16;
                    // scores two at a time: A = |mu|^2 - 2 x.mu on packed pairs, then the
                    // smaller and larger of the pair update (min, second min, winner) with
                    // three-input min / max
                    const float4 *na = reinterpret_cast<const float4 *>(n2s + c0);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float4 nn = na[q];
                        pair_update(v[4 * q], v[4 * q + 1], nn.x, nn.y, c0 + 4 * q, a1, a2, ai);
                        pair_update(v[4 * q + 2], v[4 * q + 3], nn.z, nn.w, c0 + 4 * q + 2, a1, a2, ai);
                    }
                    if (two) {
                        const float4 *nb4 = reinterpret_cast<const float4 *>(n2s + c0 + 16 * kEpiWG);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float4 nn = nb4[q];
                            pair_update(v[16 + 4 * q], v[16 + 4 * q + 1], nn.x, nn.y, c0 + 16 * kEpiWG + 4 * q, b1, b2,
                                        bi);
                            pair_update(v[16 + 4 * q + 2], v[16 + 4 * q + 3], nn.z, nn.w, c0 + 16 * kEpiWG + 4 * q + 2,
                                        b1, b2, bi);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) bar_arrive(&bars->acc_empty[buf]);
                ++g;
            }
            if (!ok) break;
            if (u + 1 == ue || tile + 1 == t.TT) {
                __syncwarp();
                if (lane == 0) bar_arrive(&bars->b_empty);
            }
            // merge the two slots (second smallest of a union = min of the second
            // smallests and the larger of the smallests)
            float m2 = fminf(fminf(a2, b2), fmaxf(a1, b1));
            int idx = b1 < a1 ? bi : ai;
            float m1 = fminf(a1, b1);
            const uint32_t mi = (uint32_t)(u - ub), slot = mi & 1;
            if (e != 0) {
                if (!warp_wait(&bars->mg_empty[slot], ((mi >> 1) & 1) ^ 1, abort_flag, a.status)) break;
                float *o = mg + ((size_t)((e - 1) * 2 + slot) * 3) * kTile;
                o[row] = m1;
                o[kTile + row] = m2;
                reinterpret_cast<int *>(o)[2 * kTile + row] = idx;
                __syncwarp();
                if (lane == 0) bar_arrive(&bars->mg_full[slot]);
            } else {
                if (!warp_wait(&bars->mg_full[slot], (mi >> 1) & 1, abort_flag, a.status)) break;
                float o1[kEpiWG - 1], o2[kEpiWG - 1];
                int oi[kEpiWG - 1];
#pragma unroll
                for (int h = 0; h < kEpiWG - 1; ++h) {
                    const float *o = mg + ((size_t)(h * 2 + slot) * 3) * kTile;
                    o1[h] = o[row];
                    o2[h] = o[kTile + row];
                    oi[h] = reinterpret_cast<const int *>(o)[2 * kTile + row];
                }
                __syncwarp();
                if (lane == 0) bar_arrive(&bars->mg_empty[slot]);
#pragma unroll
                for (int h = 0; h < kEpiWG - 1; ++h) {
                    m2 = fminf(fminf(m2, o2[h]), fmaxf(m1, o1[h]));
                    idx = o1[h] < m1 ? oi[h] : idx;
                    m1 = fminf(m1, o1[h]);
                }
                bool unsure = false;
                if (j < a.N) {
                    const float E = bound_E(ks, xn, maxnm, maxres, maxsl);
                    const bool sure = (m2 - m1) > (E + E) * (1.0f + 0x1p-20f);
                    assign[(size_t)bh * assign_bh + j] = sure ? (uint16_t)SCOPE_DCHECK(idx, Cn, a.status) : kUnsureTc;
                    unsure = !sure;
                }
                warp_append(unsure, bh * a.N + j, a.unsure_list + (size_t)r * a.BH * a.N, a.unsure_count + r);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemColsTc)
                     : "memory");
}

}  // namespace

bool km_assign_tc_supported(const KmArgs &a)
{
    if (!a.is_bf16 || (a.d != 64 && a.d != 128) || !a.cent_bf || !a.cn2p || !a.xnorm) return false;
    return tc_layout(a).total <= (size_t)kSmemLimit;
}

cudaError_t km_pack(const KmArgs &a, cudaStream_t s)
{
    const TcLayout L = tc_layout(a);
    const int P = a.BH * a.nroles;
    // the per-problem maxima are folded in with atomicMax: start them (and the rest) at 0
    const cudaError_t e = cudaMemsetAsync(a.cn2p, 0, sizeof(float) * (size_t)P * (L.Cpad + 4), s);
    if (e != cudaSuccess) return e;
    km_pack_kernel<<<dim3(P, kPackSplit), 256, 0, s>>>(a, L.Cpad);
    return cudaGetLastError();
}

cudaError_t km_norms(const KmArgs &a, cudaStream_t s)
{
    km_norms_kernel<<<dim3((a.N + 255) / 256, a.BH * a.nroles), 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t km_assign_tc(const KmArgs &a, int num_sms, cudaStream_t s)
{
    const TcLayout L = tc_layout(a);
    const int P = a.BH * a.nroles;
    CUtensorMap tq, tk, tb;
    const long long rows = (long long)a.BH * a.N;
    const bool has_q = a.role0 == 0, has_k = a.role0 + a.nroles > 1;
    const void *xq = has_q ? a.role[0].X : a.role[a.role0].X;
    const void *xk = has_k ? a.role[a.role0 + a.nroles - 1].X : xq;
    if (!bf16_tile_map(&tq, has_q ? xq : xk, rows, a.d, 64, kTile) ||
        !bf16_tile_map(&tk, xk, rows, a.d, 64, kTile) ||
        !bf16_tile_map(&tb, a.cent_bf, (long long)P * 2 * L.Cpad, a.d, 64, kBoxRows))
        return cudaErrorInvalidValue;
    TcParams t;
    t.TT = (a.N + kTile - 1) / kTile;
    t.Cpad = L.Cpad;
    t.n_units = (long long)P * t.TT;
    t.x_off = (unsigned)L.b_bytes;
    t.x_stage = (unsigned)L.x_stage;
    t.n2_off = (unsigned)L.n2_off;
    t.merge_off = (unsigned)L.merge_off;
    t.bars_off = (unsigned)L.bars_off;
    // more than half of the SM's shared memory: one CTA (and one 512-column TMEM
    // allocation) per SM
    const size_t smem = L.total > (size_t)kSmemLimit / 2 + 1024 ? L.total : (size_t)kSmemLimit / 2 + 1024;
    cudaFuncSetAttribute(km_assign_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    const int grid = (int)(t.n_units < num_sms ? t.n_units : num_sms);
    km_assign_tc_kernel<<<grid, kThreadsTc, smem, s>>>(tq, tk, tb, a, t);
    return cudaGetLastError();
}

}  // namespace scope
