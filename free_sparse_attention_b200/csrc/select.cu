// Lookup tables, proxy logits and the hybrid Top-p / fixed Top-k / online k_head
// selection of SCOPE (arXiv 2608.12780; review page, key_machinery: Eq. 6 and Eq. 9;
// major_comments[1]: Eqs. 7, 8 and 10).
//
// Per unit (b, h, query cluster c), with q_c the cluster centroid:
//   P^m[c, z] = sum_{i in m} q_c[i] mu^m_z[i]                       (LUT, shared memory)
//   s_j       = (1/sqrt d) ((P^T[z^T_j] + P^H[z^H_j]) + P^W[z^W_j])   (Eq. 6)
// Keys are ranked by s_j descending, index ascending.  Both are evaluated in binary64
// with one rounding per operation, in the order written, so logits and ranks are exact.
//
// Selection without a sort: a block-wide select finds the ranking position where the
// cumulative weight (softmax mass for Top-p, one per key for a count) first reaches
// a target.  Keys are histogrammed into 2048 bins by value; the crossing bin is
// resolved exactly (its keys gathered and ranked in shared memory) when it holds at
// most 2048 keys, otherwise it is binned again over its own value range; keys with
// identical logits are binned by index instead.  For the Top-p mass, a sample of one key
// batch in eight first narrows the first level's range to the sampled logits and predicts
// the crossing bin; the keys of a window of bins around it are gathered during the full
// pass, so the separate gather pass only runs when the crossing bin falls outside it.
//
// The softmax mass of key j is w_j = exp(s_j - s_ref), s_ref an upper bound of every
// logit: t = (s_j - s_ref) log2 e in binary64 is split into n + f (n an integer, f in
// [0, 1)) and w_j = 2^n 2^f with 2^f from the fp32 ex2 instruction (relative error of w_j
// below 3e-7, no table lookup).  Masses are accumulated as fixed-point integers (2^-63
// units, split 32/32 bits), so every sum is exact and independent of order: results are
// deterministic run to run, and a Top-p count can differ from a binary64 evaluation only
// where the mass of a prefix is within ~3e-7 (relative) of rho times the total, inside the
// 1e-6 band in which the oracle logs a near tie.
//
// The Top-p kernel saves the count histogram of its first pass, every key's bin in that
// pass (2 bytes per key) and its tables.  The mask kernel finds from the counts the bin
// where the r_c-th key of the ranking lies (or takes the bin of the Top-p boundary key when
// r_c = p_c), and one pass over the saved bins writes the selected set: keys of lower bins
// (higher logits) are set directly, and only the keys of the boundary bin get their logit
// computed again, to be compared with the boundary key or ranked exactly in shared memory.
#include "common.cuh"

#include <cfloat>

namespace scope {

namespace {

constexpr int kSelThreads = 512;
constexpr int kBins = kSelBins;
constexpr int kCap = 2048;
constexpr int kMaxLevels = 6;
constexpr int kBinsPerThread = kBins / kSelThreads;

struct SelSmem {
    double *lut, *qc;
    int *cnt;
    unsigned long long *mhi, *mlo;
    double *cs;
    int *cj;
    unsigned long long *cw;
    int *order;
    double *red;                 // reduction scratch, 32 doubles
    unsigned long long *ured;    // 3 x 32 words
    int *misc;                   // 8 ints
};

__host__ __device__ size_t sel_smem_bytes(int Cm, int d)
{
    return sizeof(double) * (3 * (size_t)Cm + d) + sizeof(int) * kBins +
           2 * sizeof(unsigned long long) * kBins + sizeof(double) * kCap + sizeof(int) * kCap +
           sizeof(unsigned long long) * kCap + sizeof(int) * kCap + sizeof(double) * 32 +
           sizeof(unsigned long long) * 96 + sizeof(int) * 8;
}

__device__ SelSmem carve(char *base, int Cm, int d)
{
    SelSmem s;
    double *dp = reinterpret_cast<double *>(base);
    s.lut = dp;
    s.qc = dp + 3 * Cm;
    s.cs = s.qc + d;
    s.red = s.cs + kCap;
    unsigned long long *up = reinterpret_cast<unsigned long long *>(s.red + 32);
    s.mhi = up;
    s.mlo = up + kBins;
    s.cw = up + 2 * kBins;
    s.ured = s.cw + kCap;
    int *ip = reinterpret_cast<int *>(s.ured + 96);
    s.cnt = ip;
    s.cj = ip + kBins;
    s.order = s.cj + kCap;
    s.misc = s.order + kCap;
    return s;
}

struct Unit {
    const uint16_t *zt, *zh, *zw;
    int Cm, N;
    double inv;          // 1/sqrt(d)
    double sref;         // logit reference of the weights (>= every logit)
    double inv_umax;     // mass normalisation
};

// Keys are visited kBatch at a time per thread (keys j0 + k * kSelThreads + tid): the codes
// and table entries of the batch are all loaded before any of them is used, so a thread
// keeps 3 kBatch independent shared-memory loads in flight instead of one key's chain, and
// every pass loads the next batch's codes (from L2) while it works on the current one.
constexpr int kBatch = 2;

// Codes of one batch, clamped to [0, Cm) so that a malformed caller-supplied code cannot read
// outside the tables (sel_check_kernel reports such codes in the status word).
struct KeyBatch {
    int zt[kBatch], zh[kBatch], zw[kBatch];
    bool v[kBatch];
};

__device__ __forceinline__ KeyBatch load_batch(const Unit &u, int j0)
{
    KeyBatch kb;
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
        const int j = j0 + k * kSelThreads + (int)threadIdx.x;
        kb.v[k] = j < u.N;
        const int jj = kb.v[k] ? j : 0;
        kb.zt[k] = min((int)u.zt[jj], u.Cm - 1);
        kb.zh[k] = min((int)u.zh[jj], u.Cm - 1);
        kb.zw[k] = min((int)u.zw[jj], u.Cm - 1);
    }
    return kb;
}

// s_j of Eq. 6 for every key of the batch
__device__ __forceinline__ void batch_scores(const SelSmem &S, const Unit &u, const KeyBatch &kb, double (&s)[kBatch])
{
    double a[kBatch], b[kBatch], c[kBatch];
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
        a[k] = S.lut[kb.zt[k]];
        b[k] = S.lut[u.Cm + kb.zh[k]];
        c[k] = S.lut[2 * u.Cm + kb.zw[k]];
    }
#pragma unroll
    for (int k = 0; k < kBatch; ++k) s[k] = __dmul_rn(u.inv, __dadd_rn(__dadd_rn(a[k], b[k]), c[k]));
}

// s_j of Eq. 6 for one key (the same operations as batch_scores)
__device__ __forceinline__ double key_score(const SelSmem &S, const Unit &u, int j)
{
    const int zt = min((int)u.zt[j], u.Cm - 1), zh = min((int)u.zh[j], u.Cm - 1),
              zw = min((int)u.zw[j], u.Cm - 1);
    return __dmul_rn(u.inv, __dadd_rn(__dadd_rn(S.lut[zt], S.lut[u.Cm + zh]), S.lut[2 * u.Cm + zw]));
}

// Softmax weight of a key of logit s: exp(s - sref) = 2^n 2^f with t = (s - sref) log2 e
// = n + f (binary64; t - n is exact) and 2^f from ex2.approx.f32 (at most 2 ulp).
__device__ __forceinline__ double key_weight(double s, const Unit &u)
{
    const double t = __dmul_rn(__dsub_rn(s, u.sref), 1.4426950408889634);
    const double n = floor(t);
    if (n < -1000.0) return 0.0;
    float p;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(p) : "f"((float)(t - n)));
    return __dmul_rn((double)p, __hiloint2double(((int)n + 1023) << 20, 0));
}

// key weights for every key of the batch (from its logit)
__device__ __forceinline__ void batch_weights(const Unit &u, const double (&s)[kBatch], double (&w)[kBatch])
{
#pragma unroll
    for (int k = 0; k < kBatch; ++k) w[k] = key_weight(s[k], u);
}

// fixed-point mass of weight w in units of 2^-63, clamped to [0, 2^63]
__device__ __forceinline__ unsigned long long weight_mass(double w, const Unit &u)
{
    return __double2ull_rn(fmin(__dmul_rn(w, u.inv_umax), 1.0) * 9223372036854775808.0);
}

__device__ __forceinline__ double mass_to_double(unsigned long long hi, unsigned long long lo)
{
    return ldexp((double)hi, -31) + ldexp((double)lo, -63);
}

__device__ __forceinline__ int vbin(double s, double hi, double scale)
{
    const double t = __dmul_rn(__dsub_rn(hi, s), scale);
    if (!(t > 0.0)) return 0;
    if (t >= (double)kBins) return kBins - 1;
    return (int)t;
}

__device__ __forceinline__ int jbin(int j, int N)
{
    return (int)(((long long)j * kBins) / N);
}

struct Levels {
    int n;
    double hi[kMaxLevels], scale[kMaxLevels];
    int bstar[kMaxLevels];
    bool jmode, jexact;
    double tie_s;
};

__device__ __forceinline__ bool in_candidates(const Levels &L, double s)
{
    for (int k = 0; k < L.n; ++k)
        if (vbin(s, L.hi[k], L.scale[k]) != L.bstar[k]) return false;
    if (L.jmode && L.jexact && s != L.tie_s) return false;
    return true;
}

// ---- block reductions (all threads call; result broadcast)
__device__ double block_max(double v, double *red)
{
    for (int o = 16; o; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) red[w] = v;
    __syncthreads();
    if (w == 0) {
        v = lane < (int)(blockDim.x >> 5) ? red[lane] : -DBL_MAX;
        for (int o = 16; o; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) red[0] = v;
    }
    __syncthreads();
    return red[0];
}

__device__ double block_min(double v, double *red)
{
    return -block_max(-v, red);
}

// inclusive warp scan of three 64-bit components
__device__ __forceinline__ void warp_scan3(unsigned long long &a, unsigned long long &b,
                                           unsigned long long &c)
{
    const int lane = threadIdx.x & 31;
    for (int o = 1; o < 32; o <<= 1) {
        unsigned long long x = __shfl_up_sync(0xffffffffu, a, o);
        unsigned long long y = __shfl_up_sync(0xffffffffu, b, o);
        unsigned long long z = __shfl_up_sync(0xffffffffu, c, o);
        if (lane >= o) {
            a += x;
            b += y;
            c += z;
        }
    }
}

// Exclusive block scan of (a, b, c); returns the block totals through tot[3].
__device__ void block_excl_scan3(unsigned long long &a, unsigned long long &b, unsigned long long &c,
                                 unsigned long long *ured, unsigned long long tot[3])
{
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    unsigned long long ia = a, ib = b, ic = c;
    warp_scan3(ia, ib, ic);
    __syncthreads();
    if (lane == 31) {
        ured[w] = ia;
        ured[32 + w] = ib;
        ured[64 + w] = ic;
    }
    __syncthreads();
    if (w == 0) {
        unsigned long long xa = lane < nw ? ured[lane] : 0ull;
        unsigned long long xb = lane < nw ? ured[32 + lane] : 0ull;
        unsigned long long xc = lane < nw ? ured[64 + lane] : 0ull;
        warp_scan3(xa, xb, xc);
        ured[lane] = xa;
        ured[32 + lane] = xb;
        ured[64 + lane] = xc;
    }
    __syncthreads();
    const unsigned long long pa = w ? ured[w - 1] : 0ull, pb = w ? ured[32 + w - 1] : 0ull,
                             pc = w ? ured[64 + w - 1] : 0ull;
    tot[0] = ured[nw - 1];
    tot[1] = ured[32 + nw - 1];
    tot[2] = ured[64 + nw - 1];
    a = pa + ia - a;
    b = pb + ib - b;
    c = pc + ic - c;
}

struct SelectOut {
    double s;
    int j;
    long long rank;   // keys before it in the ranking
    double margin;    // mass mode: min(|mass before - target|, |mass through it - target|) / Z
};

constexpr int kSampleStride = 8;     // the window sample takes one key batch in 8
constexpr int kWindowMinN = 16384;   // below this the sample would be too small to matter

// Predicts the bin of the first level's Top-p crossing from the keys of every
// kSampleStride-th batch.  The first level's value range [lo, hi] (the bounds from the
// tables on entry) is narrowed to the sampled logits' range widened by 1/64 of it on each
// side: keys outside it land in the end bins, which keeps the binning monotone, and the
// bins become fine where the keys are.  The sample's count and mass histogram then gives
// the bin where its cumulative mass reaches rho times its total, widened to a window of bins
// [wlo, whi] whose sampled counts, scaled up, stay within kCap / 2 keys.  The window is only a
// guess: the caller checks it against the full histogram.  All threads call; [wlo, whi] is
// empty (wlo > whi) when the sample finds no crossing.
__device__ void predict_window(const SelSmem &S, const Unit &u, double rho, double &hi, double &lo,
                               int &wlo, int &whi)
{
    const int tid = threadIdx.x;
    {
        double cmin = DBL_MAX, cmax = -DBL_MAX;
        for (int j0 = 0; j0 < u.N; j0 += kSampleStride * kBatch * kSelThreads) {
            const KeyBatch kb = load_batch(u, j0);
            double sc[kBatch];
            batch_scores(S, u, kb, sc);
#pragma unroll
            for (int k = 0; k < kBatch; ++k)
                if (kb.v[k]) {
                    cmin = fmin(cmin, sc[k]);
                    cmax = fmax(cmax, sc[k]);
                }
        }
        cmin = block_min(cmin, S.red);
        cmax = block_max(cmax, S.red);
        if (cmax > cmin) {
            const double pad = (cmax - cmin) * (1.0 / 64.0);
            hi = fmin(hi, cmax + pad);
            lo = fmax(lo, cmin - pad);
        }
    }
    const double scale = (double)kBins / (hi - lo);
    for (int b = tid; b < kBins; b += kSelThreads) {
        S.cnt[b] = 0;
        S.mhi[b] = 0;
        S.mlo[b] = 0;
    }
    __syncthreads();
    for (int j0 = 0; j0 < u.N; j0 += kSampleStride * kBatch * kSelThreads) {
        const KeyBatch kb = load_batch(u, j0);
        double sc[kBatch], uw[kBatch];
        batch_scores(S, u, kb, sc);
        batch_weights(u, sc, uw);
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
            if (!kb.v[k]) continue;
            const int b = vbin(sc[k], hi, scale);
            atomicAdd(&S.cnt[b], 1);
            const unsigned long long W = weight_mass(uw[k], u);
            atomicAdd(&S.mhi[b], W >> 32);
            atomicAdd(&S.mlo[b], W & 0xffffffffull);
        }
    }
    __syncthreads();
    unsigned long long th = 0, tl = 0, tc = 0;
    const int b0 = tid * kBinsPerThread;
    for (int q = 0; q < kBinsPerThread; ++q) {
        th += S.mhi[b0 + q];
        tl += S.mlo[b0 + q];
        tc += (unsigned long long)S.cnt[b0 + q];
    }
    unsigned long long tot[3];
    block_excl_scan3(th, tl, tc, S.ured, tot);
    const double target = rho * mass_to_double(tot[0], tot[1]);
    if (tid == 0) S.misc[4] = -1;
    __syncthreads();
    {
        unsigned long long eh = th, el = tl;
        for (int q = 0; q < kBinsPerThread; ++q) {
            const unsigned long long ih = eh + S.mhi[b0 + q], il = el + S.mlo[b0 + q];
            if (!(mass_to_double(eh, el) >= target) && mass_to_double(ih, il) >= target) S.misc[4] = b0 + q;
            eh = ih;
            el = il;
        }
    }
    __syncthreads();
    if (tid == 0) {
        const int bs = S.misc[4];
        int lo = bs, hi2 = bs;
        if (bs >= 0) {
            long long est = (long long)S.cnt[bs] * kSampleStride;
            for (bool grow = true; grow;) {
                grow = false;
                if (lo > 0 && est + (long long)S.cnt[lo - 1] * kSampleStride <= kCap / 2) {
                    --lo;
                    est += (long long)S.cnt[lo] * kSampleStride;
                    grow = true;
                }
                if (hi2 < kBins - 1 && est + (long long)S.cnt[hi2 + 1] * kSampleStride <= kCap / 2) {
                    ++hi2;
                    est += (long long)S.cnt[hi2] * kSampleStride;
                    grow = true;
                }
            }
            S.misc[4] = lo;
            S.misc[5] = hi2;
        } else {
            S.misc[4] = 1;
            S.misc[5] = 0;
        }
    }
    __syncthreads();
    wlo = S.misc[4];
    whi = S.misc[5];
    __syncthreads();
}

// Finds the first key of the ranking at which the cumulative weight reaches the target.
// mass_mode: weight = softmax mass, target = rho * (total mass); else weight = 1 and
// target = count (1 <= count <= N).  Called by all threads of the block.
// umax_out (mass mode): the largest key weight, found in the first histogram pass.
__device__ SelectOut block_select(const SelSmem &S, const Unit &u, bool mass_mode, double rho,
                                  long long count, double smax, double smin, int32_t *status,
                                  double *umax_out = nullptr, int32_t *save_hist = nullptr,
                                  double *range_out = nullptr, uint16_t *save_bins = nullptr)
{
    Levels L;
    L.n = 0;
    L.jmode = false;
    L.jexact = false;
    L.tie_s = 0.0;
    double hi = smax, lo = smin;
    unsigned long long bhi = 0, blo = 0;   // mass before the candidate set (fixed point)
    long long bcnt = 0;                    // keys before the candidate set
    double target = 0.0;
    bool have_target = !mass_mode;
    const int tid = threadIdx.x;
    SelectOut out{smax, 0, 0, INFINITY};
    // Mass mode: a histogram of every kSampleStride-th batch of keys predicts the bin where
    // the first level's crossing lies, and a window of bins around it (about kCap / 2 keys
    // by the sample's counts) is gathered during the first full pass, so that the separate
    // gather pass is skipped whenever the crossing bin falls inside the window.
    int wlo = 1, whi = 0;   // empty window
    if (mass_mode && u.N >= kWindowMinN && hi > lo) predict_window(S, u, rho, hi, lo, wlo, whi);
    if (range_out) {
        range_out[0] = hi;   // the first level's value range (the mask kernel bins with it)
        range_out[1] = lo;
        range_out[2] = 0.0;  // set to 1 once the first level's counts (and bins) are saved
    }

    for (int iter = 0; iter < kMaxLevels + 3; ++iter) {
        const double scale = (hi > lo) ? (double)kBins / (hi - lo) : 0.0;
        const bool gather_window = iter == 0 && wlo <= whi;
        if (tid == 0) S.misc[3] = 0;
        for (int b = tid; b < kBins; b += kSelThreads) {
            S.cnt[b] = 0;
            S.mhi[b] = 0;
            S.mlo[b] = 0;
        }
        __syncthreads();
        double cmin = DBL_MAX, cmax = -DBL_MAX, umx = 0.0;
        KeyBatch next = load_batch(u, 0);
        for (int j0 = 0; j0 < u.N; j0 += kBatch * kSelThreads) {
            const KeyBatch kb = next;
            if (j0 + kBatch * kSelThreads < u.N) next = load_batch(u, j0 + kBatch * kSelThreads);
            double sc[kBatch], uw[kBatch];
            batch_scores(S, u, kb, sc);
            if (mass_mode) batch_weights(u, sc, uw);
#pragma unroll
            for (int k = 0; k < kBatch; ++k) {
                const double s = sc[k];
                if (!kb.v[k] || !in_candidates(L, s)) continue;
                const int j = j0 + k * kSelThreads + tid;
                const int b = L.jmode ? jbin(j, u.N) : vbin(s, hi, scale);
                if (iter == 0 && save_bins) save_bins[j] = (uint16_t)b;
                atomicAdd(&S.cnt[b], 1);
                if (mass_mode) {
                    umx = fmax(umx, uw[k]);
                    const unsigned long long W = weight_mass(uw[k], u);
                    atomicAdd(&S.mhi[b], W >> 32);
                    atomicAdd(&S.mlo[b], W & 0xffffffffull);
                    if (gather_window && b >= wlo && b <= whi) {
                        const int slot = atomicAdd(&S.misc[3], 1);
                        if (slot < kCap) {
                            S.cs[slot] = s;
                            S.cj[slot] = j;
                            S.cw[slot] = W;
                        }
                    }
                }
                cmin = fmin(cmin, s);
                cmax = fmax(cmax, s);
            }
        }
        cmin = block_min(cmin, S.red);
        cmax = block_max(cmax, S.red);
        if (mass_mode && iter == 0 && umax_out) *umax_out = block_max(umx, S.red);
        if (iter == 0 && save_hist && !(cmin == cmax)) {   // the first level's counts, for the mask kernel
            for (int b = tid; b < kBins; b += kSelThreads) save_hist[b] = S.cnt[b];
            if (range_out) range_out[2] = 1.0;
        }
        if (!L.jmode && cmin == cmax) {
            // every candidate has the same logit: the ranking among them is by index
            L.jmode = true;
            L.jexact = true;
            L.tie_s = cmin;
            continue;
        }
        // per-thread sums of its bins, then block scan
        unsigned long long th = 0, tl = 0, tc = 0;
        const int b0 = tid * kBinsPerThread;
        for (int q = 0; q < kBinsPerThread; ++q) {
            th += S.mhi[b0 + q];
            tl += S.mlo[b0 + q];
            tc += (unsigned long long)S.cnt[b0 + q];
        }
        unsigned long long tot[3];
        block_excl_scan3(th, tl, tc, S.ured, tot);
        if (!have_target) {
            // first scan covers every key: its total is the softmax normaliser Z
            target = rho * mass_to_double(tot[0], tot[1]);
            have_target = true;
        }
        if (tid == 0) S.misc[0] = -1;
        __syncthreads();
        {
            unsigned long long eh = bhi + th, el = blo + tl;
            long long ec = bcnt + (long long)tc;
            for (int q = 0; q < kBinsPerThread; ++q) {
                const int b = b0 + q;
                const unsigned long long ih = eh + S.mhi[b], il = el + S.mlo[b];
                const long long ic = ec + S.cnt[b];
                bool before_ok, incl_ok;
                if (mass_mode) {
                    before_ok = mass_to_double(eh, el) >= target;
                    incl_ok = mass_to_double(ih, il) >= target;
                } else {
                    before_ok = ec >= count;
                    incl_ok = ic >= count;
                }
                if (!before_ok && incl_ok) {
                    S.misc[0] = b;
                    S.ured[0] = eh;   // safe: scan results already consumed above
                    S.ured[1] = el;
                    reinterpret_cast<long long *>(S.ured)[2] = ec;
                }
                eh = ih;
                el = il;
                ec = ic;
            }
        }
        __syncthreads();
        int bstar = S.misc[0];
        if (bstar < 0) {
            // cannot happen for consistent inputs; fall back to the last non-empty bin
            if (tid == 0) set_status(status, SCOPE_DEV_SELECT_TIE);
            return out;
        }
        bhi = S.ured[0];
        blo = S.ured[1];
        bcnt = reinterpret_cast<long long *>(S.ured)[2];
        const int nb = S.cnt[bstar];
        __syncthreads();

        if (nb <= kCap || L.jmode) {
            if (nb > kCap) {
                if (tid == 0) set_status(status, SCOPE_DEV_SELECT_TIE);
            }
            // the crossing bin's keys: from the window gathered during this pass when the
            // bin lies inside it (the window's keys of other bins are dropped), else by
            // another pass over every key
            bool have = false;
            if (gather_window && bstar >= wlo && bstar <= whi && S.misc[3] <= kCap) {
                const int nwin = S.misc[3];
                double ks[kCap / kSelThreads];
                int kj[kCap / kSelThreads];
                unsigned long long kw[kCap / kSelThreads];
                bool keep[kCap / kSelThreads];
#pragma unroll
                for (int q = 0; q < kCap / kSelThreads; ++q) {
                    const int i = q * kSelThreads + tid;
                    keep[q] = i < nwin && vbin(S.cs[i], hi, scale) == bstar;
                    if (keep[q]) {
                        ks[q] = S.cs[i];
                        kj[q] = S.cj[i];
                        kw[q] = S.cw[i];
                    }
                }
                if (tid == 0) S.misc[1] = 0;
                __syncthreads();
#pragma unroll
                for (int q = 0; q < kCap / kSelThreads; ++q)
                    if (keep[q]) {
                        const int slot = atomicAdd(&S.misc[1], 1);
                        S.cs[slot] = ks[q];
                        S.cj[slot] = kj[q];
                        S.cw[slot] = kw[q];
                    }
                __syncthreads();
                have = S.misc[1] == nb;   // every key of the bin was in the window
                __syncthreads();
            }
            if (!have) {
            if (tid == 0) S.misc[1] = 0;
            __syncthreads();
            KeyBatch next = load_batch(u, 0);
            for (int j0 = 0; j0 < u.N; j0 += kBatch * kSelThreads) {
                const KeyBatch kb = next;
                if (j0 + kBatch * kSelThreads < u.N) next = load_batch(u, j0 + kBatch * kSelThreads);
                double sc[kBatch];
                batch_scores(S, u, kb, sc);
#pragma unroll
                for (int k = 0; k < kBatch; ++k) {
                    const double s = sc[k];
                    if (!kb.v[k] || !in_candidates(L, s)) continue;
                    const int j = j0 + k * kSelThreads + tid;
                    const int b = L.jmode ? jbin(j, u.N) : vbin(s, hi, scale);
                    if (b != bstar) continue;
                    const int slot = atomicAdd(&S.misc[1], 1);
                    if (slot < kCap) {
                        S.cs[slot] = s;
                        S.cj[slot] = j;
                        if (mass_mode) S.cw[slot] = weight_mass(key_weight(s, u), u);
                    }
                }
            }
            __syncthreads();
            }
            const int n = min(S.misc[1], kCap);
            if (n == 0) {   // the gather pass always finds the crossing bin's keys
                if (tid == 0) set_status(status, SCOPE_DEV_SELECT_TIE);
                __syncthreads();
                return out;
            }
            // rank among the gathered keys: logit descending, index ascending
            for (int i = tid; i < n; i += kSelThreads) {
                const double si = S.cs[i];
                const int ji = S.cj[i];
                int r = 0;
                for (int k = 0; k < n; ++k) {
                    const double sk = S.cs[k];
                    r += (sk > si) || (sk == si && S.cj[k] < ji);
                }
                S.order[r] = i;
            }
            __syncthreads();
            int pos = -1;
            if (tid == 0) S.red[31] = INFINITY;
            __syncthreads();
            if (mass_mode) {
                if (tid < 32) {
                    unsigned long long rh = bhi, rl = blo;
                    for (int base = 0; base < n && pos < 0; base += 32) {
                        const int idx = base + tid;
                        unsigned long long W = idx < n ? S.cw[S.order[idx]] : 0ull;
                        unsigned long long h = W >> 32, l = W & 0xffffffffull, z = 0;
                        warp_scan3(h, l, z);
                        const bool ok = idx < n && mass_to_double(rh + h, rl + l) >= target;
                        const unsigned bal = __ballot_sync(0xffffffffu, ok);
                        if (bal) {
                            pos = base + __ffs(bal) - 1;
                            // the decision's closeness to a tie, as the oracle measures it:
                            // the masses before and through the crossing key against rho Z
                            if (tid == pos - base) {
                                const double incl = mass_to_double(rh + h, rl + l);
                                const double excl = mass_to_double(rh + h - (W >> 32), rl + l - (W & 0xffffffffull));
                                const double Z = target / rho;
                                S.red[31] = fmin(fabs(incl - target), fabs(excl - target)) / Z;
                            }
                        }
                        rh += __shfl_sync(0xffffffffu, h, 31);
                        rl += __shfl_sync(0xffffffffu, l, 31);
                    }
                    if (tid == 0) S.misc[2] = pos < 0 ? n - 1 : pos;
                }
            } else if (tid == 0) {
                long long q = count - 1 - bcnt;
                S.misc[2] = (int)(q < 0 ? 0 : (q >= n ? n - 1 : q));
            }
            __syncthreads();
            pos = S.misc[2];
            const int i = S.order[pos];
            out.s = S.cs[i];
            out.j = S.cj[i];
            out.rank = bcnt + pos;
            if (mass_mode) out.margin = S.red[31];
            __syncthreads();
            return out;
        }
        // refine inside the crossing bin
        if (L.n >= kMaxLevels) {
            if (tid == 0) set_status(status, SCOPE_DEV_SELECT_TIE);
            L.jmode = true;   // order the remaining candidates by index
            continue;
        }
        L.hi[L.n] = hi;
        L.scale[L.n] = scale;
        L.bstar[L.n] = bstar;
        L.n += 1;
        const double nhi = hi - (double)bstar / scale, nlo = hi - (double)(bstar + 1) / scale;
        hi = nhi;
        lo = nlo;
        __syncthreads();
    }
    if (tid == 0) set_status(status, SCOPE_DEV_SELECT_TIE);
    return out;
}

// Builds the LUT of unit c: P^m[c, z] for the three subspaces m and every code z.
__device__ void build_tables(const SelArgs &a, const SelSmem &S, int bh, int c)
{
    const int tid = threadIdx.x, Cm = a.Cm, d = a.d;
    const double *qc = a.qcent + ((size_t)bh * a.Cq + c) * d;
    for (int i = tid; i < d; i += kSelThreads) S.qc[i] = qc[i];
    __syncthreads();
    const int bnd[4] = {0, a.dt, a.dt + a.dh, d};
    const double *kc = a.kcent + (size_t)bh * Cm * d;
    for (int idx = tid; idx < 3 * Cm; idx += kSelThreads) {
        const int m = idx / Cm, z = idx - m * Cm;
        double acc = 0.0;
        for (int i = bnd[m]; i < bnd[m + 1]; ++i)
            acc = __dadd_rn(acc, __dmul_rn(S.qc[i], kc[(size_t)z * d + i]));
        S.lut[idx] = acc;
    }
    __syncthreads();
}

// ------------------------------------------------------------------------- kernels
// Reports caller-supplied codes outside [0, Cm) (the tables clamp them).
__global__ void sel_check_kernel(SelArgs a)
{
    const long long total = (long long)a.BH * 3 * a.N;
    bool bad = false;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x)
        bad |= a.codes[i] >= a.Cm;
    if (__syncthreads_or(bad) && threadIdx.x == 0) set_status(a.status, SCOPE_DEV_BAD_ASSIGN);
}

// Top-p count p_c and base count b_c (Eqs. 7-8).  grid (Cq, BH).
__global__ void __launch_bounds__(kSelThreads, 2) sel_topp_kernel(SelArgs a)
{
    extern __shared__ __align__(16) char smem_raw[];
    const SelSmem S = carve(smem_raw, a.Cm, a.d);
    const int c = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    build_tables(a, S, bh, c);
    Unit u;
    u.zt = a.codes + (size_t)bh * 3 * a.N;
    u.zh = u.zt + a.N;
    u.zw = u.zh + a.N;
    u.Cm = a.Cm;
    u.N = a.N;
    u.inv = a.inv_sqrt_d;
    // Score bounds from the tables: rounded sums and the positive scale are monotone, so
    // (1/sqrt d)((max P^T + max P^H) + max P^W) bounds every key's score from above (and
    // likewise from below); they only set the range of the first histogram.
    double tmax[3], tmin[3];
    for (int m = 0; m < 3; ++m) {
        double mx = -DBL_MAX, mn = DBL_MAX;
        for (int z = tid; z < a.Cm; z += kSelThreads) {
            mx = fmax(mx, S.lut[m * a.Cm + z]);
            mn = fmin(mn, S.lut[m * a.Cm + z]);
        }
        tmax[m] = block_max(mx, S.red);
        tmin[m] = block_min(mn, S.red);
    }
    const double smax = __dmul_rn(u.inv, __dadd_rn(__dadd_rn(tmax[0], tmax[1]), tmax[2]));
    const double smin = __dmul_rn(u.inv, __dadd_rn(__dadd_rn(tmin[0], tmin[1]), tmin[2]));
    // Key weights u_j = exp(s_j - smax) <= 1 (smax bounds every logit), so masses are
    // quantised against 1: at most N 2^-64 of absolute error in total.  That stays below
    // 1e-9 of the total mass Z >= max_j u_j unless the largest weight is tiny, in which
    // case the selection runs again normalised by the largest weight itself.
    u.sref = smax;
    u.inv_umax = 1.0;
    long long p = a.N;
    SelectOut so{smax, 0, 0};
    const size_t unit = (size_t)bh * a.Cq + c;
    int32_t *hist = a.hist ? a.hist + unit * kBins : nullptr;
    // every key's first-level bin, kept beside the counts when the mask kernel can use them
    uint16_t *bins = hist && a.bins && a.lut ? a.bins + unit * a.bins_stride : nullptr;
    if (bins)   // the unit's tables, so that the mask kernel need not build them again
        for (int i = tid; i < 3 * a.Cm; i += kSelThreads) a.lut[unit * 3 * a.Cm + i] = S.lut[i];
    // the first level's value range of the saved counts, and whether they were saved
    double range[3] = {smax, smin, 0.0};
    if (a.rho < 1.0) {
        double umax = 1.0;
        so = block_select(S, u, true, a.rho, 0, smax, smin, a.status, &umax, hist, range, bins);
        if (umax < (double)a.N * 0x1p-64 * 1e9 && umax > 0.0) {
            u.inv_umax = 1.0 / umax;
            so = block_select(S, u, true, a.rho, 0, smax, smin, a.status);
        }
        p = so.rank + 1;
        if (tid == 0 && a.stats) {
            atomicAdd(&a.stats[0], 1);
            if (so.margin < 1e-6) atomicAdd(&a.stats[1], 1);
            if (so.margin < 3e-7) atomicAdd(&a.stats[2], 1);
        }
    }
    // The counts are saved only by a first level that binned by value (not when every logit
    // is the same, and not at rho = 1, where no pass runs and r = N selects every key).
    const bool saved = hist && range[2] != 0.0;
    if (tid == 0) {
        const long long b = p > a.kfix ? p : a.kfix;
        if (a.topp) a.topp[unit] = (int32_t)p;
        a.base[unit] = (int32_t)b;
        double *st = a.state + unit * 8;
        st[0] = smax;
        st[1] = smin;
        st[2] = so.s;
        st[3] = (double)so.j;
        st[4] = (double)p;
        st[5] = saved ? 1.0 : 0.0;
        st[6] = range[0];
        st[7] = range[1];
    }
}

// k_head (Eq. 9) and final counts r_c (Eq. 10; with the online k_head switched off,
// the ablation, r_c = b_c).  grid BH.
__global__ void __launch_bounds__(256) sel_khead_kernel(SelArgs a)
{
    __shared__ long long rn[8], rd[8];
    const int bh = blockIdx.x, tid = threadIdx.x;
    long long num = 0, den = 0;
    for (int c = tid; c < a.Cq; c += 256) {
        const long long n = a.qsizes[(size_t)bh * a.Cq + c];
        num += n * (long long)a.base[(size_t)bh * a.Cq + c];
        den += n;
    }
    for (int o = 16; o; o >>= 1) {
        num += __shfl_xor_sync(0xffffffffu, num, o);
        den += __shfl_xor_sync(0xffffffffu, den, o);
    }
    if ((tid & 31) == 0) {
        rn[tid >> 5] = num;
        rd[tid >> 5] = den;
    }
    __syncthreads();
    if (tid == 0) {
        num = 0;
        den = 0;
        for (int w = 0; w < 8; ++w) {
            num += rn[w];
            den += rd[w];
        }
        rn[0] = den > 0 ? (num + den - 1) / den : a.N;
        a.khead[bh] = (int32_t)rn[0];
    }
    __syncthreads();
    const long long kh = rn[0];
    for (int c = tid; c < a.Cq; c += 256) {
        const long long b = a.base[(size_t)bh * a.Cq + c];
        a.final_cnt[(size_t)bh * a.Cq + c] = (int32_t)(b < kh && a.khead_mode == SCOPE_KHEAD_ONLINE ? kh : b);
    }
}

// Selected set S_c = the first r_c keys of the ranking, as a bitmask.  grid (Cq, BH).
__global__ void __launch_bounds__(kSelThreads) sel_mask_kernel(SelArgs a)
{
    extern __shared__ __align__(16) char smem_raw[];
    const SelSmem S = carve(smem_raw, a.Cm, a.d);
    const int c = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
    const size_t unit = (size_t)bh * a.Cq + c;
    uint32_t *row = a.mask + unit * a.nw;
    const long long r = a.final_cnt[unit];
    const int lane = tid & 31, warp = tid >> 5;
    if (r >= a.N) {
        for (int w = tid; w < a.nw; w += kSelThreads) {
            const int rem = a.N - w * 32;
            row[w] = rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u);
        }
        return;
    }
    const double *st = a.state + unit * 8;
    // With the Top-p kernel's saved bins (and its copy of the tables), the pass below reads
    // each key's first-level bin and computes a logit only for the keys of the boundary bin.
    const bool use_bins = a.bins && a.lut && a.hist && st[5] != 0.0;
    if (use_bins) {
        const double *lut = a.lut + unit * 3 * a.Cm;
        for (int i = tid; i < 3 * a.Cm; i += kSelThreads) S.lut[i] = lut[i];
        __syncthreads();
    } else {
        build_tables(a, S, bh, c);
    }
    Unit u;
    u.zt = a.codes + (size_t)bh * 3 * a.N;
    u.zh = u.zt + a.N;
    u.zw = u.zh + a.N;
    u.Cm = a.Cm;
    u.N = a.N;
    u.inv = a.inv_sqrt_d;
    u.sref = a.state[unit * 8];
    u.inv_umax = 1.0;
    const double hi = st[6], lo = st[7];   // the value range of the saved level-0 counts
    const double scale = (hi > lo) ? (double)kBins / (hi - lo) : 0.0;
    // Either the exact last selected key (s*, j*) is known -- the Top-p boundary when r_c =
    // p_c, or a count-based select -- or the level-0 counts saved by the Top-p kernel give the
    // bin b* that holds the r_c-th key: every key of a lower bin (higher logits) is selected,
    // and the keys of b* are gathered in this same pass and ranked afterwards.
    double s_star = 0.0;
    int j_star = 0, bstar = -1;
    long long before = 0;
    if ((long long)st[4] == r) {
        s_star = st[2];
        j_star = (int)st[3];
    } else {
        if (st[5] != 0.0) {
            const int32_t *h = a.hist + unit * kBins;
            unsigned long long z0 = 0, z1 = 0, tc = 0;
            const int b0 = tid * kBinsPerThread;
            int cnt[kBinsPerThread];
            for (int q = 0; q < kBinsPerThread; ++q) {
                cnt[q] = h[b0 + q];
                tc += (unsigned long long)cnt[q];
            }
            unsigned long long tot[3];
            block_excl_scan3(z0, z1, tc, S.ured, tot);
            if (tid == 0) S.misc[0] = -1;
            __syncthreads();
            long long ec = (long long)tc;
            for (int q = 0; q < kBinsPerThread; ++q) {
                if (ec < r && ec + cnt[q] >= r) {
                    S.misc[0] = b0 + q;
                    S.misc[1] = cnt[q];
                    reinterpret_cast<long long *>(S.ured)[3] = ec;
                }
                ec += cnt[q];
            }
            __syncthreads();
            if (S.misc[0] >= 0 && S.misc[1] <= kCap) {
                bstar = S.misc[0];
                before = reinterpret_cast<long long *>(S.ured)[3];
            }
            __syncthreads();
        }
        if (bstar < 0) {   // no saved counts, or a crossing bin too large to gather
            const SelectOut so = block_select(S, u, false, 0.0, r, hi, lo, a.status);
            s_star = so.s;
            j_star = so.j;
        }
    }
    if (tid == 0) S.misc[2] = 0;
    __syncthreads();
    if (use_bins) {
        // Bins are monotone in the logit (a lower bin holds strictly higher logits), so a key
        // of a bin below the boundary bin is selected, one above it is not, and only the keys
        // of the boundary bin need their logit: compared with (s*, j*), or gathered for ranking.
        const bool gather = bstar >= 0;
        const int bsel = gather ? bstar : vbin(s_star, hi, scale);
        const uint16_t *bn = a.bins + unit * a.bins_stride;
        // thread t takes keys 8 t .. 8 t + 7 of each step (one 16-byte load; rows are padded
        // to a multiple of 8 keys); lanes 4 q .. 4 q + 3 fill word q of the warp's 8 words
        constexpr int kPer = 8, kStep = kPer * kSelThreads;
        auto load8 = [&](int j0) -> uint4 {
            const int j = j0 + kPer * tid;
            return j < a.N ? *reinterpret_cast<const uint4 *>(bn + j) : make_uint4(0u, 0u, 0u, 0u);
        };
        uint4 next = load8(0), next2 = load8(kStep);
        for (int j0 = 0; j0 < a.N; j0 += kStep) {
            const uint4 cur = next;
            next = next2;
            if (j0 + 2 * kStep < a.N) next2 = load8(j0 + 2 * kStep);
            const uint32_t pair[4] = {cur.x, cur.y, cur.z, cur.w};
            const int jb = j0 + kPer * tid;
            const int nv = min(max(a.N - jb, 0), kPer);   // keys of this thread below N
            // bit i: key jb + i lies below (lt) or in (eq) the boundary bin
            uint32_t lt = 0, eq = 0;
#pragma unroll
            for (int i = 0; i < kPer; ++i) {
                const uint32_t b = (pair[i >> 1] >> (16 * (i & 1))) & 0xffffu;
                lt |= (uint32_t)(b < (uint32_t)bsel) << i;
                eq |= (uint32_t)(b == (uint32_t)bsel) << i;
            }
            const uint32_t valid = (1u << nv) - 1u;
            uint32_t m8 = lt & valid;
            eq &= valid;
            while (eq) {   // the boundary bin's keys (a few per unit)
                const int i = __ffs(eq) - 1;
                eq &= eq - 1u;
                const int j = jb + i;
                const double sj = key_score(S, u, j);
                if (gather) {
                    const int slot = atomicAdd(&S.misc[2], 1);
                    if (slot < kCap) {
                        S.cs[slot] = sj;
                        S.cj[slot] = j;
                    }
                } else if ((sj > s_star) || (sj == s_star && j <= j_star)) {
                    m8 |= 1u << i;
                }
            }
            uint32_t bits = m8 << (8 * (lane & 3));
            bits |= __shfl_xor_sync(0xffffffffu, bits, 1);
            bits |= __shfl_xor_sync(0xffffffffu, bits, 2);
            const int w = jb >> 5;
            if ((lane & 3) == 0 && w < a.nw) row[w] = bits;
        }
        if (!gather) return;
    } else {
    // word w of the row holds keys 32 w .. 32 w + 31; a batch covers kBatch x 16 words, word
    // j0 / 32 + k * 16 + warp of batch j0 from warp `warp`
    // this pass is bound by the latency of the code loads (L2): two batches are in flight
    constexpr int kStep = kBatch * kSelThreads;
    KeyBatch next = load_batch(u, 0), next2 = load_batch(u, kStep);
    for (int j0 = 0; j0 < a.N; j0 += kStep) {
        const KeyBatch kb = next;
        next = next2;
        if (j0 + 2 * kStep < a.N) next2 = load_batch(u, j0 + 2 * kStep);
        double sc[kBatch];
        batch_scores(S, u, kb, sc);
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
            const int j = j0 + k * kSelThreads + tid;
            bool sel;
            if (bstar < 0) {
                sel = kb.v[k] && ((sc[k] > s_star) || (sc[k] == s_star && j <= j_star));
            } else {
                const int b = kb.v[k] ? vbin(sc[k], hi, scale) : kBins;
                sel = b < bstar;
                if (b == bstar) {
                    const int slot = atomicAdd(&S.misc[2], 1);
                    if (slot < kCap) {
                        S.cs[slot] = sc[k];
                        S.cj[slot] = j;
                    }
                }
            }
            const unsigned bits = __ballot_sync(0xffffffffu, sel);
            const int w = (j0 + k * kSelThreads) / 32 + warp;
            if (lane == 0 && w < a.nw) row[w] = bits;
        }
    }
    }
    if (bstar < 0) return;
    // rank the keys of b* (logit descending, index ascending) and add the first r - before
    __threadfence_block();
    __syncthreads();
    const int n = min(S.misc[2], kCap);
    if (n != S.misc[1] && tid == 0) set_status(a.status, SCOPE_DEV_SELECT_TIE);   // counts disagree
    for (int i = tid; i < n; i += kSelThreads) {
        const double si = S.cs[i];
        const int ji = S.cj[i];
        int rk = 0;
        for (int k = 0; k < n; ++k) {
            const double sk = S.cs[k];
            rk += (sk > si) || (sk == si && S.cj[k] < ji);
        }
        S.order[rk] = i;
    }
    __syncthreads();
    const long long need = r - before;
    for (long long q = tid; q < need && q < n; q += kSelThreads) {
        const int j = S.cj[S.order[q]];
        atomicOr(&row[j >> 5], 1u << (j & 31));
    }
}

}  // namespace

size_t select_smem_bytes(int Cm, int d)
{
    return sel_smem_bytes(Cm, d);
}

cudaError_t select_run(const SelArgs &a, cudaStream_t s)
{
    const size_t smem = sel_smem_bytes(a.Cm, a.d);
    cudaFuncSetAttribute(sel_topp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(sel_mask_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    dim3 grid(a.Cq, a.BH);
    if (a.stats) {
        const cudaError_t e = cudaMemsetAsync(a.stats, 0, 4 * sizeof(int32_t), s);
        if (e != cudaSuccess) return e;
    }
    sel_check_kernel<<<256, 256, 0, s>>>(a);
    sel_topp_kernel<<<grid, kSelThreads, smem, s>>>(a);
    sel_khead_kernel<<<a.BH, 256, 0, s>>>(a);
    sel_mask_kernel<<<grid, kSelThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace scope
