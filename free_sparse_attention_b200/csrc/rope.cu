// 3D rotary position embedding of pre-RoPE queries and keys: the step before SCOPE's
// clustering, which works on post-RoPE q and k whose channels fall into the temporal,
// height and width ranges of 3D RoPE (SCOPE abstract; the rotation is RoFormer's, the
// page's reference [31]).
//
// Token n = t*Hg*Wg + h*Wg + w.  In channel range a (start c_a, even width d_a, position
// p_a = t, h or w) the pair (c_a + 2i, c_a + 2i + 1) turns by phi = p_a * base^(-2i/d_a):
//   y0 = x0 cos phi - x1 sin phi,   y1 = x0 sin phi + x1 cos phi.
// The result is that of binary64 arithmetic: two rounded products and a rounded sum per
// output, no fused multiply-add, then one rounding to the tensor's type.  cos and sin of
// every (axis, position, pair) are tabulated per block in shared memory (binary64 pairs,
// plus their binary32 roundings).  For bf16 a binary32 evaluation comes first: it is off
// the binary64 value by less than 3 * 2^-24 (|x0| + |x1|), so when y32 - e and y32 + e,
// e = 2^-21 (|x0| + |x1|), round to the same bf16 value, that value is the rounding of the
// binary64 result too (rounding is monotone); otherwise (rarely: y near a bf16 rounding
// boundary) the group of 8 channels is recomputed in binary64.
//
// HBM-bound: every element is read once and written once.  A persistent grid (one block
// per SM: 1024 threads for bf16, 512 for fp32) strides over rows; each thread owns 8 consecutive channels of a row (one 16-byte
// vector for bf16, two for fp32) and streams its rows through a private ring of STAGES
// shared-memory slots filled by cp.async, so that STAGES - 1 rows of loads stay in flight
// while it rotates the oldest one (no thread waits on another: each thread reads only the
// slots it filled itself, after cp.async.wait_group).
#include "common.cuh"

namespace scope {

namespace {

// threads per block: bf16 fits 64 registers, so 32 warps per SM hide the per-row chain
template <bool BF16>
constexpr int rope_threads()
{
    return BF16 ? 1024 : 512;
}

// binary64 -> bf16, one rounding to nearest even (cvt.rn.bf16.f64).
__device__ __forceinline__ uint16_t f64_to_bf16(double v)
{
    return __bfloat16_as_ushort(__double2bfloat16(v));
}

// Rotate one pair with the table entry cs = (cos phi, sin phi), binary64.
__device__ __forceinline__ void rot(double x0, double x1, double2 cs, double &y0, double &y1)
{
    y0 = __dsub_rn(__dmul_rn(x0, cs.x), __dmul_rn(x1, cs.y));
    y1 = __dadd_rn(__dmul_rn(x0, cs.y), __dmul_rn(x1, cs.x));
}

// bf16 fast path for one pair: writes the two rounded outputs and returns whether both
// were decided (see the header).
__device__ __forceinline__ bool rot_bf16_fast(uint32_t w, float2 cs, uint32_t &out)
{
    const float x0 = __uint_as_float(w << 16), x1 = __uint_as_float(w & 0xFFFF0000u);
    const float e = __fmul_rn(__fadd_rn(fabsf(x0), fabsf(x1)), 0x1p-21f);
    const float y0 = __fmaf_rn(x0, cs.x, -__fmul_rn(x1, cs.y));
    const float y1 = __fmaf_rn(x0, cs.y, __fmul_rn(x1, cs.x));
    const __nv_bfloat162 b0 = __floats2bfloat162_rn(__fsub_rn(y0, e), __fadd_rn(y0, e));
    const __nv_bfloat162 b1 = __floats2bfloat162_rn(__fsub_rn(y1, e), __fadd_rn(y1, e));
    const uint32_t u0 = *reinterpret_cast<const uint32_t *>(&b0), u1 = *reinterpret_cast<const uint32_t *>(&b1);
    out = (u0 & 0xFFFFu) | (u1 << 16);
    return ((u0 ^ (u0 >> 16)) & 0xFFFFu) == 0u && ((u1 ^ (u1 >> 16)) & 0xFFFFu) == 0u;
}

// x / d for x < 2^31 by a multiply and a shift (Granlund and Montgomery, "Division by
// invariant integers using multiplication", 1994): with l = ceil(log2 d) and
// m = floor(2^32 (2^l - d) / d) + 1, x / d = (umulhi(x, m) + x) >> l.
__device__ __forceinline__ unsigned fdiv(unsigned x, FastDiv f)
{
    return (__umulhi(x, f.m) + x) >> f.l;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_commit()
{
    asm volatile("cp.async.commit_group;\n" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Element type traits: VEC 16-byte vectors per 8-channel group.
template <bool BF16>
struct RopeElt {
    static constexpr int VEC = BF16 ? 1 : 2;
    static constexpr int BYTES = BF16 ? 2 : 4;
};

template <bool BF16, int STAGES>
__global__ void __launch_bounds__(rope_threads<BF16>(), 1) rope3d_kernel(RopeArgs a)
{
    using E = RopeElt<BF16>;
    extern __shared__ __align__(16) unsigned char smem[];
    // cos/sin table: axis a holds (positions of a) x (d_a / 2) entries, position-major,
    // axes in the order T, H, W; the binary32 copy follows the binary64 one; then the ring
    const int hT = a.dt / 2, hH = a.dh / 2, hW = a.dw / 2;
    const int o1 = a.T * hT, o2 = o1 + a.Hg * hH, o3 = o2 + a.Wg * hW;
    double2 *tab = reinterpret_cast<double2 *>(smem);
    float2 *tab32 = reinterpret_cast<float2 *>(tab + o3);
    uint4 *ring = reinterpret_cast<uint4 *>(smem + ((size_t)o3 * 24 + 15) / 16 * 16);

    // issue the first loads before the table is built: they overlap its transcendental work
    const int tpr = a.d / 8;                       // threads per row
    const int g = threadIdx.x % tpr;               // this thread's 8-channel group
    const int rpp = blockDim.x / tpr;              // rows per block pass
    const long long step = (long long)gridDim.x * rpp;
    const long long total = a.rows * a.n_tensors;  // virtual rows: tensor-major
    const long long vr0 = (long long)blockIdx.x * rpp + threadIdx.x / tpr;
    const unsigned char *X0 = static_cast<const unsigned char *>(a.X[0]);
    const unsigned char *X1 = static_cast<const unsigned char *>(a.X[1]);
    unsigned char *Y0 = static_cast<unsigned char *>(a.Y[0]);
    unsigned char *Y1 = static_cast<unsigned char *>(a.Y[1]);
    const size_t row_bytes = (size_t)a.d * E::BYTES;
    const size_t grp_off = (size_t)g * 16 * E::VEC;
    auto slot = [&](int s) { return ring + ((size_t)s * blockDim.x + threadIdx.x) * E::VEC; };
    auto issue = [&](long long vr, int s) {
        if (vr < total) {
            const bool second = vr >= a.rows;
            const long long r = vr - (second ? a.rows : 0);
            const unsigned char *src = (second ? X1 : X0) + (size_t)r * row_bytes + grp_off;
            uint4 *dst = slot(s);
#pragma unroll
            for (int j = 0; j < E::VEC; ++j)
                cp_async16((uint32_t)__cvta_generic_to_shared(dst + j), src + 16 * j);
        }
        cp_async_commit();   // one group per row, empty past the end
    };
#pragma unroll
    for (int s = 0; s < STAGES - 1; ++s) issue(vr0 + s * step, s);

    for (int e = threadIdx.x; e < o3; e += blockDim.x) {
        const int ax = e < o1 ? 0 : (e < o2 ? 1 : 2);
        const int half = ax == 0 ? hT : (ax == 1 ? hH : hW);
        const int r = e - (ax == 0 ? 0 : (ax == 1 ? o1 : o2));
        const int p = r / half, i = r - p * half;
        const double theta = pow(a.base, (double)(-2 * i) / (double)(2 * half));
        double sn, cs;
        sincos(__dmul_rn((double)p, theta), &sn, &cs);
        tab[e] = make_double2(cs, sn);
        tab32[e] = make_float2(__double2float_rn(cs), __double2float_rn(sn));
    }
    __syncthreads();

    // the 4 pairs of the group: axis, table index at position 0 and per-position stride
    int pax[4], pbase[4], pstride[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int c = 8 * g + 2 * q;
        const int ax = c < a.dt ? 0 : (c < a.dt + a.dh ? 1 : 2);
        const int c0 = ax == 0 ? 0 : (ax == 1 ? a.dt : a.dt + a.dh);
        pax[q] = ax;
        pstride[q] = ax == 0 ? hT : (ax == 1 ? hH : hW);
        pbase[q] = (ax == 0 ? 0 : (ax == 1 ? o1 : o2)) + (c - c0) / 2;
    }
    const unsigned HW = (unsigned)a.Hg * (unsigned)a.Wg;
    int s = 0;
    for (long long vr = vr0; vr < total; vr += step) {
        issue(vr + (STAGES - 1) * step, s == 0 ? STAGES - 1 : s - 1);
        cp_async_wait<STAGES - 1>();   // this thread's row vr has landed in slot s
        const uint4 *src = slot(s);
        s = s + 1 == STAGES ? 0 : s + 1;
        const bool second = vr >= a.rows;
        const unsigned ur = (unsigned)(vr - (second ? a.rows : 0));   // rows < 2^31
        unsigned char *dst = (second ? Y1 : Y0) + (size_t)ur * row_bytes + grp_off;
        const unsigned n = ur - fdiv(ur, a.div_N) * (unsigned)a.N;
        const unsigned t = fdiv(n, a.div_HW), rem = n - t * HW;
        const unsigned h = fdiv(rem, a.div_Wg), w = rem - h * (unsigned)a.Wg;
        int idx[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const unsigned p = pax[q] == 0 ? t : (pax[q] == 1 ? h : w);
            idx[q] = pbase[q] + (int)p * pstride[q];
        }
        if constexpr (BF16) {
            const uint4 v = src[0];
            const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
            uint32_t o[4];
            bool ok = true;
#pragma unroll
            for (int q = 0; q < 4; ++q) ok &= rot_bf16_fast(wv[q], tab32[idx[q]], o[q]);
            if (!ok) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    double y0, y1;
                    rot((double)__uint_as_float(wv[q] << 16), (double)__uint_as_float(wv[q] & 0xFFFF0000u),
                        tab[idx[q]], y0, y1);
                    o[q] = (uint32_t)f64_to_bf16(y0) | ((uint32_t)f64_to_bf16(y1) << 16);
                }
            }
            __stcs(reinterpret_cast<uint4 *>(dst), make_uint4(o[0], o[1], o[2], o[3]));
        } else {
            const float4 v0 = *reinterpret_cast<const float4 *>(src), v1 = *reinterpret_cast<const float4 *>(src + 1);
            const float x[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            float y[8];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                double y0, y1;
                rot((double)x[2 * q], (double)x[2 * q + 1], tab[idx[q]], y0, y1);
                y[2 * q] = __double2float_rn(y0);
                y[2 * q + 1] = __double2float_rn(y1);
            }
            float4 *d4 = reinterpret_cast<float4 *>(dst);
            __stcs(d4, make_float4(y[0], y[1], y[2], y[3]));
            __stcs(d4 + 1, make_float4(y[4], y[5], y[6], y[7]));
        }
    }
    cp_async_wait<0>();
}

template <bool BF16, int STAGES>
cudaError_t launch_rope(const RopeArgs &a, int grid, size_t table_bytes, cudaStream_t st)
{
    const size_t smem = (table_bytes + 15) / 16 * 16 + (size_t)STAGES * rope_threads<BF16>() * 16 * RopeElt<BF16>::VEC;
    cudaError_t e = cudaFuncSetAttribute(rope3d_kernel<BF16, STAGES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    rope3d_kernel<BF16, STAGES><<<grid, rope_threads<BF16>(), smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

size_t rope_table_bytes(int T, int Hg, int Wg, int dt, int dh, int dw)
{
    return (sizeof(double2) + sizeof(float2)) * ((size_t)T * (dt / 2) + (size_t)Hg * (dh / 2) + (size_t)Wg * (dw / 2));
}

FastDiv make_fastdiv(unsigned d)
{
    unsigned l = 0;
    while ((1ull << l) < d) ++l;
    FastDiv f;
    f.l = l;
    f.m = (unsigned)(((1ull << 32) * ((1ull << l) - d)) / d + 1);
    return f;
}

cudaError_t rope3d_run(const RopeArgs &a_in, int num_sms, cudaStream_t s)
{
    RopeArgs a = a_in;
    a.div_N = make_fastdiv((unsigned)a.N);
    a.div_HW = make_fastdiv((unsigned)a.Hg * (unsigned)a.Wg);
    a.div_Wg = make_fastdiv((unsigned)a.Wg);
    const size_t table = rope_table_bytes(a.T, a.Hg, a.Wg, a.dt, a.dh, a.dw);
    // ring depth: as deep as the shared memory left after the table allows (227 KB per block)
    const size_t room = (size_t)227 * 1024 - (table + 15) / 16 * 16;
    const size_t per_stage = (size_t)16 * (a.is_bf16 ? rope_threads<true>() : 2 * rope_threads<false>());
    const int stages = room >= 16 * per_stage ? 16 : (room >= 8 * per_stage ? 8 : (room >= 4 * per_stage ? 4 : 2));
    if (a.is_bf16) {
        if (stages == 16) return launch_rope<true, 16>(a, num_sms, table, s);
        if (stages == 8) return launch_rope<true, 8>(a, num_sms, table, s);
        if (stages == 4) return launch_rope<true, 4>(a, num_sms, table, s);
        return launch_rope<true, 2>(a, num_sms, table, s);
    }
    if (stages >= 8) return launch_rope<false, 8>(a, num_sms, table, s);
    if (stages == 4) return launch_rope<false, 4>(a, num_sms, table, s);
    return launch_rope<false, 2>(a, num_sms, table, s);
}

}  // namespace scope
