// 3D rotary position embedding of pre-RoPE queries and keys: the step before SCOPE's
// clustering, which works on post-RoPE q and k whose channels fall into the temporal,
// height and width ranges of 3D RoPE (SCOPE abstract; the rotation is RoFormer's, the
// page's reference [31]).
//
// Token n = t*Hg*Wg + h*Wg + w.  In channel range a (start c_a, even width d_a, position
// p_a = t, h or w) the pair (c_a + 2i, c_a + 2i + 1) turns by phi = p_a * base^(-2i/d_a):
//   y0 = x0 cos phi - x1 sin phi,   y1 = x0 sin phi + x1 cos phi.
// Arithmetic is binary64: two rounded products and a rounded sum per output, no fused
// multiply-add, then one rounding to the tensor's type.  cos and sin of every
// (axis, position, pair) are tabulated per block in shared memory (binary64 pairs).
//
// HBM-bound: every element is read once and written once.  A persistent grid (one block
// per SM) strides over rows; each thread owns 8 consecutive channels of a row
// (one 16-byte vector for bf16, two for fp32), keeps the table offsets of its 4 pairs in
// registers and has kRopeUnroll rows' loads in flight before it computes.
#include "common.cuh"

namespace scope {

namespace {

constexpr int kRopeThreads = 512;

// binary64 -> bf16 with one rounding (to nearest, ties to even): round toward zero to
// binary32, make the last bit sticky if that was inexact (round-to-odd keeps enough
// information for a second rounding 16 bits further up), then round to nearest even.
__device__ __forceinline__ uint16_t f64_to_bf16(double v)
{
    float f = __double2float_rz(v);
    uint32_t u = __float_as_uint(f);
    if ((double)f != v) u |= 1u;
    return __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(u)));
}

__device__ __forceinline__ double bf16_lo(uint32_t w)
{
    return (double)__uint_as_float(w << 16);
}

__device__ __forceinline__ double bf16_hi(uint32_t w)
{
    return (double)__uint_as_float(w & 0xFFFF0000u);
}

// Rotate one pair with the table entry cs = (cos phi, sin phi).
__device__ __forceinline__ void rot(double x0, double x1, double2 cs, double &y0, double &y1)
{
    y0 = __dsub_rn(__dmul_rn(x0, cs.x), __dmul_rn(x1, cs.y));
    y1 = __dadd_rn(__dmul_rn(x0, cs.y), __dmul_rn(x1, cs.x));
}

template <bool BF16>
struct Vec8;

template <>
struct Vec8<true> {
    uint4 v;
    __device__ __forceinline__ void load(const void *base, long long row, int d, int g)
    {
        v = __ldcs(reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(base) + row * d) + g);
    }
    __device__ __forceinline__ double get(int k) const
    {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        return (k & 1) ? bf16_hi(w[k >> 1]) : bf16_lo(w[k >> 1]);
    }
    __device__ __forceinline__ static void store(void *base, long long row, int d, int g, const double *y)
    {
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) w[q] = (uint32_t)f64_to_bf16(y[2 * q]) | ((uint32_t)f64_to_bf16(y[2 * q + 1]) << 16);
        __stcs(reinterpret_cast<uint4 *>(static_cast<uint16_t *>(base) + row * d) + g, make_uint4(w[0], w[1], w[2], w[3]));
    }
};

template <>
struct Vec8<false> {
    float4 a, b;
    __device__ __forceinline__ void load(const void *base, long long row, int d, int g)
    {
        const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(base) + row * d) + 2 * g;
        a = __ldcs(p);
        b = __ldcs(p + 1);
    }
    __device__ __forceinline__ double get(int k) const
    {
        const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        return (double)f[k];
    }
    __device__ __forceinline__ static void store(void *base, long long row, int d, int g, const double *y)
    {
        float4 *p = reinterpret_cast<float4 *>(static_cast<float *>(base) + row * d) + 2 * g;
        __stcs(p, make_float4(__double2float_rn(y[0]), __double2float_rn(y[1]), __double2float_rn(y[2]),
                              __double2float_rn(y[3])));
        __stcs(p + 1, make_float4(__double2float_rn(y[4]), __double2float_rn(y[5]), __double2float_rn(y[6]),
                                  __double2float_rn(y[7])));
    }
};

template <bool BF16>
__global__ void __launch_bounds__(kRopeThreads, 1) rope3d_kernel(RopeArgs a)
{
    constexpr int kRopeUnroll = BF16 ? 8 : 4;   // 64 KB of loads in flight per SM
    extern __shared__ double2 tab[];
    const int dims[3] = {a.dt, a.dh, a.dw};
    const int npos[3] = {a.T, a.Hg, a.Wg};
    // table: axis a holds npos[a] x (dims[a]/2) entries, position-major
    int toff[4];
    toff[0] = 0;
    for (int ax = 0; ax < 3; ++ax) toff[ax + 1] = toff[ax] + npos[ax] * (dims[ax] / 2);
    for (int e = threadIdx.x; e < toff[3]; e += blockDim.x) {
        const int ax = e < toff[1] ? 0 : (e < toff[2] ? 1 : 2);
        const int half = dims[ax] / 2, r = e - toff[ax];
        const int p = r / half, i = r - p * half;
        const double theta = pow(a.base, (double)(-2 * i) / (double)dims[ax]);
        double sn, cs;
        sincos(__dmul_rn((double)p, theta), &sn, &cs);
        tab[e] = make_double2(cs, sn);
    }
    __syncthreads();

    const int tpr = a.d / 8;                       // threads per row
    const int g = threadIdx.x % tpr;               // this thread's 8-channel group
    const int rpp = blockDim.x / tpr;              // rows per block pass
    const int r_in = threadIdx.x / tpr;
    // the 4 pairs of the group: axis, table base (position 0) and per-position stride
    int pax[4], pbase[4], pstride[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int c = 8 * g + 2 * q;
        const int ax = c < a.dt ? 0 : (c < a.dt + a.dh ? 1 : 2);
        const int c0 = ax == 0 ? 0 : (ax == 1 ? a.dt : a.dt + a.dh);
        pax[q] = ax;
        pstride[q] = dims[ax] / 2;
        pbase[q] = toff[ax] + (c - c0) / 2;
    }
    const unsigned HW = (unsigned)a.Hg * (unsigned)a.Wg;
    const long long step = (long long)gridDim.x * rpp;
    for (int k = 0; k < a.n_tensors; ++k) {
        const void *X = a.X[k];
        void *Y = a.Y[k];
        for (long long r0 = (long long)blockIdx.x * rpp + r_in; r0 < a.rows; r0 += kRopeUnroll * step) {
            Vec8<BF16> v[kRopeUnroll];
#pragma unroll
            for (int u = 0; u < kRopeUnroll; ++u) {
                const long long r = r0 + u * step;
                if (r < a.rows) v[u].load(X, r, a.d, g);
            }
#pragma unroll
            for (int u = 0; u < kRopeUnroll; ++u) {
                const long long r = r0 + u * step;
                if (r >= a.rows) break;
                const unsigned n = (unsigned)r % (unsigned)a.N;   // rows < 2^31
                const unsigned t = n / HW, rem = n - t * HW;
                const unsigned h = rem / (unsigned)a.Wg, w = rem - h * (unsigned)a.Wg;
                double y[8];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const unsigned p = pax[q] == 0 ? t : (pax[q] == 1 ? h : w);
                    const double2 cs = tab[pbase[q] + (int)p * pstride[q]];
                    rot(v[u].get(2 * q), v[u].get(2 * q + 1), cs, y[2 * q], y[2 * q + 1]);
                }
                Vec8<BF16>::store(Y, r, a.d, g, y);
            }
        }
    }
}

}  // namespace

size_t rope_table_bytes(int T, int Hg, int Wg, int dt, int dh, int dw)
{
    return sizeof(double2) * ((size_t)T * (dt / 2) + (size_t)Hg * (dh / 2) + (size_t)Wg * (dw / 2));
}

cudaError_t rope3d_run(const RopeArgs &a, int num_sms, cudaStream_t s)
{
    const size_t smem = rope_table_bytes(a.T, a.Hg, a.Wg, a.dt, a.dh, a.dw);
    const int grid = num_sms;   // one 512-thread block per SM, persistent
    cudaError_t e;
    if (a.is_bf16) {
        e = cudaFuncSetAttribute(rope3d_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        rope3d_kernel<true><<<grid, kRopeThreads, smem, s>>>(a);
    } else {
        e = cudaFuncSetAttribute(rope3d_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        rope3d_kernel<false><<<grid, kRopeThreads, smem, s>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace scope
