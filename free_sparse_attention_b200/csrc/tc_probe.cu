// Accumulation check of the tensor-core products the k-means assignment certifies.
//
// The tensor-core assignment (kmeans_tc.cu) accepts a token's nearest centroid only when
// the gap to the runner-up exceeds a bound on the error of its fp32 scores, and that
// bound includes an allowance per 16-channel tcgen05.mma step for the accumulation inside
// the tensor core (products of bf16 operands are exact in fp32; their sum with the
// accumulator is not).  NVIDIA does not document how tcgen05.mma kind::f16 aligns and
// rounds that sum, so this kernel exposes the raw accumulator of the same instruction form
// (M = 128, bf16 A and B from 128-byte swizzled K-major shared memory, fp32 accumulator in
// TMEM, one chain of K/16 steps) for a test to compare against exact sums.
//
// One CTA of 128 threads: the operands are copied into shared memory in the swizzled
// layout, one thread issues the chain and commits, and thread r reads row r (TMEM lane r)
// of the accumulator.
#include "tc_common.cuh"

namespace scope {

namespace {

constexpr int kProbeM = 128;

__global__ void __launch_bounds__(128, 1)
    tc_probe_kernel(const __nv_bfloat16 *A, const __nv_bfloat16 *B, int K, int N, float *D)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int nbox = K / 64;
    unsigned char *sa = sm;                                   // [nbox][128 rows][128 B]
    unsigned char *sb = sm + (size_t)nbox * kProbeM * 128;     // [nbox][N rows][128 B]
    uint64_t *bar = reinterpret_cast<uint64_t *>(sb + (size_t)nbox * N * 128);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar + 1);
    const int tid = threadIdx.x, warp = tid >> 5;
    // 16-byte chunk j (of K/8) of row r: box j/8, position r*128 + ((j%8) ^ (r%8))*16
    for (int i = tid; i < kProbeM * (K / 8); i += blockDim.x) {
        const int r = i / (K / 8), j = i % (K / 8);
        *reinterpret_cast<uint4 *>(sa + (j >> 3) * (kProbeM * 128) + r * 128 + (((j & 7) ^ (r & 7)) << 4)) =
            *reinterpret_cast<const uint4 *>(A + (size_t)r * K + j * 8);
    }
    for (int i = tid; i < N * (K / 8); i += blockDim.x) {
        const int r = i / (K / 8), j = i % (K / 8);
        *reinterpret_cast<uint4 *>(sb + (j >> 3) * (N * 128) + r * 128 + (((j & 7) ^ (r & 7)) << 4)) =
            *reinterpret_cast<const uint4 *>(B + (size_t)r * K + j * 8);
    }
    fence_proxy_async();   // generic-proxy stores, read by the tensor core (async proxy)
    if (tid == 0) {
        bar_init(bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(256u)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (tid == 0) {
        const uint32_t idesc = f16_idesc(kProbeM, N, false);
        const uint32_t a0 = smem_u32(sa), b0 = smem_u32(sb);
        for (int kk = 0; kk < K / 16; ++kk) {
            const uint64_t ad = sw128_desc(a0 + (kk >> 2) * (kProbeM * 128) + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = sw128_desc(b0 + (kk >> 2) * (N * 128) + (kk & 3) * 32, 16, 1024);
            mma_bf16(tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar);
        // bounded wait for the chain (a few microseconds)
        const unsigned long long t0 = global_ns();
        while (!bar_test(bar, 0) && global_ns() - t0 < kTcWaitNs) __nanosleep(64);
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    for (int c0 = 0; c0 < N; c0 += 16) {
        float v[16];
        tmem_ld16(tmem + lane_base + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) D[(size_t)tid * N + c0 + e] = v[e];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256u) : "memory");
}

}  // namespace

}  // namespace scope

extern "C" scope_status scope_tc_accumulation_probe(const void *A, const void *B, int K, int N, float *D, void *stream)
{
    using namespace scope;
    if (K < 64 || K > 512 || K % 64 || N < 16 || N > 256 || N % 16) return SCOPE_ERR_INVALID_ARGUMENT;
    const uintptr_t al = reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(B) |
                         reinterpret_cast<uintptr_t>(D);
    if (!A || !B || !D || (al & 15u)) return SCOPE_ERR_INVALID_ARGUMENT;
    const size_t smem = (size_t)(K / 64) * (kProbeM + N) * 128 + 64 + 1024;
    if (smem > 232448) return SCOPE_ERR_UNSUPPORTED;
    // more than half of the SM's shared memory: one probe CTA (and TMEM allocation) per SM
    const size_t req = smem > 232448 / 2 + 1024 ? smem : 232448 / 2 + 1024;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaFuncSetAttribute(tc_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)req) != cudaSuccess)
        return SCOPE_ERR_CUDA;
    tc_probe_kernel<<<1, 128, req, s>>>(static_cast<const __nv_bfloat16 *>(A), static_cast<const __nv_bfloat16 *>(B),
                                        K, N, D);
    return cudaGetLastError() == cudaSuccess ? SCOPE_OK : SCOPE_ERR_CUDA;
}
