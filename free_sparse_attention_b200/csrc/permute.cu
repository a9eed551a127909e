// Channel permutation of [rows, d] tensors (the random-channel-partition ablation of the
// review page, significance): every row is copied with Y[e] = X[perm[e]].  Grid-stride over
// rows; one thread per channel, the permutation in shared memory.
#include "common.cuh"

namespace scope {

namespace {

template <typename T>
__global__ void __launch_bounds__(256) permute_channels_kernel(const T *X, const int32_t *perm, T *Y,
                                                               long long rows, int d)
{
    __shared__ int pm[128];
    for (int e = threadIdx.x; e < d; e += blockDim.x) pm[e] = min(max(perm[e], 0), d - 1);
    __syncthreads();
    const int per = blockDim.x / d;   // rows per block step
    const int r0 = threadIdx.x / d, e = threadIdx.x - r0 * d;
    if (r0 >= per) return;
    for (long long r = (long long)blockIdx.x * per + r0; r < rows; r += (long long)gridDim.x * per)
        Y[r * d + e] = X[r * d + pm[e]];
}

}  // namespace

cudaError_t permute_channels_run(const void *X, const int32_t *perm, void *Y, long long rows, int d,
                                 int is_bf16, int num_sms, cudaStream_t s)
{
    const int grid = num_sms * 8;
    if (is_bf16)
        permute_channels_kernel<uint16_t><<<grid, 256, 0, s>>>(static_cast<const uint16_t *>(X), perm,
                                                               static_cast<uint16_t *>(Y), rows, d);
    else
        permute_channels_kernel<float><<<grid, 256, 0, s>>>(static_cast<const float *>(X), perm,
                                                            static_cast<float *>(Y), rows, d);
    return cudaGetLastError();
}

}  // namespace scope
