// Per-sample exact logits and proxy logits shared by the fidelity and rank-correlation
// kernels (review page: falsifier and the skeptic's concrete test).
#pragma once

#include "common.cuh"

namespace scope {

// Exact logits and Eq. 6 proxy logits of sampled query g (its cluster's LUT) for all N keys,
// computed by one block of THREADS threads; qs (d doubles) and lut (3 Cm doubles) are
// shared-memory buffers.  Logits sum the channels in order (every bf16 or fp32 product is
// exact in binary64); the proxy follows the selection's binary64 formula and order.
// Ends with the block synchronised.
template <int THREADS>
__device__ void sample_logits(const FidArgs &a, long long g, double *logit, double *proxy, double *qs, double *lut)
{
    const int tid = threadIdx.x;
    constexpr int kFidThreads = THREADS;
    const int bh = (int)(g / a.N);
    const int c = min((int)a.q_assign[g], a.Cq - 1);
        for (int e = tid; e < a.d; e += kFidThreads) qs[e] = (double)load_x(a.Q, g * a.d + e, a.is_bf16);
        // LUT of cluster c (Eq. 6): P^m[z] = sum over channels of subspace m of qc . mu_z
        const double *qc = a.qcent + ((size_t)bh * a.Cq + c) * a.d;
        const double *kc = a.kcent + (size_t)bh * a.Cm * a.d;
        const int bnd[4] = {0, a.dt, a.dt + a.dh, a.d};
        for (int idx = tid; idx < 3 * a.Cm; idx += kFidThreads) {
            const int m = idx / a.Cm, z = idx - m * a.Cm;
            double acc = 0.0;
            for (int e = bnd[m]; e < bnd[m + 1]; ++e) acc = __dadd_rn(acc, __dmul_rn(qc[e], kc[(size_t)z * a.d + e]));
            lut[idx] = acc;
        }
        __syncthreads();
        const uint16_t *zt = a.codes + (size_t)bh * 3 * a.N, *zh = zt + a.N, *zw = zh + a.N;
        for (int j = tid; j < a.N; j += kFidThreads) {
            const long long row = ((long long)bh * a.N + j) * a.d;
            double acc = 0.0;   // channels in order; every product is exact in binary64
            if (a.is_bf16) {
                const uint4 *kr = reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(a.K) + row);
                for (int e8 = 0; e8 < a.d / 8; ++e8) {
                    const uint4 v = kr[e8];
                    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float x = __uint_as_float((q & 1) ? (wv[q >> 1] & 0xFFFF0000u) : (wv[q >> 1] << 16));
                        acc = fma(qs[8 * e8 + q], (double)x, acc);
                    }
                }
            } else {
                for (int e = 0; e < a.d; ++e) acc = fma(qs[e], (double)load_x(a.K, row + e, 0), acc);
            }
            logit[j] = acc;
            const int t0 = min((int)zt[j], a.Cm - 1), t1 = min((int)zh[j], a.Cm - 1), t2 = min((int)zw[j], a.Cm - 1);
            proxy[j] = __dmul_rn(a.inv_sqrt_d, __dadd_rn(__dadd_rn(lut[t0], lut[a.Cm + t1]), lut[2 * a.Cm + t2]));
        }
    __syncthreads();
}

}  // namespace scope
