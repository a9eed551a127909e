// Tensor-core (tcgen05) sparse attention for bf16 -- routed to the CUDA-core kernel
// until the tcgen05 kernel passes its parity tests.
#include "common.cuh"

namespace scope {

cudaError_t attention_tc_run(const AttnArgs &a, cudaStream_t s)
{
    return attention_simt_run(a, s);
}

}  // namespace scope
