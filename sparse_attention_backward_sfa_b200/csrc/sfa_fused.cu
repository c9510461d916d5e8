// Fused tensor-core sparse attention backward (tcgen05 / TMEM / TMA) for sm_100a.
#include "sfa_internal.cuh"

namespace sfa {

bool fused_supported(int64_t N1) {
    (void)N1;
    return false;
}

cudaError_t launch_bwd_fused(int dtype, const GradArgs& a, cudaStream_t st) {
    (void)dtype;
    (void)a;
    (void)st;
    return cudaErrorNotSupported;
}

}  // namespace sfa
