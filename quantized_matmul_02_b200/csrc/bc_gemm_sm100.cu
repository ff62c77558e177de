// bc_gemm_sm100.cu -- tcgen05 prefill GEMM (placeholder until the kernel lands).
#include "bc_internal.cuh"

namespace bc {
bc_status launch_gemm_packed(const GemmJob *, int, int64_t, cudaStream_t) {
    return BC_ERR_UNSUPPORTED;
}
}  // namespace bc
