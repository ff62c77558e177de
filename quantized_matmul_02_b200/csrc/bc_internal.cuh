// bc_internal.cuh -- shared declarations of the CUDA library (not installed).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/bc.h"

namespace bc {

// ---------------------------------------------------------------------------
// Host-side helpers
// ---------------------------------------------------------------------------
struct DeviceInfo {
    int sm_count = 0;
    int cc_major = 0, cc_minor = 0;
    int max_smem_optin = 0;
};
// Cached per device; returns false if the CUDA runtime fails.
bool device_info(DeviceInfo *out);

inline bool aligned(const void *p, size_t a) {
    return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

inline bc_status cuda_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? BC_OK : BC_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Quantizer kernels (bc_quant.cu)
// ---------------------------------------------------------------------------
bc_status launch_group_params(const __half *W, int64_t N, int64_t K, int bits,
                              int64_t group, bool f16_out, void *scales,
                              void *zeros, cudaStream_t s);
// Per-group range (fp16 min, fp16 max) as one 32-bit word per group.
bc_status launch_group_minmax(const __half *W, int64_t N, int64_t K, int64_t group,
                              void *minmax, cudaStream_t s);
bc_status launch_quantize_codes(const __half *W, const void *scales,
                                const void *zeros, bool f16_sz, int64_t N,
                                int64_t K, int bits, int64_t group,
                                uint8_t *codes, cudaStream_t s);
bc_status launch_pack_int4(const __half *W, const __half *scales,
                           const __half *zeros, int64_t N, int64_t K,
                           uint8_t *packed, cudaStream_t s);
// Packed codes of 2, 3, 4 or 8 bits (row = little-endian bit string).
bc_status launch_pack_codes(const __half *W, const __half *scales, const __half *zeros,
                            int64_t N, int64_t K, int bits, uint8_t *packed, cudaStream_t s);

// ---------------------------------------------------------------------------
// Fused dequant GEMV (bc_gemv.cu), M < 64, fp32 x
// ---------------------------------------------------------------------------
struct GemvJob {             // one matrix of a launch
    const float *x;          // [M][K]
    const void *w;           // fp16 [N][K] or packed [N][K/2]
    const void *s;           // fp32 / fp16 [N][K/g]
    const void *z;
    float *y;                // [M][N]
    int64_t N, K;
    int64_t group;           // 64 or K
    int64_t range;           // runtime mode: s holds per-group ranges (fp16 min|max)
                             // and z is unused; the same for every job of a call
};
// Streaming decode kernels (bc_gemv_stream.cu): M <= 4 on the mma.sync
// streaming kernel; M = 5..16 on the tcgen05 decode kernel (packed, or
// runtime RTN at 2..8 bits).  Used for launches large enough to fill the GPU.
bool gemv_stream_supported(const GemvJob *jobs, int count, int M, bool packed, int bits,
                           int max_smem);
// Workspace the streaming kernels need: the activation pieces of launches
// with M > 4 (one copy per distinct non-null x; 0 otherwise).
size_t gemv_stream_workspace_bytes(const GemvJob *jobs, int count, int M, bool packed,
                                   int bits);
// early_start: programmatic dependent launch (weights known not to be
// written by pending work; x / y accesses wait for the previous kernel).
bc_status launch_gemv_stream(const GemvJob *jobs, int count, int M, int bits,
                             bool packed, cudaStream_t s, bool early_start, void *workspace,
                             size_t ws_bytes);
unsigned gemv_timeouts();
bc_status gemv_set_wait_limit(long long cycles);
// Decode GEMV over packed codes of 2, 3 or 8 bits (bc_gemv_packed.cu;
// fp32 x, any M).
bc_status launch_gemv_packed(const GemvJob *jobs, int count, int M, int bits, cudaStream_t s);
// Bytes of split-K scratch a launch over these jobs needs.
size_t gemv_workspace_bytes(const GemvJob *jobs, int count, int M, bool packed,
                            int sm_count);
bc_status launch_gemv(const GemvJob *jobs, int count, int M, int bits,
                      bool packed, void *workspace, size_t ws_bytes,
                      cudaStream_t s, bool early_start = false);

// ---------------------------------------------------------------------------
// Greedy token selection (bc_argmax.cu): per row of y [M][N] the index of
// the largest value, ties to the lowest index.
// ---------------------------------------------------------------------------
// Scratch of the reduction (partials), 256-byte multiple.
size_t argmax_partials_bytes(int64_t M, int64_t N);
bc_status launch_argmax(const float *y, int64_t M, int64_t N, void *partials,
                        int32_t *token, cudaStream_t s);

// ---------------------------------------------------------------------------
// tcgen05 prefill GEMM (bc_gemm_sm100.cu), bf16 x, M >= 64: packed int4 W,
// or fp16 W re-quantized inline (runtime mode)
// ---------------------------------------------------------------------------
struct GemmJob {
    const __nv_bfloat16 *x;  // [M][K]
    const void *w;           // packed [N][K/2] or fp16 [N][K]
    const void *s;           // fp16 [N][K/64] | fp32 [N][K/group] | ranges
    const void *z;           // fp16 | fp32 | unused (ranges)
    float *y;                // [M][N]
    int64_t N, K;
    int64_t group;           // 64, or K (runtime per channel)
};
bc_status launch_gemm(const GemmJob *jobs, int count, int64_t M, bool packed, int bits,
                      bool range, cudaStream_t s);
// Bounded waits of the GEMM that ran out on the current device since load.
unsigned gemm_timeouts();
bc_status gemm_set_wait_limit(long long cycles);

}  // namespace bc
