// bc_gemv_packed.cu -- decode GEMV over packed codes of 2, 3 or 8 bits.
//
// The int4 form has its own streaming kernels; this file serves the other
// packed widths, so that the bytes a decode step reads fall with the bit
// width (BITCRUSH BC-06, "The machine", BRAIN SIZE: 421 MB at 2 bits;
// Enargeia, "Honestly": an int8 tied embedding).  Layout: each weight row is
// a little-endian bit string, code k at bits [b k, b k + b); a 64-group takes
// 8 b bytes (16, 24 or 64), with an fp16 scale and zero point per group.
//
// Eight threads share a weight row and stride over its groups.  A thread
// loads a group's 2 b words, extracts the 64 codes with constant shifts,
// and accumulates sum (q - z) x in fp32 per x row (q - z exact), times the
// group's scale.  The eight partial sums of a row are combined with warp
// shuffles in a fixed order, so the result does not depend on timing.
// Roofline: HBM (b/8 bytes per weight plus 4 bytes of scale/zero per group).
#include "bc_internal.cuh"

#include <algorithm>
#include <vector>

namespace bc {
namespace {

constexpr int kThreads = 256;
constexpr int kRL = 8;                      // threads per weight row
constexpr int kRowsPerBlock = kThreads / kRL;
constexpr int kMaxJobs = 256;

struct PJob {
    const float *x;
    const uint8_t *w;
    const __half *s;
    const __half *z;
    float *y;
    int N, K;
    int block_begin;
};
struct PParams {
    PJob jobs[kMaxJobs];
    int count, total_blocks, M;
};
static_assert(sizeof(PParams) <= 32000, "kernel parameter space");

// The group's 8 b bytes as 2 b words (8-byte aligned: every group starts at
// a multiple of 8 b bytes of a 16-byte aligned row base).
template <int BITS>
__device__ __forceinline__ void load_group(const uint8_t *p, uint32_t (&w)[2 * BITS]) {
    if constexpr (BITS == 3) {
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            const uint2 v = __ldg(reinterpret_cast<const uint2 *>(p) + i);
            w[2 * i] = v.x;
            w[2 * i + 1] = v.y;
        }
    } else {
#pragma unroll
        for (int i = 0; i < BITS / 2; ++i) {
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p) + i);
            w[4 * i] = v.x;
            w[4 * i + 1] = v.y;
            w[4 * i + 2] = v.z;
            w[4 * i + 3] = v.w;
        }
    }
}
// code k of the group (k a compile-time constant after unrolling)
template <int BITS>
__device__ __forceinline__ uint32_t code_at(const uint32_t (&w)[2 * BITS], int k) {
    const int pos = BITS * k, wi = pos >> 5, sh = pos & 31;
    uint32_t v = w[wi] >> sh;
    if (sh + BITS > 32) v |= w[wi + 1] << (32 - sh);
    return v & ((1u << BITS) - 1u);
}

template <int BITS, int MT>
__global__ void __launch_bounds__(kThreads)
gemv_packed_kernel(const __grid_constant__ PParams P) {
    const int lr = threadIdx.x % kRL;
    for (int blk = blockIdx.x; blk < P.total_blocks; blk += gridDim.x) {
        int lo = 0, hi = P.count - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (P.jobs[mid].block_begin <= blk) lo = mid; else hi = mid - 1;
        }
        const PJob &J = P.jobs[lo];
        const int row = (blk - J.block_begin) * kRowsPerBlock + threadIdx.x / kRL;
        const int G = J.K >> 6;
        float acc[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
        if (row < J.N) {
            const uint8_t *wrow = J.w + (int64_t)row * (J.K / 8) * BITS;
            for (int g = lr; g < G; g += kRL) {
                uint32_t w[2 * BITS];
                load_group<BITS>(wrow + g * 8 * BITS, w);
                const float s = __half2float(__ldg(J.s + (int64_t)row * G + g));
                const float z = __half2float(__ldg(J.z + (int64_t)row * G + g));
                float part[MT];
#pragma unroll
                for (int m = 0; m < MT; ++m) part[m] = 0.0f;
#pragma unroll
                for (int k4 = 0; k4 < 16; ++k4) {
                    float c[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) c[i] = (float)code_at<BITS>(w, 4 * k4 + i) - z;
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        if (m >= P.M) break;
                        const float4 xv = __ldg(reinterpret_cast<const float4 *>(
                            J.x + (int64_t)m * J.K + 64 * g) + k4);
                        float p = part[m];
                        p = fmaf(c[0], xv.x, p);
                        p = fmaf(c[1], xv.y, p);
                        p = fmaf(c[2], xv.z, p);
                        p = fmaf(c[3], xv.w, p);
                        part[m] = p;
                    }
                }
#pragma unroll
                for (int m = 0; m < MT; ++m) acc[m] = fmaf(part[m], s, acc[m]);
            }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
#pragma unroll
            for (int off = kRL / 2; off > 0; off >>= 1)
                acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], off);
        }
        if (lr == 0 && row < J.N) {
#pragma unroll
            for (int m = 0; m < MT; ++m)
                if (m < P.M) J.y[(int64_t)m * J.N + row] = acc[m];
        }
    }
}

template <int BITS>
bc_status launch_bits(const PParams &P, int mt, int grid, cudaStream_t s) {
    switch (mt) {
    case 1: gemv_packed_kernel<BITS, 1><<<grid, kThreads, 0, s>>>(P); break;
    case 2: gemv_packed_kernel<BITS, 2><<<grid, kThreads, 0, s>>>(P); break;
    case 4: gemv_packed_kernel<BITS, 4><<<grid, kThreads, 0, s>>>(P); break;
    case 8: gemv_packed_kernel<BITS, 8><<<grid, kThreads, 0, s>>>(P); break;
    default: gemv_packed_kernel<BITS, 16><<<grid, kThreads, 0, s>>>(P); break;
    }
    return cuda_status();
}

}  // namespace

bc_status launch_gemv_packed(const GemvJob *jobs, int count, int M, int bits, cudaStream_t s) {
    DeviceInfo di;
    if (!device_info(&di)) return BC_ERR_CUDA;
    thread_local PParams *Pp = nullptr;
    if (!Pp) Pp = new PParams();
    PParams &P = *Pp;
    for (int m0 = 0; m0 < M; m0 += 16) {
        const int mrows = std::min(16, M - m0);
        const int mt = mrows <= 1 ? 1 : mrows <= 2 ? 2 : mrows <= 4 ? 4 : mrows <= 8 ? 8 : 16;
        for (int b = 0; b < count; b += kMaxJobs) {
            const int n = std::min(kMaxJobs, count - b);
            int blocks = 0;
            for (int i = 0; i < n; ++i) {
                const GemvJob &J = jobs[b + i];
                P.jobs[i] = PJob{J.x + (int64_t)m0 * J.K, static_cast<const uint8_t *>(J.w),
                                 static_cast<const __half *>(J.s),
                                 static_cast<const __half *>(J.z), J.y + (int64_t)m0 * J.N,
                                 (int)J.N, (int)J.K, blocks};
                blocks += (int)((J.N + kRowsPerBlock - 1) / kRowsPerBlock);
            }
            P.count = n;
            P.total_blocks = blocks;
            P.M = mrows;
            const int grid = std::max(1, std::min(blocks, 8 * di.sm_count));
            bc_status st = bits == 2 ? launch_bits<2>(P, mt, grid, s)
                         : bits == 3 ? launch_bits<3>(P, mt, grid, s)
                                     : launch_bits<8>(P, mt, grid, s);
            if (st != BC_OK) return st;
        }
    }
    return BC_OK;
}

}  // namespace bc
