// bc_argmax.cu -- greedy token selection after the LM-head matmul.
//
// Enargeia ("One decode step") ends a decode step with a single GPU -> CPU
// readback that carries one token id; BITCRUSH BC-06 decodes greedily
// throughout ("Honest notes").  bc_matmul_q_argmax therefore runs the fused
// dequant GEMV of the LM head into scratch and reduces each output row to
// the index of its largest logit, ties going to the lowest index, so the
// caller reads back M int32 values instead of M x N floats.
//
// The logits (4 bytes per output row of W, 0.2 % of the weight bytes of a
// 1024-wide fp16 head) stay in L2 between the GEMV and the reduction.  The
// reduction is two small launches with no atomics, so the result is
// deterministic: per (row, 4096-wide chunk) the best (value, index), then
// per row the best of the chunks.
#include "bc_internal.cuh"

namespace bc {
namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 4096;            // logits per partial

struct Best {
    float v;
    int i;
};
// a beats b: larger value, or equal value and lower index
__device__ __forceinline__ bool better(float av, int ai, float bv, int bi) {
    return av > bv || (av == bv && ai < bi);
}
__device__ __forceinline__ Best warp_best(Best b) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, b.v, off);
        const int oi = __shfl_xor_sync(0xffffffffu, b.i, off);
        if (better(ov, oi, b.v, b.i)) {
            b.v = ov;
            b.i = oi;
        }
    }
    return b;
}
__device__ __forceinline__ Best block_best(Best b, Best *sh) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    b = warp_best(b);
    if (lane == 0) sh[warp] = b;
    __syncthreads();
    if (warp == 0) {
        b = lane < kThreads / 32 ? sh[lane] : Best{-INFINITY, 0x7fffffff};
        b = warp_best(b);
    }
    return b;
}

// grid (chunks, M): best (value, index) of y[m][c*kChunk ...] -> part[m][c]
__global__ void __launch_bounds__(kThreads)
argmax_partial_kernel(const float *__restrict__ y, int64_t N, int chunks, float2 *part) {
    __shared__ Best sh[kThreads / 32];
    const int c = blockIdx.x, m = blockIdx.y;
    const float *row = y + (int64_t)m * N;
    const int64_t n0 = (int64_t)c * kChunk;
    const int64_t n1 = min(N, n0 + kChunk);
    Best b{-INFINITY, 0x7fffffff};
    for (int64_t n = n0 + threadIdx.x; n < n1; n += kThreads) {
        const float v = row[n];
        if (better(v, (int)n, b.v, b.i)) {
            b.v = v;
            b.i = (int)n;
        }
    }
    b = block_best(b, sh);
    if (threadIdx.x == 0)
        part[(int64_t)m * chunks + c] = make_float2(b.v, __int_as_float(b.i));
}

// one block per row: the best of its partials -> token[m]
__global__ void __launch_bounds__(kThreads)
argmax_final_kernel(const float2 *__restrict__ part, int chunks, int32_t *token) {
    __shared__ Best sh[kThreads / 32];
    const int m = blockIdx.x;
    Best b{-INFINITY, 0x7fffffff};
    for (int c = threadIdx.x; c < chunks; c += kThreads) {
        const float2 p = part[(int64_t)m * chunks + c];
        const int pi = __float_as_int(p.y);
        if (better(p.x, pi, b.v, b.i)) {
            b.v = p.x;
            b.i = pi;
        }
    }
    b = block_best(b, sh);
    if (threadIdx.x == 0) token[m] = b.i;
}

inline size_t round256(size_t b) { return (b + 255) / 256 * 256; }
inline int chunks_of(int64_t N) { return (int)((N + kChunk - 1) / kChunk); }

}  // namespace

size_t argmax_partials_bytes(int64_t M, int64_t N) {
    return round256((size_t)M * chunks_of(N) * 8);
}

bc_status launch_argmax(const float *y, int64_t M, int64_t N, void *partials,
                        int32_t *token, cudaStream_t s) {
    const int chunks = chunks_of(N);
    float2 *part = static_cast<float2 *>(partials);
    argmax_partial_kernel<<<dim3(chunks, (unsigned)M), kThreads, 0, s>>>(y, N, chunks, part);
    argmax_final_kernel<<<(unsigned)M, kThreads, 0, s>>>(part, chunks, token);
    return cuda_status();
}

}  // namespace bc
