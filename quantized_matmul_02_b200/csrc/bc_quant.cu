// bc_quant.cu -- per-group scale/zero precompute, standalone RTN codes and
// the one-time int4 packer.
//
// BITCRUSH BC-06, "Under the hood": a per-group scale/zero precompute kernel
// runs once per precision change; the codes are round-to-nearest with an
// affine (scale, zero) per group.  The same page's NAIVE / SMART row sets
// the group to one output channel or to 64 weights.  Enargeia, "Four bits
// per weight": int4 codes, 64-blocks along K, one scale and zero per block.
//
// All three kernels are HBM-bound streams over fp16 W (2 bytes per weight
// read).  Each lane moves 16-byte vectors; a 64-weight group is 128 bytes,
// i.e. 8 lanes, so one warp covers four groups per load.
#include "bc_internal.cuh"
#include "bc_rtn.cuh"

namespace bc {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ uint4 ld_stream(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

__device__ __forceinline__ void half8_to_float(const uint4 &v, float (&f)[8]) {
    const __half2 *h = reinterpret_cast<const __half2 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 t = __half22float2(h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

// scale = fl32(fl32(hi - lo) / L); a constant group c takes |c| (1 if c==0).
// fp16 storage rounds that fp32 scale to fp16 (floored at 2^-24).
// zero = round-half-even(-lo / scale) of the exact quotient: the fp64
// quotient of an fp16 numerator and an fp32 denominator never crosses a
// rounding boundary of the exact one, so rint() of it is exact.
__device__ __forceinline__ void rtn_params(float lo, float hi, int bits,
                                           bool f16, float &s, float &z) {
    const float L = (float)((1 << bits) - 1);
    s = rtn_scale(lo, hi, L);
    if (f16) {
        s = __half2float(__float2half_rn(s));
        if (s < 5.9604644775390625e-08f) s = 5.9604644775390625e-08f;  // 2^-24
    }
    double zd = rint(-(double)lo / (double)s);
    z = (float)zd;
    if (f16) z = __half2float(__float2half_rn(z));
    if (z == 0.0f) z = 0.0f;   // no negative zero
}

// Exact RTN code: clamp(round-half-even(w / s) + z, 0, L).
__device__ __forceinline__ int rtn_code_exact(float w, float s, float z, int L) {
    double q = rint((double)w / (double)s) + (double)z;
    q = fmin(fmax(q, 0.0), (double)L);
    return (int)q;
}

// LPG lanes share one group; lane handles chunks (lane % LPG) + LPG*i.
// RANGE: store the group's range instead (fp16 min | fp16 max << 16 in one
// word of `scales`; bits, f16 and zeros unused).
template <int LPG, bool RANGE>
__global__ void __launch_bounds__(kThreads)
group_params_kernel(const __half *__restrict__ W, int64_t N, int64_t K,
                    int64_t group, int bits, bool f16, void *scales,
                    void *zeros) {
    const int64_t G = K / group;
    const int64_t ngroups = N * G;
    const int64_t gt = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const int64_t gi = gt / LPG;               // flat group index n*G + j
    const int sub = (int)(gt % LPG);
    const bool valid = gi < ngroups;
    float lo = INFINITY, hi = -INFINITY;
    if (valid) {
        const int64_t n = gi / G, j = gi % G;
        const __half *base = W + n * K + j * group;
        const int chunks = (int)(group / 8);
        for (int c = sub; c < chunks; c += LPG) {
            float f[8];
            half8_to_float(ld_stream(base + c * 8), f);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                lo = fminf(lo, f[i]);
                hi = fmaxf(hi, f[i]);
            }
        }
    }
#pragma unroll
    for (int off = LPG / 2; off > 0; off >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
    }
    if (RANGE) {
        if (valid && sub == 0) {
            const __half2 r = __halves2half2(__float2half_rn(lo), __float2half_rn(hi));
            reinterpret_cast<__half2 *>(scales)[gi] = r;      // exact: fp16 values
        }
        return;
    }
    if (valid && sub == 0) {
        float s, z;
        rtn_params(lo, hi, bits, f16, s, z);
        if (f16) {
            reinterpret_cast<__half *>(scales)[gi] = __float2half_rn(s);
            reinterpret_cast<__half *>(zeros)[gi] = __float2half_rn(z);
        } else {
            reinterpret_cast<float *>(scales)[gi] = s;
            reinterpret_cast<float *>(zeros)[gi] = z;
        }
    }
}

// One thread per 8 consecutive weights (16 bytes in, 8 bytes out).
__global__ void __launch_bounds__(kThreads)
codes_kernel(const __half *__restrict__ W, const void *__restrict__ scales,
             const void *__restrict__ zeros, bool f16, int64_t N, int64_t K,
             int64_t group, int bits, uint8_t *__restrict__ codes) {
    const int64_t t = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const int64_t total = N * K / 8;
    if (t >= total) return;
    const int64_t e = t * 8;
    const int64_t n = e / K, k = e % K;
    const int64_t gi = n * (K / group) + k / group;
    float s, z;
    if (f16) {
        s = __half2float(reinterpret_cast<const __half *>(scales)[gi]);
        z = __half2float(reinterpret_cast<const __half *>(zeros)[gi]);
    } else {
        s = reinterpret_cast<const float *>(scales)[gi];
        z = reinterpret_cast<const float *>(zeros)[gi];
    }
    const int L = (1 << bits) - 1;
    float f[8];
    half8_to_float(ld_stream(W + e), f);
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        lo |= (uint32_t)rtn_code_exact(f[i], s, z, L) << (8 * i);
        hi |= (uint32_t)rtn_code_exact(f[i + 4], s, z, L) << (8 * i);
    }
    *reinterpret_cast<uint2 *>(codes + e) = make_uint2(lo, hi);
}

// One thread per 16 consecutive weights (32 bytes in, 8 bytes out).
__global__ void __launch_bounds__(kThreads)
pack_int4_kernel(const __half *__restrict__ W, const __half *__restrict__ S,
                 const __half *__restrict__ Z, int64_t N, int64_t K,
                 uint8_t *__restrict__ packed) {
    const int64_t t = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const int64_t total = N * K / 16;
    if (t >= total) return;
    const int64_t e = t * 16;
    const int64_t n = e / K, k = e % K;
    const int64_t gi = n * (K / 64) + k / 64;
    const float s = __half2float(S[gi]);
    const float z = __half2float(Z[gi]);
    float fa[8], fb[8];
    half8_to_float(ld_stream(W + e), fa);
    half8_to_float(ld_stream(W + e + 8), fb);
    uint32_t w0 = 0, w1 = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        w0 |= (uint32_t)rtn_code_exact(fa[i], s, z, 15) << (4 * i);
        w1 |= (uint32_t)rtn_code_exact(fb[i], s, z, 15) << (4 * i);
    }
    *reinterpret_cast<uint2 *>(packed + e / 2) = make_uint2(w0, w1);
}

// Packed codes of 2, 3 or 8 bits: one thread per 64-group.  The row is a
// little-endian bit string, code k at bits [BITS k, BITS k + BITS); the
// group's 8 BITS bytes are built as 2 BITS words and stored with aligned
// vector stores (8-byte for 3 bits, 16-byte otherwise).
template <int BITS>
__global__ void __launch_bounds__(kThreads)
pack_codes_kernel(const __half *__restrict__ W, const __half *__restrict__ S,
                  const __half *__restrict__ Z, int64_t N, int64_t K,
                  uint8_t *__restrict__ packed) {
    const int64_t gi = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const int64_t G = K / 64;
    if (gi >= N * G) return;
    const int64_t n = gi / G, g = gi % G;
    const float s = __half2float(S[gi]);
    const float z = __half2float(Z[gi]);
    constexpr int L = (1 << BITS) - 1;
    uint32_t w[2 * BITS];
#pragma unroll
    for (int i = 0; i < 2 * BITS; ++i) w[i] = 0;
    const __half *src = W + n * K + g * 64;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        float f[8];
        half8_to_float(ld_stream(src + 8 * c), f);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int k = 8 * c + i, pos = BITS * k, wi = pos >> 5, sh = pos & 31;
            const uint32_t q = (uint32_t)rtn_code_exact(f[i], s, z, L);
            w[wi] |= q << sh;
            if (sh + BITS > 32) w[wi + 1] |= q >> (32 - sh);
        }
    }
    uint8_t *dst = packed + n * (K / 8) * BITS + g * 8 * BITS;
    if constexpr (BITS == 3) {
#pragma unroll
        for (int i = 0; i < 3; ++i)
            reinterpret_cast<uint2 *>(dst)[i] = make_uint2(w[2 * i], w[2 * i + 1]);
    } else {
#pragma unroll
        for (int i = 0; i < BITS / 2; ++i)
            reinterpret_cast<uint4 *>(dst)[i] =
                make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
    }
}

inline unsigned blocks_for(int64_t threads) {
    return (unsigned)((threads + kThreads - 1) / kThreads);
}

}  // namespace

bc_status launch_group_params(const __half *W, int64_t N, int64_t K, int bits,
                              int64_t group, bool f16_out, void *scales,
                              void *zeros, cudaStream_t s) {
    const int64_t ngroups = N * (K / group);
    if (group == 64) {
        group_params_kernel<8, false><<<blocks_for(ngroups * 8), kThreads, 0, s>>>(
            W, N, K, group, bits, f16_out, scales, zeros);
    } else {
        group_params_kernel<32, false><<<blocks_for(ngroups * 32), kThreads, 0, s>>>(
            W, N, K, group, bits, f16_out, scales, zeros);
    }
    return cuda_status();
}

bc_status launch_group_minmax(const __half *W, int64_t N, int64_t K, int64_t group,
                              void *minmax, cudaStream_t s) {
    const int64_t ngroups = N * (K / group);
    if (group == 64) {
        group_params_kernel<8, true><<<blocks_for(ngroups * 8), kThreads, 0, s>>>(
            W, N, K, group, 2, false, minmax, nullptr);
    } else {
        group_params_kernel<32, true><<<blocks_for(ngroups * 32), kThreads, 0, s>>>(
            W, N, K, group, 2, false, minmax, nullptr);
    }
    return cuda_status();
}

bc_status launch_quantize_codes(const __half *W, const void *scales,
                                const void *zeros, bool f16_sz, int64_t N,
                                int64_t K, int bits, int64_t group,
                                uint8_t *codes, cudaStream_t s) {
    codes_kernel<<<blocks_for(N * K / 8), kThreads, 0, s>>>(
        W, scales, zeros, f16_sz, N, K, group, bits, codes);
    return cuda_status();
}

bc_status launch_pack_codes(const __half *W, const __half *scales, const __half *zeros,
                            int64_t N, int64_t K, int bits, uint8_t *packed, cudaStream_t s) {
    if (bits == 4) return launch_pack_int4(W, scales, zeros, N, K, packed, s);
    const unsigned blocks = blocks_for(N * (K / 64));
    if (bits == 2)
        pack_codes_kernel<2><<<blocks, kThreads, 0, s>>>(W, scales, zeros, N, K, packed);
    else if (bits == 3)
        pack_codes_kernel<3><<<blocks, kThreads, 0, s>>>(W, scales, zeros, N, K, packed);
    else
        pack_codes_kernel<8><<<blocks, kThreads, 0, s>>>(W, scales, zeros, N, K, packed);
    return cuda_status();
}

bc_status launch_pack_int4(const __half *W, const __half *scales,
                           const __half *zeros, int64_t N, int64_t K,
                           uint8_t *packed, cudaStream_t s) {
    pack_int4_kernel<<<blocks_for(N * K / 16), kThreads, 0, s>>>(
        W, scales, zeros, N, K, packed);
    return cuda_status();
}

}  // namespace bc
