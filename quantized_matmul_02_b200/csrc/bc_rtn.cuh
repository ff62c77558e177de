// bc_rtn.cuh -- the RTN scale and zero of a group from its range, shared by
// the precompute kernel and every kernel that derives them in place.
//
// BITCRUSH BC-06, "Under the hood": a per-group scale/zero precompute runs
// once per precision change, after which changing the bit width costs one
// kernel argument.  Storing each group's range (min, max) instead of its
// (scale, zero) makes the precompute independent of the bit width: a kernel
// that reads the range forms
//     scale = fl32(fl32(max - min) / L)     (|c| for a constant group c,
//                                            1 when c == 0)
//     zero  = round-half-even(-min / scale), of the exact quotient
// itself, with the same fp32 operations as the precompute, so its codes
// are bit-identical to those of the stored (scale, zero).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace bc {

__device__ __forceinline__ float rtn_scale(float lo, float hi, float L) {
    if (hi == lo) return (lo == 0.0f) ? 1.0f : fabsf(lo);
    return __fdiv_rn(__fsub_rn(hi, lo), L);
}

// round-half-even(-lo / s) of the exact quotient (lo fp16-valued, s fp32).
// Fast path: r = rint(-lo * rcp(s)) with the residual e of that product.
// rcp.approx is within one ulp, so |(-lo/s) - (-lo * rcp(s))| <= |lo/s| 2^-23,
// and the fma residual is within 2^-25 of (-lo * rcp(s)) - r; when
// |e| < 1/2 - (|r| + 2) 2^-23 the exact quotient lies strictly within 1/2 of
// r and rounds to it.  Otherwise the fp64 quotient decides (for an fp16
// numerator and an fp32 denominator it never crosses a rounding boundary of
// the exact one).  Beyond 2^22 the fp32 path cannot round, so fp64 as well.
static __device__ __noinline__ float rtn_zero_exact(float lo, float s) {
    return (float)rint(-(double)lo / (double)s) + 0.0f;
}
__device__ __forceinline__ float rtn_zero(float lo, float s) {
    float inv;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(inv) : "f"(s));
    const float magic = 12582912.0f;              // 1.5 * 2^23
    const float r = fmaf(-lo, inv, magic) - magic;
    const float e = fmaf(-lo, inv, -r);
    if (fabsf(r) < 4194304.0f &&
        fabsf(e) < 0.5f - (fabsf(r) + 2.0f) * 1.1920928955078125e-07f)   // 2^-23
        return r + 0.0f;                          // no negative zero
    return rtn_zero_exact(lo, s);
}

// (scale, zero) of the group with range [lo, hi] at `bits` bits (fp32
// storage convention of the runtime mode).
__device__ __forceinline__ float2 rtn_params_from_range(float lo, float hi, int bits) {
    const float L = (float)((1 << bits) - 1);
    const float s = rtn_scale(lo, hi, L);
    return make_float2(s, rtn_zero(lo, s));
}

// The range of a group as stored by bc_group_minmax: one 32-bit word, fp16
// min in the low half, fp16 max in the high half.
__device__ __forceinline__ float2 range_of_word(uint32_t w) {
    __half2 h;
    *reinterpret_cast<uint32_t *>(&h) = w;
    return __half22float2(h);
}

}  // namespace bc

namespace bc {

// q - z of one weight, exact (fp64 quotient; see rtn_zero_exact).
static __device__ __noinline__ float rtn_centered_exact(float w, float s, float z, float L) {
    double q = rint((double)w / (double)s) + (double)z;
    q = fmin(fmax(q, 0.0), (double)L);
    return (float)(q - (double)z);
}

// Centred codes q - z = clamp(rint(w / s), -z, L - z) of 8 fp16 weights.
// Fast path through the approximate reciprocal: rcp.approx is within one
// ulp, so for the quotients that matter (|w/s| <= T + 1, T = max(|z|, |L-z|))
// |w/s - w rcp(s)| <= (T + 1) 2^-23; if every residual of the chunk is below
// 1/2 - (T + 2) 2^-21 the fast result is round-half-even of the exact
// quotient.  Otherwise the chunk takes the exact quotient.
__device__ __forceinline__ void rtn_centered8(const uint4 raw, float s, float z, float L,
                                              float (&c)[8]) {
    const __half2 *h = reinterpret_cast<const __half2 *>(&raw);
    float w[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 t = __half22float2(h[i]);
        w[2 * i] = t.x;
        w[2 * i + 1] = t.y;
    }
    float inv;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(inv) : "f"(s));
    const float magic = 12582912.0f;              // 1.5 * 2^23
    const float lo_c = -z, hi_c = L - z;
    const float thr = 0.5f - (fmaxf(fabsf(lo_c), fabsf(hi_c)) + 2.0f) * 4.76837158203125e-07f;
    float emax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float v = fmaf(w[i], inv, magic);
        const float r = v - magic;
        const float e = fmaf(w[i], inv, -r);
        emax = fmaxf(emax, fabsf(e));
        c[i] = fminf(fmaxf(r, lo_c), hi_c);
    }
    if (emax > thr) {
#pragma unroll
        for (int i = 0; i < 8; ++i) c[i] = rtn_centered_exact(w[i], s, z, L);
    }
}

}  // namespace bc
