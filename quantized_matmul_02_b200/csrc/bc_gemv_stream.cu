// bc_gemv_stream.cu -- streaming decode kernels for launches that fill the
// GPU: gemv_stream_kernel (M <= 4, int8 mma.sync) described here, and the
// tcgen05 decode kernel for M = 5..16 further below (gemv_tc_kernel).
//
// A decode step touches every weight once to produce a single output row
// (Enargeia makes this point about decode): the matmul is one pass over HBM.  The kernel is a TMA pipeline that keeps
// ~130-200 KB per SM in flight, with the arithmetic per weight cut down until
// the stream, not the issue slots, sets the pace.
//
// One CTA per SM, persistent over a cost-balanced contiguous range of
// "units" (128 weight rows of one matrix) that spans every matrix of a
// grouped launch (Enargeia, "One decode step": hundreds of passes per token
// are one launch here).  Warp roles:
//   warp 0      loader: lane 0 issues the TMA of each stage (a 256-byte column
//               chunk of the unit's 128 rows as two 2D boxes of 128 rows x
//               128 bytes, 128-byte swizzle) into a ring of up to 6 stages with
//               full/empty mbarriers.
//   warp 1      activation stager: the x of each new matrix goes into one of
//               two smem slots (see below); the first slot is filled by the
//               stager and the consumers together before streaming starts.
//   warps 2-3   (packed) scale/zero stagers: the fp16 scales and zeros of each
//               stage (64 rows x 8 groups each) into a ring slot beside it,
//               with coalesced loads two stages ahead of the stores; every
//               lane of them arrives on the stage's full barrier.
//   consumers   packed: 8 warps, warp g owns rows 16g..16g+15 of each unit over
//               both 128-byte windows of every stage (tensor cores).  Runtime:
//               16 warps of 8 rows each (CUDA-core quantizer, which needs more
//               warps in flight to hide its latency).
//
// Packed int4 (Enargeia, "Four bits per weight": codes unpacked in registers,
// never written back) runs on the int8 tensor cores (mma.sync m16n8k32
// u8 x s8 -> s32).  The activations are staged as integers per 64-group g
// (max|x| < 2^E_g):  X_e = rint(x_k 2^(30-E_g)) at even k and
// X_o = rint(x_k 2^(26-E_g)) at odd k, so x_k ~= X_e 2^(E_g-30), resp.
// 16 X_o 2^(E_g-30).  ldmatrix brings the swizzled stage into A fragments;
// each code byte b = q_e + 16 q_o (two neighbouring k) fills an even-k slot
// as is and an odd-k slot as b & 0xF0 = 16 q_o, against B digits of X_e and
// of X_o - X_e respectively:
//     b X_e + 16 q_o (X_o - X_e) = q_e X_e + 16 q_o X_o.
// B values are split into four balanced int8 digits (d0 + 2^8 d1 + 2^16 d2 +
// 2^24 d3) that fill the 8 columns of B: with one x row, 2 groups x 4 digits
// (the k slots of each mma split between the two groups, block diagonal);
// with several x rows, 2 rows x 4 digits.  The integer sums are exact, so
//     y = sum_g s_g ( 2^(E_g-30) sum_d 2^(8d) C_gd - z_g sum_k x_k~ )
// carries only the rounding of x to 2^-27 of its group maximum (even k 2^-31)
// and that of the fp32 epilogue.
//
// Runtime RTN (BITCRUSH BC-06, "Under the hood": codes computed inline as
// weights are read) runs on the CUDA cores, four threads per row, with the
// exact-rounding fast path of the general GEMV (bc_gemv.cu).
//
// Every mbarrier wait is bounded; a wait that runs out stops the CTA (its
// outputs are then incomplete) and is counted for bc_device_timeouts.  A
// thread that read or wrote a shared-memory slot arrives on the slot's
// barrier itself: an arrive orders only the arriving thread's own accesses,
// so a single lane arriving for its warp could let the producer overwrite a
// slot while other lanes' loads are still in flight.
#include "bc_internal.cuh"
#include "bc_rtn.cuh"
#include "bc_tc.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <memory>
#include <mutex>
#include <vector>

namespace bc {

__device__ unsigned int g_gemv_timeouts = 0;
// Limit of the pipeline waits, in clock64 cycles (bc_set_wait_limit);
// the drains after an abort keep the fixed ~2 s limit.
__device__ long long g_gemv_wait_limit = 4000000000LL;

namespace {

constexpr int kRows = 128;              // weight rows per unit
constexpr int kChunk = 256;             // bytes of a row per stage
constexpr int kBoxBytes = kRows * 128;  // one TMA box: 128 rows x 128 bytes, SW128
constexpr int kStageBytes = 2 * kBoxBytes;
// Warp roles per mode.  Packed: loader, x stager, two scale/zero stagers
// (64 rows each), 8 consumers of 16 rows.  Runtime: loader, x stager, 16
// consumers of 8 rows (the CUDA-core quantizer wants more warps in flight).
template <bool PACKED> struct Roles {
    static constexpr int consumers = PACKED ? 8 : 16;
    static constexpr int sz_warps = PACKED ? 2 : 0;
    static constexpr int first_consumer = 2 + sz_warps;
    static constexpr int threads = 32 * (first_consumer + consumers);
    static constexpr int stagers = 1 + consumers;    // warps that fill the first x slot
};
constexpr int kSzBytes = 2 * kRows * 16;   // packed: fp16 scales + zeros of a stage
constexpr int kMaxJobs = 168;
constexpr int kMaxCtas = 160;
constexpr int kMaxM = 4;                 // rows of x held in a per-matrix smem slot
constexpr int kMaxMChunk = 16;           // packed: rows of x of the tensor-core kernel
constexpr int kXP = 26;                 // bits of the odd-k activation integers (even: +4)
constexpr long long kWaitCycles = 4000000000LL;
constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23

struct StreamJob {
    const float *x;
    const void *s;
    const void *z;
    float *y;
    int N, K, group;
    int unit_begin;
};

struct __align__(64) StreamParams {
    CUtensorMap wmap[kMaxJobs];   // weights as bytes [N][row_bytes], box 128x128, SW128
    StreamJob jobs[kMaxJobs];
    int cta_begin[kMaxCtas + 1];
    int cta_job[kMaxCtas + 1];    // job of each CTA's first unit (count-1 past the end)
    int count, total_units, M, bits;
    int xslot_bytes, stages, max_cta_jobs;
    int early;                    // launched as a programmatic dependent launch
    int xchunk_bytes;             // tensor-core kernel: bytes of one stage's x chunk
    int range;                    // runtime mode: (scale, zero) from stored ranges
};
static_assert(sizeof(StreamParams) <= 32000, "kernel parameter space");

template <bool PACKED> __host__ __device__ __forceinline__ int row_bytes_of(int K) {
    return PACKED ? K / 2 : K * 2;
}
template <bool PACKED> __host__ __device__ __forceinline__ int kchunks_of(int K) {
    return (row_bytes_of<PACKED>(K) + kChunk - 1) / kChunk;
}
// k covered by the x slot (zero-padded past K)
template <bool PACKED> __host__ __device__ __forceinline__ int kpad_of(int K) {
    return kchunks_of<PACKED>(K) * (PACKED ? 2 * kChunk : kChunk / 2);
}
// Packed x row: digit words [digit d][lane t][unit U][parity] with a row
// stride of dig_rs words (= 4 mod 32, so the 8 rows a quarter-warp reads sit
// in distinct banks), then [parity][group] float2 (f, T) tables, then per
// group the values of its side pair (float2: even k, odd k; for a group with
// several side pairs the masks of their even and odd side members) and one
// side byte (0: none; 1 + p: exactly one side pair, pair p = k 64g + 2p,
// 2p + 1; 0xFF: more than one), eight bytes to a stage chunk.
__host__ __device__ __forceinline__ int dig_rs(int kchunks) { return 32 * kchunks + 4; }
__host__ __device__ __forceinline__ int side_val_off(int kchunks) {
    return 64 * dig_rs(kchunks) + 16 * (8 * kchunks);
}
__host__ __device__ __forceinline__ int side_flag_off(int kchunks) {
    return side_val_off(kchunks) + 8 * (8 * kchunks);
}
constexpr uint8_t kSideMany = 0xFF;
// Bytes of one x row in a slot (a multiple of 16).  Runtime: x[kp] f32.
template <bool PACKED> __host__ __device__ __forceinline__ int xrow_bytes(int K) {
    const int kc = kchunks_of<PACKED>(K);
    return PACKED ? (side_flag_off(kc) + 8 * kc + 15) / 16 * 16 : 4 * kpad_of<false>(K);
}

// ---- PTX helpers -------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          volatile int *abort_flag) {
    if (mbar_try(bar, parity)) return true;
    const long long t0 = clock64();
    const long long limit = *(volatile long long *)&g_gemv_wait_limit;
    while (true) {
        if (mbar_try(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > limit) {
            if (atomicExch((int *)abort_flag, 1) == 0)
                atomicAdd(&g_gemv_timeouts, 1u);
            return false;
        }
    }
}
// Weights are read once: their lines go first when L2 needs room, which keeps
// the activations, scales and zeros (read by many CTAs or stages) resident.
__device__ __forceinline__ uint64_t evict_first_policy() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map,
                                            int x, int y, uint32_t bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
        : "memory");
}
// Contiguous global -> shared copy completing on `bar` (16-byte aligned both
// ends, size a multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}
// C (16x8 s32) += A (16x32 u8) * B (32x8 s8)
__device__ __forceinline__ void mma_i8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                       uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}
__device__ __forceinline__ float rcp_approx(float s) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s));
    return r;
}
__device__ __noinline__ float centered_code_exact(float w, float s, float z,
                                                  float L) {
    double q = rint((double)w / (double)s) + (double)z;
    q = fmin(fmax(q, 0.0), (double)L);
    return (float)(q - (double)z);
}
__device__ __forceinline__ float2 half2_bits_to_float2(uint32_t v) {
    __half2 h;
    *reinterpret_cast<uint32_t *>(&h) = v;
    return __half22float2(h);
}
// Two integer-valued fp16 (zero points) as ints.
__device__ __forceinline__ int2 half2_bits_to_int2(uint32_t v) {
    __half2 h;
    *reinterpret_cast<uint32_t *>(&h) = v;
    return make_int2(__half2int_rn(__low2half(h)), __half2int_rn(__high2half(h)));
}
// (float)(v - z t), the difference exact: in int32 when |z| <= 45 (|v| < 2^30,
// |t| < 2^25), else in int64 (single-sign groups, whose zero lies far out).
__device__ __forceinline__ float exact_dot(int v, int z, int t) {
    if (abs(z) <= 45) return (float)(v - z * t);
    return (float)((long long)v - (long long)z * (long long)t);
}

// Units are visited in increasing order, so the owning job only moves forward.
__device__ __forceinline__ int next_job(const StreamJob *jobs, int count, int j, int unit) {
    while (j + 1 < count && jobs[j + 1].unit_begin <= unit) ++j;
    return j;
}

// ---- activation staging ------------------------------------------------------
// Four balanced int8 digits of v (|v| < 2^31 - 2^23) as the bytes of one word:
// adding 0x80 to each low byte turns the digits into unsigned bytes.
__device__ __forceinline__ uint32_t digits4(int v) {
    return ((uint32_t)v + 0x00808080u) ^ 0x00808080u;
}
// Byte transpose: out[d] = byte d of w[0..3].
__device__ __forceinline__ void transpose4(const uint32_t (&w)[4], uint32_t (&o)[4]) {
    const uint32_t t0 = prmt(w[0], w[1], 0x5140), t1 = prmt(w[0], w[1], 0x7362);
    const uint32_t t2 = prmt(w[2], w[3], 0x5140), t3 = prmt(w[2], w[3], 0x7362);
    o[0] = prmt(t0, t2, 0x5410);
    o[1] = prmt(t0, t2, 0x7632);
    o[2] = prmt(t1, t3, 0x5410);
    o[3] = prmt(t1, t3, 0x7632);
}

// Digits of one 64-group held by 8 lanes (lane j has k = 8j .. 8j+7 of it):
// the digit words of this lane's even-k values (te) and odd-k slots (to,
// carrying X_odd - X_even), byte i of each at k = 8j + 2i; and, on every
// lane of the 8, the group's f = 2^(E-30), its zero-point sums T01 / T23
// and the mask of its side elements.
//
// Side elements.  The integer grid of a group is 2^(E-30) at even k and
// 2^(E-26) at odd k, so an element above 2^(E-17) (even) or 2^(E-13) (odd)
// is always held within 2^-14 of itself.  Below those bounds an element
// whose rounding misses it by more than 2^-14 of itself is left out of the
// digits (staged as 0) and flagged (about half of the small ones); the
// consumers add their products exactly, in fp32.  The values of a group's
// side pair are kept beside the digits (a group holds one side pair or none
// on almost every input; groups with more take a slower exact path that
// reads x from global memory).
// When the odd element of a (2i, 2i+1) pair is a side element, its even
// partner is one too: the odd slot then carries no part of the even value,
// which keeps every digit pair's sum below free of carries from elements
// the integers do not hold (see the epilogue).
//
// Zero-point sums.  With A = z in place of the codes (17 z in the raw-byte
// even slot, 16 z in the odd slot) the MMA would give, per digit d,
// T_d = sum over pairs (17 d(X_e) + 16 d(X_o - X_e)); the consumer forms
// C_d - z T_d, which is exactly sum (q - z) d(...).  Per digit pair
// (0,1) and (2,3): T01 = T_0 + 256 T_1, T23 = T_2 + 256 T_3, |T| < 2^25.
// max|x| < 2^E for a group with largest magnitude amax; E >= -96 keeps
// every scale below a normal float.
__device__ __forceinline__ int group_exponent(float amax) {
    const int E = amax > 0.0f ? (int)((__float_as_uint(amax) >> 23) & 0xffu) - 126 : 0;
    return max(E, -96);
}
// Side elements of the pair (ve, vo) by the staging rules of a group with
// grid exponent E: an element is a side element when its integer rounding
// misses it by more than 2^-14 of itself (only possible below 2^(E-17) at
// even k, 2^(E-13) at odd k); the even element goes with a side odd one.
__device__ __forceinline__ bool rounds_badly(float v, int E, int bits) {
    // grid 2^(E-bits); below 2^(E-bits+13) the scaled value is under 2^13,
    // so rint, the product and the fma residual are all exact
    if (v == 0.0f) return false;
    if (fabsf(v) >= __uint_as_float((uint32_t)(127 + E - bits + 13) << 23)) return false;
    const float sc = __uint_as_float((uint32_t)(127 + bits - E) << 23);
    const float grid = __uint_as_float((uint32_t)(127 + E - bits) << 23);
    const float err = fmaf(-rintf(v * sc), grid, v);
    return fabsf(err) > fabsf(v) * 6.103515625e-05f;             // 2^-14
}
__device__ __forceinline__ void side_pair(float ve, float vo, int E, bool &se, bool &so) {
    so = rounds_badly(vo, E, kXP);
    se = ve != 0.0f && (so || rounds_badly(ve, E, kXP + 4));
}
__device__ __forceinline__ int lo16(int v) {          // d0 + 256 d1 of digits4(v)
    return (int)(((uint32_t)v + 0x8080u) & 0xFFFFu) - 0x8080;
}
__device__ __forceinline__ void group_digits(const float (&v)[8], uint32_t (&te)[4],
                                             uint32_t (&to)[4], float &f, int &t01,
                                             int &t23, uint32_t &side_e, uint32_t &side_o,
                                             int &Eg) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
    const int E = group_exponent(amax);
    const float sc_e = __uint_as_float((uint32_t)(127 + kXP + 4 - E) << 23);
    const float sc_o = __uint_as_float((uint32_t)(127 + kXP - E) << 23);
    uint32_t de[4], dq[4];
    uint32_t lme = 0, lmo = 0;
    int s01 = 0, s23 = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float ve = v[2 * i], vo = v[2 * i + 1];
        bool se, so;
        side_pair(ve, vo, E, se, so);
        lme |= (se ? 1u : 0u) << i;
        lmo |= (so ? 1u : 0u) << i;
        const int xe = se ? 0 : __float2int_rn(ve * sc_e);   // |xe| <= 2^30
        const int xo = so ? 0 : __float2int_rn(vo * sc_o);   // |xo| <= 2^26
        const int dv = xo - xe;       // odd slots carry X_odd - X_even (raw-byte A)
        de[i] = digits4(xe);
        dq[i] = digits4(dv);
        const int le = lo16(xe), ld = lo16(dv);
        s01 += 17 * le + 16 * ld;
        s23 += 17 * ((xe - le) >> 16) + 16 * ((dv - ld) >> 16);
    }
    transpose4(de, te);
    transpose4(dq, to);
    s01 += __shfl_xor_sync(0xffffffffu, s01, 1);
    s01 += __shfl_xor_sync(0xffffffffu, s01, 2);
    s01 += __shfl_xor_sync(0xffffffffu, s01, 4);
    s23 += __shfl_xor_sync(0xffffffffu, s23, 1);
    s23 += __shfl_xor_sync(0xffffffffu, s23, 2);
    s23 += __shfl_xor_sync(0xffffffffu, s23, 4);
    t01 = s01;
    t23 = s23;
    // side members of the group's pairs: bit 4j + i <-> pair (8j + 2i,
    // 8j + 2i + 1), even members in side_e, odd members in side_o
    side_e = lme << (4 * (threadIdx.x & 7));
    side_o = lmo << (4 * (threadIdx.x & 7));
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
        side_e |= __shfl_xor_sync(0xffffffffu, side_e, o);
        side_o |= __shfl_xor_sync(0xffffffffu, side_o, o);
    }
    f = __uint_as_float((uint32_t)(127 + E - kXP - 4) << 23);
    Eg = E;
}

// One x row of a packed-mode slot, by warp `widx` of `nw` working together.
// Eight lanes per 64-group, each with 8 consecutive k (one 32-k unit half).
__device__ void stage_x_packed(const float *__restrict__ xr, int K, uint8_t *xm,
                               int widx, int nw, int lane) {
    const int kch = kchunks_of<true>(K);
    const int rs = dig_rs(kch);
    const int gpad = 8 * kch, G = K >> 6;
    uint32_t *dig = reinterpret_cast<uint32_t *>(xm);
    float2 *tab = reinterpret_cast<float2 *>(xm + 64 * rs);
    const int j = lane & 7;
    const int nq = gpad / 4;
    constexpr int kBatch = 4;
    for (int q0 = widx; q0 < nq; q0 += nw * kBatch) {
        float4 va[kBatch][2];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int g = 4 * (q0 + b * nw) + (lane >> 3);
            va[b][0] = va[b][1] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (q0 + b * nw < nq && g < G) {
                const float4 *p = reinterpret_cast<const float4 *>(xr + 64 * g + 8 * j);
                va[b][0] = __ldg(p);
                va[b][1] = __ldg(p + 1);
            }
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            if (q0 + b * nw >= nq) break;
            const int g = 4 * (q0 + b * nw) + (lane >> 3);
            const float v[8] = {va[b][0].x, va[b][0].y, va[b][0].z, va[b][0].w,
                                va[b][1].x, va[b][1].y, va[b][1].z, va[b][1].w};
            uint32_t te[4], to[4];
            float f;
            int t01, t23;
            uint32_t sme, smo;
            int E;
            group_digits(v, te, to, f, t01, t23, sme, smo, E);
            const uint32_t sp = sme | smo;
            const int U = 2 * g + (j >> 2), tt = j & 3;
#pragma unroll
            for (int d = 0; d < 4; ++d)
                *reinterpret_cast<uint2 *>(dig + (d * 4 + tt) * rs + 2 * U) =
                    make_uint2(te[d], to[d]);
            if (j == 0) {
                tab[g] = make_float2(f, __int_as_float(t01));
                tab[gpad + g] = make_float2(f * 65536.0f, __int_as_float(t23));
                xm[side_flag_off(kch) + g] =
                    sp == 0 ? 0 : (__popc(sp) == 1 ? (uint8_t)(__ffs(sp)) : kSideMany);
                if (__popc(sp) > 1)      // several side pairs: their members' masks
                    reinterpret_cast<uint2 *>(xm + side_val_off(kch))[g] = make_uint2(sme, smo);
            }
            if (sp != 0 && __popc(sp) == 1 && ((__ffs(sp) - 1) >> 2) == j) {
                // the lane holding the group's one side pair stores its values
                // (0 for a member the integers hold)
                const int i = (__ffs(sp) - 1) & 3;
                float ve = 0.0f, vo = 0.0f;
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (q == i) {
                        ve = v[2 * q];
                        vo = v[2 * q + 1];
                    }
                const bool se = (sme >> (__ffs(sp) - 1)) & 1u, so = (smo >> (__ffs(sp) - 1)) & 1u;
                reinterpret_cast<float2 *>(xm + side_val_off(kch))[g] =
                    make_float2(se ? ve : 0.0f, so ? vo : 0.0f);
            }
        }
    }
}

// ---- activation pre-pass tasks (tensor-core kernel) -----------------------------
// One launch before the tensor-core kernel prepares every distinct x of the
// call per stage chunk (see xpieces_kernel); tasks are numbered per x from
// task_begin.
struct XpreTask {
    const float *x;
    uint8_t *out;
    int K, task_begin;
};
struct XpreParams {
    XpreTask t[kMaxJobs];
    int count, M, MT, total;
};
// One x row of a runtime-mode slot: fp32, zero past K.
__device__ void stage_x_runtime(const float *__restrict__ xr, int K, uint8_t *xm,
                                int widx, int nw, int lane) {
    float *xf = reinterpret_cast<float *>(xm);
    const int kp = kpad_of<false>(K);
    constexpr int kBatch = 8;
    const int step = 128 * nw;
    for (int k0 = 128 * widx + 4 * lane; k0 < kp; k0 += step * kBatch) {
        float4 v[kBatch];
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {
            const int k = k0 + step * q;
            v[q] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (k < K) v[q] = __ldg(reinterpret_cast<const float4 *>(xr + k));
        }
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {
            const int k = k0 + step * q;
            if (k < kp) *reinterpret_cast<float4 *>(xf + k) = v[q];
        }
    }
}

template <bool PACKED>
__device__ __forceinline__ void stage_x(const StreamJob &J, int M, uint8_t *xs,
                                        int widx, int nw, int lane) {
    const int mb = xrow_bytes<PACKED>(J.K);
    for (int m = 0; m < M; ++m) {
        if constexpr (PACKED)
            stage_x_packed(J.x + (int64_t)m * J.K, J.K, xs + m * mb, widx, nw, lane);
        else
            stage_x_runtime(J.x + (int64_t)m * J.K, J.K, xs + m * mb, widx, nw, lane);
    }
}

// The consumer's activation slot; it moves on at a unit whose matrix reads
// a different x than the previous unit (the stager walks the same units).
struct XCursor {
    const float *cur = nullptr;
    uint32_t e = 0;
    const uint8_t *xs = nullptr;
};
__device__ __forceinline__ bool x_enter(XCursor &c, const StreamJob &J, bool first,
                                        uint8_t *xslots, int xslot_bytes,
                                        uint64_t *xfull, uint64_t *xempty,
                                        volatile int *abort_flag, int lane) {
    if (!first && J.x == c.cur) return true;
    if (!first) {
        __syncwarp();
        mbar_arrive(smem_u32(&xempty[(c.e - 1) & 1]));     // every lane, after its reads
    }
    c.cur = J.x;
    if (!mbar_wait(smem_u32(&xfull[c.e & 1]), (c.e >> 1) & 1, abort_flag)) return false;
    c.xs = xslots + (c.e & 1) * xslot_bytes;
    ++c.e;
    return true;
}

// Stage / unit walk shared by the consumers.
struct Walk {
    int u, kc, jidx, sidx;
    uint32_t sph;
    // the stage after this one; false at the end of the range
    __device__ __forceinline__ bool next(const StreamJob *jobs, int count, int u1, int kch,
                                         int S, Walk &n) const {
        n = *this;
        if (++n.kc == kch) {
            n.kc = 0;
            if (++n.u >= u1) return false;
            n.jidx = next_job(jobs, count, jidx, n.u);
        }
        if (++n.sidx == S) {
            n.sidx = 0;
            n.sph ^= 1;
        }
        return true;
    }
};
// ---- packed: scales and zeros through shared memory ----------------------------
// Warp 2 copies the fp16 scales and zeros of each stage (rows r0..r0+127,
// groups 8kc..8kc+7) into a ring slot beside the weight stage: s[128][8] then
// z[128][8].  Lane l takes 16-byte row slice word l&3 of rows l/4 + 8i, so a
// load instruction reads eight whole 16-byte slices.  Loads run one stage
// ahead of the stores (two register sets), their indices clamped into the
// matrix so no load waits on a predicate; positions past N or K/64 are stored
// as zero once the values are in.  The warp runs ahead of the consumers by
// the ring depth, and the loader has prefetched each unit's scale/zero block
// into L2, so one stage of load look-ahead suffices.
struct SzSet {
    uint32_t s[8], z[8];
};
struct SzWalk {
    int u, kc, j;
    __device__ __forceinline__ bool next(const StreamJob *jobs, int count, int u1) {
        if (++kc == kchunks_of<true>(jobs[j].K)) {
            kc = 0;
            if (++u >= u1) return false;
            j = next_job(jobs, count, j, u);
        }
        return true;
    }
};
__device__ __forceinline__ void sz_issue(const StreamJob *jobs, const SzWalk &a, int half,
                                         int lane, SzSet &o) {
    const StreamJob &J = jobs[a.j];
    const int G = J.K >> 6;
    const int r0 = (a.u - J.unit_begin) * kRows + 64 * half + (lane >> 2);
    const int c = lane & 3;
    const unsigned short *S16 = reinterpret_cast<const unsigned short *>(J.s);
    const unsigned short *Z16 = reinterpret_cast<const unsigned short *>(J.z);
    if ((G & 1) == 0) {
        const int g = min(8 * a.kc + 2 * c, G - 2);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int64_t off = (int64_t)min(r0 + 8 * i, J.N - 1) * G + g;
            o.s[i] = __ldg(reinterpret_cast<const uint32_t *>(S16 + off));
            o.z[i] = __ldg(reinterpret_cast<const uint32_t *>(Z16 + off));
        }
    } else {        // rows only 2-byte aligned: two halves per word
        const int g0 = min(8 * a.kc + 2 * c, G - 1), g1 = min(8 * a.kc + 2 * c + 1, G - 1);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int64_t off = (int64_t)min(r0 + 8 * i, J.N - 1) * G;
            o.s[i] = (uint32_t)__ldg(S16 + off + g0) | ((uint32_t)__ldg(S16 + off + g1) << 16);
            o.z[i] = (uint32_t)__ldg(Z16 + off + g0) | ((uint32_t)__ldg(Z16 + off + g1) << 16);
        }
    }
}
__device__ __forceinline__ void sz_store(const StreamJob *jobs, const SzWalk &a, int half,
                                         int lane, const SzSet &v, uint8_t *slot) {
    const StreamJob &J = jobs[a.j];
    const int G = J.K >> 6;
    const int rl = 64 * half + (lane >> 2), c = lane & 3;
    const int r0 = (a.u - J.unit_begin) * kRows + rl;
    const int g = 8 * a.kc + 2 * c;
    const uint32_t gmask = g + 1 < G ? 0xffffffffu : (g < G ? 0x0000ffffu : 0u);
    uint32_t *ss = reinterpret_cast<uint32_t *>(slot) + rl * 4 + c;
    uint32_t *zz = reinterpret_cast<uint32_t *>(slot + kSzBytes / 2) + rl * 4 + c;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t m = r0 + 8 * i < J.N ? gmask : 0u;
        ss[32 * i] = v.s[i] & m;
        zz[32 * i] = v.z[i] & m;
    }
}

// ---- packed consumer, one x row: block-diagonal groups ---------------------------
// Warp rg owns rows 16rg..16rg+15 of each unit and both 128-byte windows of a
// stage.  In window w, mma p pairs units (p, p+4): slots 0-15 take unit p's
// codes and B columns 0-3, slots 16-31 unit p+4's and columns 4-7.  Units
// (0,4) and (1,5) belong to groups (0,2), units (2,6) and (3,7) to groups
// (1,3).
//
// The loop is software-pipelined by one stage: a step releases stage n, waits
// for stage n+1 and issues its ldmatrix loads, and only then runs stage n's
// tensor-core math and epilogue, so the wait and load latency of one stage
// hide behind the arithmetic of the other.  A step reads the activation slot
// only for its own stage, before the next stage may move to another slot.
// Side products of group `sub` of a stage window (its 128-byte swizzled rows
// start at `box`), for one weight row, with the group's scale s and zero z.
// Fast path (info = 1 + p): the group's one side pair p, its values from the
// x slot, both codes from one byte of the row.
__device__ __forceinline__ float side_fast(uint32_t info, float2 vals, const uint8_t *box,
                                           int row, int sub, float s, float z) {
    const int byte = 32 * sub + (int)info - 1;
    const uint32_t b = box[row * 128 + (((byte >> 4) ^ (row & 7)) << 4) + (byte & 15)];
    return s * fmaf((float)(b >> 4) - z, vals.y, ((float)(b & 15u) - z) * vals.x);
}
// Slow path (more than one side pair in the group): the slot holds the masks
// of the group's side members (even, odd) instead of values; the values come
// from x in global memory (xg = the group's first element).
__device__ __noinline__ float side_slow(uint2 masks, const float *__restrict__ xg,
                                        const uint8_t *box, int row, int sub, float s, float z) {
    float acc = 0.0f;
    uint32_t pm = masks.x | masks.y;
    while (pm) {
        const int p = __ffs(pm) - 1;
        pm &= pm - 1;
        const float2 v = __ldg(reinterpret_cast<const float2 *>(xg) + p);
        acc += side_fast((uint32_t)p + 1, make_float2(((masks.x >> p) & 1u) ? v.x : 0.0f,
                                                      ((masks.y >> p) & 1u) ? v.y : 0.0f),
                         box, row, sub, s, z);
    }
    return acc;
}

struct StageA {
    uint32_t R[2][4][4];   // [window][j] ldmatrix fragments
    uint32_t s[2][2], z[2][2];   // [row ra / ra+8][window] fp16 pair (2eh, 2eh+1)
};
__device__ __forceinline__ void consume_packed_m1(
    const StreamParams &P, const StreamJob *jobs, int jf, int jc, uint8_t *smem,
    const uint8_t *szring, uint8_t *xslots, uint64_t *full, uint64_t *empty, uint64_t *xfull,
    uint64_t *xempty, volatile int *abort_flag, int u0, int u1, int rg, int lane) {
    const int S = P.stages;
    const int gq = lane >> 2, t = lane & 3;
    // ldmatrix: this lane gives the address of row lrow of unit (j + 4*(lane>>4))
    const int lrow = 16 * rg + (lane & 7) + ((lane >> 3) & 1) * 8;
    uint32_t a_off[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        a_off[j] = lrow * 128 + ((((lane >> 4) * 4 + j) ^ (lrow & 7)) << 4);
    // B role: column gq = 4*bh + digit bd
    const int bh = gq >> 2, bd = gq & 3;
    const uint32_t m0 = bh ? 0u : 0xffffffffu, m1 = ~m0;
    // epilogue role: groups 2*eh (+1) of each window, digit pair ep
    const int eh = t >> 1, ep = t & 1;
    const int ra = 16 * rg + gq;
    XCursor xc;
    Walk k{u0, 0, jf, 0, 0u};
    float ya = 0.0f, yb = 0.0f;
    auto load = [&](StageA &r, int s, uint32_t ph) -> bool {
        if (!mbar_wait(smem_u32(&full[s]), ph, abort_flag)) return false;
        const uint32_t box = smem_u32(smem + s * kStageBytes);
#pragma unroll
        for (int w = 0; w < 2; ++w)
#pragma unroll
            for (int j = 0; j < 4; ++j) ldsm_x4(box + w * kBoxBytes + a_off[j], r.R[w][j]);
        const uint8_t *sz = szring + s * kSzBytes + ra * 16 + 4 * eh;
#pragma unroll
        for (int w = 0; w < 2; ++w) {
            r.s[0][w] = *reinterpret_cast<const uint32_t *>(sz + 8 * w);
            r.s[1][w] = *reinterpret_cast<const uint32_t *>(sz + 128 + 8 * w);
            r.z[0][w] = *reinterpret_cast<const uint32_t *>(sz + kSzBytes / 2 + 8 * w);
            r.z[1][w] = *reinterpret_cast<const uint32_t *>(sz + kSzBytes / 2 + 128 + 8 * w);
        }
        return true;
    };
    if (!x_enter(xc, jobs[k.jidx], true, xslots, P.xslot_bytes, xfull, xempty, abort_flag, lane))
        return;
    StageA stA, stB;
    if (!load(stA, 0, 0u)) return;
    // One step on `cur` (loaded); `nxt` receives the next stage's fragments.
    // Returns true when this warp is done.
    auto step = [&](StageA &cur, StageA &nxt) -> bool {
        const StreamJob &J = jobs[k.jidx];
        const int kch = kchunks_of<true>(J.K);
        {
            // side elements of this stage's 8 groups (about one stage in ten
            // on Gaussian activations): this lane takes groups 2eh, 2eh + 1 of
            // each window for row ra (ep = 0) or ra + 8 (ep = 1), before the
            // stage is released
            const uint2 fl = *reinterpret_cast<const uint2 *>(xc.xs + side_flag_off(kch) +
                                                               8 * k.kc);
            if (fl.x | fl.y) {
                const float2 *sv =
                    reinterpret_cast<const float2 *>(xc.xs + side_val_off(kch)) + 8 * k.kc;
                const uint8_t *st = smem + k.sidx * kStageBytes;
                const int row = ra + 8 * ep;
                float v = 0.0f;
#pragma unroll
                for (int w = 0; w < 2; ++w) {
                    const uint32_t fw = w ? fl.y : fl.x;
                    if (!fw) continue;
                    const float2 s2 = half2_bits_to_float2(ep ? cur.s[1][w] : cur.s[0][w]);
                    const float2 z2 = half2_bits_to_float2(ep ? cur.z[1][w] : cur.z[0][w]);
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int sub = 2 * eh + e;
                        const uint32_t info = (fw >> (8 * sub)) & 0xffu;
                        if (!info) continue;
                        const float sc = e ? s2.y : s2.x, zc = e ? z2.y : z2.x;
                        v += info != kSideMany
                                 ? side_fast(info, sv[4 * w + sub], st + w * kBoxBytes, row, sub,
                                             sc, zc)
                                 : side_slow(reinterpret_cast<const uint2 *>(sv)[4 * w + sub],
                                             J.x + 512 * k.kc + 64 * (4 * w + sub),
                                             st + w * kBoxBytes, row, sub, sc, zc);
                    }
                }
                if (ep) yb += v; else ya += v;
            }
        }
        // stage released: the arrive's release semantics order this warp's
        // ldmatrix reads (made visible to lane 0 by the warp sync) before it
        __syncwarp();
        mbar_arrive(smem_u32(&empty[k.sidx]));       // every lane, after its reads
        Walk n;
        const bool more = k.next(jobs, jc, u1, kch, S, n);
        if (more && !load(nxt, n.sidx, n.sph)) return true;
        const int rs = dig_rs(kch);
#pragma unroll
        for (int w = 0; w < 2; ++w) {
            // activation digits and (f, X~) of this window
            const uint32_t *xd = reinterpret_cast<const uint32_t *>(xc.xs) + (bd * 4 + t) * rs +
                                 2 * (16 * k.kc + 8 * w + 4 * bh);
            const uint4 Q0 = *reinterpret_cast<const uint4 *>(xd);
            const uint4 Q1 = *reinterpret_cast<const uint4 *>(xd + 4);
            const float4 tb = *reinterpret_cast<const float4 *>(
                xc.xs + 64 * rs + 8 * (ep * 8 * kch + 8 * k.kc + 4 * w + 2 * eh));
            int CA[4] = {0, 0, 0, 0}, CB[4] = {0, 0, 0, 0};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                int (&C)[4] = j < 2 ? CA : CB;
                const uint4 &Q = j < 2 ? Q0 : Q1;
                const uint32_t bl = (j & 1) ? Q.z : Q.x, bu = (j & 1) ? Q.w : Q.y;
                const uint32_t(&R)[4] = cur.R[w][j];
                mma_i8(C, R[0], R[1], R[2], R[3], bl & m0, bl & m1);
                mma_i8(C, R[0] & 0xF0F0F0F0u, R[1] & 0xF0F0F0F0u, R[2] & 0xF0F0F0F0u,
                       R[3] & 0xF0F0F0F0u, bu & m0, bu & m1);
            }
            // digits (2ep, 2ep+1) of rows ra, ra+8 for groups 4w+2eh (A) and +1 (B):
            // y += s f (C - z T), the integer part exact
            const float2 sa = half2_bits_to_float2(cur.s[0][w]);
            const float2 sb = half2_bits_to_float2(cur.s[1][w]);
            const int2 za = half2_bits_to_int2(cur.z[0][w]);
            const int2 zb = half2_bits_to_int2(cur.z[1][w]);
            const int TA = __float_as_int(tb.y), TB = __float_as_int(tb.w);
            const float rAa = exact_dot(CA[0] + 256 * CA[1], za.x, TA);
            const float rAb = exact_dot(CA[2] + 256 * CA[3], zb.x, TA);
            const float rBa = exact_dot(CB[0] + 256 * CB[1], za.y, TB);
            const float rBb = exact_dot(CB[2] + 256 * CB[3], zb.y, TB);
            ya = fmaf(sa.x * tb.x, rAa, ya);
            yb = fmaf(sb.x * tb.x, rAb, yb);
            ya = fmaf(sa.y * tb.z, rBa, ya);
            yb = fmaf(sb.y * tb.z, rBb, yb);
        }
        if (n.kc == 0 || !more) {      // unit done: four lanes per row
            ya += __shfl_xor_sync(0xffffffffu, ya, 1);
            ya += __shfl_xor_sync(0xffffffffu, ya, 2);
            yb += __shfl_xor_sync(0xffffffffu, yb, 1);
            yb += __shfl_xor_sync(0xffffffffu, yb, 2);
            if (t == 0) {
                const int r0 = (k.u - J.unit_begin) * kRows;
                if (r0 + ra < J.N) J.y[r0 + ra] = ya;
                if (r0 + ra + 8 < J.N) J.y[r0 + ra + 8] = yb;
            }
            ya = yb = 0.0f;
        }
        if (!more) return true;
        if (n.kc == 0 && !x_enter(xc, jobs[n.jidx], false, xslots, P.xslot_bytes, xfull,
                                  xempty, abort_flag, lane))
            return true;
        k = n;
        return false;
    };
    // One copy of the step in the loop, the fragments moved from nxt to cur
    // after it (40 register moves a stage): the loop with the step inlined
    // twice (cur/nxt swapped) ran 6 % slower on instruction fetch.
    while (!step(stA, stB)) stA = stB;
}

// ---- packed consumer, 2 or 4 x rows ------------------------------------------------
// Each mma takes one 32-k unit (slots 0-15 even k, 16-31 odd k) and a pair of
// x rows as B columns (row 2*mp + h in columns 4h..4h+3), digits from the
// matrix's x slot.
template <int MT>
__device__ __forceinline__ void consume_packed_mx(
    const StreamParams &P, const StreamJob *jobs, int jf, int jc, uint8_t *smem,
    const uint8_t *szring, uint8_t *xslots, uint64_t *full, uint64_t *empty, uint64_t *xfull,
    uint64_t *xempty, volatile int *abort_flag, int u0, int u1, int rg, int lane) {
    constexpr int MP = MT / 2;
    const int S = P.stages;
    const int gq = lane >> 2, t = lane & 3;
    // ldmatrix: this lane gives the address of row lrow of unit (2j + (lane>>4))
    const int lrow = 16 * rg + (lane & 7) + ((lane >> 3) & 1) * 8;
    uint32_t a_off[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        a_off[j] = lrow * 128 + (((2 * j + (lane >> 4)) ^ (lrow & 7)) << 4);
    const int bh = gq >> 2, bd = gq & 3;
    const int eh = t >> 1, ep = t & 1;
    const int ra = 16 * rg + gq;
    XCursor xc;
    Walk k{u0, 0, jf, 0, 0u};
    float ya[MP], yb[MP];
#pragma unroll
    for (int p = 0; p < MP; ++p) ya[p] = yb[p] = 0.0f;
    if (!x_enter(xc, jobs[k.jidx], true, xslots, P.xslot_bytes, xfull, xempty, abort_flag, lane))
        return;
    auto step = [&]() -> bool {
        const StreamJob &J = jobs[k.jidx];
        const int kch = kchunks_of<true>(J.K);
        // x rows: slot rows of `mb` bytes (digit stride rs, k offset of this chunk)
        const int rs = dig_rs(kch);
        const int mb = xrow_bytes<true>(J.K);
        const uint8_t *xb = xc.xs;
        const int u_off = 16 * k.kc;            // unit offset of this chunk
        const int tab_off = 64 * rs;
        const int g_off = 8 * k.kc;              // group offset of this chunk
        const int gpad = 8 * kch;
        if (!mbar_wait(smem_u32(&full[k.sidx]), k.sph, abort_flag)) return true;
        const uint32_t box0 = smem_u32(smem + k.sidx * kStageBytes);
        // scales / zeros of rows ra, ra+8, groups 4w..4w+3 of both windows
        uint2 su[2][2], zu[2][2];
        {
            const uint8_t *sz = szring + k.sidx * kSzBytes + ra * 16;
#pragma unroll
            for (int w = 0; w < 2; ++w) {
                su[0][w] = *reinterpret_cast<const uint2 *>(sz + 8 * w);
                su[1][w] = *reinterpret_cast<const uint2 *>(sz + 128 + 8 * w);
                zu[0][w] = *reinterpret_cast<const uint2 *>(sz + kSzBytes / 2 + 8 * w);
                zu[1][w] = *reinterpret_cast<const uint2 *>(sz + kSzBytes / 2 + 128 + 8 * w);
            }
        }
        // side elements of the stage's groups, per x row (rows past M hold
        // stale data and are skipped); before the stage is released
#pragma unroll
        for (int mp = 0; mp < MP; ++mp) {
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                const int m = 2 * mp + h2;
                if (m >= P.M) continue;
                const uint8_t *xr = xb + m * mb;
                const uint2 fl = *reinterpret_cast<const uint2 *>(xr + side_flag_off(kch) +
                                                                   8 * k.kc);
                if (!(fl.x | fl.y)) continue;
                const float2 *sv =
                    reinterpret_cast<const float2 *>(xr + side_val_off(kch)) + 8 * k.kc;
                const uint8_t *st = smem + k.sidx * kStageBytes;
                const int row = ra + 8 * ep;
                float v = 0.0f;
#pragma unroll
                for (int w = 0; w < 2; ++w) {
                    const uint32_t fw = w ? fl.y : fl.x;
                    if (!fw) continue;
                    // lanes of x row parity eh = h2; ep = 0 row ra, 1 row ra + 8
                    const uint2 svw = ep ? su[1][w] : su[0][w];
                    const uint2 zvw = ep ? zu[1][w] : zu[0][w];
#pragma unroll 1
                    for (int sub = 0; sub < 4; ++sub) {
                        const uint32_t info = (fw >> (8 * sub)) & 0xffu;
                        if (!info) continue;
                        const float2 s2 = half2_bits_to_float2(sub < 2 ? svw.x : svw.y);
                        const float2 z2 = half2_bits_to_float2(sub < 2 ? zvw.x : zvw.y);
                        const float sc = (sub & 1) ? s2.y : s2.x, zc = (sub & 1) ? z2.y : z2.x;
                        v += info != kSideMany
                                 ? side_fast(info, sv[4 * w + sub], st + w * kBoxBytes, row, sub,
                                             sc, zc)
                                 : side_slow(reinterpret_cast<const uint2 *>(sv)[4 * w + sub],
                                             J.x + (int64_t)m * J.K + 512 * k.kc +
                                                 64 * (4 * w + sub),
                                             st + w * kBoxBytes, row, sub, sc, zc);
                    }
                }
                if (eh == h2) {
                    if (ep) yb[mp] += v; else ya[mp] += v;
                }
            }
        }
#pragma unroll
        for (int w = 0; w < 2; ++w) {
            uint32_t R[4][4];
#pragma unroll
            for (int j = 0; j < 4; ++j) ldsm_x4(box0 + w * kBoxBytes + a_off[j], R[j]);
            uint32_t hi[4][4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int i = 0; i < 4; ++i) hi[j][i] = R[j][i] & 0xF0F0F0F0u;
            if (w == 1) {
                __syncwarp();
                mbar_arrive(smem_u32(&empty[k.sidx]));   // stage consumed (every lane)
            }
            float sa[4], sb[4];
            int za[4], zb[4];
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                const float2 a2 = half2_bits_to_float2(p ? su[0][w].y : su[0][w].x);
                const float2 b2 = half2_bits_to_float2(p ? su[1][w].y : su[1][w].x);
                const int2 c2 = half2_bits_to_int2(p ? zu[0][w].y : zu[0][w].x);
                const int2 d2 = half2_bits_to_int2(p ? zu[1][w].y : zu[1][w].x);
                sa[2 * p] = a2.x; sa[2 * p + 1] = a2.y;
                sb[2 * p] = b2.x; sb[2 * p + 1] = b2.y;
                za[2 * p] = c2.x; za[2 * p + 1] = c2.y;
                zb[2 * p] = d2.x; zb[2 * p + 1] = d2.y;
            }
#pragma unroll
            for (int mp = 0; mp < MP; ++mp) {
                // B: this lane's words for units 0..7 of the window, both parities
                const uint32_t *xd =
                    reinterpret_cast<const uint32_t *>(xb + (2 * mp + bh) * mb) +
                    (bd * 4 + t) * rs + 2 * (u_off + 8 * w);
                uint4 Q[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) Q[j] = reinterpret_cast<const uint4 *>(xd)[j];
                int C[4][4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    C[j][0] = C[j][1] = C[j][2] = C[j][3] = 0;
                    mma_i8(C[j], R[j][0], R[j][1], hi[j][0], hi[j][1], Q[j].x, Q[j].y);
                    mma_i8(C[j], R[j][2], R[j][3], hi[j][2], hi[j][3], Q[j].z, Q[j].w);
                }
                const float *tb = reinterpret_cast<const float *>(
                    xb + (2 * mp + eh) * mb + tab_off + 8 * (ep * gpad + g_off + 4 * w));
                const float4 t01 = reinterpret_cast<const float4 *>(tb)[0];
                const float4 t23 = reinterpret_cast<const float4 *>(tb)[1];
                const float f[4] = {t01.x, t01.z, t23.x, t23.z};
                const int T[4] = {__float_as_int(t01.y), __float_as_int(t01.w),
                                  __float_as_int(t23.y), __float_as_int(t23.w)};
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const float ra = exact_dot(C[g][0] + 256 * C[g][1], za[g], T[g]);
                    const float rb = exact_dot(C[g][2] + 256 * C[g][3], zb[g], T[g]);
                    ya[mp] = fmaf(sa[g] * f[g], ra, ya[mp]);
                    yb[mp] = fmaf(sb[g] * f[g], rb, yb[mp]);
                }
            }
        }
        Walk n;
        const bool more = k.next(jobs, jc, u1, kch, S, n);
        if (n.kc == 0 || !more) {      // unit done: two lanes per row and x row
            const int r0 = (k.u - J.unit_begin) * kRows;
#pragma unroll
            for (int mp = 0; mp < MP; ++mp) {
                ya[mp] += __shfl_xor_sync(0xffffffffu, ya[mp], 1);
                yb[mp] += __shfl_xor_sync(0xffffffffu, yb[mp], 1);
                const int m = 2 * mp + eh;
                if (ep == 0 && m < P.M) {
                    if (r0 + ra < J.N) J.y[(int64_t)m * J.N + r0 + ra] = ya[mp];
                    if (r0 + ra + 8 < J.N) J.y[(int64_t)m * J.N + r0 + ra + 8] = yb[mp];
                }
                ya[mp] = yb[mp] = 0.0f;
            }
        }
        if (!more) return true;
        if (n.kc == 0 &&
            !x_enter(xc, jobs[n.jidx], false, xslots, P.xslot_bytes, xfull, xempty, abort_flag,
                     lane))
            return true;
        k = n;
        return false;
    };
    while (!step()) {
    }
}

// ---- runtime (RTN) consumer --------------------------------------------------
// Warp cw owns rows 8cw..8cw+7 of each unit.  Lane (row r8 = lane & 7, part
// p = lane >> 3) takes 32 of the 128 k of a stage: window p >> 1, half p & 1.
// A quarter-warp thus reads eight different rows at one 16-byte offset,
// which the 128-byte swizzle spreads over all banks.
template <int MT>
__device__ __forceinline__ void consume_runtime(
    const StreamParams &P, const StreamJob *jobs, int jf, int jc, uint8_t *smem,
    uint8_t *xslots, uint64_t *full, uint64_t *empty, uint64_t *xfull, uint64_t *xempty,
    volatile int *abort_flag, int u0, int u1, int cw, int lane) {
    const int S = P.stages;
    const int r8 = lane & 7, part = lane >> 3;
    const int w = part >> 1, half = part & 1;
    const int rr = 8 * cw + r8;
    const float L = (float)((1 << P.bits) - 1);
    const bool pass = P.bits == 16;
    XCursor xc;
    Walk k{u0, 0, jf, 0, 0u};
    // (scale, zero) of this lane's 32 k for a stage
    auto load_sz = [&](const Walk &q, float2 &o) {
        const StreamJob &J = jobs[q.jidx];
        const int row = (q.u - J.unit_begin) * kRows + rr;
        const int k0 = q.kc * 128 + w * 64 + half * 32;
        o = make_float2(1.0f, 0.0f);
        if (pass || row >= J.N || k0 >= J.K) return;
        const int64_t gi = (int64_t)row * (J.K / J.group) + k0 / J.group;
        if (P.range) {
            const float2 r =
                range_of_word(__ldg(reinterpret_cast<const uint32_t *>(J.s) + gi));
            o = rtn_params_from_range(r.x, r.y, P.bits);
        } else {
            o.x = __ldg(reinterpret_cast<const float *>(J.s) + gi);
            o.y = __ldg(reinterpret_cast<const float *>(J.z) + gi);
        }
    };
    float2 sz_a, sz_b = make_float2(1.0f, 0.0f);
    load_sz(k, sz_a);
    float yacc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) yacc[m] = 0.0f;
    if (!x_enter(xc, jobs[k.jidx], true, xslots, P.xslot_bytes, xfull, xempty, abort_flag, lane))
        return;
    auto step = [&](const float2 use, float2 &fill) -> bool {
        const StreamJob &J = jobs[k.jidx];
        const int row = (k.u - J.unit_begin) * kRows + rr;
        const int kchunks = kchunks_of<false>(J.K);
        Walk n;
        const bool more = k.next(jobs, jc, u1, kchunks, S, n);
        if (more) load_sz(n, fill);
        if (!mbar_wait(smem_u32(&full[k.sidx]), k.sph, abort_flag)) return true;
        const uint8_t *box = smem + k.sidx * kStageBytes + w * kBoxBytes;
        const int kp = kpad_of<false>(J.K);
        const float s_cur = use.x, z_cur = use.y;
        const int k0 = k.kc * 128 + w * 64 + half * 32;     // this lane's 32 k
        float part_acc[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) part_acc[m] = 0.0f;
        if (row < J.N && k0 < J.K) {
            const float inv = rcp_approx(s_cur);
            const float lo_c = -z_cur, hi_c = L - z_cur;
            const float thr = 0.5f - (fmaxf(fabsf(lo_c), fabsf(hi_c)) + 2.0f) *
                                         4.76837158203125e-07f;   // 2^-21
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
                const int u16 = half * 4 + c8;
                const uint4 raw = *reinterpret_cast<const uint4 *>(
                    box + rr * 128 + ((u16 ^ (rr & 7)) << 4));
                const __half2 *h2 = reinterpret_cast<const __half2 *>(&raw);
                float wv[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f2 = __half22float2(h2[i]);
                    wv[2 * i] = f2.x;
                    wv[2 * i + 1] = f2.y;
                }
                float cq[8];
                if (pass) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) cq[i] = wv[i];
                } else {
                    float emax = 0.0f;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float v = fmaf(wv[i], inv, kMagic);
                        const float r = v - kMagic;
                        const float ee = fmaf(wv[i], inv, -r);
                        emax = fmaxf(emax, fabsf(ee));
                        cq[i] = fminf(fmaxf(r, lo_c), hi_c);
                    }
                    if (emax > thr) {
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            cq[i] = centered_code_exact(wv[i], s_cur, z_cur, L);
                    }
                }
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    const float *xr = reinterpret_cast<const float *>(xc.xs) +
                                      (int64_t)m * kp + k0 + c8 * 8;
                    const float4 xa = *reinterpret_cast<const float4 *>(xr);
                    const float4 xb = *reinterpret_cast<const float4 *>(xr + 4);
                    float p = part_acc[m];
                    p = fmaf(xa.x, cq[0], p);
                    p = fmaf(xa.y, cq[1], p);
                    p = fmaf(xa.z, cq[2], p);
                    p = fmaf(xa.w, cq[3], p);
                    p = fmaf(xb.x, cq[4], p);
                    p = fmaf(xb.y, cq[5], p);
                    p = fmaf(xb.z, cq[6], p);
                    p = fmaf(xb.w, cq[7], p);
                    part_acc[m] = p;
                }
            }
        }
        mbar_arrive(smem_u32(&empty[k.sidx]));       // every lane, after its reads
#pragma unroll
        for (int m = 0; m < MT; ++m) yacc[m] = fmaf(part_acc[m], s_cur, yacc[m]);
        if (n.kc == 0 || !more) {       // unit done: the four lanes of a row
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                yacc[m] += __shfl_xor_sync(0xffffffffu, yacc[m], 8);
                yacc[m] += __shfl_xor_sync(0xffffffffu, yacc[m], 16);
                if (part == 0 && row < J.N && m < P.M) J.y[(int64_t)m * J.N + row] = yacc[m];
                yacc[m] = 0.0f;
            }
        }
        if (!more) return true;
        if (n.kc == 0 && !x_enter(xc, jobs[n.jidx], false, xslots, P.xslot_bytes, xfull,
                                  xempty, abort_flag, lane))
            return true;
        k = n;
        return false;
    };
    while (!step(sz_a, sz_b)) sz_a = sz_b;       // one copy of the step (see above)
}

// Prefetch of the CTA's activations into L2 by staging warp `wi` of `nw`.
__device__ __forceinline__ void prefetch_xs(const StreamParams &P, const StreamJob *jobs, int jf,
                                            int jc, int wi, int nw, int lane) {
    for (int j = jf; j < jc; ++j) {
        const StreamJob &J = jobs[j];
        if (j > jf && jobs[j - 1].x == J.x) continue;
        const int lines = (int)(((int64_t)P.M * J.K * 4 + 127) / 128);
        for (int l = 32 * wi + lane; l < lines; l += 32 * nw)
            prefetch_l2(reinterpret_cast<const char *>(J.x) + (int64_t)l * 128);
    }
}

// Warps 2-3 of a packed launch: the scale / zero slice of every stage of the
// CTA's range, in ring order, gated by the same empty barriers as the loader;
// every lane arrives on the stage's full barrier after its stores.
__device__ __forceinline__ void sz_stager(const StreamParams &P, const StreamJob *jobs, int jf,
                                       int jc, uint8_t *szring, uint64_t *full, uint64_t *empty,
                                       volatile int *abort_flag, int u0, int u1, int half,
                                       int lane) {
    const int S = P.stages;
    SzWalk st{u0, 0, jf};   // stage stored next
    SzWalk ld = st;                                     // stage loaded next
    bool ld_ok = true;
    SzSet A, B, C;
    sz_issue(jobs, ld, half, lane, A);
    ld_ok = ld.next(jobs, jc, u1);
    if (ld_ok) {
        sz_issue(jobs, ld, half, lane, B);
        ld_ok = ld.next(jobs, jc, u1);
    }
    int sidx = 0;
    uint32_t sph = 0;
    // start the loads of the stage two later, then store `cur` (stage st)
    auto step = [&](const SzSet &cur, SzSet &fill) -> bool {
        if (ld_ok) {
            sz_issue(jobs, ld, half, lane, fill);
            ld_ok = ld.next(jobs, jc, u1);
        }
        bool got = true;
        if (lane == 0) got = mbar_wait(smem_u32(&empty[sidx]), sph ^ 1, abort_flag);
        got = __shfl_sync(0xffffffffu, got, 0);
        __syncwarp();
        if (!got) return true;
        sz_store(jobs, st, half, lane, cur, szring + sidx * kSzBytes);
        // every lane arrives after its own stores (an arrive orders the
        // arriving thread's accesses only)
        mbar_arrive(smem_u32(&full[sidx]));
        if (++sidx == S) {
            sidx = 0;
            sph ^= 1;
        }
        return !st.next(jobs, jc, u1);
    };
    while (!step(A, C)) {      // one copy of the step; the sets move down by one
        A = B;
        B = C;
    }
}

// Loader warp: the TMA of every stage of the CTA's unit range (the weights
// of 128 rows x 256 bytes as two 128-byte boxes), gated by the empty
// barriers.  For the tensor-core kernel (xslots > 0) it also loads each
// stage's activation chunk, `xchunk` bytes from job.x + kc * xchunk, into a
// ring of `xslots` slots at xring + slot * xstride with barriers xfull /
// xempty.  It then waits (bounded) for its copies in flight, so none lands
// after the CTA has exited.
template <bool PACKED>
__device__ void load_stages(const StreamParams &P, const StreamJob *jobs, int jf, int jc,
                            int u0, int u1, uint8_t *smem, uint8_t *xring, int xchunk,
                            int xstride, uint64_t *full, uint64_t *empty,
                            volatile int *abort_flag, int lane, int xslots = 0,
                            uint64_t *xfull = nullptr, uint64_t *xempty = nullptr) {
    const int S = P.stages;
    const uint64_t policy = evict_first_policy();
    uint32_t g = 0, armed = 0;
    int jw = jf;
    int pidx = 0;
    uint32_t pph = 0;
    bool ok = true;
    for (int u = u0; u < u1 && ok; ++u) {
        jw = next_job(jobs, jc, jw, u);
        const int j = jw;
        const StreamJob &J = jobs[j];
        const int r0 = (u - J.unit_begin) * kRows;
        const int rbytes = row_bytes_of<PACKED>(J.K);
        const int kchunks = kchunks_of<PACKED>(J.K);
        for (int kc = 0; kc < kchunks; ++kc, ++g) {
            const int s = pidx;
            bool got = true;
            if (lane == 0) got = mbar_wait(smem_u32(&empty[s]), pph ^ 1, abort_flag);
            got = __shfl_sync(0xffffffffu, got, 0);
            __syncwarp();
            if (!got) {
                ok = false;
                break;
            }
            if (++pidx == S) {
                pidx = 0;
                pph ^= 1;
            }
            const uint32_t fb = smem_u32(&full[s]);
            if (lane == 0) {
                // a window wholly past the row end is not loaded: its codes
                // meet zero activations (packed) or are skipped (runtime)
                const int nbox = (rbytes - kc * kChunk) > 128 ? 2 : 1;
                mbar_expect_tx(fb, (uint32_t)(nbox * kBoxBytes));
                const uint32_t st = smem_u32(smem + s * kStageBytes);
                for (int b = 0; b < nbox; ++b)
                    tma_load_2d(st + b * kBoxBytes, &P.wmap[j], kc * kChunk + b * 128, r0, fb,
                                policy);
                if (xslots) {      // job.x holds this matrix's x chunks
                    const uint8_t *xsrc =
                        reinterpret_cast<const uint8_t *>(J.x) + (int64_t)kc * xchunk;
                    const int xs = (int)(g % (uint32_t)xslots);
                    const uint32_t use = g / (uint32_t)xslots;
                    got = use == 0 || mbar_wait(smem_u32(&xempty[xs]), (use - 1) & 1, abort_flag);
                    if (got) {
                        const uint32_t xb = smem_u32(&xfull[xs]);
                        mbar_expect_tx(xb, (uint32_t)xchunk);
                        bulk_load(smem_u32(xring + xs * xstride), xsrc, (uint32_t)xchunk, xb);
                    }
                }
            }
            if (xslots) {
                got = __shfl_sync(0xffffffffu, got, 0);
                if (!got) {
                    ok = false;
                    armed |= 1u << s;
                    ++g;
                    break;
                }
            }
            armed |= 1u << s;
            if (PACKED && kc == 0) {
                // the unit's scales and zeros (one contiguous block each)
                // go to L2 behind its first weights; the scale/zero
                // stagers read them a few stages later
                const int G = J.K >> 6;
                const int64_t b0 = (int64_t)r0 * G * 2;
                const int64_t b1 = (int64_t)min(r0 + kRows, J.N) * G * 2;
                const int lines = (int)((b1 - b0 + 127) >> 7) + 1;
                const int64_t a0 = b0 & ~(int64_t)127;
                const char *sb = reinterpret_cast<const char *>(J.s) + a0;
                const char *zb = reinterpret_cast<const char *>(J.z) + a0;
                const int64_t limit = (int64_t)J.N * G * 2 - a0;
                for (int l = lane; l < lines && (int64_t)l * 128 < limit; l += 32) {
                    prefetch_l2(sb + (int64_t)l * 128);
                    prefetch_l2(zb + (int64_t)l * 128);
                }
            }
        }
    }
    // drain: copies in flight land before the CTA exits
    if (lane == 0 && g > 0) {
        for (int q = 0; q < S; ++q) {
            if (!(armed & (1u << q))) continue;
            const uint32_t gl = (g - 1) - (((g - 1) % S + S - q) % S);
            const long long t0 = clock64();
            while (!mbar_try(smem_u32(&full[q]), (gl / S) & 1) &&
                   clock64() - t0 < kWaitCycles) {
            }
        }
        // the activation ring: the last x load of each slot (an x load was
        // issued for every stage below g, except perhaps the last)
        for (uint32_t k = 0; xslots && k < (uint32_t)xslots && k < g; ++k) {
            const uint32_t gl = g - 1 - k;
            const long long t0 = clock64();
            while (!mbar_try(smem_u32(&xfull[gl % xslots]), (gl / xslots) & 1) &&
                   clock64() - t0 < kWaitCycles) {
            }
        }
    }
    __syncwarp();
}

template <bool PACKED, int MT>
__global__ void __launch_bounds__(Roles<PACKED>::threads, 1)
gemv_stream_kernel(const __grid_constant__ StreamParams P) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int S = P.stages;
    uint8_t *szring = smem + S * kStageBytes;
    uint8_t *xslots = szring + (PACKED ? S * kSzBytes : 0);
    uint64_t *bars = reinterpret_cast<uint64_t *>(xslots + 2 * P.xslot_bytes);
    uint64_t *full = bars, *empty = bars + S;
    uint64_t *xfull = bars + 2 * S, *xempty = xfull + 2;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(xempty + 2);
    uint64_t *xfirst = xempty + 3;      // the first x slot is complete
    StreamJob *jobs_sm = reinterpret_cast<StreamJob *>(bars + 2 * S + 8);

    using RL = Roles<PACKED>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u0 = P.cta_begin[blockIdx.x], u1 = P.cta_begin[blockIdx.x + 1];
    // the next launch on the stream may start as SMs free up (no-op unless it
    // was launched as a programmatic dependent launch)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // This CTA's jobs (those its unit range touches) into shared memory; the
    // table is indexed by global job number through a rebased pointer.
    const int jf = P.cta_job[blockIdx.x];
    const int jc = min(P.count, P.cta_job[blockIdx.x + 1] + 1);
    {
        const uint4 *src = reinterpret_cast<const uint4 *>(&P.jobs[jf]);
        uint4 *dst = reinterpret_cast<uint4 *>(jobs_sm);
        const int n16 = (jc - jf) * (int)(sizeof(StreamJob) / 16);
        for (int i = threadIdx.x; i < n16; i += RL::threads) dst[i] = src[i];
    }
    const StreamJob *jobs = jobs_sm - jf;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&full[s]), 1 + RL::sz_warps * 32);
            mbar_init(smem_u32(&empty[s]), RL::consumers * 32);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&xfull[b]), 32);
            mbar_init(smem_u32(&xempty[b]), RL::consumers * 32);
        }
        mbar_init(smem_u32(xfirst), RL::stagers * 32);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    // The activations of this CTA's matrices go to L2 ahead of the weight
    // stream: queued behind the first ring fill they would hold up the start.
    // (After an early start they may not be written yet: the staging warps
    // prefetch them once the previous kernel has completed.)
    if (!P.early && warp >= 1 && warp < 1 + RL::stagers && u0 < u1)
        prefetch_xs(P, jobs, jf, jc, warp - 1, RL::stagers, lane);
    if (!P.early) __syncthreads();

    if (warp == 0) {
        // ---------------- loader ----------------
        load_stages<PACKED>(P, jobs, jf, jc, u0, u1, smem, nullptr, 0, 0, full, empty,
                            abort_flag, lane);
    } else if (warp >= 2 && warp < RL::first_consumer) {
        // ---------------- scale / zero stagers (packed) ----------------
        if constexpr (PACKED) {
            if (u0 < u1)
                sz_stager(P, jobs, jf, jc, szring, full, empty, abort_flag, u0, u1, warp - 2, lane);
        }
    } else {
        // The first two x slots (the CTA's first two activations, in the order
        // its units meet them), by the x stager and the consumers together:
        // each warp reports on `xfirst`, and the stager turns that into the
        // slots' first xfull phases once all have.  A lone stager needs ~8k
        // cycles for a 4864-wide x; consumers that reach a matrix switch early
        // would wait for it.
        bool first_ok = true;
        int j2 = -1;                     // job of the second activation, if any
        for (int j = jf + 1; j < jc && jobs[j].unit_begin < u1; ++j)
            if (jobs[j].x != jobs[j - 1].x) {
                j2 = j;
                break;
            }
        // x and y belong to the previous kernel until it completes (every CTA
        // waits here, so this grid completes only after it)
        asm volatile("griddepcontrol.wait;" ::: "memory");
        if (P.early && u0 < u1)
            prefetch_xs(P, jobs, jf, jc, warp == 1 ? 0 : warp - RL::first_consumer + 1,
                        RL::stagers, lane);
        if (u0 < u1) {
            const int wi = warp == 1 ? 0 : warp - RL::first_consumer + 1;
            stage_x<PACKED>(jobs[jf], P.M, xslots, wi, RL::stagers, lane);
            if (j2 >= 0)
                stage_x<PACKED>(jobs[j2], P.M, xslots + P.xslot_bytes, wi, RL::stagers, lane);
            __syncwarp();
            mbar_arrive(smem_u32(xfirst));       // every lane, after its writes
            if (warp == 1) {
                first_ok = mbar_wait(smem_u32(xfirst), 0, abort_flag);
                if (first_ok) {
                    mbar_arrive(smem_u32(&xfull[0]));
                    if (j2 >= 0) mbar_arrive(smem_u32(&xfull[1]));
                }
            }
        }
        if (warp == 1) {
            // ---------------- activation stager (slot mode) ----------------
            const float *cur = nullptr;
            uint32_t e = 0;
            const uint32_t pre = j2 >= 0 ? 2u : 1u;     // slots filled above
            int js = jf;
            for (int u = u0; u < u1 && first_ok && !*abort_flag; ++u) {
                js = next_job(jobs, jc, js, u);
                const StreamJob &J = jobs[js];
                if (u != u0 && J.x == cur) continue;
                cur = J.x;
                if (e < pre) {
                    ++e;
                    continue;
                }
                const int slot = e & 1;
                if (!mbar_wait(smem_u32(&xempty[slot]), ((e >> 1) & 1) ^ 1, abort_flag)) break;
                stage_x<PACKED>(J, P.M, xslots + slot * P.xslot_bytes, 0, 1, lane);
                mbar_arrive(smem_u32(&xfull[slot]));     // every lane, after its writes
                ++e;
            }
        } else {
            // ---------------- consumers ----------------
            const int rg = warp - RL::first_consumer;
            if (u0 < u1) {
                if constexpr (PACKED) {
                    if constexpr (MT == 1)
                        consume_packed_m1(P, jobs, jf, jc, smem, szring, xslots, full, empty,
                                          xfull, xempty, abort_flag, u0, u1, rg, lane);
                    else
                        consume_packed_mx<MT>(P, jobs, jf, jc, smem, szring, xslots, full,
                                              empty, xfull, xempty, abort_flag, u0, u1, rg,
                                              lane);
                } else {
                    consume_runtime<MT>(P, jobs, jf, jc, smem, xslots, full, empty, xfull,
                                        xempty, abort_flag, u0, u1, rg, lane);
                }
            }
        }
    }
    __syncthreads();
}

// ---- tensor-core decode (tcgen05), 5..16 x rows -------------------------------
// Swap-AB: the unit's 128 weight rows are the MMA's M (TMEM lanes) and the x
// rows its N.  Per 64-group of K:
//   * A holds the codes in bf16 (exact), written by transform warps straight
//     into tensor memory (32 columns per group):
//       - packed: A = 1 + q/16, unpacked from the swizzled stage of int4 codes;
//       - runtime: A = q, the RTN code of each fp16 weight (BITCRUSH BC-06,
//         "Under the hood": codes formed as the weights are read), exact by
//         the same fast path and fallback as the other decode kernels;
//   * B = x split into two bf16 pieces, hi = bf16(x), lo = bf16(x - hi), so
//     x~ = hi + lo carries 16 significant bits; a pre-pass writes them per
//     stage chunk in the MMA's K-major 128-byte-swizzled layout, with
//     X~ = sum over the group of x~ (fp64 sum, rounded once);
//   * tcgen05.mma.kind::f16 (A from TMEM, B from smem, fp32 in TMEM) gives
//     D = sum_k A_k x~_k per group, and the epilogue warps form
//         s sum_k (q_k - z) x~_k = 16 s D - s (16 + z) X~   (packed)
//                                 =    s D - s z X~         (runtime),
//     two FMAs per output and group.
// Both pieces share one MMA: B rows 0..MT-1 hold hi, MT..2MT-1 lo (N = 2 MT),
// added in the epilogue.  Products are exact; D carries fp32 accumulation
// only.  The codes enter A in the order (k_i, k_i+4) per TMEM column of each
// 8-k block; the pre-pass writes x~ in that same order.
//
// Tensor memory holds two sets of A (up to 4 groups x 32 columns) and of D
// (groups x 2 MT columns), so the transform, the MMAs and the epilogue work
// on different sets; within a set the MMAs of its groups are interleaved,
// so one group's dependent accumulation hides behind the others.  A packed
// stage (512 k) is two sets of 4 groups, a runtime stage (128 k) one set of
// 2.  The activation chunks have a ring of their own (two slots), which
// leaves shared memory for a deeper weight ring.
namespace tcd {
constexpr int kTmemCols = 512;
constexpr int kAcol = 0;                    // A: 2 sets x up to 4 groups x 32 columns
constexpr int kDcol = 256;                  // D: 2 sets x up to 4 groups x 2 MT columns
constexpr int kLoaderWarp = 0, kMmaWarp = 1, kSzWarp0 = 2, kTrWarp0 = 4, kTrWarps = 8;
constexpr int kEpWarp0 = 12, kEpWarps = 8;
constexpr int kThreads = 32 * (kEpWarp0 + kEpWarps);
constexpr int kXSlots = 2;                      // activation-chunk ring
template <bool PACKED> struct Geo {
    static constexpr int kGroups = PACKED ? 8 : 2;         // 64-groups per stage
    static constexpr int kSetGroups = PACKED ? 4 : 2;      // groups per TMEM set
    static constexpr int kSets = kGroups / kSetGroups;     // sets per stage
};
template <bool PACKED, int MT> struct Chunk {
    static constexpr int kGroups = Geo<PACKED>::kGroups;
    static constexpr int kTile = 2 * MT * 128;             // 2 MT rows x 128 bytes
    static constexpr int kTab = kGroups * kTile;           // X~ [group][MT] f32
    static constexpr int kBytes = kTab + kGroups * MT * 4;
    static constexpr int kStride = (kBytes + 1023) / 1024 * 1024;   // smem slot
};
// B row of x row m, piece p (0 hi, 1 lo) of group gl within a chunk: byte
// offset of its 128-byte row.
template <int MT> __host__ __device__ __forceinline__ int brow_off(int gl, int m, int p) {
    const int row = p * MT + m;
    return gl * (2 * MT * 128) + (row >> 3) * 1024 + (row & 7) * 128;
}
}  // namespace tcd

// Pre-pass: the bf16 pieces of every distinct x of the launch, per stage
// chunk, into the workspace.  A warp does one (x, chunk, row m, quad) task:
// up to 4 groups of 64 k, 8 lanes per group, 8 k per lane (one 16-byte piece
// of a B row).  Rows m >= M and groups past K/64 are zero.
template <bool PACKED, int MT>
__global__ void __launch_bounds__(256) xpieces_kernel(const __grid_constant__ XpreParams P) {
    using C = tcd::Chunk<PACKED, MT>;
    constexpr int Q = (C::kGroups + 3) / 4;          // quads per chunk
    const int lane = threadIdx.x & 31, j = lane & 7;
    const int nw = (gridDim.x * blockDim.x) >> 5;
    for (int task = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; task < P.total; task += nw) {
        int lo = 0, hi = P.count - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (P.t[mid].task_begin <= task) lo = mid; else hi = mid - 1;
        }
        const XpreTask &T = P.t[lo];
        int r = task - T.task_begin;
        const int quad = r % Q;
        r /= Q;
        const int m = r % MT, kc = r / MT;
        const int gl = 4 * quad + (lane >> 3);
        const int g = C::kGroups * kc + gl;
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0.0f;
        if (m < P.M && gl < C::kGroups && g < (T.K >> 6)) {
            const float4 *p = reinterpret_cast<const float4 *>(T.x + (int64_t)m * T.K + 64 * g + 8 * j);
            const float4 a = __ldg(p), b = __ldg(p + 1);
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
            v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
        }
        uint32_t wh[4], wl[4];
        double sum = 0.0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat16 h0 = __float2bfloat16_rn(v[i]), h1 = __float2bfloat16_rn(v[i + 4]);
            const float r0 = v[i] - __bfloat162float(h0), r1 = v[i + 4] - __bfloat162float(h1);
            const __nv_bfloat16 l0 = __float2bfloat16_rn(r0), l1 = __float2bfloat16_rn(r1);
            wh[i] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
            wl[i] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
            sum += (double)__bfloat162float(h0) + (double)__bfloat162float(l0);
            sum += (double)__bfloat162float(h1) + (double)__bfloat162float(l1);
        }
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
        sum += __shfl_xor_sync(0xffffffffu, sum, 4);
        if (gl >= C::kGroups) continue;
        uint8_t *chunk = T.out + (int64_t)kc * C::kBytes;
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const int row = p * MT + m;
            uint8_t *dst = chunk + tcd::brow_off<MT>(gl, m, p) + ((j ^ (row & 7)) << 4);
            *reinterpret_cast<uint4 *>(dst) = p ? make_uint4(wl[0], wl[1], wl[2], wl[3])
                                                : make_uint4(wh[0], wh[1], wh[2], wh[3]);
        }
        if (j == 0) reinterpret_cast<float *>(chunk + C::kTab)[gl * MT + m] = (float)sum;
    }
}

// (bf16 1 + q/16) pairs for the codes of one 32-bit word (k0..k7, low nibble
// first): word i holds (k_i, k_i+4).
__device__ __forceinline__ void unpack_a(uint32_t w, uint32_t *o) {
    uint32_t t;
    asm("lop3.b32 %0, %1, 0x00780078, 0x3F803F80, 0xEA;" : "=r"(t) : "r"(w << 3));
    o[0] = t;
    asm("lop3.b32 %0, %1, 0x00780078, 0x3F803F80, 0xEA;" : "=r"(t) : "r"(w >> 1));
    o[1] = t;
    asm("lop3.b32 %0, %1, 0x00780078, 0x3F803F80, 0xEA;" : "=r"(t) : "r"(w >> 5));
    o[2] = t;
    asm("lop3.b32 %0, %1, 0x00780078, 0x3F803F80, 0xEA;" : "=r"(t) : "r"(w >> 9));
    o[3] = t;
}

// Runtime RTN: codes q of 8 fp16 weights (one 16-byte chunk, k0..k7) as
// bf16 pairs (k_i, k_i+4).  Fast path: q - z = clamp(rint(w / s), -z, L - z)
// through the approximate reciprocal, exact unless some |w/s - w rcp(s)|
// could reach a rounding boundary (then the chunk takes the exact quotient);
// q = (q - z) + z in exact integer arithmetic.
__device__ __forceinline__ void rtn_codes8(uint4 raw, float s, float z, float L,
                                           bool centered, uint32_t *o) {
    const __half2 *h2 = reinterpret_cast<const __half2 *>(&raw);
    float wv[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f2 = __half22float2(h2[i]);
        wv[2 * i] = f2.x;
        wv[2 * i + 1] = f2.y;
    }
    const float inv = rcp_approx(s);
    const float lo_c = -z, hi_c = L - z;
    const float thr = 0.5f - (fmaxf(fabsf(lo_c), fabsf(hi_c)) + 2.0f) * 4.76837158203125e-07f;
    float cq[8];
    float emax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float v = fmaf(wv[i], inv, kMagic);
        const float r = v - kMagic;
        const float ee = fmaf(wv[i], inv, -r);
        emax = fmaxf(emax, fabsf(ee));
        cq[i] = fminf(fmaxf(r, lo_c), hi_c);
    }
    if (emax > thr) {
#pragma unroll
        for (int i = 0; i < 8; ++i) cq[i] = centered_code_exact(wv[i], s, z, L);
    }
    const float zb = centered ? 0.0f : z;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 p = __floats2bfloat162_rn(cq[i] + zb, cq[i + 4] + zb);
        o[i] = *reinterpret_cast<const uint32_t *>(&p);
    }
}
// The A operand holds centred codes q - z (bf16) when they are exact in bf16
// (|q - z| <= 256 for every code, i.e. max(|z|, |L - z|) <= 256; packed:
// |z| <= 224, where 1 + z/16 and (q - z)/16 are exact as well), so that
// D = sum (q - z) x~ and an activation that meets q = z adds exactly
// nothing.  Otherwise (a single-sign group whose zero lies far outside
// [0, L]) A holds q (packed: 1 + q/16) and the epilogue subtracts z X~; then
// |z| X~ is within a small factor of sum |q - z| |x~| and loses nothing.
__device__ __forceinline__ bool centered_rt(float z, float L) {
    return fmaxf(fabsf(z), fabsf(L - z)) <= 256.0f;
}
__device__ __forceinline__ bool centered_pk(float z) { return fabsf(z) <= 224.0f; }

template <bool PACKED, int MT>
__global__ void __launch_bounds__(tcd::kThreads, 1)
gemv_tc_kernel(const __grid_constant__ StreamParams P) {
    using C = tcd::Chunk<PACKED, MT>;
    using G = tcd::Geo<PACKED>;
    constexpr int NB = 2 * MT;                       // MMA N: hi and lo rows of B
    constexpr int MH = MT / 2;                       // x rows per epilogue warp
    constexpr int SG = G::kSetGroups;
    constexpr uint32_t kIdesc = tc::idesc_bf16(128, NB);
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int S = P.stages;
    uint8_t *szring = smem + S * kStageBytes;
    uint8_t *xring = szring + (PACKED ? S * kSzBytes : 0);     // 1024-aligned slots
    uint64_t *bars = reinterpret_cast<uint64_t *>(xring + tcd::kXSlots * C::kStride);
    uint64_t *full = bars, *empty = bars + S;
    uint64_t *xfull = bars + 2 * S, *xempty = xfull + tcd::kXSlots;
    uint64_t *afull = xempty + tcd::kXSlots;            // A set written (8 warps)
    uint64_t *done = afull + 2;                         // MMAs of a set complete
    uint64_t *dempty = done + 2;                        // D set read (8 warps)
    uint64_t *mma_final = dempty + 2;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(mma_final + 1);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_final + 1) + 1;
    StreamJob *jobs_sm = reinterpret_cast<StreamJob *>(bars + 2 * S + 16);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u0 = P.cta_begin[blockIdx.x], u1 = P.cta_begin[blockIdx.x + 1];
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int jf = P.cta_job[blockIdx.x];
    const int jc = min(P.count, P.cta_job[blockIdx.x + 1] + 1);
    {
        const uint4 *src = reinterpret_cast<const uint4 *>(&P.jobs[jf]);
        uint4 *dst = reinterpret_cast<uint4 *>(jobs_sm);
        const int n16 = (jc - jf) * (int)(sizeof(StreamJob) / 16);
        for (int i = threadIdx.x; i < n16; i += tcd::kThreads) dst[i] = src[i];
    }
    const StreamJob *jobs = jobs_sm - jf;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            // loader, plus every lane of the two scale/zero stagers (packed)
            mbar_init(smem_u32(&full[s]), PACKED ? 1 + 2 * 32 : 1);
            // one arrival per transform warp (its reads of the stage are
            // consumed by its tensor-memory stores, which it waits for), and
            // one per epilogue lane (each lane's own scale/zero reads)
            mbar_init(smem_u32(&empty[s]), tcd::kTrWarps + 32 * tcd::kEpWarps);
        }
        for (int b = 0; b < tcd::kXSlots; ++b) {
            mbar_init(smem_u32(&xfull[b]), 1);
            // the MMAs' commit + every epilogue lane (each lane's own X~ reads)
            mbar_init(smem_u32(&xempty[b]), 1 + 32 * tcd::kEpWarps);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&afull[b]), tcd::kTrWarps);
            mbar_init(smem_u32(&done[b]), 1);
            mbar_init(smem_u32(&dempty[b]), tcd::kEpWarps);
        }
        mbar_init(smem_u32(mma_final), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == tcd::kMmaWarp) tc::alloc(smem_u32(tmem_slot), tcd::kTmemCols);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *tmem_slot;
    // warp-uniform bounded wait
    auto wait_all = [&](uint64_t *bar, uint32_t parity) -> bool {
        return __all_sync(0xffffffffu, mbar_wait(smem_u32(bar), parity, abort_flag));
    };
    // runtime mode: (scale, zero) of weight row `row`, group gg of job J
    auto rt_sz = [&](const StreamJob &J, int row, int gg) -> float2 {
        if (row >= J.N || 64 * gg >= J.K) return make_float2(0.0f, 0.0f);
        const int64_t gi = (int64_t)row * (J.K / J.group) + (64 * gg) / J.group;
        if (P.range) {
            const float2 r =
                range_of_word(__ldg(reinterpret_cast<const uint32_t *>(J.s) + gi));
            return rtn_params_from_range(r.x, r.y, P.bits);
        }
        return make_float2(__ldg(reinterpret_cast<const float *>(J.s) + gi),
                           __ldg(reinterpret_cast<const float *>(J.z) + gi));
    };

    if (u0 < u1) {
        if (warp == tcd::kLoaderWarp) {
            // activation chunks: written by the pre-pass kernel just before
            asm volatile("griddepcontrol.wait;" ::: "memory");
            load_stages<PACKED>(P, jobs, jf, jc, u0, u1, smem, xring, C::kBytes, C::kStride, full,
                                empty, abort_flag, lane, tcd::kXSlots, xfull, xempty);
        } else if (warp == tcd::kMmaWarp) {
            // The whole warp walks the stages and waits; one elected lane issues
            // a set's MMAs, interleaved over its groups.  Descriptors are formed
            // once and advanced by constant offsets (16-byte units of the start
            // address).
            const uint64_t bdesc0 = tc::sw128_desc(smem_u32(xring));
            uint32_t g = 0;
            int j = jf;
            bool ok = true;
            for (int u = u0; u < u1 && ok; ++u) {
                j = next_job(jobs, jc, j, u);
                const int kch = kchunks_of<PACKED>(jobs[j].K);
                for (int kc = 0; kc < kch && ok; ++kc, ++g) {
                    const int xs = (int)(g % tcd::kXSlots);
                    if (!wait_all(&xfull[xs], (g / tcd::kXSlots) & 1)) {
                        ok = false;
                        break;
                    }
                    const uint64_t bs = bdesc0 + (uint64_t)((xs * C::kStride) >> 4);
#pragma unroll
                    for (int hs = 0; hs < G::kSets; ++hs) {
                        const uint32_t t = g * G::kSets + hs, b = t & 1, k = t >> 1;
                        bool w = mbar_wait(smem_u32(&afull[b]), k & 1, abort_flag);
                        if (w && k > 0) w = mbar_wait(smem_u32(&dempty[b]), (k - 1) & 1, abort_flag);
                        if (!__all_sync(0xffffffffu, w)) {
                            ok = false;
                            break;
                        }
                        tc::fence_after();
                        if (tc::elect_one()) {
                            const uint32_t d0 = tmem + tcd::kDcol + b * SG * NB;
                            const uint32_t a0 = tmem + tcd::kAcol + b * SG * 32;
                            const uint64_t b0 = bs + (uint64_t)((hs * SG * C::kTile) >> 4);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                                for (int gi = 0; gi < SG; ++gi)
                                    tc::mma_bf16_ts(d0 + gi * NB, a0 + gi * 32 + 8 * kk,
                                                    b0 + (uint64_t)((gi * C::kTile) >> 4) + 2 * kk,
                                                    kIdesc, kk ? 1u : 0u);
                            tc::commit(smem_u32(&done[b]));
                            if (hs == G::kSets - 1) tc::commit(smem_u32(&xempty[xs]));  // x read
                        }
                        __syncwarp();
                    }
                }
            }
            // every MMA issued has completed before TMEM is freed
            if (tc::elect_one()) tc::commit(smem_u32(mma_final));
            __syncwarp();
            if (lane == 0) {
                const long long t0 = clock64();
                while (!mbar_try(smem_u32(mma_final), 0) && clock64() - t0 < kWaitCycles) {
                }
            }
            __syncwarp();
        } else if (warp < tcd::kTrWarp0) {
            if constexpr (PACKED)
                sz_stager(P, jobs, jf, jc, szring, full, empty, abort_flag, u0, u1,
                          warp - tcd::kSzWarp0, lane);
        } else if (warp < tcd::kEpWarp0) {
            // ---- transform: codes -> A (bf16) in TMEM ----
            // Warp (quarter q = warp & 3, parity par) writes lanes 32q..32q+31
            // (its rows) for groups par, par + 2, ... of each set.
            const int q = warp & 3, par = (warp - tcd::kTrWarp0) >> 2;
            const int r = 32 * q + lane;
            const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16) + tcd::kAcol;
            const float L = (float)((1 << P.bits) - 1);
            uint32_t g = 0;
            int j = jf;
            bool ok = true;
            for (int u = u0; u < u1 && ok; ++u) {
                j = next_job(jobs, jc, j, u);
                const StreamJob &J = jobs[j];
                const int kch = kchunks_of<PACKED>(J.K);
                const int row = (u - J.unit_begin) * kRows + r;
                for (int kc = 0; kc < kch && ok; ++kc, ++g) {
                    const int s = (int)(g % (uint32_t)S);
                    float2 szv[SG / 2];
                    if constexpr (!PACKED) {       // this warp's groups of the stage
#pragma unroll
                        for (int i = 0; i < SG / 2; ++i)
                            szv[i] = rt_sz(J, row, G::kGroups * kc + par + 2 * i);
                    }
                    if (!wait_all(&full[s], (g / S) & 1)) {
                        ok = false;
                        break;
                    }
                    const uint8_t *st = smem + s * kStageBytes;
#pragma unroll
                    for (int hs = 0; hs < G::kSets; ++hs) {
                        const uint32_t t = g * G::kSets + hs, b = t & 1, k = t >> 1;
                        // the A set is free once the MMAs of its previous use are done
                        if (k > 0 && !wait_all(&done[b], (k - 1) & 1)) {
                            ok = false;
                            break;
                        }
                        tc::fence_after();
#pragma unroll
                        for (int i = 0; i < SG / 2; ++i) {
                            const int gi = 2 * i + par;          // group within the set
                            uint32_t o[32];
                            if constexpr (PACKED) {
                                const uint8_t *box = st + hs * kBoxBytes + r * 128;
                                const uint4 v0 = *reinterpret_cast<const uint4 *>(
                                    box + (((2 * gi) ^ (r & 7)) << 4));
                                const uint4 v1 = *reinterpret_cast<const uint4 *>(
                                    box + (((2 * gi + 1) ^ (r & 7)) << 4));
                                unpack_a(v0.x, o + 0);
                                unpack_a(v0.y, o + 4);
                                unpack_a(v0.z, o + 8);
                                unpack_a(v0.w, o + 12);
                                unpack_a(v1.x, o + 16);
                                unpack_a(v1.y, o + 20);
                                unpack_a(v1.z, o + 24);
                                unpack_a(v1.w, o + 28);
                                // centred: (1 + q/16) - (1 + z/16) = (q - z)/16, exact
                                const float zc = __half2float(__ushort_as_half(
                                    reinterpret_cast<const unsigned short *>(
                                        szring + s * kSzBytes + kSzBytes / 2 +
                                        r * 16)[hs * SG + gi]));
                                if (centered_pk(zc)) {
                                    const __nv_bfloat162 zz = __float2bfloat162_rn(1.0f + zc * 0.0625f);
#pragma unroll
                                    for (int c = 0; c < 32; ++c) {
                                        const __nv_bfloat162 a =
                                            __hsub2(*reinterpret_cast<const __nv_bfloat162 *>(&o[c]), zz);
                                        o[c] = *reinterpret_cast<const uint32_t *>(&a);
                                    }
                                }
                            } else {
                                // group gi is the stage's box gi: 64 fp16 of row r
                                const uint8_t *box = st + gi * kBoxBytes + r * 128;
#pragma unroll
                                for (int c = 0; c < 8; ++c) {
                                    const uint4 raw =
                                        *reinterpret_cast<const uint4 *>(box + ((c ^ (r & 7)) << 4));
                                    rtn_codes8(raw, szv[i].x, szv[i].y, L,
                                               centered_rt(szv[i].y, L), o + 4 * c);
                                }
                            }
                            // tcgen05.st is warp-collective: reconverge after
                            // the lanes that took the exact quotient
                            __syncwarp();
                            tc::st32(lane_base + b * SG * 32 + gi * 32, o);
                        }
                        tc::fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(smem_u32(&afull[b]));
                    }
                    if (!ok) break;
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&empty[s]));   // codes read
                }
            }
        } else {
            // ---- epilogue: y[m][row] += sc D - sz X~ ----
            // Warp (quarter q, half h) takes x rows h*MT/2 .. of its 32 weight
            // rows, over every group.
            const int q = warp & 3, h = (warp - tcd::kEpWarp0) >> 2, m0 = h * MH;
            const int r = 32 * q + lane;
            const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16) + tcd::kDcol;
            float y[MH];
#pragma unroll
            for (int i = 0; i < MH; ++i) y[i] = 0.0f;
            uint32_t g = 0;
            int j = jf;
            bool ok = true;
            for (int u = u0; u < u1 && ok; ++u) {
                j = next_job(jobs, jc, j, u);
                const StreamJob &J = jobs[j];
                const int kch = kchunks_of<PACKED>(J.K);
                const int row = (u - J.unit_begin) * kRows + r;
                for (int kc = 0; kc < kch && ok; ++kc, ++g) {
                    const int s = (int)(g % (uint32_t)S);
                    // scale and zero of each group of the stage: packed fp16 words
                    // from the stage's scale/zero slot, runtime fp32 (sc, -sc z)
                    uint32_t sw[4], zw[4];
                    float2 rcoef[PACKED ? 1 : G::kGroups];
                    if constexpr (!PACKED) {
                        const float L = (float)((1 << P.bits) - 1);
#pragma unroll
                        for (int gl = 0; gl < G::kGroups; ++gl) {
                            const float2 v = rt_sz(J, row, G::kGroups * kc + gl);
                            rcoef[gl] = make_float2(v.x, centered_rt(v.y, L) ? 0.0f : -v.x * v.y);
                        }
                    }
                    if (!wait_all(&full[s], (g / S) & 1)) {
                        ok = false;
                        break;
                    }
                    if constexpr (PACKED) {
                        const uint4 sv =
                            *reinterpret_cast<const uint4 *>(szring + s * kSzBytes + r * 16);
                        const uint4 zv = *reinterpret_cast<const uint4 *>(
                            szring + s * kSzBytes + kSzBytes / 2 + r * 16);
                        sw[0] = sv.x; sw[1] = sv.y; sw[2] = sv.z; sw[3] = sv.w;
                        zw[0] = zv.x; zw[1] = zv.y; zw[2] = zv.z; zw[3] = zv.w;
                    }
                    // (multiplier of D, multiplier of X~) of group gl
                    auto coef = [&](int gl) -> float2 {
                        if constexpr (PACKED) {
                            const float2 s2 = half2_bits_to_float2(sw[gl >> 1]);
                            const float2 z2 = half2_bits_to_float2(zw[gl >> 1]);
                            const float sc = (gl & 1) ? s2.y : s2.x, zc = (gl & 1) ? z2.y : z2.x;
                            return make_float2(16.0f * sc,
                                               centered_pk(zc) ? 0.0f : -sc * (16.0f + zc));
                        } else {
                            return rcoef[gl];
                        }
                    };
                    const int xs = (int)(g % tcd::kXSlots);
                    if (!wait_all(&xfull[xs], (g / tcd::kXSlots) & 1)) {
                        ok = false;
                        break;
                    }
                    const float *tab =
                        reinterpret_cast<const float *>(xring + xs * C::kStride + C::kTab) + m0;
#pragma unroll
                    for (int hs = 0; hs < G::kSets; ++hs) {
                        const uint32_t t = g * G::kSets + hs, b = t & 1, k = t >> 1;
                        // X~ of the set's groups for this warp's x rows, read into
                        // registers before the set's tensor-memory loads
                        float4 tx[SG][MH / 4];
#pragma unroll
                        for (int gi = 0; gi < SG; ++gi)
#pragma unroll
                            for (int m4 = 0; m4 < MH / 4; ++m4)
                                tx[gi][m4] =
                                    reinterpret_cast<const float4 *>(tab + (hs * SG + gi) * MT)[m4];
                        if (!wait_all(&done[b], k & 1)) {
                            ok = false;
                            break;
                        }
                        tc::fence_after();
#pragma unroll
                        for (int pr = 0; pr < SG / 2; ++pr) {
                            float D[2][MH];
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const uint32_t col = lane_base + (b * SG + 2 * pr + e) * NB + m0;
                                if constexpr (MH == 8) {
                                    uint32_t a[8], c2[8];
                                    tc::ld8x2(col, col + MT, a, c2);
#pragma unroll
                                    for (int i = 0; i < MH; ++i)
                                        D[e][i] = __uint_as_float(a[i]) + __uint_as_float(c2[i]);
                                } else {
                                    uint32_t a[4], c2[4];
                                    tc::ld4x2(col, col + MT, a, c2);
#pragma unroll
                                    for (int i = 0; i < MH; ++i)
                                        D[e][i] = __uint_as_float(a[i]) + __uint_as_float(c2[i]);
                                }
                            }
                            if (pr == SG / 2 - 1) {   // this warp's reads of the D set are done
                                tc::fence_before();
                                __syncwarp();
                                if (lane == 0) mbar_arrive(smem_u32(&dempty[b]));
                            }
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const int gl = hs * SG + 2 * pr + e;
                                const float2 cf = coef(gl);
#pragma unroll
                                for (int m4 = 0; m4 < MH / 4; ++m4) {
                                    const float4 X = tx[2 * pr + e][m4];
                                    const float Xm[4] = {X.x, X.y, X.z, X.w};
#pragma unroll
                                    for (int i = 0; i < 4; ++i)
                                        y[4 * m4 + i] = fmaf(cf.x, D[e][4 * m4 + i],
                                                             fmaf(cf.y, Xm[i], y[4 * m4 + i]));
                                }
                            }
                        }
                    }
                    if (!ok) break;
                    // every lane releases the slots after its own reads: an
                    // arrive orders only the arriving thread's accesses, and a
                    // lane's shared-memory load may still be in flight when
                    // another lane of the warp arrives
                    mbar_arrive(smem_u32(&empty[s]));        // scales read
                    mbar_arrive(smem_u32(&xempty[xs]));      // X~ read
                    if (kc + 1 == kch) {
#pragma unroll
                        for (int i = 0; i < MH; ++i) {
                            if (m0 + i < P.M && row < J.N) J.y[(int64_t)(m0 + i) * J.N + row] = y[i];
                            y[i] = 0.0f;
                        }
                    }
                }
            }
        }
    }
    tc::fence_before();
    __syncthreads();
    if (warp == tcd::kMmaWarp) {
        tc::fence_after();
        tc::dealloc(tmem, tcd::kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
constexpr int kBarBytes = 256 + kMaxJobs * (int)sizeof(StreamJob);

template <bool PACKED, int MT>
bc_status launch_one(const StreamParams &P, int grid, int smem, cudaStream_t s) {
    // P.early: programmatic dependent launch (see the kernel's start)
    static std::mutex mu;
    static int attr_smem[64] = {};      // per device: largest size already allowed
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return BC_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (smem > attr_smem[dev]) {
            if (cudaFuncSetAttribute(gemv_stream_kernel<PACKED, MT>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     smem) != cudaSuccess)
                return BC_ERR_CUDA;
            attr_smem[dev] = smem;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(Roles<PACKED>::threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = P.early ? 1 : 0;
    if (cudaLaunchKernelEx(&cfg, gemv_stream_kernel<PACKED, MT>, P) != cudaSuccess) {
        (void)cudaGetLastError();
        return BC_ERR_CUDA;
    }
    return cuda_status();
}

template <bool PACKED, int MT>
bc_status launch_tc(const StreamParams &P, int grid, int smem, cudaStream_t s) {
    static std::mutex mu;
    static int attr_smem[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return BC_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (smem > attr_smem[dev]) {
            if (cudaFuncSetAttribute(gemv_tc_kernel<PACKED, MT>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     smem) != cudaSuccess)
                return BC_ERR_CUDA;
            attr_smem[dev] = smem;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(tcd::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = P.early ? 1 : 0;
    if (cudaLaunchKernelEx(&cfg, gemv_tc_kernel<PACKED, MT>, P) != cudaSuccess) {
        (void)cudaGetLastError();
        return BC_ERR_CUDA;
    }
    return cuda_status();
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault,
                                    &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Weights viewed as bytes [N][row_bytes]; box 128 bytes x 128 rows, 128B swizzle.
bool encode_weights(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap *m,
                    const void *w, int64_t N, int64_t row_bytes) {
    cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)N};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {128, (cuuint32_t)kRows};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(w), dims,
               strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Slots hold MT x rows (M rounded up to the kernel's 1, 2 or 4): the
// consumers of M = 3 read a fourth row whose results are never stored.
size_t xslot_bytes_for(const GemvJob *jobs, int count, int M, bool packed) {
    M = M <= 1 ? 1 : M <= 2 ? 2 : 4;
    size_t xmax = 0;
    for (int i = 0; i < count; ++i) {
        const int K = (int)jobs[i].K;
        const size_t rb = packed ? xrow_bytes<true>(K) : xrow_bytes<false>(K);
        xmax = std::max(xmax, (size_t)M * rb);
    }
    return (xmax + 127) / 128 * 128;
}

// Chunk mode: launches with 5..16 x rows (packed, or runtime RTN at 2..8
// bits) run the tensor-core decode kernel, which streams x per stage from
// the workspace.
bool chunk_mode(int M, bool packed, int bits) {
    return M > kMaxM && M <= kMaxMChunk && (packed || bits <= 8);
}
int chunk_mt(int M) { return M <= 8 ? 8 : 16; }
size_t chunk_bytes(int M, bool packed) {
    if (packed)
        return chunk_mt(M) == 8 ? tcd::Chunk<true, 8>::kBytes : tcd::Chunk<true, 16>::kBytes;
    return chunk_mt(M) == 8 ? tcd::Chunk<false, 8>::kBytes : tcd::Chunk<false, 16>::kBytes;
}
size_t chunk_stride(int M, bool packed) {
    if (packed)
        return chunk_mt(M) == 8 ? tcd::Chunk<true, 8>::kStride : tcd::Chunk<true, 16>::kStride;
    return chunk_mt(M) == 8 ? tcd::Chunk<false, 8>::kStride : tcd::Chunk<false, 16>::kStride;
}
int kchunks_mode(int K, bool packed) {
    return packed ? kchunks_of<true>(K) : kchunks_of<false>(K);
}

// Workspace layout of the chunk-mode activation pieces: each distinct
// (x, K) of the launch once, in job order; off[i] is job i's offset.  A null
// x (a size query without pointers) is never shared, which bounds any call.
size_t xpieces_layout(const GemvJob *jobs, int count, int M, bool packed,
                   std::vector<size_t> *off, std::vector<int> *first) {
    const size_t mtb = chunk_bytes(M, packed);
    size_t total = 0;
    if (off) off->assign(count, 0);
    if (first) first->clear();
    for (int i = 0; i < count; ++i) {
        int prev = -1;
        for (int q = 0; q < i && prev < 0 && jobs[i].x; ++q)
            if (jobs[q].x == jobs[i].x && jobs[q].K == jobs[i].K) prev = q;
        if (prev >= 0) {
            if (off) (*off)[i] = (*off)[prev];
            continue;
        }
        if (off) (*off)[i] = total;
        if (first) first->push_back(i);
        total += (size_t)kchunks_mode((int)jobs[i].K, packed) * mtb;
    }
    return total;
}

// Contiguous unit ranges, one per CTA, that minimise the largest range's cost
// (the classic linear partition: binary search on the bound, greedy fill).
// A unit costs its weight bytes plus a fixed share for its end-of-unit work,
// and a matrix whose x differs from the previous one adds the cost of staging
// it.  Units of one matrix cost the same, so the greedy fill works matrix by
// matrix: O(matrices + CTAs) per probe of the bound.
constexpr double kUnitOverheadBytes = 4096.0;
constexpr double kXSwitchBytes = 16384.0;

void partition_units(StreamParams &P, int n, bool packed, int grid) {
    std::vector<double> ucost(n), jextra(n);
    std::vector<int> nunits(n);
    double total = 0, umax = 0;
    for (int i = 0; i < n; ++i) {
        const StreamJob &J = P.jobs[i];
        ucost[i] = (double)kRows * (packed ? J.K / 2 : J.K * 2) + kUnitOverheadBytes;
        jextra[i] = (i == 0 || P.jobs[i - 1].x != J.x) ? kXSwitchBytes : 0.0;
        nunits[i] = (J.N + kRows - 1) / kRows;
        total += ucost[i] * nunits[i] + jextra[i];
        umax = std::max(umax, ucost[i] + jextra[i]);
    }
    // CTAs a bound needs; fills cta_begin when `out` is set
    auto fill = [&](double T, bool out) -> int {
        int ctas = 1, unit = 0;
        double cur = 0;
        if (out) P.cta_begin[0] = 0;
        for (int i = 0; i < n; ++i) {
            int left = nunits[i];
            double extra = jextra[i];
            while (left > 0) {
                const double room = T - cur - extra;
                int fit = room >= ucost[i] ? (int)std::min<double>(left, room / ucost[i]) : 0;
                if (fit == 0 && cur == 0) fit = 1;       // a unit above T still goes somewhere
                cur += extra + fit * ucost[i];
                extra = 0;
                left -= fit;
                unit += fit;
                if (left > 0) {                          // next CTA starts here
                    if (out && ctas < grid) P.cta_begin[ctas] = unit;
                    ++ctas;
                    cur = 0;
                    extra = kXSwitchBytes;               // it stages this x itself
                }
            }
        }
        return ctas;
    };
    double lo = std::max(umax, total / grid), hi = total + umax;
    for (int it = 0; it < 48 && hi - lo > 1.0; ++it) {
        const double mid = 0.5 * (lo + hi);
        if (fill(mid, false) <= grid) hi = mid; else lo = mid;
    }
    const int used = fill(hi, true);
    // CTAs past the last range get empty ranges
    for (int c = std::min(used, grid); c < grid; ++c) P.cta_begin[c] = P.total_units;
}

}  // namespace

bool gemv_stream_supported(const GemvJob *jobs, int count, int M, bool packed, int bits,
                           int max_smem) {
    const bool xc = chunk_mode(M, packed, bits);
    if (M < 1 || (M > kMaxM && !xc) || count < 1) return false;
    for (int i = 0; i < count; ++i)
        if (jobs[i].N >= (1 << 30) || jobs[i].K >= (1 << 24)) return false;
    const size_t xs = xc ? 0 : xslot_bytes_for(jobs, count, M, packed);
    const size_t fixed =
        2 * xs + kBarBytes + 1024 + (xc ? tcd::kXSlots * chunk_stride(M, packed) : 0);
    const size_t per_stage = kStageBytes + (packed ? kSzBytes : 0);
    if (fixed + 2 * per_stage > (size_t)max_smem) return false;
    return tensor_map_encoder() != nullptr;
}

size_t gemv_stream_workspace_bytes(const GemvJob *jobs, int count, int M, bool packed,
                                   int bits) {
    if (!chunk_mode(M, packed, bits)) return 0;
    // launches above kMaxJobs matrices reuse the space batch by batch
    size_t worst = 0;
    for (int b = 0; b < count; b += kMaxJobs)
        worst = std::max(worst, xpieces_layout(jobs + b, std::min(kMaxJobs, count - b), M, packed,
                                            nullptr, nullptr));
    return worst ? worst + 256 : 0;
}

namespace {
// Prepared launches of recent calls (per host thread).  A decode step calls
// with the same matrices every time; a hit skips the tensor-map encoding and
// the partition, leaving only the launch itself.
struct StreamPlan {
    std::vector<GemvJob> key;
    int M = 0, bits = 0, dev = -1;
    bool packed = false;
    const void *ws = nullptr;    // chunk mode: the workspace the chunk pointers point into
    StreamParams P;
    int grid = 0, smem = 0;
    XpreParams X;                // chunk mode: the pre-pass over the distinct x
    int xgrid = 0;
};
constexpr int kPlanCache = 4;

bool same_call(const StreamPlan &p, const GemvJob *jobs, int count, int M, int bits,
               bool packed, int dev, bool early, const void *ws) {
    return p.dev == dev && p.M == M && p.bits == bits && p.packed == packed &&
           (p.P.early != 0) == early && (!chunk_mode(M, packed, bits) || p.ws == ws) &&
           (int)p.key.size() == count &&
           std::memcmp(p.key.data(), jobs, sizeof(GemvJob) * count) == 0;
}

bc_status launch_plan(const StreamPlan &p, cudaStream_t s) {
    if (chunk_mode(p.M, p.packed, p.bits)) {
        const int mt = chunk_mt(p.M);
        if (p.packed && mt == 8) xpieces_kernel<true, 8><<<p.xgrid, 256, 0, s>>>(p.X);
        if (p.packed && mt == 16) xpieces_kernel<true, 16><<<p.xgrid, 256, 0, s>>>(p.X);
        if (!p.packed && mt == 8) xpieces_kernel<false, 8><<<p.xgrid, 256, 0, s>>>(p.X);
        if (!p.packed && mt == 16) xpieces_kernel<false, 16><<<p.xgrid, 256, 0, s>>>(p.X);
        const bc_status st = cuda_status();
        if (st != BC_OK) return st;
        if (p.packed)
            return mt == 8 ? launch_tc<true, 8>(p.P, p.grid, p.smem, s)
                           : launch_tc<true, 16>(p.P, p.grid, p.smem, s);
        return mt == 8 ? launch_tc<false, 8>(p.P, p.grid, p.smem, s)
                       : launch_tc<false, 16>(p.P, p.grid, p.smem, s);
    }
    if (p.packed)
        return p.M <= 1 ? launch_one<true, 1>(p.P, p.grid, p.smem, s)
             : p.M <= 2 ? launch_one<true, 2>(p.P, p.grid, p.smem, s)
                        : launch_one<true, 4>(p.P, p.grid, p.smem, s);
    return p.M <= 1 ? launch_one<false, 1>(p.P, p.grid, p.smem, s)
         : p.M <= 2 ? launch_one<false, 2>(p.P, p.grid, p.smem, s)
                    : launch_one<false, 4>(p.P, p.grid, p.smem, s);
}
}  // namespace

bc_status launch_gemv_stream(const GemvJob *jobs, int count, int M, int bits,
                             bool packed, cudaStream_t s, bool early_start, void *workspace,
                             size_t ws_bytes) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BC_ERR_CUDA;
    const bool xc = chunk_mode(M, packed, bits);
    if (xc) {
        const size_t need = gemv_stream_workspace_bytes(jobs, count, M, packed, bits);
        if (!workspace || ws_bytes < need) return BC_ERR_WORKSPACE;
    }
    thread_local std::vector<std::unique_ptr<StreamPlan>> plans;
    if (count <= kMaxJobs) {
        for (size_t i = 0; i < plans.size(); ++i) {
            if (!same_call(*plans[i], jobs, count, M, bits, packed, dev, early_start, workspace))
                continue;
            if (i) std::rotate(plans.begin(), plans.begin() + i, plans.begin() + i + 1);
            return launch_plan(*plans[0], s);
        }
    }
    DeviceInfo di;
    if (!device_info(&di)) return BC_ERR_CUDA;
    auto enc = tensor_map_encoder();
    if (!enc) return BC_ERR_CUDA;
    std::unique_ptr<StreamPlan> plan(new StreamPlan());
    StreamParams &P = plan->P;
    for (int b0 = 0; b0 < count; b0 += kMaxJobs) {
        const int n = std::min(kMaxJobs, count - b0);
        int units = 0;
        for (int i = 0; i < n; ++i) {
            const GemvJob &G0 = jobs[b0 + i];
            StreamJob &J = P.jobs[i];
            J.x = G0.x; J.s = G0.s; J.z = G0.z; J.y = G0.y;
            J.N = (int)G0.N; J.K = (int)G0.K; J.group = (int)G0.group;
            const int rbytes = packed ? J.K / 2 : J.K * 2;
            J.unit_begin = units;
            units += (J.N + kRows - 1) / kRows;
            if (!encode_weights(enc, &P.wmap[i], G0.w, J.N, rbytes)) return BC_ERR_CUDA;
        }
        P.xchunk_bytes = 0;
        if (xc) {       // the jobs' x point at their chunks in the workspace
            const int MT = chunk_mt(M);
            std::vector<size_t> off;
            std::vector<int> first;
            xpieces_layout(jobs + b0, n, M, packed, &off, &first);
            uint8_t *ws = reinterpret_cast<uint8_t *>(
                (reinterpret_cast<uintptr_t>(workspace) + 255) & ~uintptr_t(255));
            for (int i = 0; i < n; ++i) P.jobs[i].x = reinterpret_cast<const float *>(ws + off[i]);
            XpreParams &X = plan->X;
            int tasks = 0;
            X.count = (int)first.size();
            for (int q = 0; q < X.count; ++q) {
                const GemvJob &G0 = jobs[b0 + first[q]];
                X.t[q].x = G0.x;
                X.t[q].out = ws + off[first[q]];
                X.t[q].K = (int)G0.K;
                X.t[q].task_begin = tasks;
                tasks += kchunks_mode((int)G0.K, packed) * MT * (packed ? 2 : 1);
            }
            X.M = M;
            X.MT = MT;
            X.total = tasks;
            plan->xgrid = std::max(1, std::min((tasks + 7) / 8, 4 * di.sm_count));
            plan->ws = workspace;
            P.xchunk_bytes = (int)chunk_bytes(M, packed);
        }
        const size_t xs = xc ? 0 : xslot_bytes_for(jobs + b0, n, M, packed);
        const int grid = std::max(1, std::min({units, di.sm_count, kMaxCtas}));
        P.total_units = units;
        partition_units(P, n, packed, grid);
        P.cta_begin[grid] = units;
        P.count = n;
        // first job of each CTA's range, and the most jobs one range touches
        {
            int jj = 0, most = 1;
            for (int c = 0; c <= grid; ++c) {
                const int u = std::min(P.cta_begin[c], units - 1);
                while (jj + 1 < n && P.jobs[jj + 1].unit_begin <= u) ++jj;
                P.cta_job[c] = jj;
                if (c > 0) most = std::max(most, P.cta_job[c] - P.cta_job[c - 1] + 1);
            }
            P.max_cta_jobs = most;
        }
        const int fixed = (int)(2 * xs) +
                          (xc ? 512 + tcd::kXSlots * (int)chunk_stride(M, packed) : 256) +
                          P.max_cta_jobs * (int)sizeof(StreamJob) + 1024;
        const int per_stage = kStageBytes + (packed ? kSzBytes : 0);
        int stages = (di.max_smem_optin - fixed) / per_stage;
        stages = std::min(stages, 6);
        if (stages < 2) return BC_ERR_UNSUPPORTED;
        P.M = M;
        P.bits = bits;
        P.range = (int)jobs[0].range;
        P.xslot_bytes = (int)xs;
        P.stages = stages;
        P.early = early_start ? 1 : 0;
        plan->M = M;
        plan->bits = bits;
        plan->packed = packed;
        plan->dev = dev;
        plan->grid = grid;
        plan->smem = stages * per_stage + fixed;
        const bc_status st = launch_plan(*plan, s);
        if (st != BC_OK) return st;
    }
    if (count <= kMaxJobs) {
        plan->key.assign(jobs, jobs + count);
        plans.insert(plans.begin(), std::move(plan));
        if ((int)plans.size() > kPlanCache) plans.pop_back();
    }
    return BC_OK;
}

bc_status gemv_set_wait_limit(long long cycles) {
    if (cudaMemcpyToSymbol(g_gemv_wait_limit, &cycles, sizeof(cycles)) != cudaSuccess)
        return BC_ERR_CUDA;
    return BC_OK;
}

unsigned gemv_timeouts() {
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_gemv_timeouts, sizeof(v)) != cudaSuccess) return ~0u;
    return v;
}

}  // namespace bc
