// bc_gemv_stream.cu -- streaming fused dequant GEMV for decode (M <= 4).
//
// Decode "reads every weight in the model to write one word" (Enargeia):
// the matmul is one pass over HBM.  The kernel is a TMA pipeline that keeps
// ~130-200 KB per SM in flight, with the arithmetic per weight cut down until
// the stream, not the issue slots, sets the pace.
//
// One CTA per SM, persistent over a byte-balanced contiguous range of
// "units" (128 weight rows of one matrix) that spans every matrix of a
// grouped launch (Enargeia, "One decode step": hundreds of passes per token
// are one launch here).  Warp roles:
//   warp 0      loader: lane 0 issues the TMA of each stage (a 256-byte column
//               chunk of the unit's 128 rows as two 2D boxes of 128 rows x
//               128 bytes, 128-byte swizzle) into a ring of up to 6 stages with
//               full/empty mbarriers.
//   warp 1      activation stager: the x of each new matrix goes into one of
//               two smem slots (see below); the first slot is filled by every
//               warp but the loader together before streaming starts.
//   warps 2-17  consumers: warp (window w, row group g) handles 16 rows and
//               the w-th 128-byte window of every stage; the two windows'
//               partial row sums meet in smem at the end of each unit.  Each
//               lane loads its own fp16 scales and zeros from global memory two
//               stages ahead (small scattered copies cost the loader more issue
//               time than the stage itself).
//
// Packed int4 (Enargeia, "Four bits per weight": codes unpacked in registers,
// never written back) runs on the int8 tensor cores (mma.sync m16n8k32
// u8 x s8 -> s32).  ldmatrix brings the swizzled stage into A fragments; one
// AND per register gives the even-k codes (q) and one the odd-k codes (16 q)
// as unsigned bytes.  The activations are staged as integers per 64-group,
//     x_k ~= X_k * 2^(E_g - 27),  X_k = rint(x_k 2^(27 - E_g)) (even k),
//                                 X_k = 16 rint(x_k 2^(23 - E_g)) (odd k),
// with max|x| < 2^E_g over the group, each split into four balanced int8
// digits (X = d0 + 2^8 d1 + 2^16 d2 + 2^24 d3) that fill the 8 columns of B.
// With one x row the columns hold 2 groups x 4 digits, the k slots of each
// mma split between the two groups (block diagonal); with several x rows
// they hold 2 rows x 4 digits.  The integer dot products are exact, so
//     y = sum_g s_g ( 2^(E_g-27) sum_d 2^(8d) C_gd - z_g sum_k x_k~ )
// carries only the rounding of x to 23-27 bits and of the fp32 epilogue.
//
// Runtime RTN (BITCRUSH BC-06, "Under the hood": codes computed inline as
// weights are read) runs on the CUDA cores, four threads per row, with the
// exact-rounding fast path of the general GEMV (bc_gemv.cu).
//
// Every mbarrier wait is bounded; a wait that runs out stops the CTA (its
// outputs are then incomplete) and is counted for bc_device_timeouts.
#include "bc_internal.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>
#include <vector>

namespace bc {

__device__ unsigned int g_gemv_timeouts = 0;

namespace {

constexpr int kRows = 128;              // weight rows per unit
constexpr int kChunk = 256;             // bytes of a row per stage
constexpr int kBoxBytes = kRows * 128;  // one TMA box: 128 rows x 128 bytes, SW128
constexpr int kStageBytes = 2 * kBoxBytes;
constexpr int kConsumers = 16;
constexpr int kStagers = 1 + kConsumers;   // warps that fill the first x slot
constexpr int kThreads = 32 * (2 + kConsumers);
constexpr int kMaxJobs = 168;
constexpr int kMaxCtas = 160;
constexpr int kMaxM = 4;
constexpr int kXP = 23;                 // bits of the odd-k activation integers
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
    int count, total_units, M, bits;
    int xslot_bytes, stages;
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
// in distinct banks), then [parity][group] float2 (f, X~) tables.
__host__ __device__ __forceinline__ int dig_rs(int kchunks) { return 32 * kchunks + 4; }
// Bytes of one x row in a slot.  Runtime: x[kp] f32.
template <bool PACKED> __host__ __device__ __forceinline__ int xrow_bytes(int K) {
    const int kc = kchunks_of<PACKED>(K);
    return PACKED ? 64 * dig_rs(kc) + 16 * (8 * kc) : 4 * kpad_of<false>(K);
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
    while (true) {
        if (mbar_try(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > kWaitCycles) {
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
__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}
__device__ __forceinline__ void named_bar(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
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

// The job table is copied into shared memory at kernel start: dynamically
// indexed reads of a ~30 KB parameter block miss the constant cache.
__device__ __forceinline__ int find_job(const StreamJob *jobs, int count, int unit) {
    int lo = 0, hi = count - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (jobs[mid].unit_begin <= unit) lo = mid; else hi = mid - 1;
    }
    return lo;
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
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
            // max|x| < 2^E; E >= -96 keeps every scale below a normal float
            int E = amax > 0.0f ? (int)((__float_as_uint(amax) >> 23) & 0xffu) - 126 : 0;
            E = max(E, -96);
            const float sc_e = __uint_as_float((uint32_t)(127 + kXP + 4 - E) << 23);
            const float sc_o = __uint_as_float((uint32_t)(127 + kXP - E) << 23);
            uint32_t de[4], dq[4];
            int sum = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int xe = __float2int_rn(v[2 * i] * sc_e);      // |xe| <= 2^27
                const int xo = __float2int_rn(v[2 * i + 1] * sc_o);  // |xo| <= 2^23
                sum += xe + 16 * xo;
                de[i] = digits4(xe);
                dq[i] = digits4(xo);
            }
            uint32_t te[4], to[4];
            transpose4(de, te);
            transpose4(dq, to);
            const int U = 2 * g + (j >> 2), tt = j & 3;
#pragma unroll
            for (int d = 0; d < 4; ++d)
                *reinterpret_cast<uint2 *>(dig + (d * 4 + tt) * rs + 2 * U) =
                    make_uint2(te[d], to[d]);
            float fs = (float)sum;
            fs += __shfl_xor_sync(0xffffffffu, fs, 1);
            fs += __shfl_xor_sync(0xffffffffu, fs, 2);
            fs += __shfl_xor_sync(0xffffffffu, fs, 4);
            if (j == 0) {
                const float f = __uint_as_float((uint32_t)(127 + E - kXP - 4) << 23);
                tab[g] = make_float2(f, f * fs);
                tab[gpad + g] = make_float2(f * 65536.0f, 0.0f);
            }
        }
    }
}

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
        if (lane == 0) mbar_arrive(smem_u32(&xempty[(c.e - 1) & 1]));
    }
    c.cur = J.x;
    if (!mbar_wait(smem_u32(&xfull[c.e & 1]), (c.e >> 1) & 1, abort_flag)) return false;
    c.xs = xslots + (c.e & 1) * xslot_bytes;
    ++c.e;
    return true;
}

// Cross-window sums: the window-1 warp of a row group hands its 16 row
// partials to the window-0 warp through smem, double-buffered by unit, with
// an mbarrier pair per buffer (bounded waits, so a warp that stops early on
// an abort leaves no partner blocked).
struct Xchg {
    float *base;       // [8 row groups][2 parity][16 rows][kMaxM]
    uint64_t *bars;    // [8 row groups][2 parity] {full, empty}
    __device__ __forceinline__ float *slot(int rg, int parity, int r16) const {
        return base + ((rg * 2 + parity) * 16 + r16) * kMaxM;
    }
    __device__ __forceinline__ uint32_t bar(int rg, int parity, int which) const {
        return smem_u32(&bars[(rg * 2 + parity) * 2 + which]);
    }
    // window 1, unit n of this warp: wait until slot n&1 was read two units ago
    __device__ __forceinline__ bool put_begin(int rg, uint32_t n, volatile int *ab) const {
        return mbar_wait(bar(rg, n & 1, 1), ((n >> 1) & 1) ^ 1, ab);
    }
    __device__ __forceinline__ void put_end(int rg, uint32_t n, int lane) const {
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(rg, n & 1, 0));
    }
    // window 0: wait for the partials of unit n, then hand the slot back
    __device__ __forceinline__ bool get_begin(int rg, uint32_t n, volatile int *ab) const {
        return mbar_wait(bar(rg, n & 1, 0), (n >> 1) & 1, ab);
    }
    __device__ __forceinline__ void get_end(int rg, uint32_t n, int lane) const {
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(rg, n & 1, 1));
    }
};

// Stage / unit walk shared by the consumers.
struct Walk {
    int u, kc, jidx, sidx;
    uint32_t sph;
};
// A second walk, two stages ahead, tells which scales and zeros to prefetch
// (it stays on the last stage of the range once it gets there).  It keeps
// this lane's two scale rows and two zero rows as pointers, renewed once per
// unit, so a fetch is four loads.  Rows past N are clamped to the last row:
// they only feed outputs that are never stored.
struct Ahead {
    int u, kc, j, G;
    const unsigned short *s0, *s1, *z0, *z1;
    __device__ __forceinline__ void rows(const StreamJob *jobs, int ra) {
        const StreamJob &J = jobs[j];
        G = J.K >> 6;
        const int r = (u - J.unit_begin) * kRows + ra;
        const int64_t b0 = (int64_t)min(r, J.N - 1) * G, b1 = (int64_t)min(r + 8, J.N - 1) * G;
        s0 = reinterpret_cast<const unsigned short *>(J.s) + b0;
        s1 = reinterpret_cast<const unsigned short *>(J.s) + b1;
        z0 = reinterpret_cast<const unsigned short *>(J.z) + b0;
        z1 = reinterpret_cast<const unsigned short *>(J.z) + b1;
    }
    __device__ __forceinline__ void start(const StreamJob *jobs, int u0, int j0, int ra) {
        u = u0;
        kc = 0;
        j = j0;
        rows(jobs, ra);
    }
    __device__ __forceinline__ void advance(const StreamJob *jobs, int count, int u1, int ra) {
        if (++kc == kchunks_of<true>(jobs[j].K)) {
            if (u + 1 >= u1) {
                --kc;
                return;
            }
            kc = 0;
            ++u;
            j = next_job(jobs, count, j, u);
            rows(jobs, ra);
        }
    }
};

// This lane's fp16 scales and zeros for one stage: rows ra and ra+8 of the
// unit, NG consecutive groups from 8*kc + gw, packed in pairs (g, g+1).
// Issued two stages before use so the loads are in flight while the stages
// in between are consumed.  Groups are clamped into the row instead of
// predicated, so the loads go straight into the registers read two stages
// later; a group past K/64 multiplies an exactly zero code sum and
// activation sum.
template <int NG>
struct SzRegs {
    uint32_t s[2][NG / 2], z[2][NG / 2];
};
template <int NG>
__device__ __forceinline__ void fetch_sz(const Ahead &a, int gw, SzRegs<NG> &o) {
    const int g = 8 * a.kc + gw;
#pragma unroll
    for (int p = 0; p < NG / 2; ++p) {
        if ((a.G & 1) == 0) {         // pair (gg, gg+1) is 4-byte aligned
            const int gg = min(g + 2 * p, a.G - 2);
            o.s[0][p] = __ldg(reinterpret_cast<const uint32_t *>(a.s0 + gg));
            o.s[1][p] = __ldg(reinterpret_cast<const uint32_t *>(a.s1 + gg));
            o.z[0][p] = __ldg(reinterpret_cast<const uint32_t *>(a.z0 + gg));
            o.z[1][p] = __ldg(reinterpret_cast<const uint32_t *>(a.z1 + gg));
        } else {
            const int g0 = min(g + 2 * p, a.G - 1), g1 = min(g + 2 * p + 1, a.G - 1);
            o.s[0][p] = (uint32_t)__ldg(a.s0 + g0) | ((uint32_t)__ldg(a.s0 + g1) << 16);
            o.s[1][p] = (uint32_t)__ldg(a.s1 + g0) | ((uint32_t)__ldg(a.s1 + g1) << 16);
            o.z[0][p] = (uint32_t)__ldg(a.z0 + g0) | ((uint32_t)__ldg(a.z0 + g1) << 16);
            o.z[1][p] = (uint32_t)__ldg(a.z1 + g0) | ((uint32_t)__ldg(a.z1 + g1) << 16);
        }
    }
}

// Window 0 folds window 1's partial row sums of a unit into y one unit
// later, when they are long written, instead of waiting at the unit's end.
struct PendingY {
    bool on = false;
    uint32_t n = 0;            // unit index (this warp's count) it belongs to
    float *ya = nullptr;       // y + row of this lane's first row (or null)
    float *yb = nullptr;       // ... second row (or null)
    float va[kMaxM / 2 + 1], vb[kMaxM / 2 + 1];
};

// ---- packed consumer, one x row: block-diagonal groups ---------------------------
// mma p of a step pairs window units (p, p+4): slots 0-15 take unit p's codes
// and B columns 0-3, slots 16-31 unit p+4's and columns 4-7.  Units (0,4) and
// (1,5) belong to groups (0,2), units (2,6) and (3,7) to groups (1,3).
__device__ __forceinline__ void consume_packed_m1(
    const StreamParams &P, const StreamJob *jobs, uint8_t *smem, uint8_t *xslots,
    uint64_t *full, uint64_t *empty, uint64_t *xfull, uint64_t *xempty,
    volatile int *abort_flag, const Xchg &xg, int u0, int u1, int cw, int lane) {
    const int S = P.stages;
    const int rg = cw & 7, w = cw >> 3;
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
    // epilogue role: groups 2*eh (+1), digit pair ep
    const int eh = t >> 1, ep = t & 1;
    const int ra = 16 * rg + gq;
    XCursor xc;
    Walk k{u0, 0, find_job(jobs, P.count, u0), 0, 0u};
    Ahead ah;
    ah.start(jobs, u0, k.jidx, ra);
    SzRegs<2> sz0, sz1, sz2;
    fetch_sz<2>(ah, 4 * w + 2 * eh, sz0);
    ah.advance(jobs, P.count, u1, ra);
    fetch_sz<2>(ah, 4 * w + 2 * eh, sz1);
    ah.advance(jobs, P.count, u1, ra);
    float ya = 0.0f, yb = 0.0f;
    int parity = 0;
    uint32_t nunit = 0;
    PendingY pend;
    // window 0: add window 1's partials of the pending unit and store
    auto flush = [&]() -> bool {
        if (!pend.on) return true;
        if (!xg.get_begin(rg, pend.n, abort_flag)) return false;
        if (t == 0) {
            if (pend.ya) *pend.ya = pend.va[0] + xg.slot(rg, pend.n & 1, gq)[0];
            if (pend.yb) *pend.yb = pend.vb[0] + xg.slot(rg, pend.n & 1, gq + 8)[0];
        }
        xg.get_end(rg, pend.n, lane);
        pend.on = false;
        return true;
    };
    // One stage; `use` holds its scales/zeros, `fill` receives those of the
    // stage two ahead.  Returns true when this warp is done.
    auto step = [&](const SzRegs<2> &use, SzRegs<2> &fill) -> bool {
        fetch_sz<2>(ah, 4 * w + 2 * eh, fill);
        ah.advance(jobs, P.count, u1, ra);
        const StreamJob &J = jobs[k.jidx];
        if (k.kc == 0 && !x_enter(xc, J, k.u == u0, xslots, P.xslot_bytes, xfull, xempty,
                                  abort_flag, lane))
            return true;
        const int kch = kchunks_of<true>(J.K);
        const int rs = dig_rs(kch);
        const int s = k.sidx;
        if (!mbar_wait(smem_u32(&full[s]), k.sph, abort_flag)) return true;
        const uint32_t box = smem_u32(smem + s * kStageBytes + w * kBoxBytes);
        uint32_t R[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) ldsm_x4(box + a_off[j], R[j]);
        const uint32_t *xd = reinterpret_cast<const uint32_t *>(xc.xs) + (bd * 4 + t) * rs +
                             2 * (16 * k.kc + 8 * w + 4 * bh);
        const uint4 Q0 = *reinterpret_cast<const uint4 *>(xd);
        const uint4 Q1 = *reinterpret_cast<const uint4 *>(xd + 4);
        const float4 tb = *reinterpret_cast<const float4 *>(
            xc.xs + 64 * rs + 8 * (ep * 8 * kch + 8 * k.kc + 4 * w + 2 * eh));
        uint32_t lo[4][4], hi[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                lo[j][i] = R[j][i] & 0x0F0F0F0Fu;
                hi[j][i] = R[j][i] & 0xF0F0F0F0u;
            }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[s]));   // stage consumed
        int CA[4] = {0, 0, 0, 0}, CB[4] = {0, 0, 0, 0};
        mma_i8(CA, lo[0][0], lo[0][1], lo[0][2], lo[0][3], Q0.x & m0, Q0.x & m1);
        mma_i8(CB, lo[2][0], lo[2][1], lo[2][2], lo[2][3], Q1.x & m0, Q1.x & m1);
        mma_i8(CA, hi[0][0], hi[0][1], hi[0][2], hi[0][3], Q0.y & m0, Q0.y & m1);
        mma_i8(CB, hi[2][0], hi[2][1], hi[2][2], hi[2][3], Q1.y & m0, Q1.y & m1);
        mma_i8(CA, lo[1][0], lo[1][1], lo[1][2], lo[1][3], Q0.z & m0, Q0.z & m1);
        mma_i8(CB, lo[3][0], lo[3][1], lo[3][2], lo[3][3], Q1.z & m0, Q1.z & m1);
        mma_i8(CA, hi[1][0], hi[1][1], hi[1][2], hi[1][3], Q0.w & m0, Q0.w & m1);
        mma_i8(CB, hi[3][0], hi[3][1], hi[3][2], hi[3][3], Q1.w & m0, Q1.w & m1);
        // this lane: digits (2ep, 2ep+1) of rows ra, ra+8 for groups 2eh (A), 2eh+1 (B)
        const float2 sa = half2_bits_to_float2(use.s[0][0]), sb = half2_bits_to_float2(use.s[1][0]);
        const float2 za = half2_bits_to_float2(use.z[0][0]), zb = half2_bits_to_float2(use.z[1][0]);
        const float vAa = (float)(CA[0] + 256 * CA[1]), vAb = (float)(CA[2] + 256 * CA[3]);
        const float vBa = (float)(CB[0] + 256 * CB[1]), vBb = (float)(CB[2] + 256 * CB[3]);
        ya = fmaf(sa.x, fmaf(tb.x, vAa, -za.x * tb.y), ya);
        yb = fmaf(sb.x, fmaf(tb.x, vAb, -zb.x * tb.y), yb);
        ya = fmaf(sa.y, fmaf(tb.z, vBa, -za.y * tb.w), ya);
        yb = fmaf(sb.y, fmaf(tb.z, vBb, -zb.y * tb.w), yb);

        int nu = k.u, nkc = k.kc + 1, nj = k.jidx;
        if (nkc == kch) {
            nu = k.u + 1;
            nkc = 0;
            if (nu < u1) nj = next_job(jobs, P.count, k.jidx, nu);
        }
        if (nkc == 0) {       // unit done: four lanes per row, then two windows
            ya += __shfl_xor_sync(0xffffffffu, ya, 1);
            ya += __shfl_xor_sync(0xffffffffu, ya, 2);
            yb += __shfl_xor_sync(0xffffffffu, yb, 1);
            yb += __shfl_xor_sync(0xffffffffu, yb, 2);
            if (w == 1) {
                if (!xg.put_begin(rg, nunit, abort_flag)) return true;
                if (t == 0) {
                    xg.slot(rg, parity, gq)[0] = ya;
                    xg.slot(rg, parity, gq + 8)[0] = yb;
                }
                xg.put_end(rg, nunit, lane);
            } else {
                if (!flush()) return true;
                const int r0 = (k.u - J.unit_begin) * kRows;
                pend.on = true;
                pend.n = nunit;
                pend.ya = r0 + ra < J.N ? J.y + r0 + ra : nullptr;
                pend.yb = r0 + ra + 8 < J.N ? J.y + r0 + ra + 8 : nullptr;
                pend.va[0] = ya;
                pend.vb[0] = yb;
            }
            ya = yb = 0.0f;
            parity ^= 1;
            ++nunit;
        }
        if (nu >= u1) return true;
        k.u = nu;
        k.kc = nkc;
        k.jidx = nj;
        if (++k.sidx == S) {      // ring position of the next stage
            k.sidx = 0;
            k.sph ^= 1;
        }
        return false;
    };
    while (!step(sz0, sz2) && !step(sz1, sz0) && !step(sz2, sz1)) {
    }
    if (w == 0) flush();
}

// ---- packed consumer, 2 or 4 x rows ------------------------------------------------
// Each mma takes one 32-k unit (slots 0-15 even k, 16-31 odd k) and a pair of
// x rows as B columns (row 2*mp + h in columns 4h..4h+3).
template <int MT>
__device__ __forceinline__ void consume_packed_mx(
    const StreamParams &P, const StreamJob *jobs, uint8_t *smem, uint8_t *xslots,
    uint64_t *full, uint64_t *empty, uint64_t *xfull, uint64_t *xempty,
    volatile int *abort_flag, const Xchg &xg, int u0, int u1, int cw, int lane) {
    constexpr int MP = MT / 2;
    const int S = P.stages;
    const int rg = cw & 7, w = cw >> 3;
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
    Walk k{u0, 0, find_job(jobs, P.count, u0), 0, 0u};
    Ahead ah;
    ah.start(jobs, u0, k.jidx, ra);
    SzRegs<4> sz0, sz1, sz2;
    fetch_sz<4>(ah, 4 * w, sz0);
    ah.advance(jobs, P.count, u1, ra);
    fetch_sz<4>(ah, 4 * w, sz1);
    ah.advance(jobs, P.count, u1, ra);
    float ya[MP], yb[MP];
#pragma unroll
    for (int p = 0; p < MP; ++p) ya[p] = yb[p] = 0.0f;
    int parity = 0;
    uint32_t nunit = 0;
    auto step = [&](const SzRegs<4> &use, SzRegs<4> &fill) -> bool {
        fetch_sz<4>(ah, 4 * w, fill);
        ah.advance(jobs, P.count, u1, ra);
        const StreamJob &J = jobs[k.jidx];
        if (k.kc == 0 && !x_enter(xc, J, k.u == u0, xslots, P.xslot_bytes, xfull, xempty,
                                  abort_flag, lane))
            return true;
        const int kch = kchunks_of<true>(J.K);
        const int rs = dig_rs(kch);
        const int mb = xrow_bytes<true>(J.K);
        const int s = k.sidx;
        if (!mbar_wait(smem_u32(&full[s]), k.sph, abort_flag)) return true;
        const uint32_t box = smem_u32(smem + s * kStageBytes + w * kBoxBytes);
        uint32_t R[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) ldsm_x4(box + a_off[j], R[j]);
        uint32_t lo[4][4], hi[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                lo[j][i] = R[j][i] & 0x0F0F0F0Fu;
                hi[j][i] = R[j][i] & 0xF0F0F0F0u;
            }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[s]));   // stage consumed
        float sa[4], sb[4], za[4], zb[4];
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const float2 a2 = half2_bits_to_float2(use.s[0][p]), b2 = half2_bits_to_float2(use.s[1][p]);
            const float2 c2 = half2_bits_to_float2(use.z[0][p]), d2 = half2_bits_to_float2(use.z[1][p]);
            sa[2 * p] = a2.x; sa[2 * p + 1] = a2.y;
            sb[2 * p] = b2.x; sb[2 * p + 1] = b2.y;
            za[2 * p] = c2.x; za[2 * p + 1] = c2.y;
            zb[2 * p] = d2.x; zb[2 * p + 1] = d2.y;
        }
#pragma unroll
        for (int mp = 0; mp < MP; ++mp) {
            // B: this lane's words for units 0..7 of the window, both parities
            const uint32_t *xd = reinterpret_cast<const uint32_t *>(xc.xs + (2 * mp + bh) * mb) +
                                 (bd * 4 + t) * rs + 2 * (16 * k.kc + 8 * w);
            uint4 Q[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) Q[j] = reinterpret_cast<const uint4 *>(xd)[j];
            int C[4][4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                C[j][0] = C[j][1] = C[j][2] = C[j][3] = 0;
                mma_i8(C[j], lo[j][0], lo[j][1], hi[j][0], hi[j][1], Q[j].x, Q[j].y);
                mma_i8(C[j], lo[j][2], lo[j][3], hi[j][2], hi[j][3], Q[j].z, Q[j].w);
            }
            const float *tb = reinterpret_cast<const float *>(
                xc.xs + (2 * mp + eh) * mb + 64 * rs + 8 * (ep * 8 * kch + 8 * k.kc + 4 * w));
            const float4 t01 = reinterpret_cast<const float4 *>(tb)[0];
            const float4 t23 = reinterpret_cast<const float4 *>(tb)[1];
            const float f[4] = {t01.x, t01.z, t23.x, t23.z};
            const float X[4] = {t01.y, t01.w, t23.y, t23.w};
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                const float va = (float)(C[g][0] + 256 * C[g][1]);
                const float vb = (float)(C[g][2] + 256 * C[g][3]);
                ya[mp] = fmaf(sa[g], fmaf(f[g], va, -za[g] * X[g]), ya[mp]);
                yb[mp] = fmaf(sb[g], fmaf(f[g], vb, -zb[g] * X[g]), yb[mp]);
            }
        }

        int nu = k.u, nkc = k.kc + 1, nj = k.jidx;
        if (nkc == kch) {
            nu = k.u + 1;
            nkc = 0;
            if (nu < u1) nj = next_job(jobs, P.count, k.jidx, nu);
        }
        if (nkc == 0) {       // unit done: two lanes per row and x row, then two windows
#pragma unroll
            for (int mp = 0; mp < MP; ++mp) {
                ya[mp] += __shfl_xor_sync(0xffffffffu, ya[mp], 1);
                yb[mp] += __shfl_xor_sync(0xffffffffu, yb[mp], 1);
            }
            if (w == 1) {
                if (!xg.put_begin(rg, nunit, abort_flag)) return true;
                if (ep == 0) {
#pragma unroll
                    for (int mp = 0; mp < MP; ++mp) {
                        xg.slot(rg, parity, gq)[2 * mp + eh] = ya[mp];
                        xg.slot(rg, parity, gq + 8)[2 * mp + eh] = yb[mp];
                    }
                }
                xg.put_end(rg, nunit, lane);
            } else {
                if (!xg.get_begin(rg, nunit, abort_flag)) return true;
                if (ep == 0) {
                    const int r0 = (k.u - J.unit_begin) * kRows;
#pragma unroll
                    for (int mp = 0; mp < MP; ++mp) {
                        const int m = 2 * mp + eh;
                        if (m >= P.M) continue;
                        if (r0 + ra < J.N)
                            J.y[(int64_t)m * J.N + r0 + ra] =
                                ya[mp] + xg.slot(rg, parity, gq)[m];
                        if (r0 + ra + 8 < J.N)
                            J.y[(int64_t)m * J.N + r0 + ra + 8] =
                                yb[mp] + xg.slot(rg, parity, gq + 8)[m];
                    }
                }
                xg.get_end(rg, nunit, lane);
            }
#pragma unroll
            for (int mp = 0; mp < MP; ++mp) ya[mp] = yb[mp] = 0.0f;
            parity ^= 1;
            ++nunit;
        }
        if (nu >= u1) return true;
        k.u = nu;
        k.kc = nkc;
        k.jidx = nj;
        if (++k.sidx == S) {
            k.sidx = 0;
            k.sph ^= 1;
        }
        return false;
    };
    while (!step(sz0, sz2) && !step(sz1, sz0) && !step(sz2, sz1)) {
    }
}

// ---- runtime (RTN) consumer --------------------------------------------------
template <int MT>
__device__ __forceinline__ void consume_runtime(
    const StreamParams &P, const StreamJob *jobs, uint8_t *smem, uint8_t *xslots,
    uint64_t *full, uint64_t *empty, uint64_t *xfull, uint64_t *xempty,
    volatile int *abort_flag, const Xchg &xg, int u0, int u1, int cw, int lane) {
    const int S = P.stages;
    const int rg = cw & 7, w = cw >> 3;
    const int r16 = lane >> 1, part = lane & 1;       // row in group, 32-k half
    const int rr = 16 * rg + r16;
    const float L = (float)((1 << P.bits) - 1);
    const bool pass = P.bits == 16;
    XCursor xc;
    int u = u0, kc = 0, jidx = find_job(jobs, P.count, u);
    int sidx = 0;              // stage slot and its mbarrier phase
    uint32_t sph = 0;
    auto load_sz = [&](const StreamJob &J, int uu, int kk, float &sv, float &zv) {
        const int row = (uu - J.unit_begin) * kRows + rr;
        const int k0 = kk * 128 + w * 64;
        sv = 1.0f;
        zv = 0.0f;
        if (!pass && row < J.N && k0 < J.K) {
            const int64_t gi = (int64_t)row * (J.K / J.group) + k0 / J.group;
            sv = __ldg(reinterpret_cast<const float *>(J.s) + gi);
            zv = __ldg(reinterpret_cast<const float *>(J.z) + gi);
        }
    };
    float2 sz_a, sz_b = make_float2(1.0f, 0.0f);     // (scale, zero) ping-pong
    load_sz(jobs[jidx], u, 0, sz_a.x, sz_a.y);
    float yacc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) yacc[m] = 0.0f;
    int parity = 0;
    uint32_t nunit = 0;
    auto step = [&](const float2 use, float2 &fill) -> bool {
        const float s_cur = use.x, z_cur = use.y;
        const StreamJob &J = jobs[jidx];
        const int row = (u - J.unit_begin) * kRows + rr;
        if (kc == 0 && !x_enter(xc, J, u == u0, xslots, P.xslot_bytes, xfull,
                                xempty, abort_flag, lane))
            return true;
        const int kchunks = kchunks_of<false>(J.K);
        int nu = u, nkc = kc + 1, nj = jidx;
        if (nkc == kchunks) {
            nu = u + 1;
            nkc = 0;
            if (nu < u1) nj = next_job(jobs, P.count, jidx, nu);
        }
        if (nu < u1) load_sz(jobs[nj], nu, nkc, fill.x, fill.y);
        const int s = sidx;
        if (!mbar_wait(smem_u32(&full[s]), sph, abort_flag)) return true;
        const int k0 = kc * 128 + w * 64 + part * 32;     // this thread's 32 k
        float part_acc[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) part_acc[m] = 0.0f;
        if (row < J.N && k0 < J.K) {
            const int kp = kpad_of<false>(J.K);
            const uint8_t *box = smem + s * kStageBytes + w * kBoxBytes;
            const float inv = rcp_approx(s_cur);
            const float lo_c = -z_cur, hi_c = L - z_cur;
            const float thr = 0.5f - (fmaxf(fabsf(lo_c), fabsf(hi_c)) + 2.0f) *
                                         4.76837158203125e-07f;   // 2^-21
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
                const int u16 = part * 4 + c8;
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
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
#pragma unroll
        for (int m = 0; m < MT; ++m) yacc[m] = fmaf(part_acc[m], s_cur, yacc[m]);
        if (nkc == 0) {
#pragma unroll
            for (int m = 0; m < MT; ++m)
                yacc[m] += __shfl_xor_sync(0xffffffffu, yacc[m], 1);
            if (w == 1) {
                if (!xg.put_begin(rg, nunit, abort_flag)) return true;
                if (part == 0) {
#pragma unroll
                    for (int m = 0; m < MT; ++m) xg.slot(rg, parity, r16)[m] = yacc[m];
                }
                xg.put_end(rg, nunit, lane);
            } else {
                if (!xg.get_begin(rg, nunit, abort_flag)) return true;
                if (part == 0 && row < J.N) {
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        if (m >= P.M) break;
                        J.y[(int64_t)m * J.N + row] = yacc[m] + xg.slot(rg, parity, r16)[m];
                    }
                }
                xg.get_end(rg, nunit, lane);
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) yacc[m] = 0.0f;
            parity ^= 1;
            ++nunit;
        }
        if (nu >= u1) return true;
        u = nu;
        kc = nkc;
        jidx = nj;
        if (++sidx == S) {      // ring position of the next stage
            sidx = 0;
            sph ^= 1;
        }
        return false;
    };
    while (!step(sz_a, sz_b) && !step(sz_b, sz_a)) {
    }
}

template <bool PACKED, int MT>
__global__ void __launch_bounds__(kThreads, 1)
gemv_stream_kernel(const __grid_constant__ StreamParams P) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int S = P.stages;
    uint8_t *xslots = smem + S * kStageBytes;
    float *xchg = reinterpret_cast<float *>(xslots + 2 * P.xslot_bytes);
    uint64_t *bars = reinterpret_cast<uint64_t *>(xchg + 8 * 2 * 16 * kMaxM);
    uint64_t *full = bars, *empty = bars + S;
    uint64_t *xfull = bars + 2 * S, *xempty = xfull + 2;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(xempty + 2);
    uint64_t *xbars = bars + 2 * S + 8;                 // 8 row groups x 2 x {full, empty}
    StreamJob *jobs = reinterpret_cast<StreamJob *>(bars + 2 * S + 8 + 32);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u0 = P.cta_begin[blockIdx.x], u1 = P.cta_begin[blockIdx.x + 1];
    // The activations of this CTA's matrices go to L2 ahead of the weight
    // stream: queued behind the first ring fill they would hold up the start.
    if (warp >= 1 && u0 < u1) {
        const int jf = find_job(P.jobs, P.count, u0), jl = find_job(P.jobs, P.count, u1 - 1);
        for (int j = jf; j <= jl; ++j) {
            const StreamJob &J = P.jobs[j];
            if (j > jf && P.jobs[j - 1].x == J.x) continue;
            const int lines = (int)(((int64_t)P.M * J.K * 4 + 127) / 128);
            for (int l = 32 * (warp - 1) + lane; l < lines; l += 32 * kStagers)
                prefetch_l2(reinterpret_cast<const char *>(J.x) + (int64_t)l * 128);
        }
    }
    {
        const uint32_t *src = reinterpret_cast<const uint32_t *>(P.jobs);
        uint32_t *dst = reinterpret_cast<uint32_t *>(jobs);
        const int words = P.count * (int)(sizeof(StreamJob) / 4);
        for (int i = threadIdx.x; i < words; i += kThreads) dst[i] = src[i];
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), kConsumers);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&xfull[b]), 32);
            mbar_init(smem_u32(&xempty[b]), kConsumers);
        }
        for (int b = 0; b < 32; ++b) mbar_init(smem_u32(&xbars[b]), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp == 0) {
        // ---------------- loader ----------------
        const uint64_t policy = evict_first_policy();
        uint32_t g = 0, armed = 0;
        int jw = u0 < u1 ? find_job(jobs, P.count, u0) : 0;
        int pidx = 0;
        uint32_t pph = 0;
        bool ok = true;
        for (int u = u0; u < u1 && ok; ++u) {
            jw = next_job(jobs, P.count, jw, u);
            const int j = jw;
            const StreamJob &J = jobs[j];
            const int r0 = (u - J.unit_begin) * kRows;
            const int rbytes = row_bytes_of<PACKED>(J.K);
            const int kchunks = kchunks_of<PACKED>(J.K);
            if constexpr (PACKED) {
                // the unit's scales and zeros (one contiguous block each) go to
                // L2 with its weights; consumers read them a few stages later
                const int G = J.K >> 6;
                const int64_t b0 = (int64_t)r0 * G * 2;
                const int64_t b1 = (int64_t)min(r0 + kRows, J.N) * G * 2;
                const int lines = (int)((b1 - b0 + 127) >> 7) + 1;
                const char *sb = reinterpret_cast<const char *>(J.s) + (b0 & ~(int64_t)127);
                const char *zb = reinterpret_cast<const char *>(J.z) + (b0 & ~(int64_t)127);
                const int64_t limit = (int64_t)J.N * G * 2 - (b0 & ~(int64_t)127);
                for (int l = lane; l < lines; l += 32) {
                    if ((int64_t)l * 128 >= limit) break;
                    prefetch_l2(sb + (int64_t)l * 128);
                    prefetch_l2(zb + (int64_t)l * 128);
                }
            }
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
                    // meet zero activation digits (packed) or are skipped (runtime)
                    const int nbox = (rbytes - kc * kChunk) > 128 ? 2 : 1;
                    mbar_expect_tx(fb, (uint32_t)(nbox * kBoxBytes));
                    const uint32_t st = smem_u32(smem + s * kStageBytes);
                    for (int b = 0; b < nbox; ++b)
                        tma_load_2d(st + b * kBoxBytes, &P.wmap[j], kc * kChunk + b * 128, r0, fb,
                                    policy);
                }
                armed |= 1u << s;
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
        }
        __syncwarp();
    } else {
        // the first x slot, by every warp but the loader
        if (u0 < u1) {
            const StreamJob &J0 = jobs[find_job(jobs, P.count, u0)];
            stage_x<PACKED>(J0, P.M, xslots, warp - 1, kStagers, lane);
            named_bar(9, 32 * kStagers);
            if (warp == 1) mbar_arrive(smem_u32(&xfull[0]));
        }
        if (warp == 1) {
            // ---------------- activation stager ----------------
            const float *cur = nullptr;
            uint32_t e = 0;
            int js = u0 < u1 ? find_job(jobs, P.count, u0) : 0;
            for (int u = u0; u < u1 && !*abort_flag; ++u) {
                js = next_job(jobs, P.count, js, u);
                const StreamJob &J = jobs[js];
                if (u != u0 && J.x == cur) continue;
                cur = J.x;
                if (u == u0) {     // filled above
                    e = 1;
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
            const int cw = warp - 2;
            const Xchg xg{xchg, xbars};
            if (u0 < u1) {
                if constexpr (PACKED) {
                    if constexpr (MT == 1)
                        consume_packed_m1(P, jobs, smem, xslots, full, empty, xfull, xempty,
                                          abort_flag, xg, u0, u1, cw, lane);
                    else
                        consume_packed_mx<MT>(P, jobs, smem, xslots, full, empty, xfull,
                                              xempty, abort_flag, xg, u0, u1, cw, lane);
                } else {
                    consume_runtime<MT>(P, jobs, smem, xslots, full, empty, xfull, xempty,
                                        abort_flag, xg, u0, u1, cw, lane);
                }
            }
        }
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
constexpr int kXchgBytes = 8 * 2 * 16 * kMaxM * 4;
constexpr int kBarBytes = 512 + kMaxJobs * (int)sizeof(StreamJob);

template <bool PACKED, int MT>
bc_status launch_one(const StreamParams &P, int grid, int smem, cudaStream_t s) {
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
    gemv_stream_kernel<PACKED, MT><<<grid, kThreads, smem, s>>>(P);
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

}  // namespace

bool gemv_stream_supported(const GemvJob *jobs, int count, int M, bool packed,
                           int max_smem) {
    if (M < 1 || M > kMaxM || count < 1) return false;
    for (int i = 0; i < count; ++i)
        if (jobs[i].N >= (1 << 30) || jobs[i].K >= (1 << 24)) return false;
    const size_t xs = xslot_bytes_for(jobs, count, M, packed);
    const size_t fixed = 2 * xs + kXchgBytes + kBarBytes + 1024;
    if (fixed + 2 * (size_t)kStageBytes > (size_t)max_smem) return false;
    return tensor_map_encoder() != nullptr;
}

bc_status launch_gemv_stream(const GemvJob *jobs, int count, int M, int bits,
                             bool packed, cudaStream_t s) {
    DeviceInfo di;
    if (!device_info(&di)) return BC_ERR_CUDA;
    auto enc = tensor_map_encoder();
    if (!enc) return BC_ERR_CUDA;
    thread_local StreamParams *Pp = nullptr;
    if (!Pp) Pp = new StreamParams();
    StreamParams &P = *Pp;
    for (int b0 = 0; b0 < count; b0 += kMaxJobs) {
        const int n = std::min(kMaxJobs, count - b0);
        int units = 0;
        std::vector<double> jbytes(n);
        for (int i = 0; i < n; ++i) {
            const GemvJob &G0 = jobs[b0 + i];
            StreamJob &J = P.jobs[i];
            J.x = G0.x; J.s = G0.s; J.z = G0.z; J.y = G0.y;
            J.N = (int)G0.N; J.K = (int)G0.K; J.group = (int)G0.group;
            const int rbytes = packed ? J.K / 2 : J.K * 2;
            J.unit_begin = units;
            units += (J.N + kRows - 1) / kRows;
            if (!encode_weights(enc, &P.wmap[i], G0.w, J.N, rbytes)) return BC_ERR_CUDA;
            jbytes[i] = (double)J.N * rbytes;
        }
        const size_t xs = xslot_bytes_for(jobs + b0, n, M, packed);
        const int fixed = (int)(2 * xs) + kXchgBytes + kBarBytes + 1024;
        int stages = (di.max_smem_optin - fixed) / kStageBytes;
        stages = std::min(stages, 6);
        if (stages < 2) return BC_ERR_UNSUPPORTED;
        const int grid = std::max(1, std::min({units, di.sm_count, kMaxCtas}));
        // byte-balanced contiguous unit ranges
        double total = 0;
        for (int i = 0; i < n; ++i) total += jbytes[i];
        P.cta_begin[0] = 0;
        int j = 0;
        double before = 0;     // bytes of jobs < j
        for (int c = 1; c < grid; ++c) {
            const double target = total * c / grid;
            while (j < n - 1 && before + jbytes[j] <= target) before += jbytes[j++];
            const StreamJob &J = P.jobs[j];
            const double ub = (double)kRows * (packed ? J.K / 2 : J.K * 2);
            int lu = (int)((target - before) / ub + 0.5);
            const int nu = (J.N + kRows - 1) / kRows;
            lu = std::min(std::max(lu, 0), nu);
            P.cta_begin[c] = std::max(P.cta_begin[c - 1], J.unit_begin + lu);
        }
        P.cta_begin[grid] = units;
        P.count = n;
        P.total_units = units;
        P.M = M;
        P.bits = bits;
        P.xslot_bytes = (int)xs;
        P.stages = stages;
        const int smem = stages * kStageBytes + fixed;
        bc_status st;
        if (packed) {
            st = M <= 1 ? launch_one<true, 1>(P, grid, smem, s)
               : M <= 2 ? launch_one<true, 2>(P, grid, smem, s)
                        : launch_one<true, 4>(P, grid, smem, s);
        } else {
            const int mt = M <= 1 ? 1 : M <= 2 ? 2 : 4;
            st = mt == 1 ? launch_one<false, 1>(P, grid, smem, s)
               : mt == 2 ? launch_one<false, 2>(P, grid, smem, s)
                         : launch_one<false, 4>(P, grid, smem, s);
        }
        if (st != BC_OK) return st;
    }
    return BC_OK;
}

unsigned gemv_timeouts() {
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_gemv_timeouts, sizeof(v)) != cudaSuccess) return ~0u;
    return v;
}

}  // namespace bc
