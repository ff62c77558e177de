// bc_gemv_stream.cu -- streaming fused dequant GEMV for decode (M <= 4).
//
// Decode "reads every weight in the model to write one word" (Enargeia):
// the matmul is one pass over HBM.  The kernel is a TMA pipeline that keeps
// ~160 KB per SM in flight, with the arithmetic kept well under the SM's
// issue budget so that the stream, not the ALUs, sets the pace.
//
// One CTA per SM, persistent over a byte-balanced contiguous range of
// "units" (128 weight rows of one matrix) that spans every matrix of a
// grouped launch (Enargeia, "One decode step": hundreds of passes per token
// are one launch here).  Warp roles:
//   warp 0      TMA producer: each stage is a 256-byte column chunk of the
//               unit's 128 rows, loaded as two 2D boxes of 128 rows x 128
//               bytes with the 128-byte swizzle (ring of up to 6 stages,
//               full/empty mbarriers);
//   warp 1      activation stager: the x of each new matrix goes into one of
//               two smem slots -- fp32 rows (runtime mode), or fp16 hi + lo
//               pieces (x = hi + lo to 2^-22) in mma.sync fragment order
//               plus per-64-group sums of the even-k and odd-k pieces
//               (packed mode);
//   warps 2-17  consumers: warp (window w, row group g) handles 16 rows and
//               the w-th 128-byte window of every stage; the two windows'
//               partial row sums meet in smem at the end of each unit.
//
// Packed int4 (Enargeia, "Four bits per weight": codes unpacked in
// registers, never written back).  Two shifts and four LOP3 turn 8 nibbles
// into exact fp16 pairs (256 + q) for even k and (16 + q) for odd k, which
// feed mma.sync.m16n8k16 A fragments straight from registers.  B holds the
// x pieces of the window's four 64-groups block-diagonally (8 columns = 4
// groups x {hi, lo}), so every group's dot product lands in its own column:
//     sum_k x_k (q_k - z) = C_hi + C_lo - (256 + z) X_even - (16 + z) X_odd
// then one multiply by the group's scale.  About one instruction per weight.
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
constexpr int kThreads = 32 * (2 + kConsumers);
constexpr int kMaxJobs = 168;
constexpr int kMaxCtas = 160;
constexpr int kMaxM = 4;
constexpr int kPiecePad = 32;           // bytes between the hi and lo pieces
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
// Bytes of one x row in a slot.  Packed: hi[kp] f16, pad, lo[kp] f16,
// sums[kp/64] x {even, odd} f32.  Runtime: x[kp] f32.
template <bool PACKED> __host__ __device__ __forceinline__ int xrow_bytes(int K) {
    const int kp = kpad_of<PACKED>(K);
    return PACKED ? 4 * kp + kPiecePad + (kp / 64) * 8 : 4 * kp;
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
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map,
                                            int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void named_bar(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
// Byte offset of 16-byte unit `u` of row `r` inside a 128B-swizzled box.
__device__ __forceinline__ int sw_off(int r, int u) {
    return r * 128 + ((u ^ (r & 7)) << 4);
}
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                         uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// (t & mask) | bias: fp16 pairs built from nibbles already at mantissa bits.
template <uint32_t MASK, uint32_t BIAS>
__device__ __forceinline__ uint32_t lop_or(uint32_t t) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(t), "n"(MASK), "n"(BIAS));
    return r;
}
// 8 packed codes (nibble j = k_j) -> fp16 pairs R_j = (k_j, k_{j+4}):
// even j as 256 + q (mantissa bits 2-5), odd j as 16 + q (bits 6-9).
__device__ __forceinline__ void unpack8(uint32_t w, uint32_t (&R)[4]) {
    const uint32_t t0 = w << 2, t1 = w >> 6;
    R[0] = lop_or<0x003C003Cu, 0x5C005C00u>(t0);
    R[1] = lop_or<0x03C003C0u, 0x4C004C00u>(t0);
    R[2] = lop_or<0x003C003Cu, 0x5C005C00u>(t1);
    R[3] = lop_or<0x03C003C0u, 0x4C004C00u>(t1);
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
// partials to the window-0 warp through smem (double-buffered by unit).
struct Xchg {
    float *base;       // [8 row groups][2 parity][16 rows][kMaxM]
    __device__ __forceinline__ float *slot(int rg, int parity, int r16) const {
        return base + ((rg * 2 + parity) * 16 + r16) * kMaxM;
    }
};

// ---- packed consumer -----------------------------------------------------------
// Scale / zero of one group for this lane's rows ra, rb.
struct SzP {
    float sa, za, sb, zb;
};
__device__ __forceinline__ void load_sz_packed(const StreamJob &J, int ra, int rb,
                                               int grp, SzP &o) {
    const __half *S16 = reinterpret_cast<const __half *>(J.s);
    const __half *Z16 = reinterpret_cast<const __half *>(J.z);
    const int G = J.K >> 6;
    const bool gv = grp < G;
    const bool va = gv && ra < J.N, vb = gv && rb < J.N;
    const int64_t ia = (int64_t)ra * G + grp, ib = (int64_t)rb * G + grp;
    o.sa = va ? __half2float(__ldg(S16 + ia)) : 0.f;
    o.za = va ? __half2float(__ldg(Z16 + ia)) : 0.f;
    o.sb = vb ? __half2float(__ldg(S16 + ib)) : 0.f;
    o.zb = vb ? __half2float(__ldg(Z16 + ib)) : 0.f;
}

template <int MT>
__device__ __forceinline__ void consume_packed(
    const StreamParams &P, const StreamJob *jobs, uint8_t *smem, uint8_t *xslots,
    uint64_t *full, uint64_t *empty, uint64_t *xfull, uint64_t *xempty,
    volatile int *abort_flag, const Xchg &xg, int u0, int u1, int cw, int lane) {
    const int S = P.stages;
    const int rg = cw & 7, w = cw >> 3;               // row group, window
    const int gq = lane >> 2, t = lane & 3;          // A/C fragment role
    // mma row gq <-> unit row 16*rg + perm(gq): rows 4 apart share a 16-byte
    // load phase, so their swizzled units land in different banks
    const int ra_l = 16 * rg + ((gq >> 1) | ((gq & 1) << 2));
    const int rb_l = ra_l + 8;
    const int piece = (lane >> 2) & 1, gsb = lane >> 3;    // B role: column lane>>2
    const bool act0 = gsb == (t >> 1), act1 = gsb == 2 + (t >> 1);
    XCursor xc;
    int u = u0, kc = 0, jidx = find_job(jobs, P.count, u);
    int sidx = 0;              // stage slot and its mbarrier phase
    uint32_t sph = 0;
    SzP cur, nxt;
    {
        const StreamJob &J = jobs[jidx];
        const int r0 = (u - J.unit_begin) * kRows;
        load_sz_packed(J, r0 + ra_l, r0 + rb_l, w * 4 + t, cur);
    }
    float yacc[MT][2];
#pragma unroll
    for (int m = 0; m < MT; ++m) yacc[m][0] = yacc[m][1] = 0.0f;
    int parity = 0;
    // One stage.  `use` holds this stage's scale/zero (loaded a stage ago);
    // `fill` receives the next stage's.  The two sets swap roles every call,
    // so no register copy ever waits on an outstanding load.  Returns true
    // when this warp is done.
    auto step = [&](const SzP &use, SzP &fill) -> bool {
        const StreamJob &J = jobs[jidx];
        const int r0 = (u - J.unit_begin) * kRows;
        if (kc == 0 && !x_enter(xc, J, u == u0, xslots, P.xslot_bytes, xfull,
                                xempty, abort_flag, lane))
            return true;
        const int kchunks = kchunks_of<true>(J.K);
        int nu = u, nkc = kc + 1, nj = jidx;
        if (nkc == kchunks) {
            nu = u + 1;
            nkc = 0;
            if (nu < u1) nj = next_job(jobs, P.count, jidx, nu);
        }
        if (nu < u1) {          // next stage's scale / zero, fetched early
            const StreamJob &Jn = jobs[nj];
            const int nr0 = (nu - Jn.unit_begin) * kRows;
            load_sz_packed(Jn, nr0 + ra_l, nr0 + rb_l, nkc * 8 + w * 4 + t, fill);
        }
        const int s = sidx;
        if (!mbar_wait(smem_u32(&full[s]), sph, abort_flag)) return true;
        const int kp = kpad_of<true>(J.K);
        const int mb = xrow_bytes<true>(J.K);
        const uint8_t *box = smem + s * kStageBytes + w * kBoxBytes;
        // independent accumulator chains hide the MMA latency (fewer when
        // several x rows already give independent work)
        constexpr int NCH = MT == 1 ? 4 : 2;
        float acc[MT][NCH][4];
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
            for (int a = 0; a < NCH; ++a)
                acc[m][a][0] = acc[m][a][1] = acc[m][a][2] = acc[m][a][3] = 0.0f;
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
            const uint4 qa = *reinterpret_cast<const uint4 *>(box + sw_off(ra_l, ch * 4 + t));
            const uint4 qb = *reinterpret_cast<const uint4 *>(box + sw_off(rb_l, ch * 4 + t));
            const bool act = ch == 0 ? act0 : act1;
            const uint32_t wa[4] = {qa.x, qa.y, qa.z, qa.w};
            const uint32_t wb[4] = {qb.x, qb.y, qb.z, qb.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t A[4], B[4];
                unpack8(wa[i], A);
                unpack8(wb[i], B);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    // x pieces at k = kc*512 + w*256 + ch*128 + 32*t + 8*i
                    const uint8_t *bp = xc.xs + m * mb + piece * (2 * kp + kPiecePad) +
                                        (kc * 512 + w * 256 + ch * 128 + 32 * t + 8 * i) * 2;
                    uint4 bv = make_uint4(0u, 0u, 0u, 0u);
                    if (act) bv = *reinterpret_cast<const uint4 *>(bp);
                    constexpr int base = 0;
                    const int c0 = NCH == 4 ? ch * 2 : base, c1 = c0 + 1;
                    mma16816(acc[m][c0], A[0], B[0], A[1], B[1], bv.x, bv.y);
                    mma16816(acc[m][c1], A[2], B[2], A[3], B[3], bv.z, bv.w);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[s]));   // stage consumed
        const int grp = kc * 8 + w * 4 + t;
        if (grp < (J.K >> 6)) {
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                float c[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    c[q] = acc[m][0][q] + acc[m][1][q];
                    if constexpr (NCH == 4) c[q] += acc[m][2][q] + acc[m][3][q];
                }
                const float2 xsum = reinterpret_cast<const float2 *>(
                    xc.xs + m * mb + 4 * kp + kPiecePad)[grp];
                const float v0 = (c[0] + c[1]) - (256.0f + use.za) * xsum.x -
                                 (16.0f + use.za) * xsum.y;
                const float v1 = (c[2] + c[3]) - (256.0f + use.zb) * xsum.x -
                                 (16.0f + use.zb) * xsum.y;
                yacc[m][0] = fmaf(use.sa, v0, yacc[m][0]);
                yacc[m][1] = fmaf(use.sb, v1, yacc[m][1]);
            }
        }
        if (nkc == 0) {       // unit done: four group lanes, then two windows
#pragma unroll
            for (int m = 0; m < MT; ++m)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float v = yacc[m][h];
                    v += __shfl_xor_sync(0xffffffffu, v, 1);
                    v += __shfl_xor_sync(0xffffffffu, v, 2);
                    yacc[m][h] = v;
                }
            if (w == 1 && t == 0) {
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    xg.slot(rg, parity, 2 * gq)[m] = yacc[m][0];
                    xg.slot(rg, parity, 2 * gq + 1)[m] = yacc[m][1];
                }
            }
            named_bar(1 + rg, 64);
            if (w == 0 && t == 0) {
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m >= P.M) break;
                    const float ya = yacc[m][0] + xg.slot(rg, parity, 2 * gq)[m];
                    const float yb = yacc[m][1] + xg.slot(rg, parity, 2 * gq + 1)[m];
                    if (r0 + ra_l < J.N) J.y[(int64_t)m * J.N + r0 + ra_l] = ya;
                    if (r0 + rb_l < J.N) J.y[(int64_t)m * J.N + r0 + rb_l] = yb;
                }
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) yacc[m][0] = yacc[m][1] = 0.0f;
            parity ^= 1;
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
    while (!step(cur, nxt) && !step(nxt, cur)) {
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
                const uint4 raw =
                    *reinterpret_cast<const uint4 *>(box + sw_off(rr, part * 4 + c8));
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
            if (w == 1 && part == 0) {
#pragma unroll
                for (int m = 0; m < MT; ++m) xg.slot(rg, parity, r16)[m] = yacc[m];
            }
            named_bar(1 + rg, 64);
            if (w == 0 && part == 0 && row < J.N) {
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m >= P.M) break;
                    J.y[(int64_t)m * J.N + row] = yacc[m] + xg.slot(rg, parity, r16)[m];
                }
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) yacc[m] = 0.0f;
            parity ^= 1;
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
    StreamJob *jobs = reinterpret_cast<StreamJob *>(bars + 2 * S + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u0 = P.cta_begin[blockIdx.x], u1 = P.cta_begin[blockIdx.x + 1];
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
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp == 0) {
        // ---------------- weight producer (one thread) ----------------
        uint32_t g = 0, armed = 0;
        int jw = u0 < u1 ? find_job(jobs, P.count, u0) : 0;
        int pidx = 0;
        uint32_t pph = 0;
        for (int u = u0; u < u1 && lane == 0 && !*abort_flag; ++u) {
            jw = next_job(jobs, P.count, jw, u);
            const int j = jw;
            const StreamJob &J = jobs[j];
            const int r0 = (u - J.unit_begin) * kRows;
            const int rbytes = row_bytes_of<PACKED>(J.K);
            const int kchunks = kchunks_of<PACKED>(J.K);
            bool ok = true;
            for (int kc = 0; kc < kchunks; ++kc, ++g) {
                const int s = pidx;
                if (!mbar_wait(smem_u32(&empty[s]), pph ^ 1, abort_flag)) {
                    ok = false;
                    break;
                }
                if (++pidx == S) {
                    pidx = 0;
                    pph ^= 1;
                }
                // a window wholly past the row end is not loaded: its weights
                // meet zero activations (packed) or are skipped (runtime)
                const int nbox = (rbytes - kc * kChunk) > 128 ? 2 : 1;
                const uint32_t fb = smem_u32(&full[s]);
                mbar_expect_tx(fb, (uint32_t)(nbox * kBoxBytes));
                const uint32_t st = smem_u32(smem + s * kStageBytes);
                for (int b = 0; b < nbox; ++b)
                    tma_load_2d(st + b * kBoxBytes, &P.wmap[j], kc * kChunk + b * 128, r0, fb);
                armed |= 1u << s;
            }
            if (!ok) break;
        }
        // drain: loads in flight land before the CTA exits
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
    } else if (warp == 1) {
        // ---------------- activation stager ----------------
        const float *cur = nullptr;
        uint32_t e = 0;
        int js = u0 < u1 ? find_job(jobs, P.count, u0) : 0;
        for (int u = u0; u < u1 && !*abort_flag; ++u) {
            js = next_job(jobs, P.count, js, u);
            const StreamJob &J = jobs[js];
            if (u != u0 && J.x == cur) continue;
            cur = J.x;
            const int slot = e & 1;
            if (!mbar_wait(smem_u32(&xempty[slot]), ((e >> 1) & 1) ^ 1, abort_flag)) break;
            uint8_t *xs = xslots + slot * P.xslot_bytes;
            const int K = J.K;
            const int kp = kpad_of<PACKED>(K);
            const int mb = xrow_bytes<PACKED>(K);
            for (int m = 0; m < P.M; ++m) {
                const float *xr = J.x + (int64_t)m * K;
                uint8_t *xm = xs + m * mb;
                if constexpr (PACKED) {
                    __half *hi = reinterpret_cast<__half *>(xm);
                    __half *lo = reinterpret_cast<__half *>(xm + 2 * kp + kPiecePad);
                    float2 *sums = reinterpret_cast<float2 *>(xm + 4 * kp + kPiecePad);
                    // 8-blocks; lanes 8q..8q+7 hold one 64-group.  Loads are
                    // issued kBatch blocks ahead so the stager pays one memory
                    // round trip per batch, not per block.
                    constexpr int kBatch = 4;
                    for (int b00 = 0; b00 < kp / 8; b00 += 32 * kBatch) {
                      float4 pre[kBatch][2];
#pragma unroll
                      for (int q = 0; q < kBatch; ++q) {
                          const int b = b00 + 32 * q + lane;
                          pre[q][0] = pre[q][1] = make_float4(0.f, 0.f, 0.f, 0.f);
                          if (8 * b < K) {
                              pre[q][0] = __ldg(reinterpret_cast<const float4 *>(xr + 8 * b));
                              pre[q][1] = __ldg(reinterpret_cast<const float4 *>(xr + 8 * b + 4));
                          }
                      }
#pragma unroll
                      for (int q = 0; q < kBatch; ++q) {
                        const int b = b00 + 32 * q + lane;
                        if (b00 + 32 * q >= kp / 8) break;
                        float v[8];
                        v[0] = pre[q][0].x; v[1] = pre[q][0].y; v[2] = pre[q][0].z; v[3] = pre[q][0].w;
                        v[4] = pre[q][1].x; v[5] = pre[q][1].y; v[6] = pre[q][1].z; v[7] = pre[q][1].w;
                        __half h[8], l[8];
                        float se = 0.0f, so = 0.0f;
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            h[i] = __float2half_rn(v[i]);
                            const float hf = __half2float(h[i]);
                            l[i] = __float2half_rn(v[i] - hf);
                            const float xt = hf + __half2float(l[i]);
                            if (i & 1) so += xt; else se += xt;
                        }
                        // fragment order of an 8-block: k0 k4 k1 k5 k2 k6 k3 k7
                        const __half2 H0 = __halves2half2(h[0], h[4]), H1 = __halves2half2(h[1], h[5]);
                        const __half2 H2 = __halves2half2(h[2], h[6]), H3 = __halves2half2(h[3], h[7]);
                        const __half2 L0 = __halves2half2(l[0], l[4]), L1 = __halves2half2(l[1], l[5]);
                        const __half2 L2 = __halves2half2(l[2], l[6]), L3 = __halves2half2(l[3], l[7]);
                        uint4 hv, lv;
                        hv.x = *reinterpret_cast<const uint32_t *>(&H0);
                        hv.y = *reinterpret_cast<const uint32_t *>(&H1);
                        hv.z = *reinterpret_cast<const uint32_t *>(&H2);
                        hv.w = *reinterpret_cast<const uint32_t *>(&H3);
                        lv.x = *reinterpret_cast<const uint32_t *>(&L0);
                        lv.y = *reinterpret_cast<const uint32_t *>(&L1);
                        lv.z = *reinterpret_cast<const uint32_t *>(&L2);
                        lv.w = *reinterpret_cast<const uint32_t *>(&L3);
                        *reinterpret_cast<uint4 *>(hi + 8 * b) = hv;
                        *reinterpret_cast<uint4 *>(lo + 8 * b) = lv;
#pragma unroll
                        for (int off = 1; off < 8; off <<= 1) {
                            se += __shfl_xor_sync(0xffffffffu, se, off);
                            so += __shfl_xor_sync(0xffffffffu, so, off);
                        }
                        if ((lane & 7) == 0) sums[b / 8] = make_float2(se, so);
                      }
                    }
                } else {
                    float *xf = reinterpret_cast<float *>(xm);
                    constexpr int kBatch = 8;
                    for (int k0 = 4 * lane; k0 < kp; k0 += 128 * kBatch) {
                        float4 v[kBatch];
#pragma unroll
                        for (int q = 0; q < kBatch; ++q) {
                            const int k = k0 + 128 * q;
                            v[q] = make_float4(0.f, 0.f, 0.f, 0.f);
                            if (k < K) v[q] = __ldg(reinterpret_cast<const float4 *>(xr + k));
                        }
#pragma unroll
                        for (int q = 0; q < kBatch; ++q) {
                            const int k = k0 + 128 * q;
                            if (k < kp) *reinterpret_cast<float4 *>(xf + k) = v[q];
                        }
                    }
                }
            }
            mbar_arrive(smem_u32(&xfull[slot]));     // every lane, after its writes
            ++e;
        }
    } else {
        // ---------------- consumers ----------------
        const int cw = warp - 2;
        const Xchg xg{xchg};
        if (u0 < u1) {
            if constexpr (PACKED)
                consume_packed<MT>(P, jobs, smem, xslots, full, empty, xfull, xempty,
                                   abort_flag, xg, u0, u1, cw, lane);
            else
                consume_runtime<MT>(P, jobs, smem, xslots, full, empty, xfull, xempty,
                                    abort_flag, xg, u0, u1, cw, lane);
        }
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
constexpr int kXchgBytes = 8 * 2 * 16 * kMaxM * 4;
constexpr int kBarBytes = 256 + kMaxJobs * (int)sizeof(StreamJob);

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

size_t xslot_bytes_for(const GemvJob *jobs, int count, int M, bool packed) {
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
        const int mt = M <= 1 ? 1 : M <= 2 ? 2 : 4;
        bc_status st;
        if (packed) {
            st = mt == 1 ? launch_one<true, 1>(P, grid, smem, s)
               : mt == 2 ? launch_one<true, 2>(P, grid, smem, s)
                         : launch_one<true, 4>(P, grid, smem, s);
        } else {
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
