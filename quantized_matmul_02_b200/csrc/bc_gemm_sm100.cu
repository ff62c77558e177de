// bc_gemm_sm100.cu -- prefill GEMM on the 5th-generation tensor cores.
//
// y[m,n] = sum_k x[m,k] * w'[n,k] for M >= 64 prompt rows, bf16 x, and
// weights in either form of the method:
//   * packed int4 with fp16 scale/zero per 64-block along K (Enargeia,
//     "Four bits per weight": int4 weights unpacked on chip, never written
//     back; its benchmark table measures prefill at 128 and 2048 tokens);
//   * fp16 weights re-quantized as they are read, group-wise (64) or per
//     channel, at 2..8 bits or passed through at 16 (BITCRUSH BC-06, "Under
//     the hood": matmul_q computes the RTN codes inline at any lever
//     position, so a prompt can be prefilled at any precision).
// Enargeia's tiled-matmul ladder: tiling and register blocking decide
// matmul speed; here the tiles feed tcgen05 from shared memory and TMEM.
//
// Tile = 128 weight rows (the MMA's M, i.e. TMEM lanes) x BNX activation
// rows (the MMA's N) x 64 along K (one quantization block, one 128-byte
// swizzle atom row of bf16).  Per 64-block of K:
//   * one thread (warp 0) issues the TMA loads of a stage: the bf16 x tile
//     (128B-swizzled, K-major) and the weights -- 128 x 32 bytes of packed
//     codes, or the 128 x 64 fp16 weights themselves, landed 128B-swizzled
//     in the stage's A tile;
//   * eight dequant warps form bf16 w' = (q - z) * s in the same
//     128B-swizzled K-major layout the MMA reads (packed: exact q - z in
//     bf16 arithmetic and one rounding for the scale; runtime: the exact RTN
//     code of each fp16 weight, then one rounding of (q - z) s, written over
//     the weight it came from), then fence the generic-proxy writes for the
//     tensor core;
//   * one thread (warp 1) issues four tcgen05.mma.kind::f16 (K = 16 each)
//     accumulating fp32 in TMEM, and tcgen05.commit frees the stage;
//   * eight epilogue warps (two per TMEM lane quarter, each half of the
//     columns) drain the finished accumulator (tcgen05.ld) and store y with
//     128-byte coalesced rows, while the next tile accumulates into the
//     second TMEM buffer.
// The kernel is persistent (one CTA per SM) and spans every matrix of a
// grouped launch.  Each CTA owns a contiguous range of tiles chosen on the
// host so that the ranges cost about the same (a tile costs its K/64 stages
// plus its epilogue), instead of a round-robin stride that leaves SMs idle
// when matrices of very different K share a launch.  All waits are bounded:
// a wait that runs out records a timeout, the CTA stops, waits (bounded) for
// its own copies and MMAs in flight and frees its TMEM.
#include "bc_internal.cuh"
#include "bc_rtn.cuh"
#include "bc_tc.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>
#include <vector>

namespace bc {

__device__ unsigned int g_gemm_timeouts = 0;
// Limit of the pipeline waits, in clock64 cycles (bc_set_wait_limit);
// the drains after an abort keep the fixed ~2 s limit.
__device__ long long g_gemm_wait_limit = 4000000000LL;

namespace {

constexpr int kBM = 128;                    // weight rows per tile
constexpr int kBK = 64;                     // K per stage (one quant block)
constexpr int kTmaWarp = 0, kMmaWarp = 1;
constexpr int kDqWarp0 = 2, kDqWarps = 8;   // warps 2..9
constexpr int kEpWarp0 = 10, kEpWarps = 8;  // warps 10..17 (two per TMEM lane quarter)
constexpr int kThreads = 32 * (kEpWarp0 + kEpWarps);
constexpr int kMaxJobs = 80;
constexpr int kMaxCtas = 160;
constexpr long long kWaitCycles = 4000000000LL;   // ~2 s at 2 GHz

// Weight forms.
constexpr int kPacked = 0;    // int4 codes, fp16 scale/zero per 64-block
constexpr int kRuntime = 1;   // fp16 W, RTN inline (fp32 scale/zero or ranges)

struct GemmJobDev {
    const void *s;         // packed: fp16 [N][K/64]; runtime: fp32 [N][K/g] or ranges
    const void *z;         // packed: fp16; runtime: fp32 (unused with ranges)
    float *y;
    int N, K, group;       // group: 64, or K (runtime per channel)
    int tile_begin;
    int xblocks;           // ceil(M / BNX)
};

struct __align__(64) GemmParams {
    CUtensorMap xmap[kMaxJobs];     // bf16 x [M][K], box {64, BNX}, SW128
    CUtensorMap wmap[kMaxJobs];     // packed u8 [N][K/2] box {32, 128}; fp16 W [N][K] box {64, 128} SW128
    GemmJobDev jobs[kMaxJobs];
    int cta_begin[kMaxCtas + 1];    // tile range of each CTA
    int count, total_tiles, M;
    int bits;                       // runtime: 2..8 or 16 (passthrough)
    int range;                      // runtime: s holds per-group ranges
};
static_assert(sizeof(GemmParams) <= 32000, "kernel parameter space");

template <int BNX, int WF> struct Cfg {
    static constexpr int kABytes = kBM * 128;          // 16 KB (runtime: W lands here)
    static constexpr int kBBytes = BNX * 128;
    static constexpr int kCBytes = WF == kPacked ? kBM * 32 : 0;   // 4 KB of codes
    static constexpr int kStageBytes = kABytes + kBBytes + kCBytes;  // multiple of 1024
    static constexpr int kBarBytes = 4096;     // barriers + job table copy
    static constexpr int kStages =
        std::min(6, (227 * 1024 - kBarBytes - 1024) / kStageBytes);
    static constexpr int kTmemCols = 2 * BNX;
    static constexpr int kSmem = kStages * kStageBytes + kBarBytes + 1024;
    // instruction descriptor: D f32, A/B bf16, K-major both, N, M = 128
    static constexpr uint32_t kIdesc = tc::idesc_bf16(kBM, BNX);
    static_assert(kStageBytes % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
};

// ---- small PTX wrappers ----------------------------------------------------
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
// The same test, letting the thread sleep (up to a hint of 20 us) until the
// phase completes: a waiting warp then takes no issue slots from the warps
// doing the work.
__device__ __forceinline__ bool mbar_try_sleep(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(bar), "r"(parity), "r"(20000u) : "memory");
    return ok != 0;
}
// Bounded wait; false (and a recorded timeout, once per CTA) if it ran out
// or if another role of this CTA already gave up.  SLEEP lets the thread
// sleep between tests (the dequant and epilogue warps, which wait long and
// would otherwise take issue slots); the producer and the MMA issuer spin,
// since a wake-up delay there lengthens every stage.
template <bool SLEEP = true>
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          volatile int *abort_flag) {
    if (mbar_try(bar, parity)) return true;
    const long long t0 = clock64();
    const long long limit = *(volatile long long *)&g_gemm_wait_limit;
    while (true) {
        if (SLEEP ? mbar_try_sleep(bar, parity) : mbar_try(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > limit) {
            if (atomicExch((int *)abort_flag, 1) == 0)
                atomicAdd(&g_gemm_timeouts, 1u);
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
// Bring one weight box of a later tile into L2 (no shared memory, no
// barrier): the TMA of that stage then meets L2 instead of HBM latency.
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap *map, int x, int y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y) : "memory");
}
__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ uint32_t lop3_nib(uint32_t w) {
    // ((w & 0x000F000F) | 0x43004300): two bf16 values 128 + nibble
    uint32_t r;
    asm("lop3.b32 %0, %1, 0x000F000F, 0x43004300, 0xEA;" : "=r"(r) : "r"(w));
    return r;
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}
__device__ __forceinline__ uint32_t bf2_as_u32(__nv_bfloat162 v) {
    return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ __nv_bfloat162 u32_as_bf2(uint32_t v) {
    return *reinterpret_cast<__nv_bfloat162 *>(&v);
}

// 8 packed codes (k0..k7 of one 32-bit word, low nibble = even k) -> 8 bf16
// w' = (q - z) * s as 4 bf16x2 words in k order.
__device__ __forceinline__ uint4 dequant8(uint32_t w, __nv_bfloat162 zb,
                                          __nv_bfloat162 sb) {
    const uint32_t r0 = lop3_nib(w);          // (k0, k4)
    const uint32_t r1 = lop3_nib(w >> 4);     // (k1, k5)
    const uint32_t r2 = lop3_nib(w >> 8);     // (k2, k6)
    const uint32_t r3 = lop3_nib(w >> 12);    // (k3, k7)
    const uint32_t p[4] = {prmt(r0, r1, 0x5410), prmt(r2, r3, 0x5410),
                           prmt(r0, r1, 0x7632), prmt(r2, r3, 0x7632)};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)   // (128 + q) - (128 + z) is exact; one rounding
        o[i] = bf2_as_u32(__hmul2(__hsub2(u32_as_bf2(p[i]), zb), sb));
    return make_uint4(o[0], o[1], o[2], o[3]);
}
// Same in fp32 for blocks whose zero lies outside [-128, 128].
__device__ __noinline__ uint4 dequant8_wide(uint32_t w, float z, float s) {
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float a = ((float)((w >> (8 * i)) & 0xF) - z) * s;
        const float b = ((float)((w >> (8 * i + 4)) & 0xF) - z) * s;
        o[i] = bf2_as_u32(__floats2bfloat162_rn(a, b));
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}
// Runtime mode: 8 fp16 weights -> 8 bf16 w' = (q - z) s (or w itself at 16
// bits), k order kept.
__device__ __forceinline__ uint4 requant8(uint4 raw, float s, float z, float L, bool pass) {
    uint32_t o[4];
    if (pass) {
        const __half2 *h = reinterpret_cast<const __half2 *>(&raw);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __half22float2(h[i]);
            o[i] = bf2_as_u32(__floats2bfloat162_rn(f.x, f.y));
        }
    } else {
        float c[8];
        rtn_centered8(raw, s, z, L, c);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            o[i] = bf2_as_u32(__floats2bfloat162_rn(c[2 * i] * s, c[2 * i + 1] * s));
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// Job descriptors are read from a shared-memory copy (sjobs): dynamically
// indexed reads of the parameter block miss the constant cache.
__device__ __forceinline__ int find_job(const GemmJobDev *jobs, int count, int tile) {
    int lo = 0, hi = count - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (jobs[mid].tile_begin <= tile) lo = mid; else hi = mid - 1;
    }
    return lo;
}

constexpr int kLook = 4;     // scale/zero look-ahead, in 64-blocks of K

// Walks the (tile, 64-block) sequence a dequant thread consumes and loads
// the scale and zero of its weight row for each position.
template <int WF> struct SzCursor {
    int tile, t_end, kb, kblocks, group;
    const void *srow;
    const void *zrow;
    const GemmJobDev *jobs;
    __device__ __forceinline__ void bind(const GemmParams &P, int r) {
        if (tile >= t_end) {
            srow = zrow = nullptr;
            kblocks = 1;
            return;
        }
        const GemmJobDev &J = jobs[find_job(jobs, P.count, tile)];
        const int nb = (tile - J.tile_begin) / J.xblocks;
        const int row = nb * kBM + r;
        kblocks = J.K / kBK;
        group = J.group;
        const int64_t G = J.K / J.group;
        if (row < J.N) {
            const size_t es = (WF == kPacked) ? 2 : 4;
            srow = static_cast<const uint8_t *>(J.s) + (int64_t)row * G * es;
            zrow = J.z ? static_cast<const uint8_t *>(J.z) + (int64_t)row * G * es : nullptr;
        } else {
            srow = zrow = nullptr;
        }
    }
    __device__ __forceinline__ void init(const GemmParams &P, const GemmJobDev *sj, int first,
                                         int last, int r) {
        jobs = sj;
        tile = first;
        t_end = last;
        kb = 0;
        bind(P, r);
    }
    __device__ __forceinline__ void advance(const GemmParams &P, int r) {
        if (++kb == kblocks) {
            kb = 0;
            ++tile;
            bind(P, r);
        }
    }
    // (s, z) of the current position
    __device__ __forceinline__ void load(const GemmParams &P, float &s, float &z) const {
        s = 0.0f;
        z = 0.0f;
        if (!srow) return;
        if constexpr (WF == kPacked) {
            s = __half2float(__ldg(static_cast<const __half *>(srow) + kb));
            z = __half2float(__ldg(static_cast<const __half *>(zrow) + kb));
        } else {
            if (P.bits == 16) return;
            const int gi = (kb * kBK) / group;
            if (P.range) {
                const float2 rg =
                    range_of_word(__ldg(static_cast<const uint32_t *>(srow) + gi));
                const float2 sz = rtn_params_from_range(rg.x, rg.y, P.bits);
                s = sz.x;
                z = sz.y;
            } else {
                s = __ldg(static_cast<const float *>(srow) + gi);
                z = __ldg(static_cast<const float *>(zrow) + gi);
            }
        }
    }
};

template <int BNX, int WF>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ GemmParams P) {
    using C = Cfg<BNX, WF>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *bar_area = smem + C::kStages * C::kStageBytes;
    uint64_t *full_tma = reinterpret_cast<uint64_t *>(bar_area);
    uint64_t *full_dq = full_tma + C::kStages;
    uint64_t *empty = full_dq + C::kStages;
    uint64_t *acc_full = empty + C::kStages;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *mma_done = acc_empty + 2;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(mma_done + 1);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1) + 1;
    GemmJobDev *sjobs = reinterpret_cast<GemmJobDev *>(mma_done + 2);
    {
        const uint32_t *src = reinterpret_cast<const uint32_t *>(P.jobs);
        uint32_t *dst = reinterpret_cast<uint32_t *>(sjobs);
        const int words = P.count * (int)(sizeof(GemmJobDev) / 4);
        for (int i = threadIdx.x; i < words; i += kThreads) dst[i] = src[i];
    }

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t_begin = P.cta_begin[blockIdx.x], t_end = P.cta_begin[blockIdx.x + 1];

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(smem_u32(&full_tma[s]), 1);
            mbar_init(smem_u32(&full_dq[s]), kDqWarps);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&acc_full[b]), 1);
            mbar_init(smem_u32(&acc_empty[b]), kEpWarps);
        }
        mbar_init(smem_u32(mma_done), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kMmaWarp) {
        tc::alloc(smem_u32(tmem_slot), C::kTmemCols);
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == kTmaWarp) {
        if (lane == 0) {
            uint32_t g = 0;                       // k-block counter over tiles
            uint32_t armed = 0;                   // stages with a load issued
            for (int tile = t_begin; tile < t_end && !*abort_flag; ++tile) {
                const int j = find_job(sjobs, P.count, tile);
                const GemmJobDev &J = sjobs[j];
                const int local = tile - J.tile_begin;
                const int nb = local / J.xblocks, xb = local % J.xblocks;
                const int kblocks = J.K / kBK;
                if (tile + 1 < t_end) {
                    // the next tile's weights (and their scales/zeros) to L2
                    // while this one streams, unless it reuses these rows
                    const int j2 = find_job(sjobs, P.count, tile + 1);
                    const GemmJobDev &J2 = sjobs[j2];
                    const int nb2 = (tile + 1 - J2.tile_begin) / J2.xblocks;
                    if (j2 != j || nb2 != nb) {
                        const int kb2 = J2.K / kBK;
                        for (int q = 0; q < kb2; ++q)
                            tma_prefetch_2d(&P.wmap[j2], WF == kPacked ? q * (kBK / 2) : q * kBK,
                                            nb2 * kBM);
                        const int64_t G2 = J2.K / J2.group;
                        const int rows = min(kBM, J2.N - nb2 * kBM);
                        const int64_t es = WF == kPacked ? 2 : 4;
                        const int64_t bytes = rows * G2 * es;
                        const char *sb = static_cast<const char *>(J2.s) + (int64_t)nb2 * kBM * G2 * es;
                        const char *zb = J2.z ? static_cast<const char *>(J2.z) +
                                                    (int64_t)nb2 * kBM * G2 * es
                                              : nullptr;
                        for (int64_t o = 0; o < bytes; o += 128) {
                            if (P.bits != 16 || WF == kPacked) {
                                prefetch_l2(sb + o);
                                if (zb) prefetch_l2(zb + o);
                            }
                        }
                    }
                }
                for (int kb = 0; kb < kblocks; ++kb, ++g) {
                    const int s = g % C::kStages;
                    const uint32_t ph = (g / C::kStages) & 1;
                    if (!mbar_wait<false>(smem_u32(&empty[s]), ph ^ 1, abort_flag)) break;
                    uint8_t *st = smem + s * C::kStageBytes;
                    const uint32_t fb = smem_u32(&full_tma[s]);
                    if constexpr (WF == kPacked) {
                        mbar_expect_tx(fb, C::kBBytes + C::kCBytes);
                        tma_load_2d(smem_u32(st + C::kABytes + C::kBBytes), &P.wmap[j],
                                    kb * (kBK / 2), nb * kBM, fb);
                    } else {
                        mbar_expect_tx(fb, C::kBBytes + C::kABytes);
                        tma_load_2d(smem_u32(st), &P.wmap[j], kb * kBK, nb * kBM, fb);
                    }
                    tma_load_2d(smem_u32(st + C::kABytes), &P.xmap[j], kb * kBK, xb * BNX, fb);
                    armed |= 1u << s;
                }
            }
            // drain: every load this thread issued has landed before exit
            // (on the normal path each stage was consumed, so these pass)
            for (uint32_t q = 0; q < (uint32_t)C::kStages && g > 0; ++q) {
                if (!(armed & (1u << q))) continue;
                // the last use of stage q had index g_last = largest g' < g with
                // g' % kStages == q
                const uint32_t gl = (g - 1) - (((g - 1) % C::kStages + C::kStages - q) %
                                               C::kStages);
                const long long t0 = clock64();
                while (!mbar_try(smem_u32(&full_tma[q]), (gl / C::kStages) & 1) &&
                       clock64() - t0 < kWaitCycles) {
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // The whole warp walks the tiles and waits; one elected lane issues a
        // stage's four MMAs and commits.  Descriptors are formed once and
        // advanced by constant offsets (16-byte units of the start address):
        // an MMA issued from a lone diverged lane with descriptors rebuilt per
        // instruction costs several times the tensor core's own time.
        const uint64_t adesc0 = tc::sw128_desc(smem_u32(smem));
        const uint64_t bdesc0 = tc::sw128_desc(smem_u32(smem + C::kABytes));
        uint32_t g = 0;
        int lt = 0;
        for (int tile = t_begin;
             tile < t_end && !__shfl_sync(0xffffffffu, (int)*abort_flag, 0); ++tile, ++lt) {
            const int j = find_job(sjobs, P.count, tile);
            const int kblocks = sjobs[j].K / kBK;
            const int buf = lt & 1;
            const uint32_t aph = (lt >> 1) & 1;
            if (!__all_sync(0xffffffffu,
                            mbar_wait<false>(smem_u32(&acc_empty[buf]), aph ^ 1, abort_flag)))
                break;
            tc::fence_after();
            const uint32_t d_tmem = tmem_base + buf * BNX;
            bool ok = true;
            for (int kb = 0; kb < kblocks; ++kb, ++g) {
                const int s = g % C::kStages;
                const uint32_t ph = (g / C::kStages) & 1;
                bool w = mbar_wait<false>(smem_u32(&full_tma[s]), ph, abort_flag);
                if (w) w = mbar_wait<false>(smem_u32(&full_dq[s]), ph, abort_flag);
                if (!__all_sync(0xffffffffu, w)) {
                    ok = false;
                    break;
                }
                tc::fence_after();
                const uint64_t so = (uint64_t)((s * C::kStageBytes) >> 4);
                if (tc::elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        tc::mma_bf16_ss(d_tmem, adesc0 + so + 2 * kk, bdesc0 + so + 2 * kk,
                                        C::kIdesc, (kb > 0 || kk > 0) ? 1u : 0u);
                    tc::commit(smem_u32(&empty[s]));        // stage reusable
                }
                __syncwarp();
            }
            if (!ok) break;
            if (tc::elect_one()) tc::commit(smem_u32(&acc_full[buf]));   // tile accumulated
            __syncwarp();
        }
        // every MMA issued has finished before TMEM is freed
        if (tc::elect_one()) tc::commit(smem_u32(mma_done));
        __syncwarp();
        if (lane == 0) {
            const long long t0 = clock64();
            while (!mbar_try(smem_u32(mma_done), 0) && clock64() - t0 < kWaitCycles) {
            }
        }
        __syncwarp();
    } else if (warp < kDqWarp0 + kDqWarps) {
        // dequant: thread -> (row r, half h) of the 128 x 64 weight tile.
        // Scale/zero come from global memory.  They are fetched kLook blocks
        // ahead into a window of kLook register slots indexed at compile
        // time (slot j serves blocks g with g % kLook == j), so no register
        // copy waits on a load that is still in flight.
        const int t = threadIdx.x - 32 * kDqWarp0;
        const int r = t & (kBM - 1), h = t >> 7;
        const float L = (float)((1 << (P.bits & 15)) - 1);
        const bool pass = WF == kRuntime && P.bits == 16;
        SzCursor<WF> la;                    // look-ahead cursor
        la.init(P, sjobs, t_begin, t_end, r);
        float sq[kLook], zq[kLook];
#pragma unroll
        for (int i = 0; i < kLook; ++i) {
            la.load(P, sq[i], zq[i]);
            la.advance(P, r);
        }
        int tile = t_begin, kb = 0, kblocks = 1;
        bool valid = false;
        auto bind = [&]() {
            if (tile >= t_end) return;
            const GemmJobDev &J = sjobs[find_job(sjobs, P.count, tile)];
            const int nb = (tile - J.tile_begin) / J.xblocks;
            kblocks = J.K / kBK;
            valid = nb * kBM + r < J.N;
        };
        bind();
        uint32_t g = 0;
        bool ok = true;
        while (ok && tile < t_end && !*abort_flag) {
#pragma unroll
            for (int j = 0; j < kLook; ++j) {
                if (tile >= t_end) break;
                const float sf = sq[j], zf = zq[j];
                la.load(P, sq[j], zq[j]);          // refill slot j, kLook ahead
                la.advance(P, r);
                const int s = g % C::kStages;
                const uint32_t ph = (g / C::kStages) & 1;
                if (!mbar_wait(smem_u32(&full_tma[s]), ph, abort_flag)) {
                    ok = false;
                    break;
                }
                uint8_t *st = smem + s * C::kStageBytes;
                uint8_t *arow = st + (r >> 3) * 1024 + (r & 7) * 128;
                if (!valid) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int chunk = h * 4 + i;
                        *reinterpret_cast<uint4 *>(arow + ((chunk ^ (r & 7)) << 4)) =
                            make_uint4(0, 0, 0, 0);
                    }
                } else if constexpr (WF == kRuntime) {
                    // the 8 fp16 of each chunk are replaced by their 8 bf16 w'
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        uint4 *p = reinterpret_cast<uint4 *>(arow + (((h * 4 + i) ^ (r & 7)) << 4));
                        *p = requant8(*p, sf, zf, L, pass);
                    }
                } else {
                    const uint4 codes = *reinterpret_cast<const uint4 *>(
                        st + C::kABytes + C::kBBytes + r * 32 + h * 16);
                    const uint32_t cw[4] = {codes.x, codes.y, codes.z, codes.w};
                    if (fabsf(zf) <= 128.0f) {
                        const __nv_bfloat16 zb1 = __float2bfloat16_rn(128.0f + zf);
                        const __nv_bfloat16 sb1 = __float2bfloat16_rn(sf);
                        const __nv_bfloat162 zb = __halves2bfloat162(zb1, zb1);
                        const __nv_bfloat162 sb = __halves2bfloat162(sb1, sb1);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int chunk = h * 4 + i;
                            *reinterpret_cast<uint4 *>(arow + ((chunk ^ (r & 7)) << 4)) =
                                dequant8(cw[i], zb, sb);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int chunk = h * 4 + i;
                            *reinterpret_cast<uint4 *>(arow + ((chunk ^ (r & 7)) << 4)) =
                                dequant8_wide(cw[i], zf, sf);
                        }
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&full_dq[s]));
                ++g;
                if (++kb == kblocks) {
                    kb = 0;
                    ++tile;
                    bind();
                }
            }
        }
    } else {
        // epilogue: warp quarter q reads TMEM lanes 32q..32q+31 (weight rows),
        // half hh of the accumulator's columns (x rows)
        const int q = warp & 3, hh = (warp - kEpWarp0) >> 2;
        int lt = 0;
        for (int tile = t_begin; tile < t_end && !*abort_flag; ++tile, ++lt) {
            const int j = find_job(sjobs, P.count, tile);
            const GemmJobDev &J = sjobs[j];
            const int local = tile - J.tile_begin;
            const int nb = local / J.xblocks, xb = local % J.xblocks;
            const int buf = lt & 1;
            const uint32_t aph = (lt >> 1) & 1;
            if (!mbar_wait(smem_u32(&acc_full[buf]), aph, abort_flag)) break;
            tc::fence_after();
            const int n = nb * kBM + 32 * q + lane;
            const int m0 = xb * BNX;
#pragma unroll 1
            for (int c = hh * (BNX / 64); c < (hh + 1) * (BNX / 64); ++c) {
                uint32_t v[32];
                tc::ld32(tmem_base + ((uint32_t)(32 * q) << 16) + buf * BNX + c * 32, v);
                if (n < J.N) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int m = m0 + c * 32 + i;
                        if (m < P.M) J.y[(int64_t)m * J.N + n] = __uint_as_float(v[i]);
                    }
                }
            }
            tc::fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&acc_empty[buf]));
        }
    }

    tc::fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc::fence_after();
        tc::dealloc(tmem_base, C::kTmemCols);
    }
}

// ---- host side ---------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 get_encoder() {
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

bool encode_x(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap *m,
              const __nv_bfloat16 *x, int64_t M, int64_t K, int bnx) {
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)bnx};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (void *)x, dims, strides,
               box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_codes(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap *m,
                  const void *w, int64_t N, int64_t K) {
    cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)N};
    cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    cuuint32_t box[2] = {(cuuint32_t)(kBK / 2), (cuuint32_t)kBM};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(w), dims, strides,
               box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp16 W [N][K], box 64 x 128 rows, 128B swizzle (the A tile's layout)
bool encode_w16(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap *m, const void *w,
                int64_t N, int64_t K) {
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)N};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)kBM};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(w), dims, strides,
               box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Contiguous tile ranges per CTA that minimise the costliest range (binary
// search on the bound, greedy fill).  A tile costs its K/64 stages plus a
// fixed share for its epilogue.
void partition_tiles(GemmParams &P, const std::vector<double> &tcost, int grid) {
    const int n = (int)tcost.size();
    double total = 0, tmax = 0;
    for (double c : tcost) {
        total += c;
        tmax = std::max(tmax, c);
    }
    auto fill = [&](double T, bool out) -> int {
        int ctas = 1;
        double cur = 0;
        if (out) P.cta_begin[0] = 0;
        for (int i = 0; i < n; ++i) {
            if (cur > 0 && cur + tcost[i] > T) {
                if (out && ctas < grid) P.cta_begin[ctas] = i;
                ++ctas;
                cur = 0;
            }
            cur += tcost[i];
        }
        return ctas;
    };
    double lo = std::max(tmax, total / grid), hi = total + tmax;
    for (int it = 0; it < 60 && hi - lo > 0.5; ++it) {
        const double mid = 0.5 * (lo + hi);
        if (fill(mid, false) <= grid) hi = mid; else lo = mid;
    }
    const int used = std::min(fill(hi, true), grid);
    for (int c = used; c <= grid; ++c) P.cta_begin[c] = n;
}

template <int BNX, int WF>
bc_status launch_cfg(const GemmJob *jobs, int count, int64_t M, int bits, bool range,
                     cudaStream_t s, int sm_count) {
    using C = Cfg<BNX, WF>;
    auto enc = get_encoder();
    if (!enc) return BC_ERR_CUDA;
    static std::mutex mu;
    static int attr_set[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return BC_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!attr_set[dev]) {
            if (cudaFuncSetAttribute(gemm_kernel<BNX, WF>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     C::kSmem) != cudaSuccess)
                return BC_ERR_CUDA;
            attr_set[dev] = 1;
        }
    }
    thread_local GemmParams *Pp = nullptr;
    if (!Pp) Pp = new GemmParams();
    GemmParams &P = *Pp;
    std::vector<double> tcost;
    for (int b = 0; b < count; b += kMaxJobs) {
        const int n = std::min(kMaxJobs, count - b);
        int tiles = 0;
        const int xblocks = (int)((M + BNX - 1) / BNX);
        tcost.clear();
        for (int i = 0; i < n; ++i) {
            const GemmJob &J = jobs[b + i];
            if (!encode_x(enc, &P.xmap[i], J.x, M, J.K, BNX)) return BC_ERR_CUDA;
            const bool ok = WF == kPacked ? encode_codes(enc, &P.wmap[i], J.w, J.N, J.K)
                                          : encode_w16(enc, &P.wmap[i], J.w, J.N, J.K);
            if (!ok) return BC_ERR_CUDA;
            P.jobs[i] = GemmJobDev{J.s, J.z, J.y, (int)J.N, (int)J.K, (int)J.group, tiles,
                                   xblocks};
            const int nt = (int)((J.N + kBM - 1) / kBM) * xblocks;
            tiles += nt;
            // cost in stages: K/64 of MMA plus the epilogue (BNX/32 loads of
            // 32 columns and their stores), about two stages' worth
            tcost.insert(tcost.end(), nt, (double)(J.K / kBK) + 2.0 * BNX / 128.0);
        }
        P.count = n;
        P.total_tiles = tiles;
        P.M = (int)M;
        P.bits = bits;
        P.range = range ? 1 : 0;
        const int grid = std::max(1, std::min({tiles, sm_count, kMaxCtas}));
        partition_tiles(P, tcost, grid);
        gemm_kernel<BNX, WF><<<grid, kThreads, C::kSmem, s>>>(P);
        bc_status st = cuda_status();
        if (st != BC_OK) return st;
    }
    return BC_OK;
}

}  // namespace

bc_status launch_gemm(const GemmJob *jobs, int count, int64_t M, bool packed, int bits,
                      bool range, cudaStream_t s) {
    DeviceInfo di;
    if (!device_info(&di)) return BC_ERR_CUDA;
    if (di.cc_major != 10) return BC_ERR_UNSUPPORTED;
    for (int i = 0; i < count; ++i) {
        const uintptr_t xa = reinterpret_cast<uintptr_t>(jobs[i].x);
        const uintptr_t wa = reinterpret_cast<uintptr_t>(jobs[i].w);
        if (xa % 16 || wa % 16) return BC_ERR_ALIGNMENT;
        if (M >= (int64_t)1 << 31) return BC_ERR_UNSUPPORTED;
    }
    if (packed)
        return M <= 128 ? launch_cfg<128, kPacked>(jobs, count, M, bits, false, s, di.sm_count)
                        : launch_cfg<256, kPacked>(jobs, count, M, bits, false, s, di.sm_count);
    return M <= 128 ? launch_cfg<128, kRuntime>(jobs, count, M, bits, range, s, di.sm_count)
                    : launch_cfg<256, kRuntime>(jobs, count, M, bits, range, s, di.sm_count);
}

bc_status gemm_set_wait_limit(long long cycles) {
    if (cudaMemcpyToSymbol(g_gemm_wait_limit, &cycles, sizeof(cycles)) != cudaSuccess)
        return BC_ERR_CUDA;
    return BC_OK;
}

unsigned gemm_timeouts() {
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_gemm_timeouts, sizeof(v)) != cudaSuccess) return ~0u;
    return v;
}

}  // namespace bc
