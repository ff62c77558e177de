// bc_gemm_sm100.cu -- prefill GEMM on the 5th-generation tensor cores.
//
// y[m,n] = sum_k x[m,k] * w'[n,k] for M >= 64 prompt rows, bf16 x, packed
// int4 W with fp16 scale/zero per 64-block along K (Enargeia, "Four bits per
// weight": int4 weights unpacked on chip, never written back to memory;
// Enargeia's benchmark table: prefill at 128 and 2048 tokens; the tiled
// matmul ladder on the same page: tiling and register blocking decide
// matmul speed).
//
// Tile = 128 weight rows (the MMA's M, i.e. TMEM lanes) x BNX activation
// rows (the MMA's N) x 64 along K (one quantization block, one 128-byte
// swizzle atom row of bf16).  Per 64-block of K:
//   * one thread (warp 0) issues two TMA loads into a smem stage: the bf16
//     x tile (128B-swizzled, K-major) and the 128 x 32-byte packed codes;
//   * eight dequant warps turn the codes into bf16 w' = (q - z) * s in the
//     same 128B-swizzled K-major layout the MMA reads (exact q - z in bf16
//     arithmetic, one rounding for the scale), then fence the generic-proxy
//     writes for the tensor core;
//   * one thread (warp 1) issues four tcgen05.mma.kind::f16 (K = 16 each)
//     accumulating fp32 in TMEM, and tcgen05.commit frees the stage;
//   * four epilogue warps drain the finished accumulator (tcgen05.ld) and
//     store y with 128-byte coalesced rows, while the next tile accumulates
//     into the second TMEM buffer.
// The kernel is persistent (one CTA per SM, tiles strided over the grid)
// and spans every matrix of a grouped launch.  All waits are bounded: a
// wait that runs out records a timeout, the CTA stops, waits (bounded) for
// its own TMA copies in flight and frees its TMEM.
#include "bc_internal.cuh"
#include "bc_tc.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>
#include <vector>

namespace bc {

__device__ unsigned int g_gemm_timeouts = 0;

namespace {

constexpr int kBM = 128;                    // weight rows per tile
constexpr int kBK = 64;                     // K per stage (one quant block)
constexpr int kTmaWarp = 0, kMmaWarp = 1;
constexpr int kDqWarp0 = 2, kDqWarps = 8;   // warps 2..9
constexpr int kEpWarp0 = 10, kEpWarps = 4;  // warps 10..13
constexpr int kThreads = 32 * (kEpWarp0 + kEpWarps);
constexpr int kMaxJobs = 80;
constexpr long long kWaitCycles = 4000000000LL;   // ~2 s at 2 GHz

struct GemmJobDev {
    const __half *s;
    const __half *z;
    float *y;
    int N, K;
    int tile_begin;
    int xblocks;           // ceil(M / BNX)
};

struct __align__(64) GemmParams {
    CUtensorMap xmap[kMaxJobs];     // bf16 x [M][K], box {64, BNX}, SW128
    CUtensorMap cmap[kMaxJobs];     // u8 packed [N][K/2], box {32, 128}
    GemmJobDev jobs[kMaxJobs];
    int count, total_tiles, M;
};
static_assert(sizeof(GemmParams) <= 32000, "kernel parameter space");

template <int BNX> struct Cfg {
    static constexpr int kABytes = kBM * 128;          // 16 KB
    static constexpr int kBBytes = BNX * 128;
    static constexpr int kCBytes = kBM * 32;           // 4 KB
    static constexpr int kStageBytes = kABytes + kBBytes + kCBytes;
    static constexpr int kStages = BNX == 256 ? 4 : 6;
    static constexpr int kTmemCols = 2 * BNX;
    static constexpr int kBarBytes = 4096;     // barriers + job table copy
    static constexpr int kSmem = kStages * kStageBytes + kBarBytes + 1024;
    // instruction descriptor: D f32, A/B bf16, K-major both, N, M = 128
    static constexpr uint32_t kIdesc = tc::idesc_bf16(kBM, BNX);
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
// Bounded wait; false (and a recorded timeout, once per CTA) if it ran out
// or if another role of this CTA already gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          volatile int *abort_flag) {
    if (mbar_try(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > kWaitCycles) {
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
// the scale/zero of its weight row for each position.
struct SzCursor {
    int tile, kb, kblocks;
    const __half *srow, *zrow;
    const GemmJobDev *jobs;
    __device__ __forceinline__ void bind(const GemmParams &P, int r) {
        if (tile >= P.total_tiles) {
            srow = zrow = nullptr;
            kblocks = 1;
            return;
        }
        const GemmJobDev &J = jobs[find_job(jobs, P.count, tile)];
        const int nb = (tile - J.tile_begin) / J.xblocks;
        const int row = nb * kBM + r;
        kblocks = J.K / kBK;
        if (row < J.N) {
            srow = J.s + (int64_t)row * kblocks;
            zrow = J.z + (int64_t)row * kblocks;
        } else {
            srow = zrow = nullptr;
        }
    }
    __device__ __forceinline__ void init(const GemmParams &P, const GemmJobDev *sj,
                                         int first, int, int r) {
        jobs = sj;
        tile = first;
        kb = 0;
        bind(P, r);
    }
    __device__ __forceinline__ void advance(const GemmParams &P, int stride, int r) {
        if (++kb == kblocks) {
            kb = 0;
            tile += stride;
            bind(P, r);
        }
    }
    __device__ __forceinline__ void load(float &s, float &z) const {
        if (srow) {
            s = __half2float(__ldg(srow + kb));
            z = __half2float(__ldg(zrow + kb));
        } else {
            s = 0.0f;
            z = 0.0f;
        }
    }
};

template <int BNX>
__global__ void __launch_bounds__(kThreads, 1)
gemm_packed_kernel(const __grid_constant__ GemmParams P) {
    using C = Cfg<BNX>;
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
    const int K_tiles_dummy = 0;
    (void)K_tiles_dummy;

    if (warp == kTmaWarp) {
        if (lane == 0) {
            uint32_t g = 0;                       // k-block counter over tiles
            uint32_t armed = 0;                   // stages with a load issued
            for (int tile = blockIdx.x; tile < P.total_tiles && !*abort_flag;
                 tile += gridDim.x) {
                const int j = find_job(sjobs, P.count, tile);
                const GemmJobDev &J = sjobs[j];
                const int local = tile - J.tile_begin;
                const int nb = local / J.xblocks, xb = local % J.xblocks;
                const int kblocks = J.K / kBK;
                for (int kb = 0; kb < kblocks; ++kb, ++g) {
                    const int s = g % C::kStages;
                    const uint32_t ph = (g / C::kStages) & 1;
                    if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1, abort_flag)) break;
                    uint8_t *st = smem + s * C::kStageBytes;
                    const uint32_t fb = smem_u32(&full_tma[s]);
                    mbar_expect_tx(fb, C::kBBytes + C::kCBytes);
                    tma_load_2d(smem_u32(st + C::kABytes), &P.xmap[j], kb * kBK,
                                xb * BNX, fb);
                    tma_load_2d(smem_u32(st + C::kABytes + C::kBBytes), &P.cmap[j],
                                kb * (kBK / 2), nb * kBM, fb);
                    armed |= 1u << s;
                }
            }
            // drain: every load this thread issued has landed before exit
            // (on the normal path each stage was consumed, so these pass)
            for (uint32_t q = 0; q < (uint32_t)C::kStages; ++q) {
                if (!(armed & (1u << q))) continue;
                // the last use of stage q had index g_last = largest g' < g with
                // g' % kStages == q
                if (g == 0) break;
                uint32_t gl = (g - 1) - (((g - 1) % C::kStages + C::kStages - q) %
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
        for (int tile = blockIdx.x;
             tile < P.total_tiles && !__shfl_sync(0xffffffffu, (int)*abort_flag, 0);
             tile += gridDim.x, ++lt) {
            const int j = find_job(sjobs, P.count, tile);
            const int kblocks = sjobs[j].K / kBK;
            const int buf = lt & 1;
            const uint32_t aph = (lt >> 1) & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&acc_empty[buf]), aph ^ 1, abort_flag)))
                break;
            tc::fence_after();
            const uint32_t d_tmem = tmem_base + buf * BNX;
            bool ok = true;
            for (int kb = 0; kb < kblocks; ++kb, ++g) {
                const int s = g % C::kStages;
                const uint32_t ph = (g / C::kStages) & 1;
                bool w = mbar_wait(smem_u32(&full_tma[s]), ph, abort_flag);
                if (w) w = mbar_wait(smem_u32(&full_dq[s]), ph, abort_flag);
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
        SzCursor la;                        // look-ahead cursor
        la.init(P, sjobs, blockIdx.x, gridDim.x, r);
        float sq[kLook], zq[kLook];
#pragma unroll
        for (int i = 0; i < kLook; ++i) {
            la.load(sq[i], zq[i]);
            la.advance(P, gridDim.x, r);
        }
        int tile = blockIdx.x, kb = 0, kblocks = 1;
        bool valid = false;
        auto bind = [&]() {
            if (tile >= P.total_tiles) return;
            const GemmJobDev &J = sjobs[find_job(sjobs, P.count, tile)];
            const int nb = (tile - J.tile_begin) / J.xblocks;
            kblocks = J.K / kBK;
            valid = nb * kBM + r < J.N;
        };
        bind();
        uint32_t g = 0;
        bool ok = true;
        while (ok && tile < P.total_tiles && !*abort_flag) {
#pragma unroll
            for (int j = 0; j < kLook; ++j) {
                if (tile >= P.total_tiles) break;
                const float sf = sq[j], zf = zq[j];
                la.load(sq[j], zq[j]);             // refill slot j, kLook ahead
                la.advance(P, gridDim.x, r);
                const int s = g % C::kStages;
                const uint32_t ph = (g / C::kStages) & 1;
                if (!mbar_wait(smem_u32(&full_tma[s]), ph, abort_flag)) {
                    ok = false;
                    break;
                }
                uint8_t *st = smem + s * C::kStageBytes;
                const uint4 codes = *reinterpret_cast<const uint4 *>(
                    st + C::kABytes + C::kBBytes + r * 32 + h * 16);
                const uint32_t cw[4] = {codes.x, codes.y, codes.z, codes.w};
                uint8_t *arow = st + (r >> 3) * 1024 + (r & 7) * 128;
                if (!valid) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int chunk = h * 4 + i;
                        *reinterpret_cast<uint4 *>(arow + ((chunk ^ (r & 7)) << 4)) =
                            make_uint4(0, 0, 0, 0);
                    }
                } else if (fabsf(zf) <= 128.0f) {
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
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&full_dq[s]));
                ++g;
                if (++kb == kblocks) {
                    kb = 0;
                    tile += gridDim.x;
                    bind();
                }
            }
        }
    } else {
        // epilogue: warp quarter q reads TMEM lanes 32q..32q+31 (weight rows)
        const int q = warp & 3;
        int lt = 0;
        for (int tile = blockIdx.x; tile < P.total_tiles && !*abort_flag;
             tile += gridDim.x, ++lt) {
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
            for (int c = 0; c < BNX / 32; ++c) {
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
                  const uint8_t *w, int64_t N, int64_t K) {
    cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)N};
    cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    cuuint32_t box[2] = {(cuuint32_t)(kBK / 2), (cuuint32_t)kBM};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, (void *)w, dims, strides, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BNX>
bc_status launch_bnx(const GemmJob *jobs, int count, int64_t M, cudaStream_t s,
                     int sm_count) {
    using C = Cfg<BNX>;
    auto enc = get_encoder();
    if (!enc) return BC_ERR_CUDA;
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(gemm_packed_kernel<BNX>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        C::kSmem);
    });
    if (attr_err != cudaSuccess) return BC_ERR_CUDA;
    thread_local GemmParams *Pp = nullptr;
    if (!Pp) Pp = new GemmParams();
    GemmParams &P = *Pp;
    for (int b = 0; b < count; b += kMaxJobs) {
        const int n = std::min(kMaxJobs, count - b);
        int tiles = 0;
        const int xblocks = (int)((M + BNX - 1) / BNX);
        for (int i = 0; i < n; ++i) {
            const GemmJob &J = jobs[b + i];
            if (!encode_x(enc, &P.xmap[i], J.x, M, J.K, BNX) ||
                !encode_codes(enc, &P.cmap[i], J.w, J.N, J.K))
                return BC_ERR_CUDA;
            P.jobs[i] = GemmJobDev{J.s, J.z, J.y, (int)J.N, (int)J.K, tiles, xblocks};
            tiles += (int)((J.N + kBM - 1) / kBM) * xblocks;
        }
        P.count = n;
        P.total_tiles = tiles;
        P.M = (int)M;
        const int grid = std::max(1, std::min(tiles, sm_count));
        gemm_packed_kernel<BNX><<<grid, kThreads, C::kSmem, s>>>(P);
        bc_status st = cuda_status();
        if (st != BC_OK) return st;
    }
    return BC_OK;
}

}  // namespace

bc_status launch_gemm_packed(const GemmJob *jobs, int count, int64_t M,
                             cudaStream_t s) {
    DeviceInfo di;
    if (!device_info(&di)) return BC_ERR_CUDA;
    if (di.cc_major != 10) return BC_ERR_UNSUPPORTED;
    for (int i = 0; i < count; ++i) {
        const uintptr_t xa = reinterpret_cast<uintptr_t>(jobs[i].x);
        const uintptr_t wa = reinterpret_cast<uintptr_t>(jobs[i].w);
        if (xa % 16 || wa % 16) return BC_ERR_ALIGNMENT;
        if (M >= (int64_t)1 << 31) return BC_ERR_UNSUPPORTED;
    }
    if (M <= 128) return launch_bnx<128>(jobs, count, M, s, di.sm_count);
    return launch_bnx<256>(jobs, count, M, s, di.sm_count);
}

unsigned gemm_timeouts() {
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_gemm_timeouts, sizeof(v)) != cudaSuccess) return ~0u;
    return v;
}

}  // namespace bc
