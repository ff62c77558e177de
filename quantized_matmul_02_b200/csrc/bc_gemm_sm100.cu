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
// Two SMs (a cluster of two CTAs) share one tile of 256 weight rows x BNX
// activation rows: one tcgen05.mma.cta_group::2 (M = 256, N = BNX, K = 16)
// reads the 128 dequantized weight rows of each CTA (A) and the BNX/2
// activation rows each CTA loaded (B), and accumulates fp32 into the TMEM
// of both.  Each SM therefore loads half the activation tile that a
// one-SM tile of the same shape would: on 128 x 256 one-SM tiles the
// activation traffic from L2 set the pace (each 64-wide K step waited
// about 3400 cycles for its loads), not the tensor cores.
//
// Per CTA, per 64-block of K (one quantization block):
//   * a code producer (warp 0) loads the CTA's weights into a ring of
//     their own (they are read once, by the dequant warps): packed codes
//     four blocks at a time (128 rows of 128 bytes: whole L2 lines, where
//     one block's 32 bytes per row made 32-byte requests), or the 128 x 64
//     fp16 weights of one block;
//   * an activation producer (warp 2) loads the CTA's BNX/2 rows of bf16 x
//     (128B-swizzled, K-major) into the activation ring, which the MMA
//     frees;
//   * sixteen dequant warps form bf16 w' = (q - z) * s into one of the A
//     buffers (six for packed codes, four for the runtime form) in the
//     128B-swizzled K-major layout the MMA reads (packed: two groups of
//     eight warps on alternate blocks, exact q - z in bf16 arithmetic and
//     one rounding for the scale; runtime: one group of sixteen, the exact
//     RTN code of each fp16 weight, then one rounding of (q - z) s), fence
//     the generic-proxy writes for the tensor core and arrive on the first
//     CTA's "A ready" barrier (a cluster address);
//   * the first CTA's MMA warp waits for both CTAs' A buffers and its own
//     activation stage (the second CTA's dequant warps wait for theirs
//     before they arrive), issues four MMAs and commits to the "free"
//     barriers of both CTAs at once (commit multicast);
//   * eight epilogue warps per CTA drain the finished accumulator
//     (tcgen05.ld) and store y with coalesced rows while the next tile
//     accumulates into the second TMEM buffer.
// The kernel is persistent (one cluster per SM pair) and spans every matrix
// of a grouped launch; the pairs walk one tile list side by side (see
// pair_tile), so that the tiles in flight share their activation block.
// All waits are bounded: a wait that runs out records a timeout, the CTA
// stops, waits (bounded) for its own copies and MMAs in flight, meets its
// partner at the cluster barrier and frees its TMEM.  No load uses cluster
// multicast: every CTA loads its own tiles.
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

constexpr int kBM = 128;                    // weight rows per CTA (TMEM lanes)
constexpr int kPairRows = 2 * kBM;          // weight rows per tile (the MMA's M)
constexpr int kBK = 64;                     // K per stage (one quant block)
constexpr int kCodeWarp = 0, kMmaWarp = 1, kXWarp = 2;
constexpr int kDqWarp0 = 3, kDqWarps = 16;  // warps 3..18
constexpr int kEpWarp0 = 19, kEpWarps = 8;  // warps 19..26 (two per TMEM lane quarter)
constexpr int kThreads = 32 * (kEpWarp0 + kEpWarps);
constexpr int kMaxJobs = 80;
constexpr int kMaxPairs = 80;
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
    int nblocks;           // ceil(N / 256): weight blocks (fastest in the tile order)
};

struct __align__(64) GemmParams {
    CUtensorMap xmap[kMaxJobs];     // bf16 x [M][K], box {64, BNX/2}, SW128
    CUtensorMap wmap[kMaxJobs];     // packed u8 [N][K/2] box {128, 128}; fp16 W [N][K] box {64, 128}; SW128
    GemmJobDev jobs[kMaxJobs];
    int count, total_tiles, M;
    int pairs;                      // CTA pairs launched
    int ranges;                     // 1: pair p takes tiles [pair_begin[p], pair_begin[p+1])
    int pair_begin[kMaxPairs + 1];
    int bits;                       // runtime: 2..8 or 16 (passthrough)
    int range;                      // runtime: s holds per-group ranges
};
static_assert(sizeof(GemmParams) <= 32000, "kernel parameter space");

template <int BNX, int WF> struct Cfg {
    static constexpr int kXHalf = BNX / 2;                       // x rows per CTA
    static constexpr int kXBytes = kXHalf * 128;                 // 16 or 8 KB
    // One weight box covers kGroup 64-blocks of K: packed codes of four
    // blocks are 128-byte rows (whole L2 lines; one 32-byte piece per block
    // would be a 32-byte request per row), fp16 weights one block.
    static constexpr int kGroup = WF == kPacked ? 4 : 1;
    static constexpr int kDqGroups = WF == kPacked ? 2 : 1;     // dequant warp groups
    static constexpr int kWRow = WF == kPacked ? 32 * kGroup : 128;   // bytes per row
    static constexpr int kWBytes = kBM * kWRow;                   // 16 KB
    static constexpr int kABytes = kBM * 128;                    // 16 KB
    static constexpr int kAStages = WF == kPacked ? 6 : 4;
    // even: each dequant group sees every other phase of an x (and A)
    // barrier, and the parity test is sound only if the ring depth keeps a
    // slot's stages in one group
    static constexpr int kXStages = BNX == 256 ? 4 : (WF == kPacked ? 6 : 8);
    static constexpr int kWStages = WF == kPacked ? (BNX == 256 ? 3 : 4) : 5;
    static constexpr int kAOff = 0;
    static constexpr int kXOff = kAOff + kAStages * kABytes;
    static constexpr int kWOff = kXOff + kXStages * kXBytes;
    static constexpr int kBarOff = kWOff + kWStages * kWBytes;
    static constexpr int kBarBytes = 5120;     // barriers + job table copy
    static constexpr int kSmem = kBarOff + kBarBytes + 1024;
    static constexpr int kTmemCols = 2 * BNX;  // two accumulators of BNX columns
    // instruction descriptor: D f32, A/B bf16, K-major both, M = 256, N = BNX
    static constexpr uint32_t kIdesc = tc::idesc_bf16(kPairRows, BNX);
    static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
    static_assert(kXStages % 2 == 0 && kAStages % 2 == 0, "rings of even depth");
    static_assert(kXBytes % 1024 == 0 && kWBytes % 1024 == 0 && kABytes % 1024 == 0,
                  "rings keep the 1024-byte swizzle alignment");
};

// ---- small PTX wrappers ----------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_id() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
// The address of the same shared-memory location in the pair's first CTA.
__device__ __forceinline__ uint32_t in_leader(uint32_t local) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(r) : "r"(local));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// Arrive on a barrier of the pair (cluster address).  Default semantics
// (release at CTA scope): the data it announces is this CTA's own shared
// memory, already fenced for the tensor core (fence.proxy.async), which the
// MMA reads on this CTA's SM; a cluster-scope release would also wait for
// this thread's outstanding global loads (the scale/zero look-ahead).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cbar) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cbar) : "memory");
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
// How a role waits.  kSpin polls without pause (the MMA issuer: a late
// wake-up lengthens every stage).  kSleep lets the thread sleep with a
// suspend hint until the phase completes (waits on this CTA's own loads).
// kBackoff polls with a short nanosleep between tests: the producers and
// the epilogue, which wait long on barriers that the partner CTA may
// complete (a thread sleeping with a hint there wakes thousands of cycles
// late) and which, spinning, take issue slots from the dequant warps that
// share their scheduler.
constexpr int kSpin = 0, kSleep = 1, kBackoff = 2;

// Bounded wait; false (and a recorded timeout, once per CTA) if it ran out
// or if another role of this CTA already gave up.
template <int MODE = kSleep>
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          volatile int *abort_flag) {
    if (mbar_try(bar, parity)) return true;
    const long long t0 = clock64();
    const long long limit = *(volatile long long *)&g_gemm_wait_limit;
    while (true) {
        if (MODE == kSleep ? mbar_try_sleep(bar, parity) : mbar_try(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > limit) {
            if (atomicExch((int *)abort_flag, 1) == 0)
                atomicAdd(&g_gemm_timeouts, 1u);
            return false;
        }
        if (MODE == kBackoff) __nanosleep(128);
    }
}
// Drain wait of the exit paths: fixed limit, no abort test.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
    const long long t0 = clock64();
    while (!mbar_try(bar, parity) && clock64() - t0 < kWaitCycles) {
    }
}
// tcgen05 forms of the pair (cta_group::2).
__device__ __forceinline__ void mma_pair(uint32_t d_tmem, uint64_t a, uint64_t b,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(accumulate) : "memory");
}
// Arrive once on `bar` (same offset) in both CTAs of the pair when every
// MMA issued so far has completed.
__device__ __forceinline__ void commit_pair(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;"
        ::"r"(bar), "h"((uint16_t)0x3) : "memory");
}
// Arrive once on this CTA's `bar` when every MMA issued so far has completed.
__device__ __forceinline__ void commit_local(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];"
        ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t slot_smem, uint32_t cols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(slot_smem), "r"(cols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t base, uint32_t cols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;"
                 ::"r"(base), "r"(cols) : "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map,
                                            int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
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

// The tiles of a launch form one list: matrices by decreasing K, within a
// matrix x block by x block, and within an x block its 256-row weight
// blocks.  Pair p takes the list in rounds of `pairs` tiles, forward in even
// rounds and backward in odd ones (tile i * pairs + p, or + pairs - 1 - p):
// the pairs run through the list side by side, so at any time they work on
// neighbouring tiles, which share one x block (read from DRAM once, then
// from L2 by every pair), and the snake order evens out the extra cost of
// the long-K tiles dealt first.  (Contiguous per-pair ranges put every pair
// on a different matrix: at M = 2048 their x blocks did not fit in L2 and
// were re-read from DRAM, 4.8 GB of reads per 24-layer step against 0.9 GB
// of inputs.)
// With one x block per matrix (M <= BNX) nothing is shared between tiles of
// a matrix, and pair p instead takes a contiguous range of the list chosen
// on the host so that the ranges cost about the same (a round-robin deal of
// 76-block and 14-block tiles left a fifth of the time idle at M = 128).
// Returns total_tiles past the pair's last tile.
__device__ __forceinline__ int pair_tile(const GemmParams &P, int pair, int i) {
    if (P.ranges) {
        const int t = P.pair_begin[pair] + i;
        return t < P.pair_begin[pair + 1] ? t : P.total_tiles;
    }
    return min(i * P.pairs + ((i & 1) ? P.pairs - 1 - pair : pair), P.total_tiles);
}

// Position of a tile: matrix j, 256-row weight block nb, BNX-row x block xb.
struct TilePos {
    int j, nb, xb, kblocks;
};
__device__ __forceinline__ TilePos tile_pos(const GemmJobDev *jobs, int count, int tile) {
    TilePos t;
    t.j = find_job(jobs, count, tile);
    const GemmJobDev &J = jobs[t.j];
    const int local = tile - J.tile_begin;
    t.nb = local % J.nblocks;
    t.xb = local / J.nblocks;
    t.kblocks = J.K / kBK;
    return t;
}

constexpr int kLook = 4;     // scale/zero look-ahead, in 64-blocks of K
static_assert(kLook % 2 == 0, "two dequant groups take alternate look-ahead slots");

// Walks the (tile, 64-block) sequence a dequant thread consumes and loads
// the scale and zero of its weight row for each position.
template <int WF> struct SzCursor {
    int it, tile, pair, kb, kblocks, group, row0;
    const void *srow;
    const void *zrow;
    const GemmJobDev *jobs;
    __device__ __forceinline__ void bind(const GemmParams &P, int r) {
        if (tile >= P.total_tiles) {
            srow = zrow = nullptr;
            kblocks = 1;
            return;
        }
        const GemmJobDev &J = jobs[find_job(jobs, P.count, tile)];
        const int nb = (tile - J.tile_begin) % J.nblocks;
        const int row = nb * kPairRows + row0 + r;
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
    __device__ __forceinline__ void init(const GemmParams &P, const GemmJobDev *sj, int pr,
                                         int rank_rows, int r) {
        jobs = sj;
        it = 0;
        pair = pr;
        tile = pair_tile(P, pair, 0);
        kb = 0;
        row0 = rank_rows;
        bind(P, r);
    }
    __device__ __forceinline__ void advance(const GemmParams &P, int r) {
        if (++kb == kblocks) {
            kb = 0;
            tile = pair_tile(P, pair, ++it);
            bind(P, r);
        }
    }
    // Raw words of the scale and zero at the current position (fp16 bits,
    // fp32 bits, or the packed range word).  Only the load is issued here;
    // decode() converts them when the block is dequantized, kLook blocks
    // later: converting at once would stall the warp on the load.
    __device__ __forceinline__ void load(const GemmParams &P, uint32_t &sw, uint32_t &zw) const {
        sw = 0u;
        zw = 0u;
        if (!srow) return;
        if constexpr (WF == kPacked) {
            sw = __ldg(static_cast<const unsigned short *>(srow) + kb);
            zw = __ldg(static_cast<const unsigned short *>(zrow) + kb);
        } else {
            if (P.bits == 16) return;
            const int gi = (kb * kBK) / group;
            if (P.range) {
                sw = __ldg(static_cast<const uint32_t *>(srow) + gi);
                zw = 1u;          // marks a loaded range (a zero word is a valid range)
            } else {
                sw = __ldg(static_cast<const uint32_t *>(srow) + gi);
                zw = __ldg(static_cast<const uint32_t *>(zrow) + gi);
            }
        }
    }
};

template <int WF>
__device__ __forceinline__ void decode_sz(const GemmParams &P, uint32_t sw, uint32_t zw,
                                          float &s, float &z) {
    if constexpr (WF == kPacked) {
        s = __half2float(__ushort_as_half((unsigned short)sw));
        z = __half2float(__ushort_as_half((unsigned short)zw));
    } else if (P.range) {
        s = 0.0f;
        z = 0.0f;
        if (zw) {
            const float2 rg = range_of_word(sw);
            const float2 sz = rtn_params_from_range(rg.x, rg.y, P.bits);
            s = sz.x;
            z = sz.y;
        }
    } else {
        s = __uint_as_float(sw);
        z = __uint_as_float(zw);
    }
}

// Offset of 16-byte chunk c (0..7) of row r in a 128B-swizzled K-major tile
// of 128-byte rows (8-row atoms of 1024 bytes): the layout a TMA box with
// SWIZZLE_128B writes and the MMA's shared-memory descriptor reads.
__device__ __forceinline__ int sw128_off(int r, int c) {
    return (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4);
}

template <int BNX, int WF>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ GemmParams P) {
    using C = Cfg<BNX, WF>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *a_ring = smem + C::kAOff;
    uint8_t *x_ring = smem + C::kXOff;
    uint8_t *w_ring = smem + C::kWOff;
    uint64_t *w_full = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
    uint64_t *w_empty = w_full + C::kWStages;
    uint64_t *x_full = w_empty + C::kWStages;
    uint64_t *x_empty = x_full + C::kXStages;
    uint64_t *a_full = x_empty + C::kXStages;    // used in the first CTA of the pair
    uint64_t *a_empty = a_full + C::kAStages;
    uint64_t *acc_full = a_empty + C::kAStages;
    uint64_t *acc_empty = acc_full + 2;          // used in the first CTA of the pair
    uint64_t *mma_done = acc_empty + 2;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(mma_done + 1);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1) + 1;
    GemmJobDev *sjobs = reinterpret_cast<GemmJobDev *>(smem + C::kBarOff + 512);
    static_assert((2 * C::kWStages + 2 * C::kXStages + 2 * C::kAStages + 5) * 8 + 8 <= 512,
                  "barrier block");
    static_assert(512 + kMaxJobs * sizeof(GemmJobDev) <= C::kBarBytes, "job table");
    {
        const uint32_t *src = reinterpret_cast<const uint32_t *>(P.jobs);
        uint32_t *dst = reinterpret_cast<uint32_t *>(sjobs);
        const int words = P.count * (int)(sizeof(GemmJobDev) / 4);
        for (int i = threadIdx.x; i < words; i += kThreads) dst[i] = src[i];
    }

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = (int)cluster_rank();           // 0: issues the MMAs
    const int pair = (int)cluster_id();
    const int t_first = pair_tile(P, pair, 0), T = P.total_tiles;
    const int rank_rows = rank * kBM;               // this CTA's weight rows in a tile
    const int rank_xrows = rank * C::kXHalf;        // this CTA's x rows in a tile

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kWStages; ++s) {
            mbar_init(smem_u32(&w_full[s]), 1);
            mbar_init(smem_u32(&w_empty[s]), kDqWarps);
        }
        for (int s = 0; s < C::kXStages; ++s) {
            mbar_init(smem_u32(&x_full[s]), 1);
            mbar_init(smem_u32(&x_empty[s]), 1);
        }
        for (int s = 0; s < C::kAStages; ++s) {
            mbar_init(smem_u32(&a_full[s]), 2 * kDqWarps / C::kDqGroups);  // one group per CTA
            mbar_init(smem_u32(&a_empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&acc_full[b]), 1);
            mbar_init(smem_u32(&acc_empty[b]), 2 * kEpWarps);
        }
        mbar_init(smem_u32(mma_done), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kMmaWarp) tmem_alloc_pair(smem_u32(tmem_slot), C::kTmemCols);
    tc::fence_before();
    __syncthreads();
    cluster_sync();      // the partner's barriers exist before anything arrives on them
    tc::fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == kCodeWarp || warp == kXWarp) {
        // producers: one lane each; the code producer fills the weight
        // ring, the activation producer the x ring
        if (lane == 0) {
            const bool codes = warp == kCodeWarp;
            const int stages = codes ? C::kWStages : C::kXStages;
            uint64_t *full = codes ? w_full : x_full;
            uint64_t *empty = codes ? w_empty : x_empty;
            uint8_t *ring = codes ? w_ring : x_ring;
            const int bytes = codes ? C::kWBytes : C::kXBytes;
            uint32_t g = 0;
            for (int i = 0, tile = t_first; tile < T && !*abort_flag;
                 tile = pair_tile(P, pair, ++i)) {
                const TilePos tp = tile_pos(sjobs, P.count, tile);
                const int tile2 = pair_tile(P, pair, i + 1);
                if (codes && tile2 < T) {
                    // scales/zeros of the next tile's rows to L2 (the dequant
                    // warps read them a few stages ahead)
                    const TilePos tn = tile_pos(sjobs, P.count, tile2);
                    if (tn.j != tp.j || tn.nb != tp.nb) {
                        const GemmJobDev &J2 = sjobs[tn.j];
                        const int row = tn.nb * kPairRows + rank_rows;
                        if (row < J2.N && !(WF == kRuntime && P.bits == 16)) {
                            const int64_t G2 = J2.K / J2.group;
                            const int64_t es = WF == kPacked ? 2 : 4;
                            const int64_t n = (int64_t)min(kBM, J2.N - row) * G2 * es;
                            const char *sb = static_cast<const char *>(J2.s) + row * G2 * es;
                            const char *zb =
                                J2.z ? static_cast<const char *>(J2.z) + row * G2 * es : nullptr;
                            for (int64_t o = 0; o < n; o += 128) {
                                prefetch_l2(sb + o);
                                if (zb) prefetch_l2(zb + o);
                            }
                        }
                    }
                }
                bool ok = true;
                const int step = codes ? C::kGroup : 1;
                for (int kb = 0; kb < tp.kblocks; kb += step, ++g) {
                    const int s = g % stages;
                    const uint32_t ph = (g / stages) & 1;
                    if (!mbar_wait<kBackoff>(smem_u32(&empty[s]), ph ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&full[s]);
                    mbar_expect_tx(fb, bytes);
                    const uint32_t dst = smem_u32(ring + s * bytes);
                    if (codes)
                        tma_load_2d(dst, &P.wmap[tp.j],
                                    WF == kPacked ? kb * (kBK / 2) : kb * kBK,
                                    tp.nb * kPairRows + rank_rows, fb);
                    else
                        tma_load_2d(dst, &P.xmap[tp.j], kb * kBK,
                                    tp.xb * BNX + rank_xrows, fb);
                }
                if (!ok) break;
            }
            // drain: every load this thread issued has landed before exit
            // (on the normal path each stage was consumed, so these pass)
            for (uint32_t q = 0; q < (uint32_t)stages && g > 0; ++q) {
                if (q >= g) break;
                // the last use of stage q had index gl = largest g' < g with
                // g' % stages == q
                const uint32_t gl = (g - 1) - (((g - 1) % stages + stages - q) % stages);
                mbar_drain(smem_u32(&full[q]), (gl / stages) & 1);
            }
        }
    } else if (warp == kMmaWarp) {
        if (rank == 0) {
            // The whole warp walks the tiles and waits; one elected lane
            // issues a stage's four MMAs and commits.  Descriptors are formed
            // once and advanced by constant offsets (16-byte units of the
            // start address): an MMA issued from a lone diverged lane with
            // descriptors rebuilt per instruction costs several times the
            // tensor core's own time.
            const uint64_t adesc0 = tc::sw128_desc(smem_u32(a_ring));
            const uint64_t bdesc0 = tc::sw128_desc(smem_u32(x_ring));
            uint32_t g = 0;
            int lt = 0;
            for (int i = 0, tile = t_first;
                 tile < T && !__shfl_sync(0xffffffffu, (int)*abort_flag, 0);
                 tile = pair_tile(P, pair, ++i), ++lt) {
                const int kblocks = sjobs[find_job(sjobs, P.count, tile)].K / kBK;
                const int buf = lt & 1;
                const uint32_t aph = (lt >> 1) & 1;
                if (!__all_sync(0xffffffffu, mbar_wait<kSpin>(smem_u32(&acc_empty[buf]),
                                                                     aph ^ 1, abort_flag)))
                    break;
                tc::fence_after();
                const uint32_t d_tmem = tmem_base + buf * BNX;
                bool ok = true;
                for (int kb = 0; kb < kblocks; ++kb, ++g) {
                    const int sx = g % C::kXStages, sa = g % C::kAStages;
                    bool w = mbar_wait<kSpin>(smem_u32(&x_full[sx]), (g / C::kXStages) & 1,
                                              abort_flag);
                    if (w)
                        w = mbar_wait<kSpin>(smem_u32(&a_full[sa]),
                                                   (g / C::kAStages) & 1, abort_flag);
                    if (!__all_sync(0xffffffffu, w)) {
                        ok = false;
                        break;
                    }
                    tc::fence_after();
                    const uint64_t ao = (uint64_t)((sa * C::kABytes) >> 4);
                    const uint64_t bo = (uint64_t)((sx * C::kXBytes) >> 4);
                    if (tc::elect_one()) {
#pragma unroll
                        for (int kk = 0; kk < kBK / 16; ++kk)
                            mma_pair(d_tmem, adesc0 + ao + 2 * kk, bdesc0 + bo + 2 * kk,
                                     C::kIdesc, (kb > 0 || kk > 0) ? 1u : 0u);
                        commit_pair(smem_u32(&x_empty[sx]));    // x stage reusable
                        commit_pair(smem_u32(&a_empty[sa]));    // A buffer reusable
                    }
                    __syncwarp();
                }
                if (!ok) break;
                if (tc::elect_one()) commit_pair(smem_u32(&acc_full[buf]));   // tile done
                __syncwarp();
            }
            // every MMA issued has finished before TMEM is freed
            if (tc::elect_one()) commit_local(smem_u32(mma_done));
            __syncwarp();
            if (lane == 0) mbar_drain(smem_u32(mma_done), 0);
            __syncwarp();
        }
    } else if (warp < kDqWarp0 + kDqWarps) {
        // dequant: kDqGroups groups of warps take alternate stages (group
        // gi the stages g with g % kDqGroups == gi), so with two groups a
        // group has two stages' time for one (packed codes; the runtime
        // requantization, heavier in registers, runs one group).  Thread ->
        // (row r, part) of the 128 x 64 weight tile, kCpt 16-byte chunks
        // (8 k values each) per thread.  Scale/zero come from
        // global memory, fetched kLook blocks ahead into a window of kLook
        // register slots indexed at compile time (slot j serves blocks g
        // with g % kLook == j), so no register copy waits on a load in flight.
        constexpr int kGroupWarps = kDqWarps / C::kDqGroups;
        constexpr int kCpt = 2 * C::kDqGroups;          // chunks per thread
        const int dw = warp - kDqWarp0;
        const int gi = dw / kGroupWarps;
        const int t = (dw % kGroupWarps) * 32 + lane;
        const int r = t & (kBM - 1), part = t >> 7;
        const float L = (float)((1 << (P.bits & 15)) - 1);
        const bool pass = WF == kRuntime && P.bits == 16;
        // In the second CTA the first warp of each group also waits for the
        // CTA's own x stage before arriving: the MMA issued by the first CTA
        // reads it.
        const bool x_gate = rank == 1 && dw % kGroupWarps == 0;
        SzCursor<WF> la;                    // look-ahead cursor
        la.init(P, sjobs, pair, rank_rows, r);
        uint32_t sq[kLook], zq[kLook];
#pragma unroll
        for (int i = 0; i < kLook; ++i) {
            la.load(P, sq[i], zq[i]);
            la.advance(P, r);
        }
        int it = 0, tile = t_first, kb = 0, kblocks = 1;
        bool valid = false;
        auto bind = [&]() {
            if (tile >= T) return;
            const GemmJobDev &J = sjobs[find_job(sjobs, P.count, tile)];
            const int nb = (tile - J.tile_begin) % J.nblocks;
            kblocks = J.K / kBK;
            valid = nb * kPairRows + rank_rows + r < J.N;
        };
        bind();
        uint32_t g = 0, cg = 0;            // stages, weight boxes consumed
        bool ok = true;
        int aoff[kCpt];
#pragma unroll
        for (int i = 0; i < kCpt; ++i) aoff[i] = sw128_off(r, kCpt * part + i);
        while (ok && tile < T && !*abort_flag) {
#pragma unroll
            for (int j = 0; j < kLook; ++j) {
                if (tile >= T) break;
                const int sw = cg % C::kWStages;
                // Both groups wait for every weight box, the one whose blocks
                // they skip too: a barrier's parity test is only sound for a
                // waiter at most one phase ahead, and a group that skipped
                // boxes could otherwise release a slot's next phase early.
                if (!mbar_wait(smem_u32(&w_full[sw]), (cg / C::kWStages) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                if (j % C::kDqGroups == gi) {   // kLook % kDqGroups == 0: g ≡ j
                    float sf, zf;
                    decode_sz<WF>(P, sq[j], zq[j], sf, zf);
                    const uint8_t *wt = w_ring + sw * C::kWBytes;
                    uint4 o[kCpt];
#pragma unroll
                    for (int i = 0; i < kCpt; ++i) o[i] = make_uint4(0, 0, 0, 0);
                    if (valid) {
                        if constexpr (WF == kRuntime) {
#pragma unroll
                            for (int i = 0; i < kCpt; ++i)
                                o[i] = requant8(*reinterpret_cast<const uint4 *>(wt + aoff[i]), sf,
                                                zf, L, pass);
                        } else {
                            static_assert(C::kDqGroups == 2, "packed: one 16-byte code chunk");
                            // 16 bytes at (kb % 4) * 32 + part * 16 of the row's
                            // 128 (128B-swizzled)
                            const int chunk = (kb % C::kGroup) * 2 + part;
                            const uint4 cw = *reinterpret_cast<const uint4 *>(
                                wt + r * 128 + ((chunk ^ (r & 7)) << 4));
                            const uint32_t w4[4] = {cw.x, cw.y, cw.z, cw.w};
                            if (fabsf(zf) <= 128.0f) {
                                const __nv_bfloat16 zb1 = __float2bfloat16_rn(128.0f + zf);
                                const __nv_bfloat16 sb1 = __float2bfloat16_rn(sf);
                                const __nv_bfloat162 zb = __halves2bfloat162(zb1, zb1);
                                const __nv_bfloat162 sb = __halves2bfloat162(sb1, sb1);
#pragma unroll
                                for (int i = 0; i < 4; ++i) o[i] = dequant8(w4[i], zb, sb);
                            } else {
#pragma unroll
                                for (int i = 0; i < 4; ++i) o[i] = dequant8_wide(w4[i], zf, sf);
                            }
                        }
                    }
                    const int sa = g % C::kAStages;
                    // completed by the first CTA's commit (multicast): polled, the
                    // MMA waits on what this warp writes next
                    if (!mbar_wait<kSpin>(smem_u32(&a_empty[sa]), ((g / C::kAStages) & 1) ^ 1,
                                             abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t *at = a_ring + sa * C::kABytes;
#pragma unroll
                    for (int i = 0; i < kCpt; ++i) *reinterpret_cast<uint4 *>(at + aoff[i]) = o[i];
                    fence_proxy_async_smem();
                    if (x_gate && !mbar_wait(smem_u32(&x_full[g % C::kXStages]),
                                             (g / C::kXStages) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(in_leader(smem_u32(&a_full[sa])));
                }
                la.load(P, sq[j], zq[j]);          // refill slot j, kLook ahead
                la.advance(P, r);
                // the weight box is released by both groups after its last
                // block (this group's values are in registers or stored)
                if (kb % C::kGroup == C::kGroup - 1 || kb == kblocks - 1) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&w_empty[sw]));
                    ++cg;
                }
                ++g;
                if (++kb == kblocks) {
                    kb = 0;
                    tile = pair_tile(P, pair, ++it);
                    bind();
                }
            }
        }
    } else {
        // epilogue: warp quarter q reads TMEM lanes 32q..32q+31 (weight rows),
        // half hh of the accumulator's columns (x rows)
        const int q = warp & 3, hh = (warp - kEpWarp0) >> 2;
        int lt = 0;
        for (int i = 0, tile = t_first; tile < T && !*abort_flag;
             tile = pair_tile(P, pair, ++i), ++lt) {
            const TilePos tp = tile_pos(sjobs, P.count, tile);
            const GemmJobDev &J = sjobs[tp.j];
            const int buf = lt & 1;
            const uint32_t aph = (lt >> 1) & 1;
            if (!mbar_wait<kBackoff>(smem_u32(&acc_full[buf]), aph, abort_flag)) break;
            tc::fence_after();
            const int n = tp.nb * kPairRows + rank_rows + 32 * q + lane;
            const int m0 = tp.xb * BNX;
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
            if (lane == 0) mbar_arrive_cluster(in_leader(smem_u32(&acc_empty[buf])));
        }
    }

    tc::fence_before();
    __syncthreads();
    // neither CTA leaves (or frees TMEM) while the pair's MMAs, commits or
    // arrivals may still touch its memory
    cluster_sync();
    if (warp == kMmaWarp) {
        tc::fence_after();
        tmem_dealloc_pair(tmem_base, C::kTmemCols);
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
    // four 64-blocks (128 bytes) of 128 rows, 128B-swizzled
    cuuint32_t box[2] = {(cuuint32_t)(2 * kBK), (cuuint32_t)kBM};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(w), dims, strides,
               box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
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

// Contiguous tile ranges per CTA pair that minimise the costliest range
// (binary search on the bound, greedy fill).  A tile costs its K/64 stages
// plus a fixed share for its epilogue.
void partition_tiles(GemmParams &P, const std::vector<double> &tcost, int pairs) {
    const int n = (int)tcost.size();
    double total = 0, tmax = 0;
    for (double c : tcost) {
        total += c;
        tmax = std::max(tmax, c);
    }
    auto fill = [&](double T, bool out) -> int {
        int used = 1;
        double cur = 0;
        if (out) P.pair_begin[0] = 0;
        for (int i = 0; i < n; ++i) {
            if (cur > 0 && cur + tcost[i] > T) {
                if (out && used < pairs) P.pair_begin[used] = i;
                ++used;
                cur = 0;
            }
            cur += tcost[i];
        }
        return used;
    };
    double lo = std::max(tmax, total / pairs), hi = total + tmax;
    for (int it = 0; it < 60 && hi - lo > 0.5; ++it) {
        const double mid = 0.5 * (lo + hi);
        if (fill(mid, false) <= pairs) hi = mid; else lo = mid;
    }
    const int used = std::min(fill(hi, true), pairs);
    for (int c = used; c <= pairs; ++c) P.pair_begin[c] = n;
}

template <int BNX, int WF>
bc_status launch_cfg(const GemmJob *jobs, int count, int64_t M, int bits, bool range,
                     cudaStream_t s, int sm_count) {
    using C = Cfg<BNX, WF>;
    auto enc = get_encoder();
    if (!enc) return BC_ERR_CUDA;
    static std::mutex mu;
    static int max_pairs[64] = {};     // per device, 0 = not yet set up
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return BC_ERR_CUDA;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::kSmem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!max_pairs[dev]) {
            if (cudaFuncSetAttribute(gemm_kernel<BNX, WF>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     C::kSmem) != cudaSuccess)
                return BC_ERR_CUDA;
            // pairs that can be resident at once (one CTA per SM)
            cfg.gridDim = dim3(2 * kMaxPairs);
            int clusters = 0;
            if (cudaOccupancyMaxActiveClusters(&clusters, gemm_kernel<BNX, WF>, &cfg) !=
                    cudaSuccess ||
                clusters < 1)
                return BC_ERR_CUDA;
            max_pairs[dev] = std::min({clusters, std::max(1, sm_count / 2), kMaxPairs});
        }
    }
    thread_local GemmParams *Pp = nullptr;
    if (!Pp) Pp = new GemmParams();
    GemmParams &P = *Pp;
    std::vector<int> order;
    std::vector<double> tcost;
    for (int b = 0; b < count; b += kMaxJobs) {
        const int n = std::min(kMaxJobs, count - b);
        int tiles = 0;
        const int xblocks = (int)((M + BNX - 1) / BNX);
        // matrices by decreasing K (stable): the long-K tiles are dealt first
        order.resize(n);
        tcost.clear();
        for (int i = 0; i < n; ++i) order[i] = b + i;
        std::stable_sort(order.begin(), order.end(),
                         [&](int p, int q) { return jobs[p].K > jobs[q].K; });
        for (int i = 0; i < n; ++i) {
            const GemmJob &J = jobs[order[i]];
            if (!encode_x(enc, &P.xmap[i], J.x, M, J.K, C::kXHalf)) return BC_ERR_CUDA;
            const bool ok = WF == kPacked ? encode_codes(enc, &P.wmap[i], J.w, J.N, J.K)
                                          : encode_w16(enc, &P.wmap[i], J.w, J.N, J.K);
            if (!ok) return BC_ERR_CUDA;
            const int nblocks = (int)((J.N + kPairRows - 1) / kPairRows);
            P.jobs[i] = GemmJobDev{J.s, J.z, J.y, (int)J.N, (int)J.K, (int)J.group, tiles,
                                   nblocks};
            tiles += nblocks * xblocks;
            // cost in stages: K/64 of MMA plus the epilogue (BNX/32 loads of
            // 32 columns and their stores), about two stages' worth
            tcost.insert(tcost.end(), nblocks * xblocks, (double)(J.K / kBK) + 2.0 * BNX / 128.0);
        }
        P.count = n;
        P.total_tiles = tiles;
        P.M = (int)M;
        P.bits = bits;
        P.range = range ? 1 : 0;
        const int pairs = std::max(1, std::min(tiles, max_pairs[dev]));
        P.pairs = pairs;
        P.ranges = xblocks == 1 ? 1 : 0;
        if (P.ranges) partition_tiles(P, tcost, pairs);
        cfg.gridDim = dim3(2 * pairs);
        if (cudaLaunchKernelEx(&cfg, gemm_kernel<BNX, WF>, P) != cudaSuccess) return BC_ERR_CUDA;
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
