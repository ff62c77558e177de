// bc_gemv.cu -- fused dequant GEMV for decode shapes (M < 64, fp32 x).
//
// y[m,n] = sum_k x[m,k] * w'[n,k] with w' formed in registers as the weights
// stream in (BITCRUSH BC-06, "Under the hood": matmul_q computes the
// group-wise affine RTN inline as weights are read; Enargeia, "Four bits per
// weight": int4 codes unpacked in registers and never written back).
// A decode step touches every weight once for one output row (Enargeia's
// point about decode), so the kernel is an HBM stream: 16-byte vector loads that skip L1, one
// 16-byte chunk per lane per step (8 fp16 weights, or 32 int4 codes),
// `lpr` lanes per weight row, 8 warps per CTA, a persistent grid over a
// work list that spans every matrix of a grouped launch (Enargeia, "One
// decode step": hundreds of passes per token, so launches are batched).
//
// Runtime mode re-derives each code from fp16 w and the fp32 (scale, zero):
//   q - z = clamp(rne(w / s), -z, L - z)
// The exact real quotient must be rounded (codes are bit-exact).  The fast
// path rounds w * rcp(s) with the 1.5*2^23 trick and keeps the residual
// e = w*rcp(s) - c; when |e| comes within the rcp/rounding error of 1/2 for
// any weight of a chunk, the chunk is recomputed with an fp64 quotient.
//
// Split-K (single small matrices): each k-split writes a partial row block
// to the caller's workspace; the last CTA to finish a row block (ticket
// counter) sums the partials in split order, so results are deterministic.
#include "bc_internal.cuh"
#include "bc_rtn.cuh"

#include <algorithm>
#include <vector>

namespace bc {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxJobs = 368;
constexpr float kMagic = 12582912.0f;       // 1.5 * 2^23

struct JobDev {
    const float *x;
    const void *w;
    const void *s;
    const void *z;
    float *y;
    int N, K, group;
    int item_begin;        // first work item of this job
    int rows_per_item;     // kWarps * 32 / lpr
    int splits;            // k-splits (1 = none)
    int lpr_log2;          // lanes per row = 1 << lpr_log2
    int ws_offset;         // split-K partials: float offset in workspace
    int ticket_offset;     // split-K tickets: index in ticket array
};

struct GemvParams {
    int count, total_items, M, bits;
    int range;             // runtime mode: (scale, zero) derived from stored ranges
    float *ws_partial;
    unsigned *ws_ticket;
    JobDev jobs[kMaxJobs];
};
static_assert(sizeof(GemvParams) <= 32000, "kernel parameter space");

__device__ __forceinline__ uint4 ld_stream(const void *p) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

__device__ __forceinline__ float rcp_approx(float s) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s));
    return r;
}

// q - z for one weight, exact (fp64 quotient, see bc_quant.cu).
__device__ __noinline__ float centered_code_exact(float w, float s, float z,
                                                  float L) {
    double q = rint((double)w / (double)s) + (double)z;
    q = fmin(fmax(q, 0.0), (double)L);
    return (float)(q - (double)z);
}

// Runtime mode: 8 fp16 weights of one group -> 8 centered codes (q - z),
// or the weights themselves for the fp16 passthrough (bits == 16).
__device__ __forceinline__ void runtime_codes(const uint4 raw, float s, float z,
                                              float L, bool passthrough,
                                              float (&c)[8]) {
    const __half2 *h = reinterpret_cast<const __half2 *>(&raw);
    float w[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 t = __half22float2(h[i]);
        w[2 * i] = t.x;
        w[2 * i + 1] = t.y;
    }
    if (passthrough) {
#pragma unroll
        for (int i = 0; i < 8; ++i) c[i] = w[i];
        return;
    }
    const float inv = rcp_approx(s);
    const float lo_c = -z, hi_c = L - z;
    // |w/s - w*inv| <= |w/s| * 2^-22 (rcp.approx is within 1 ulp); codes
    // that matter have |w/s| <= max(|z|, |L - z|) + 1.
    const float thr = 0.5f - (fmaxf(fabsf(lo_c), fabsf(hi_c)) + 2.0f) *
                                 4.76837158203125e-07f;   // 2^-21
    float emax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float v = fmaf(w[i], inv, kMagic);
        const float r = v - kMagic;                 // nearest integer to w*inv
        const float e = fmaf(w[i], inv, -r);        // residual, |e| <= 1/2
        emax = fmaxf(emax, fabsf(e));
        c[i] = fminf(fmaxf(r, lo_c), hi_c);
    }
    if (emax > thr) {                               // near a half-way point
#pragma unroll
        for (int i = 0; i < 8; ++i) c[i] = centered_code_exact(w[i], s, z, L);
    }
}

template <bool PACKED, int MT>
__global__ void __launch_bounds__(kThreads)
gemv_kernel(const __grid_constant__ GemvParams P) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float L = (float)((1 << P.bits) - 1);
    const bool passthrough = P.bits == 16;
    __shared__ int s_last;

    for (int item = blockIdx.x; item < P.total_items; item += gridDim.x) {
        int lo = 0, hi = P.count - 1;                 // job owning this item
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (P.jobs[mid].item_begin <= item) lo = mid; else hi = mid - 1;
        }
        const JobDev &J = P.jobs[lo];
        const int local = item - J.item_begin;
        const int split = local % J.splits;
        const int rb = local / J.splits;
        const int lpr_log2 = J.lpr_log2;
        const int lpr = 1 << lpr_log2;
        const int row = rb * J.rows_per_item + warp * (32 >> lpr_log2) +
                        (lane >> lpr_log2);
        const int sub = lane & (lpr - 1);
        const int K = J.K, N = J.N;
        const int cpr = PACKED ? K / 32 : K / 8;       // 16-byte chunks per row
        const int c_begin = (int)((int64_t)split * cpr / J.splits);
        const int c_end = (int)((int64_t)(split + 1) * cpr / J.splits);
        const int G = K / J.group;
        const int chunks_per_group = PACKED ? 2 : J.group / 8;

        float acc[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[m] = 0.0f;

        if (row < N) {
            const uint8_t *wrow = reinterpret_cast<const uint8_t *>(J.w) +
                                  (int64_t)row * (PACKED ? K / 2 : K * 2);
            for (int c0 = c_begin + sub; c0 < c_end; c0 += 4 * lpr) {
                uint4 raw[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int c = c0 + u * lpr;
                    if (c < c_end) raw[u] = ld_stream(wrow + (int64_t)c * 16);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int c = c0 + u * lpr;
                    if (c >= c_end) break;
                    const int gi = row * G + c / chunks_per_group;
                    if constexpr (PACKED) {
                        const float s = __half2float(
                            __ldg(reinterpret_cast<const __half *>(J.s) + gi));
                        const float z = __half2float(
                            __ldg(reinterpret_cast<const __half *>(J.z) + gi));
                        const float bias = 8388608.0f + z;    // 2^23 + z
                        const uint32_t wd[4] = {raw[u].x, raw[u].y, raw[u].z,
                                                raw[u].w};
                        float part[MT];
#pragma unroll
                        for (int m = 0; m < MT; ++m) part[m] = 0.0f;
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            float cq[8];
#pragma unroll
                            for (int j = 0; j < 8; ++j)
                                cq[j] = __int_as_float(0x4B000000u |
                                                       ((wd[q4] >> (4 * j)) & 0xFu)) -
                                        bias;
#pragma unroll
                            for (int m = 0; m < MT; ++m) {
                                if (m >= P.M) break;
                                const float4 *xp = reinterpret_cast<const float4 *>(
                                    J.x + (int64_t)m * K + c * 32 + q4 * 8);
                                const float4 xa = __ldg(xp), xb = __ldg(xp + 1);
                                float p = part[m];
                                p = fmaf(xa.x, cq[0], p);
                                p = fmaf(xa.y, cq[1], p);
                                p = fmaf(xa.z, cq[2], p);
                                p = fmaf(xa.w, cq[3], p);
                                p = fmaf(xb.x, cq[4], p);
                                p = fmaf(xb.y, cq[5], p);
                                p = fmaf(xb.z, cq[6], p);
                                p = fmaf(xb.w, cq[7], p);
                                part[m] = p;
                            }
                        }
#pragma unroll
                        for (int m = 0; m < MT; ++m) acc[m] = fmaf(part[m], s, acc[m]);
                    } else {
                        float s = 1.0f, z = 0.0f;
                        if (!passthrough) {
                            if (P.range) {
                                const float2 r = range_of_word(
                                    __ldg(reinterpret_cast<const uint32_t *>(J.s) + gi));
                                const float2 sz = rtn_params_from_range(r.x, r.y, P.bits);
                                s = sz.x;
                                z = sz.y;
                            } else {
                                s = __ldg(reinterpret_cast<const float *>(J.s) + gi);
                                z = __ldg(reinterpret_cast<const float *>(J.z) + gi);
                            }
                        }
                        float cq[8];
                        runtime_codes(raw[u], s, z, L, passthrough, cq);
#pragma unroll
                        for (int m = 0; m < MT; ++m) {
                            if (m >= P.M) break;
                            const float4 *xp = reinterpret_cast<const float4 *>(
                                J.x + (int64_t)m * K + c * 8);
                            const float4 xa = __ldg(xp), xb = __ldg(xp + 1);
                            float p = xa.x * cq[0];
                            p = fmaf(xa.y, cq[1], p);
                            p = fmaf(xa.z, cq[2], p);
                            p = fmaf(xa.w, cq[3], p);
                            p = fmaf(xb.x, cq[4], p);
                            p = fmaf(xb.y, cq[5], p);
                            p = fmaf(xb.z, cq[6], p);
                            p = fmaf(xb.w, cq[7], p);
                            acc[m] = fmaf(p, s, acc[m]);
                        }
                    }
                }
            }
        }
        // reduce over the lpr lanes of each row (all lanes take part)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            for (int off = lpr >> 1; off > 0; off >>= 1)
                acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], off);
        }
        if (J.splits == 1) {
            if (sub == 0 && row < N) {
#pragma unroll
                for (int m = 0; m < MT; ++m)
                    if (m < P.M) J.y[(int64_t)m * N + row] = acc[m];
            }
            continue;
        }
        // ---- split-K: partials, ticket, ordered reduction by the last CTA
        float *part_base = P.ws_partial + J.ws_offset;
        if (sub == 0 && row < N) {
#pragma unroll
            for (int m = 0; m < MT; ++m)
                if (m < P.M)
                    part_base[((int64_t)split * P.M + m) * N + row] = acc[m];
        }
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) {
            const unsigned prev =
                atomicAdd(&P.ws_ticket[J.ticket_offset + rb], 1u);
            s_last = (prev == (unsigned)(J.splits - 1));
        }
        __syncthreads();
        if (s_last) {
            __threadfence();
            const int r0 = rb * J.rows_per_item;
            const int nr = min(J.rows_per_item, N - r0);
            for (int t = threadIdx.x; t < nr * P.M; t += kThreads) {
                const int m = t / nr, r = r0 + t % nr;
                float sum = 0.0f;
                for (int sp = 0; sp < J.splits; ++sp)
                    sum += __ldcg(part_base + ((int64_t)sp * P.M + m) * N + r);
                J.y[(int64_t)m * N + r] = sum;
            }
            if (threadIdx.x == 0) P.ws_ticket[J.ticket_offset + rb] = 0u;
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Host-side planning
// ---------------------------------------------------------------------------
struct Plan {
    std::vector<JobDev> jobs;
    int total_items = 0;
    size_t partial_floats = 0;     // split-K partials
    size_t tickets = 0;
};

int pick_lpr_log2(int cpr) {
    for (int l = 5; l >= 0; --l)
        if (cpr % (1 << l) == 0 && cpr / (1 << l) >= 4) return l;
    for (int l = 5; l >= 0; --l)
        if (cpr % (1 << l) == 0) return l;
    return 0;
}

constexpr int kCtasPerSm = 4;

Plan make_plan(const GemvJob *jobs, int count, int M, bool packed, int sm_count) {
    Plan p;
    p.jobs.resize(count);
    int64_t items_nosplit = 0;
    for (int i = 0; i < count; ++i) {
        const int K = (int)jobs[i].K;
        const int cpr = packed ? K / 32 : K / 8;
        JobDev &d = p.jobs[i];
        d.lpr_log2 = pick_lpr_log2(cpr);
        d.rows_per_item = kWarps * (32 >> d.lpr_log2);
        items_nosplit += (jobs[i].N + d.rows_per_item - 1) / d.rows_per_item;
    }
    // Split K only when the whole launch cannot fill the GPU.
    const int64_t target = (int64_t)kCtasPerSm * sm_count;
    int want = 1;
    if (items_nosplit < target)
        want = (int)std::min<int64_t>(16, (target + items_nosplit - 1) / items_nosplit);
    int item = 0;
    for (int i = 0; i < count; ++i) {
        JobDev &d = p.jobs[i];
        const GemvJob &j = jobs[i];
        d.x = j.x; d.w = j.w; d.s = j.s; d.z = j.z; d.y = j.y;
        d.N = (int)j.N; d.K = (int)j.K; d.group = (int)j.group;
        const int cpr = packed ? d.K / 32 : d.K / 8;
        const int lpr = 1 << d.lpr_log2;
        const int max_splits = std::max(1, cpr / (lpr * 4));
        d.splits = std::max(1, std::min(want, max_splits));
        const int rblocks = (d.N + d.rows_per_item - 1) / d.rows_per_item;
        d.item_begin = item;
        item += rblocks * d.splits;
        d.ws_offset = 0;
        d.ticket_offset = 0;
        if (d.splits > 1) {
            d.ws_offset = (int)p.partial_floats;
            p.partial_floats += (size_t)d.splits * M * d.N;
            d.ticket_offset = (int)p.tickets;
            p.tickets += rblocks;
        }
    }
    p.total_items = item;
    return p;
}

size_t ws_bytes_of(const Plan &p) {
    if (p.tickets == 0) return 0;
    const size_t part = (p.partial_floats * 4 + 255) / 256 * 256;
    return part + p.tickets * 4;
}

template <bool PACKED>
bc_status launch_mt(const GemvParams &P, int mt, int grid, cudaStream_t s) {
    switch (mt) {
    case 1: gemv_kernel<PACKED, 1><<<grid, kThreads, 0, s>>>(P); break;
    case 2: gemv_kernel<PACKED, 2><<<grid, kThreads, 0, s>>>(P); break;
    case 4: gemv_kernel<PACKED, 4><<<grid, kThreads, 0, s>>>(P); break;
    case 8: gemv_kernel<PACKED, 8><<<grid, kThreads, 0, s>>>(P); break;
    default: gemv_kernel<PACKED, 16><<<grid, kThreads, 0, s>>>(P); break;
    }
    return cuda_status();
}

// Whole launches with at least half an SM's worth of 128-row units per SM
// go to the streaming kernels (M <= 4; M <= 16 for packed codes and for
// runtime RTN below 16 bits); lone small matrices keep the split-K GEMV.
bool use_stream(const GemvJob *jobs, int count, int M, bool packed, int bits,
                const DeviceInfo &di) {
    if (M > (packed || bits <= 8 ? 16 : 4)) return false;
    int64_t units = 0;
    for (int i = 0; i < count; ++i) units += (jobs[i].N + 127) / 128;
    if (units < di.sm_count / 2) return false;
    return gemv_stream_supported(jobs, count, M, packed, bits, di.max_smem_optin);
}

}  // namespace

size_t gemv_workspace_bytes(const GemvJob *jobs, int count, int M, bool packed,
                            int sm_count) {
    // The bit width is not known here: a runtime launch that the tensor-core
    // decode kernel would take at 2..8 bits uses the general GEMV at 16.
    DeviceInfo di;
    size_t worst = 0;
    if (device_info(&di) && use_stream(jobs, count, M, packed, 8, di)) {
        worst = gemv_stream_workspace_bytes(jobs, count, M, packed, 8);
        if (packed || M <= 4) return worst;
    }
    for (int b = 0; b < count; b += kMaxJobs) {
        const int n = std::min(kMaxJobs, count - b);
        Plan p = make_plan(jobs + b, n, std::min(M, 16), packed, sm_count);
        worst = std::max(worst, ws_bytes_of(p));
    }
    return worst;
}

bc_status launch_gemv(const GemvJob *jobs, int count, int M, int bits,
                      bool packed, void *workspace, size_t ws_bytes,
                      cudaStream_t s, bool early_start) {
    DeviceInfo di;
    if (!device_info(&di)) return BC_ERR_CUDA;
    if (use_stream(jobs, count, M, packed, bits, di))
        return launch_gemv_stream(jobs, count, M, bits, packed, s, early_start, workspace,
                                  ws_bytes);
    // ~32 KB of kernel parameters, kept off the stack; the launch copies it.
    thread_local GemvParams *Pp = nullptr;
    if (!Pp) Pp = new GemvParams();
    GemvParams &Q = *Pp;
    std::vector<GemvJob> sub(jobs, jobs + count);
    for (int m0 = 0; m0 < M; m0 += 16) {
        const int mrows = std::min(16, M - m0);
        const int mt = mrows <= 1 ? 1 : mrows <= 2 ? 2 : mrows <= 4 ? 4
                                   : mrows <= 8 ? 8 : 16;
        for (int b = 0; b < count; b += kMaxJobs) {
            const int n = std::min(kMaxJobs, count - b);
            for (int i = 0; i < n; ++i) {
                sub[i] = jobs[b + i];
                sub[i].x = jobs[b + i].x + (int64_t)m0 * jobs[b + i].K;
                sub[i].y = jobs[b + i].y + (int64_t)m0 * jobs[b + i].N;
            }
            Plan p = make_plan(sub.data(), n, mrows, packed, di.sm_count);
            const size_t need = ws_bytes_of(p);
            if (need > ws_bytes) return BC_ERR_WORKSPACE;
            Q.count = n;
            Q.total_items = p.total_items;
            Q.M = mrows;
            Q.bits = bits;
            Q.range = (int)jobs[0].range;
            Q.ws_partial = reinterpret_cast<float *>(workspace);
            Q.ws_ticket = nullptr;
            if (p.tickets) {
                const size_t part = (p.partial_floats * 4 + 255) / 256 * 256;
                Q.ws_ticket = reinterpret_cast<unsigned *>(
                    reinterpret_cast<uint8_t *>(workspace) + part);
                if (cudaMemsetAsync(Q.ws_ticket, 0, p.tickets * 4, s) != cudaSuccess)
                    return BC_ERR_CUDA;
            }
            for (int i = 0; i < n; ++i) Q.jobs[i] = p.jobs[i];
            const int grid = std::max(1, std::min(p.total_items,
                                                  kCtasPerSm * di.sm_count));
            bc_status st = packed ? launch_mt<true>(Q, mt, grid, s)
                                  : launch_mt<false>(Q, mt, grid, s);
            if (st != BC_OK) return st;
        }
    }
    return BC_OK;
}

}  // namespace bc
