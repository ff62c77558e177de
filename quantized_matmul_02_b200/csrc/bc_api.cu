// bc_api.cu -- the C ABI: argument validation and kernel choice.
//
// Every entry point validates on the host, then enqueues kernels on the
// caller's stream.  Nothing here allocates device memory or synchronises.
#include "bc_internal.cuh"

#include <algorithm>
#include <mutex>
#include <vector>

namespace bc {

bool device_info(DeviceInfo *out) {
    static std::mutex mu;
    static std::vector<DeviceInfo> cache;
    static std::vector<bool> have;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::lock_guard<std::mutex> lock(mu);
    if ((int)cache.size() <= dev) {
        cache.resize(dev + 1);
        have.resize(dev + 1, false);
    }
    if (!have[dev]) {
        DeviceInfo d;
        if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount,
                                   dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor,
                                   dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor,
                                   dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.max_smem_optin,
                                   cudaDevAttrMaxSharedMemoryPerBlockOptin,
                                   dev) != cudaSuccess)
            return false;
        cache[dev] = d;
        have[dev] = true;
    }
    *out = cache[dev];
    return true;
}

namespace {

// Shape/precision rules shared by the single and batched matmul calls.
bc_status check_matmul_common(int64_t M, int bits, int64_t group_norm,
                              bc_mode mode, bc_dtype x_dtype) {
    if (M <= 0 || M > (int64_t)1 << 24) return BC_ERR_INVALID_ARG;
    if (mode == BC_MODE_RUNTIME || mode == BC_MODE_RUNTIME_RANGE) {
        if (!((bits >= 2 && bits <= 8) || bits == 16)) return BC_ERR_UNSUPPORTED;
        if (x_dtype == BC_BF16) {
            if (M < 64) return BC_ERR_UNSUPPORTED;
        } else if (x_dtype != BC_F32) {
            return BC_ERR_UNSUPPORTED;
        }
    } else if (mode == BC_MODE_PACKED_INT4) {
        // packed codes: int4 everywhere; 2, 3 and 8 bits on the decode GEMV
        if (!(bits == 2 || bits == 3 || bits == 4 || bits == 8) || group_norm != 64)
            return BC_ERR_UNSUPPORTED;
        if (x_dtype == BC_BF16) {
            if (M < 64 || bits != 4) return BC_ERR_UNSUPPORTED;
        } else if (x_dtype != BC_F32) {
            return BC_ERR_UNSUPPORTED;
        }
    } else {
        return BC_ERR_UNSUPPORTED;
    }
    return BC_OK;
}

bc_status check_nk(int64_t N, int64_t K) {
    if (N <= 0 || K <= 0 || K % 64) return BC_ERR_INVALID_ARG;
    if (N >= ((int64_t)1 << 31) / 2 || K >= ((int64_t)1 << 24))
        return BC_ERR_UNSUPPORTED;
    if (N * K >= ((int64_t)1 << 31) * 16) return BC_ERR_UNSUPPORTED;
    return BC_OK;
}

// group as given -> 64 or K (per channel); -1 if not offered.
int64_t normalize_group(int64_t group, int64_t K) {
    if (group == 64) return 64;
    if (group == BC_GROUP_PER_CHANNEL || group == K) return K;
    return -1;
}

bc_status check_matmul_ptrs(const void *x, bc_dtype x_dtype, const void *w,
                            const void *s, const void *z, const float *y,
                            int bits, bc_mode mode) {
    if (!x || !w || !y) return BC_ERR_INVALID_ARG;
    const bool need_sz = !(mode != BC_MODE_PACKED_INT4 && bits == 16);
    const bool need_z = need_sz && mode != BC_MODE_RUNTIME_RANGE;   // ranges: one array
    if ((need_sz && !s) || (need_z && !z)) return BC_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(w, 16) || !aligned(y, 4))
        return BC_ERR_ALIGNMENT;
    (void)x_dtype;
    if (need_sz) {
        const size_t a = mode == BC_MODE_PACKED_INT4 ? 2 : 4;
        if (!aligned(s, a) || (need_z && !aligned(z, a))) return BC_ERR_ALIGNMENT;
    }
    return BC_OK;
}

}  // namespace
}  // namespace bc

using namespace bc;

extern "C" {

const char *bc_status_string(bc_status st) {
    switch (st) {
    case BC_OK: return "ok";
    case BC_ERR_INVALID_ARG: return "invalid argument (null pointer, bad size, or K not a multiple of 64)";
    case BC_ERR_UNSUPPORTED: return "unsupported bits/group/mode/dtype combination";
    case BC_ERR_ALIGNMENT: return "misaligned pointer";
    case BC_ERR_WORKSPACE: return "workspace too small";
    case BC_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

int bc_version(void) { return 100; }

bc_status bc_device_timeouts(unsigned *count) {
    if (!count) return BC_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return BC_ERR_CUDA;
    const unsigned a = gemm_timeouts(), b = gemv_timeouts();
    if (a == ~0u || b == ~0u) return BC_ERR_CUDA;
    *count = a + b;
    return BC_OK;
}

bc_status bc_set_wait_limit(uint64_t cycles) {
    const long long v = cycles == 0 ? 4000000000LL
                                    : (long long)std::min<uint64_t>(cycles, 4000000000ull);
    if (cudaDeviceSynchronize() != cudaSuccess) return BC_ERR_CUDA;
    bc_status st = gemv_set_wait_limit(v);
    if (st == BC_OK) st = gemm_set_wait_limit(v);
    return st;
}

bc_status bc_group_params(const void *W, int64_t N, int64_t K, int bits,
                          int64_t group, bc_dtype out_dtype, void *scales,
                          void *zeros, bc_stream_t stream) {
    if (!W || !scales || !zeros) return BC_ERR_INVALID_ARG;
    bc_status st = check_nk(N, K);
    if (st != BC_OK) return st;
    if (bits < 2 || bits > 8) return BC_ERR_UNSUPPORTED;
    const int64_t g = normalize_group(group, K);
    if (g < 0) return BC_ERR_UNSUPPORTED;
    if (out_dtype != BC_F32 && out_dtype != BC_F16) return BC_ERR_UNSUPPORTED;
    const size_t a = out_dtype == BC_F32 ? 4 : 2;
    if (!aligned(W, 16) || !aligned(scales, a) || !aligned(zeros, a))
        return BC_ERR_ALIGNMENT;
    return launch_group_params(static_cast<const __half *>(W), N, K, bits, g,
                               out_dtype == BC_F16, scales, zeros,
                               reinterpret_cast<cudaStream_t>(stream));
}

bc_status bc_group_minmax(const void *W, int64_t N, int64_t K, int64_t group,
                          void *ranges, bc_stream_t stream) {
    if (!W || !ranges) return BC_ERR_INVALID_ARG;
    bc_status st = check_nk(N, K);
    if (st != BC_OK) return st;
    const int64_t g = normalize_group(group, K);
    if (g < 0) return BC_ERR_UNSUPPORTED;
    if (!aligned(W, 16) || !aligned(ranges, 4)) return BC_ERR_ALIGNMENT;
    return launch_group_minmax(static_cast<const __half *>(W), N, K, g, ranges,
                               reinterpret_cast<cudaStream_t>(stream));
}

bc_status bc_quantize_codes(const void *W, const void *scales,
                            const void *zeros, bc_dtype sz_dtype, int64_t N,
                            int64_t K, int bits, int64_t group,
                            uint8_t *codes, bc_stream_t stream) {
    if (!W || !scales || !zeros || !codes) return BC_ERR_INVALID_ARG;
    bc_status st = check_nk(N, K);
    if (st != BC_OK) return st;
    if (bits < 2 || bits > 8) return BC_ERR_UNSUPPORTED;
    const int64_t g = normalize_group(group, K);
    if (g < 0) return BC_ERR_UNSUPPORTED;
    if (sz_dtype != BC_F32 && sz_dtype != BC_F16) return BC_ERR_UNSUPPORTED;
    const size_t a = sz_dtype == BC_F32 ? 4 : 2;
    if (!aligned(W, 16) || !aligned(scales, a) || !aligned(zeros, a) ||
        !aligned(codes, 8))
        return BC_ERR_ALIGNMENT;
    return launch_quantize_codes(static_cast<const __half *>(W), scales, zeros,
                                 sz_dtype == BC_F16, N, K, bits, g, codes,
                                 reinterpret_cast<cudaStream_t>(stream));
}

bc_status bc_pack_int4(const void *W, const void *scales_f16,
                       const void *zeros_f16, int64_t N, int64_t K,
                       uint8_t *packed, bc_stream_t stream) {
    if (!W || !scales_f16 || !zeros_f16 || !packed) return BC_ERR_INVALID_ARG;
    bc_status st = check_nk(N, K);
    if (st != BC_OK) return st;
    if (!aligned(W, 16) || !aligned(scales_f16, 2) || !aligned(zeros_f16, 2) ||
        !aligned(packed, 16))
        return BC_ERR_ALIGNMENT;
    return launch_pack_int4(static_cast<const __half *>(W),
                            static_cast<const __half *>(scales_f16),
                            static_cast<const __half *>(zeros_f16), N, K,
                            packed, reinterpret_cast<cudaStream_t>(stream));
}

bc_status bc_pack_codes(const void *W, const void *scales_f16, const void *zeros_f16,
                        int64_t N, int64_t K, int bits, uint8_t *packed, bc_stream_t stream) {
    if (!W || !scales_f16 || !zeros_f16 || !packed) return BC_ERR_INVALID_ARG;
    bc_status st = check_nk(N, K);
    if (st != BC_OK) return st;
    if (!(bits == 2 || bits == 3 || bits == 4 || bits == 8)) return BC_ERR_UNSUPPORTED;
    if (!aligned(W, 16) || !aligned(scales_f16, 2) || !aligned(zeros_f16, 2) ||
        !aligned(packed, 16))
        return BC_ERR_ALIGNMENT;
    return launch_pack_codes(static_cast<const __half *>(W),
                             static_cast<const __half *>(scales_f16),
                             static_cast<const __half *>(zeros_f16), N, K, bits, packed,
                             reinterpret_cast<cudaStream_t>(stream));
}

size_t bc_workspace_size_batched(const bc_matmul_desc *descs, int count,
                                 int64_t M, bc_mode mode, bc_dtype x_dtype) {
    if (!descs || count <= 0 || M <= 0) return 0;
    if (x_dtype == BC_BF16) return 0;      // tensor-core path needs none
    DeviceInfo di;
    if (!device_info(&di)) return 0;
    std::vector<GemvJob> jobs(count);
    for (int i = 0; i < count; ++i) {
        jobs[i].x = static_cast<const float *>(descs[i].x);   // may be null
        jobs[i].N = descs[i].N;
        jobs[i].K = descs[i].K;
        jobs[i].group = 64;
    }
    return gemv_workspace_bytes(jobs.data(), count, (int)M,
                                mode == BC_MODE_PACKED_INT4, di.sm_count);
}

size_t bc_workspace_size(int64_t M, int64_t N, int64_t K, bc_mode mode) {
    bc_matmul_desc d{};
    d.N = N;
    d.K = K;
    return bc_workspace_size_batched(&d, 1, M, mode, BC_F32);
}

bc_status bc_matmul_q_batched(const bc_matmul_desc *descs, int count,
                              int64_t M, int bits, int64_t group,
                              bc_mode mode, bc_dtype x_dtype, void *workspace,
                              size_t workspace_bytes, bc_stream_t stream) {
    return bc_matmul_q_batched_ex(descs, count, M, bits, group, mode, x_dtype, workspace,
                                  workspace_bytes, 0u, stream);
}

bc_status bc_matmul_q_batched_ex(const bc_matmul_desc *descs, int count,
                                 int64_t M, int bits, int64_t group,
                                 bc_mode mode, bc_dtype x_dtype, void *workspace,
                                 size_t workspace_bytes, unsigned flags,
                                 bc_stream_t stream) {
    if (!descs || count <= 0) return BC_ERR_INVALID_ARG;
    if (flags & ~BC_FLAG_STATIC_WEIGHTS) return BC_ERR_INVALID_ARG;
    // group rule: 64, or per channel (0)
    if (group != 64 && group != BC_GROUP_PER_CHANNEL) return BC_ERR_UNSUPPORTED;
    bc_status st = check_matmul_common(M, bits, group, mode, x_dtype);
    if (st != BC_OK) return st;
    for (int i = 0; i < count; ++i) {
        const bc_matmul_desc &d = descs[i];
        if ((st = check_nk(d.N, d.K)) != BC_OK) return st;
        if ((st = check_matmul_ptrs(d.x, x_dtype, d.W_or_packed, d.scales,
                                    d.zeros, d.y, bits, mode)) != BC_OK)
            return st;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (x_dtype == BC_BF16) {
        std::vector<GemmJob> jobs(count);
        for (int i = 0; i < count; ++i) {
            const bc_matmul_desc &d = descs[i];
            jobs[i] = GemmJob{static_cast<const __nv_bfloat16 *>(d.x), d.W_or_packed,
                              d.scales, d.zeros, d.y, d.N, d.K,
                              group == 64 ? (int64_t)64 : d.K};
        }
        return launch_gemm(jobs.data(), count, M, mode == BC_MODE_PACKED_INT4, bits,
                           mode == BC_MODE_RUNTIME_RANGE, s);
    }
    if (workspace_bytes && !workspace) return BC_ERR_INVALID_ARG;
    if (workspace && !aligned(workspace, 256)) return BC_ERR_ALIGNMENT;
    std::vector<GemvJob> jobs(count);
    for (int i = 0; i < count; ++i) {
        const bc_matmul_desc &d = descs[i];
        jobs[i] = GemvJob{static_cast<const float *>(d.x), d.W_or_packed,
                          d.scales, d.zeros, d.y, d.N, d.K,
                          group == 64 ? (int64_t)64 : d.K,
                          mode == BC_MODE_RUNTIME_RANGE ? (int64_t)1 : (int64_t)0};
    }
    if (mode == BC_MODE_PACKED_INT4 && bits != 4)
        return launch_gemv_packed(jobs.data(), count, (int)M, bits, s);
    return launch_gemv(jobs.data(), count, (int)M, bits,
                       mode == BC_MODE_PACKED_INT4, workspace, workspace_bytes,
                       s, (flags & BC_FLAG_STATIC_WEIGHTS) != 0);
}

bc_status bc_matmul_q(const void *x, bc_dtype x_dtype, const void *W_or_packed,
                      const void *scales, const void *zeros, int64_t M,
                      int64_t N, int64_t K, int bits, int64_t group,
                      bc_mode mode, float *y, void *workspace,
                      size_t workspace_bytes, bc_stream_t stream) {
    bc_status st = check_nk(N, K);
    if (st != BC_OK) return st;
    const int64_t g = normalize_group(group, K);
    if (g < 0) return BC_ERR_UNSUPPORTED;
    bc_matmul_desc d{x, W_or_packed, scales, zeros, y, N, K};
    return bc_matmul_q_batched(&d, 1, M, bits,
                               g == 64 ? 64 : BC_GROUP_PER_CHANNEL, mode,
                               x_dtype, workspace, workspace_bytes, stream);
}

size_t bc_workspace_size_argmax(int64_t M, int64_t N, int64_t K, bc_mode mode,
                                bc_dtype x_dtype) {
    if (M <= 0 || M > 65535 || N <= 0 || K <= 0 || check_nk(N, K) != BC_OK) return 0;
    const size_t yb = ((size_t)M * N * 4 + 255) / 256 * 256;
    const size_t gemv = x_dtype == BC_F32 ? bc_workspace_size(M, N, K, mode) : 0;
    return yb + argmax_partials_bytes(M, N) + gemv;
}

bc_status bc_matmul_q_argmax(const void *x, bc_dtype x_dtype, const void *W_or_packed,
                             const void *scales, const void *zeros, int64_t M,
                             int64_t N, int64_t K, int bits, int64_t group,
                             bc_mode mode, int32_t *token, void *workspace,
                             size_t workspace_bytes, bc_stream_t stream) {
    if (!token) return BC_ERR_INVALID_ARG;
    if (!aligned(token, 4)) return BC_ERR_ALIGNMENT;
    bc_status st = check_nk(N, K);
    if (st != BC_OK) return st;
    if (M <= 0 || M > 65535) return BC_ERR_INVALID_ARG;
    const size_t need = bc_workspace_size_argmax(M, N, K, mode, x_dtype);
    if (!workspace || workspace_bytes < need) return BC_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return BC_ERR_ALIGNMENT;
    // scratch: logits y [M][N], then the reduction's partials, then the
    // matmul's own workspace
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const size_t yb = ((size_t)M * N * 4 + 255) / 256 * 256;
    const size_t pb = argmax_partials_bytes(M, N);
    float *y = reinterpret_cast<float *>(ws);
    st = bc_matmul_q(x, x_dtype, W_or_packed, scales, zeros, M, N, K, bits, group, mode, y,
                     ws + yb + pb, workspace_bytes - yb - pb, stream);
    if (st != BC_OK) return st;
    return launch_argmax(y, M, N, ws + yb, token, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
