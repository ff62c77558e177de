// bc_noalloc.cu -- bc_matmul_q_noalloc: the decode matmul for callers that
// cannot allocate device memory.
//
// Some callers have no way to hand the library a workspace: code that runs
// where cudaMalloc is forbidden or unavailable (inside a host callback, under
// an allocator that must not grow, in a plugin that only receives its input
// and output pointers).  bc_matmul_q needs caller-provided scratch when it
// splits K for a small matrix; this entry point instead uses a fixed scratch
// array that lives in the library image itself.
//
// The array below is a file-scope __device__ object: every GPU that loads
// this library holds its kNoAllocScratchBytes until the process exits.  In
// host code its name is only a host-side stand-in, not a device address, so
// the address passed to kernels comes from cudaGetSymbolAddress, looked up
// once per device (with that device current) on the first call made on it.
#include "bc_internal.cuh"

#include <mutex>

namespace bc {
namespace {

// Upper bound of split-K scratch (partial sums + tickets) one call may use.
constexpr size_t kNoAllocScratchBytes = 4u << 20;     // 4 MiB per device

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (set-up on the
// first call per device).  Returns nullptr on failure.
void *scratch_on_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess)
            return nullptr;
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace bc

using namespace bc;

extern "C" bc_status bc_matmul_q_noalloc(const void *x, const void *W_or_packed,
                                         const void *scales, const void *zeros,
                                         int64_t M, int64_t N, int64_t K, int bits,
                                         int64_t group, bc_mode mode, float *y,
                                         bc_stream_t stream) {
    if (N <= 0 || K <= 0 || K % 64 || M <= 0 || !x || !W_or_packed || !y)
        return BC_ERR_INVALID_ARG;
    // Sizes whose split-K scratch would exceed the fixed array are refused.
    if (bc_workspace_size(M, N, K, mode) > kNoAllocScratchBytes)
        return BC_ERR_WORKSPACE;
    void *scratch = scratch_on_current_device();
    if (!scratch) return BC_ERR_CUDA;
    return bc_matmul_q(x, BC_F32, W_or_packed, scales, zeros, M, N, K, bits,
                       group, mode, y, scratch, kNoAllocScratchBytes, stream);
}
