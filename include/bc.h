/*
 * bc.h -- C ABI of the B200 fused group-wise quantize/dequantize matmul.
 *
 * The operation (BITCRUSH BC-06, "Under the hood"): matmul_q multiplies an
 * activation by a weight matrix whose entries are re-quantized group-wise
 * with an affine round-to-nearest (RTN) code as they are read; a separate
 * kernel precomputes one scale and one zero point per group.  The NAIVE /
 * SMART row of the same page's "The machine" table fixes the two group
 * shapes: one scale per output channel (group = K) or one per 64-weight
 * group.  Enargeia ("Four bits per weight") fixes the packed mode: int4
 * codes in blocks of 64 along the reduction axis, each block with its own
 * scale and zero point, unpacked in registers and never written back.
 *
 * Arithmetic convention (the pages leave it open):
 *   L      = 2^bits - 1
 *   scale  = fl32(fl32(max - min) / L)            over the group's fp16 weights
 *            (a constant group c takes scale |c|, or 1 when c == 0)
 *   zero   = round(-min / scale)
 *   q      = clamp(round(w / scale) + zero, 0, L)
 *   w'     = (q - zero) * scale
 *   y[m,n] = sum_k x[m,k] * w'[n,k]
 * round() is round-half-to-even of the EXACT real quotient.  fp16-stored
 * parameters (packed mode) round the fp32 scale to fp16 (RNE, floored at
 * 2^-24), derive zero and codes from that stored scale, and store zero as
 * fp16 (RNE).
 *
 * Layouts (all row-major, C order):
 *   W       fp16 [N][K]            (PyTorch Linear weight: N = out, K = in)
 *   scales  [N][K/group]           fp32 (runtime mode) or fp16 (packed mode)
 *   zeros   [N][K/group]           same dtype as scales
 *   codes   uint8 [N][K]
 *   packed  uint8 [N][K/2]         byte = q[n][2i] | q[n][2i+1] << 4
 *   x       [M][K]                 fp32, or bf16 for the tensor-core path
 *   y       fp32 [M][N]
 *
 * Conventions shared by every call:
 *   - Pointers named W, x, y, scales, zeros, codes, packed, workspace are
 *     DEVICE pointers owned by the caller; the library never allocates,
 *     frees or keeps them, and keeps no per-call device state.
 *   - Calls only enqueue work on `stream` (NULL = legacy default stream)
 *     and return without synchronising.  Arguments are validated on the
 *     host before anything is enqueued; a rejected call enqueues nothing.
 *   - Launch failures are reported as BC_ERR_CUDA (cudaGetLastError); an
 *     asynchronous fault surfaces at the caller's next synchronisation.
 *   - K must be a multiple of 64; W, x and packed must be 16-byte aligned;
 *     scales/zeros aligned to their element size; y 4-byte aligned.
 *   - Inputs must be finite (no NaN / Inf weights or activations).
 *   - No call throws; nothing falls back to the CPU.
 */
#ifndef BC_H_
#define BC_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define BC_API __attribute__((visibility("default")))
#else
#define BC_API
#endif

/* Same object as cudaStream_t. */
typedef struct CUstream_st *bc_stream_t;

typedef enum bc_status {
    BC_OK = 0,
    BC_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, K % 64 != 0 */
    BC_ERR_UNSUPPORTED = 2,   /* bits / group / mode / dtype combination not offered */
    BC_ERR_ALIGNMENT = 3,     /* a pointer is not aligned as stated above */
    BC_ERR_WORKSPACE = 4,     /* workspace smaller than bc_workspace_size() */
    BC_ERR_CUDA = 5           /* a CUDA launch or runtime call failed */
} bc_status;

typedef enum bc_dtype { BC_F32 = 0, BC_F16 = 1, BC_BF16 = 2 } bc_dtype;

typedef enum bc_mode {
    BC_MODE_RUNTIME = 0,      /* fp16 W re-quantized inline to `bits` (2..8), or 16 = passthrough */
    BC_MODE_PACKED_INT4 = 1,  /* pre-packed codes, fp16 scale/zero per 64-block: int4, or
                                 2, 3 and 8 bits (bc_pack_codes) on the decode path */
    BC_MODE_PACKED = 1,       /* the same mode under its width-neutral name */
    BC_MODE_RUNTIME_RANGE = 2 /* as BC_MODE_RUNTIME, but `scales` holds each group's range
                                 (bc_group_minmax) and the kernel derives scale and zero
                                 for `bits` itself; `zeros` is unused (may be NULL) */
} bc_mode;

/* Per-channel grouping may be requested as group == K or group == 0. */
#define BC_GROUP_PER_CHANNEL 0

/*
 * bc_group_params -- per-group scale/zero precompute (BITCRUSH BC-06,
 * "Under the hood": the per-group scale/zero precompute kernel; a change
 * of bit width reruns it once, then decoding only passes the new bits).
 *   W          fp16 [N][K], device
 *   bits       2..8
 *   group      64, or K / 0 for per-channel
 *   out_dtype  BC_F32 (runtime mode) or BC_F16 (packed int4 mode)
 *   scales     [N][K/group] of out_dtype, device, written
 *   zeros      [N][K/group] of out_dtype, device, written
 */
BC_API bc_status bc_group_params(const void *W, int64_t N, int64_t K, int bits,
                          int64_t group, bc_dtype out_dtype, void *scales,
                          void *zeros, bc_stream_t stream);

/*
 * bc_group_minmax -- the bit-width-independent form of the precompute
 * (BITCRUSH BC-06, "Under the hood": after the precompute, a change of bit
 * width costs one kernel argument).  Stores each group's range, so that
 * BC_MODE_RUNTIME_RANGE matmuls derive scale and zero for any `bits` from it
 * with the fp32 arithmetic of bc_group_params: their codes are bit-identical
 * to those of the (scale, zero) that bc_group_params(..., bits, ..., BC_F32)
 * stores, and moving the lever reruns nothing.
 *   W       fp16 [N][K], device
 *   group   64, or K / 0 for per-channel
 *   ranges  uint32 [N][K/group], device, written: fp16 min in the low half,
 *           fp16 max in the high half (both exact: they are weights)
 */
BC_API bc_status bc_group_minmax(const void *W, int64_t N, int64_t K, int64_t group,
                                 void *ranges, bc_stream_t stream);

/*
 * bc_quantize_codes -- the RTN codes q = clamp(round(w/scale)+zero, 0, L)
 * as a standalone output (the same codes matmul_q forms inline; BITCRUSH
 * BC-06, "Under the hood").  Used for validation and the WEIGHT SCOPE-style
 * code histogram.
 *   W        fp16 [N][K], device
 *   scales, zeros  [N][K/group], dtype sz_dtype (BC_F32 or BC_F16), device
 *   codes    uint8 [N][K], device, written
 */
BC_API bc_status bc_quantize_codes(const void *W, const void *scales,
                            const void *zeros, bc_dtype sz_dtype, int64_t N,
                            int64_t K, int bits, int64_t group,
                            uint8_t *codes, bc_stream_t stream);

/*
 * bc_pack_int4 -- one-time int4 packing (Enargeia, "Four bits per weight":
 * four bits per weight, blocks of 64 along K with their own scale and
 * zero point).
 *   W                  fp16 [N][K], device
 *   scales_f16, zeros_f16  fp16 [N][K/64] from bc_group_params(..., BC_F16)
 *   packed             uint8 [N][K/2], device, written; low nibble = even k
 */
BC_API bc_status bc_pack_int4(const void *W, const void *scales_f16,
                       const void *zeros_f16, int64_t N, int64_t K,
                       uint8_t *packed, bc_stream_t stream);

/*
 * bc_pack_codes -- one-time packing at other code widths (Enargeia,
 * "Honestly": an int8 tied embedding; BITCRUSH BC-06, "The machine", BRAIN
 * SIZE: 2-bit weights), so that decode bytes fall with the bit width.
 *   W                  fp16 [N][K], device
 *   scales_f16, zeros_f16  fp16 [N][K/64] from bc_group_params(..., bits,
 *                      64, BC_F16, ...)
 *   bits               2, 3, 4 or 8
 *   packed             uint8 [N][K*bits/8], device, written: each row a
 *                      little-endian bit string, code k at bits
 *                      [bits*k, bits*k + bits) (bits = 4 is bc_pack_int4's
 *                      layout; a 64-group takes 8*bits bytes)
 * Matmuls over these codes use BC_MODE_PACKED with the same `bits`; widths
 * other than 4 take fp32 x (the decode GEMV, any M).
 */
BC_API bc_status bc_pack_codes(const void *W, const void *scales_f16,
                               const void *zeros_f16, int64_t N, int64_t K, int bits,
                               uint8_t *packed, bc_stream_t stream);

/*
 * bc_matmul_q -- y = x . deq(W)^T (BITCRUSH BC-06 matmul_q; Enargeia int4
 * weights unpacked in registers).
 *   x, x_dtype   [M][K]: BC_F32 for any M; BC_BF16 for M >= 64 in every
 *                mode (tensor-core prefill, fp32 accumulate: packed codes, or
 *                fp16 weights re-quantized inline at 2..8 bits / passed
 *                through at 16)
 *   W_or_packed  fp16 W [N][K] (runtime) or packed uint8 [N][K*bits/8] (packed)
 *   scales, zeros  fp32 [N][K/group] (runtime) or fp16 [N][K/64] (packed);
 *                BC_MODE_RUNTIME_RANGE: scales = uint32 ranges [N][K/group]
 *                from bc_group_minmax, zeros unused;
 *                ignored (may be NULL) when bits == 16
 *   bits         runtime: 2..8 or 16 (fp16 passthrough); packed: 4, or 2, 3, 8
 *                with fp32 x
 *   group        runtime: 64, or K / 0 (per channel); packed: 64
 *   y            fp32 [M][N], device, written (not accumulated into)
 *   workspace    device scratch of at least bc_workspace_size() bytes
 *                (may be NULL when that size is 0); its contents on entry
 *                do not matter; overlapping calls must not share it
 * Decode shapes (M < 64, fp32 x) use the fused dequant GEMV: launches that
 * can fill the GPU run the streaming decode kernels (M <= 4 on the int8
 * tensor cores; M = 5..16 on the tcgen05 decode kernel, packed or runtime at
 * 2..8 bits, whose workspace holds the split activations of each x); M >= 64
 * with bf16 x uses the tcgen05 tensor-core GEMM (no workspace).
 */
BC_API bc_status bc_matmul_q(const void *x, bc_dtype x_dtype, const void *W_or_packed,
                      const void *scales, const void *zeros, int64_t M,
                      int64_t N, int64_t K, int bits, int64_t group,
                      bc_mode mode, float *y, void *workspace,
                      size_t workspace_bytes, bc_stream_t stream);

/* Workspace bytes bc_matmul_q needs for this shape (0 if none). */
BC_API size_t bc_workspace_size(int64_t M, int64_t N, int64_t K, bc_mode mode);

/*
 * One matrix of a grouped launch.  All pointers are device pointers with
 * the layouts above; several descriptors may share one x.
 */
typedef struct bc_matmul_desc {
    const void *x;
    const void *W_or_packed;
    const void *scales;
    const void *zeros;
    float *y;
    int64_t N;
    int64_t K;
} bc_matmul_desc;

/*
 * bc_matmul_q_batched -- one grouped launch over many independent matrices
 * that share M, bits, group rule, mode and x dtype (a whole layer set).
 * Enargeia ("One decode step") shows that a decode step is a list of
 * hundreds of small passes; launching them one by one costs more than the
 * work of the small ones.
 *   descs   HOST array of `count` descriptors (read before return)
 *   group   64, or 0 for per-channel (each matrix uses its own K)
 *   workspace  as for bc_matmul_q, at least bc_workspace_size_batched()
 */
BC_API bc_status bc_matmul_q_batched(const bc_matmul_desc *descs, int count,
                              int64_t M, int bits, int64_t group,
                              bc_mode mode, bc_dtype x_dtype, void *workspace,
                              size_t workspace_bytes, bc_stream_t stream);

/*
 * bc_workspace_size_batched -- scratch bytes a bc_matmul_q_batched call over
 * these descriptors needs.  Reads N, K and x of each descriptor: matrices
 * that name the same non-null x (and K) share scratch, and a size computed
 * with x = NULL holds for any x pointers of a later call with the same N, K.
 * Returns 0 for arguments the call would reject, and for calls that need no
 * scratch (bf16 x, and the streaming decode kernel at M <= 4).
 */
BC_API size_t bc_workspace_size_batched(const bc_matmul_desc *descs, int count,
                                 int64_t M, bc_mode mode, bc_dtype x_dtype);

/*
 * Flags of bc_matmul_q_batched_ex.
 *   BC_FLAG_STATIC_WEIGHTS  the caller promises that no work still pending
 *     (on `stream` or elsewhere) writes any descriptor's weights, scales or
 *     zeros -- the usual case for a model's weights during decoding.  The
 *     decode kernel is then launched as a programmatic dependent launch: its
 *     CTAs may start, and stream weights, scales and zeros, while the kernel
 *     before it on the stream is still finishing; every read of x and write
 *     of y still waits until that kernel has completed.  Back-to-back decode
 *     steps then overlap one step's start with the previous step's end.
 *     Ignored by the prefill (bf16 x) path and the small-launch GEMV.
 */
#define BC_FLAG_STATIC_WEIGHTS 1u

/*
 * bc_matmul_q_batched_ex -- bc_matmul_q_batched with `flags` (a bitwise OR
 * of BC_FLAG_* values; unknown bits are rejected with BC_ERR_INVALID_ARG).
 * flags = 0 is exactly bc_matmul_q_batched.
 */
BC_API bc_status bc_matmul_q_batched_ex(const bc_matmul_desc *descs, int count,
                                 int64_t M, int bits, int64_t group,
                                 bc_mode mode, bc_dtype x_dtype, void *workspace,
                                 size_t workspace_bytes, unsigned flags,
                                 bc_stream_t stream);

/*
 * bc_matmul_q_noalloc -- the decode matmul (fp32 x, the GEMV path of
 * bc_matmul_q) for callers that cannot allocate device memory: code that
 * must not call cudaMalloc (a host callback, a fixed-pool allocator, a
 * plugin that only receives its input and output pointers) and so cannot
 * supply bc_matmul_q's workspace.  The paper has no counterpart; this is a
 * deployment variant of the same computation.
 *   Arguments mean what they mean for bc_matmul_q with x_dtype = BC_F32.
 *   Scratch: instead of a caller workspace, the split-K partial sums and
 *   tickets (and the split activations of the tcgen05 decode kernel) live
 *   in a fixed 4 MiB array inside the library (a __device__
 *   object that every GPU loading the library holds until process exit).
 *   Shapes whose scratch would exceed it are rejected with
 *   BC_ERR_WORKSPACE before anything is enqueued.  The call allocates
 *   nothing (no cudaMalloc/cudaFree, no allocating library routine).
 *   Set-up: the first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture on that device.
 *   Sharing: all calls share the one array, which keeps the last call's
 *   contents (the counters that must start at zero are cleared by each
 *   call).  Calls that can overlap on the GPU -- on different streams, or
 *   from different threads without ordering -- race on the array and give
 *   wrong results; serialise them (e.g. one stream).
 *   Device reset: the looked-up address belongs to the device's context at
 *   the time of the first call; after cudaDeviceReset on that device this
 *   entry point (like the library's other cached per-device state, such as
 *   kernel shared-memory attributes) is not valid in this process.
 */
BC_API bc_status bc_matmul_q_noalloc(const void *x, const void *W_or_packed,
                                     const void *scales, const void *zeros,
                                     int64_t M, int64_t N, int64_t K, int bits,
                                     int64_t group, bc_mode mode, float *y,
                                     bc_stream_t stream);

/*
 * bc_matmul_q_argmax -- greedy token selection: for each row m of
 * y = x . deq(W)^T, the index n of its largest value (ties go to the lowest
 * index).  Enargeia ("One decode step"): a decode step ends in a single
 * GPU -> CPU readback that carries one token id; BITCRUSH BC-06 ("Honest
 * notes") decodes greedily.  Typically W is the LM head (Qwen3-0.6B's tied
 * head: K = 1024, N = 151936, fp16 passthrough with bits = 16).
 *   Arguments other than `token` mean what they mean for bc_matmul_q
 *   (M <= 65535).
 *   token      int32 [M], device, written
 *   workspace  device scratch of at least bc_workspace_size_argmax() bytes,
 *              256-byte aligned: it holds the logits (M x N fp32), the
 *              reduction's partials and the matmul's own workspace; its
 *              contents on entry do not matter
 * Enqueues the matmul and two reduction kernels on `stream`.
 */
BC_API bc_status bc_matmul_q_argmax(const void *x, bc_dtype x_dtype, const void *W_or_packed,
                                    const void *scales, const void *zeros, int64_t M,
                                    int64_t N, int64_t K, int bits, int64_t group,
                                    bc_mode mode, int32_t *token, void *workspace,
                                    size_t workspace_bytes, bc_stream_t stream);

/* Workspace bytes bc_matmul_q_argmax needs for this shape (0 if the shape
 * would be rejected). */
BC_API size_t bc_workspace_size_argmax(int64_t M, int64_t N, int64_t K, bc_mode mode,
                                       bc_dtype x_dtype);

/*
 * bc_device_timeouts -- number of bounded in-kernel waits (tensor-core
 * pipeline barriers) that ran out on the current device since the library
 * was loaded.  A kernel whose wait runs out stops early, frees its tensor
 * memory and leaves its outputs incomplete instead of hanging the GPU; a
 * nonzero count means some earlier output is not valid.  Synchronises the
 * device.  `count` is a HOST pointer.
 */
BC_API bc_status bc_device_timeouts(unsigned *count);

/*
 * bc_set_wait_limit -- limit of the bounded in-kernel pipeline waits on the
 * current device, in SM clock cycles (0 restores the default of about 2 s,
 * the maximum).  For tests of the failure path: a limit shorter than a
 * pipeline stage makes the kernels' waits run out, so they record timeouts
 * (bc_device_timeouts), stop early and leave their outputs incomplete --
 * after waiting, with the default limit, for their own copies and MMAs in
 * flight and freeing their tensor memory.  Synchronises the device.
 */
BC_API bc_status bc_set_wait_limit(uint64_t cycles);

/* Static description of a status code. */
BC_API const char *bc_status_string(bc_status status);

/* Library version, major*10000 + minor*100 + patch. */
BC_API int bc_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BC_H_ */
