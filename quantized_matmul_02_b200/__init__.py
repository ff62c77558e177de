"""Python binding of libbc.so, the B200 fused group-wise dequant matmul.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/bc.h``.  PyTorch supplies the
device memory and the current stream.  There is no CPU fallback: importing
this package on a machine without the built library raises.

Functions (same names as the C entry points, without the ``bc_`` prefix):
    group_params, quantize_codes, pack_int4, matmul_q, matmul_q_batched,
    workspace_size, workspace_size_batched
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbc.so")

BC_OK, BC_ERR_INVALID_ARG, BC_ERR_UNSUPPORTED, BC_ERR_ALIGNMENT, \
    BC_ERR_WORKSPACE, BC_ERR_CUDA = range(6)
BC_F32, BC_F16, BC_BF16 = 0, 1, 2
BC_MODE_RUNTIME, BC_MODE_PACKED_INT4, BC_MODE_RUNTIME_RANGE = 0, 1, 2
BC_MODE_PACKED = BC_MODE_PACKED_INT4
GROUP_PER_CHANNEL = 0
BC_FLAG_STATIC_WEIGHTS = 1

# Every symbol include/bc.h declares.
EXPORTS = ("bc_group_params", "bc_group_minmax", "bc_quantize_codes", "bc_pack_int4",
           "bc_pack_codes",
           "bc_matmul_q", "bc_workspace_size", "bc_matmul_q_batched",
           "bc_matmul_q_batched_ex",
           "bc_workspace_size_batched", "bc_matmul_q_noalloc",
           "bc_matmul_q_argmax", "bc_workspace_size_argmax",
           "bc_device_timeouts", "bc_set_wait_limit",
           "bc_status_string", "bc_version")


class BCError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} (status {status})")
        self.status = status


class MatmulDesc(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("W_or_packed", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("zeros", ctypes.c_void_p),
                ("y", ctypes.c_void_p), ("N", ctypes.c_int64),
                ("K", ctypes.c_int64)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python quantized_matmul_02_b200/build.py` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    P, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    lib.bc_group_params.argtypes = [P, i64, i64, i32, i64, i32, P, P, P]
    lib.bc_quantize_codes.argtypes = [P, P, P, i32, i64, i64, i32, i64, P, P]
    lib.bc_group_minmax.argtypes = [P, i64, i64, i64, P, P]
    lib.bc_group_minmax.restype = i32
    lib.bc_pack_int4.argtypes = [P, P, P, i64, i64, P, P]
    lib.bc_pack_codes.argtypes = [P, P, P, i64, i64, i32, P, P]
    lib.bc_pack_codes.restype = i32
    lib.bc_matmul_q.argtypes = [P, i32, P, P, P, i64, i64, i64, i32, i64, i32,
                                P, P, sz, P]
    lib.bc_workspace_size.argtypes = [i64, i64, i64, i32]
    lib.bc_workspace_size.restype = sz
    lib.bc_matmul_q_batched.argtypes = [ctypes.POINTER(MatmulDesc), i32, i64,
                                        i32, i64, i32, i32, P, sz, P]
    lib.bc_matmul_q_batched_ex.argtypes = [ctypes.POINTER(MatmulDesc), i32, i64,
                                           i32, i64, i32, i32, P, sz, ctypes.c_uint, P]
    lib.bc_workspace_size_batched.argtypes = [ctypes.POINTER(MatmulDesc), i32,
                                              i64, i32, i32]
    lib.bc_workspace_size_batched.restype = sz
    lib.bc_matmul_q_noalloc.argtypes = [P, P, P, P, i64, i64, i64, i32, i64,
                                        i32, P, P]
    lib.bc_matmul_q_noalloc.restype = i32
    lib.bc_matmul_q_argmax.argtypes = [P, i32, P, P, P, i64, i64, i64, i32, i64, i32,
                                       P, P, sz, P]
    lib.bc_matmul_q_argmax.restype = i32
    lib.bc_workspace_size_argmax.argtypes = [i64, i64, i64, i32, i32]
    lib.bc_workspace_size_argmax.restype = sz
    lib.bc_set_wait_limit.argtypes = [ctypes.c_uint64]
    lib.bc_set_wait_limit.restype = i32
    lib.bc_device_timeouts.argtypes = [ctypes.POINTER(ctypes.c_uint)]
    lib.bc_device_timeouts.restype = i32
    lib.bc_status_string.argtypes = [i32]
    lib.bc_status_string.restype = ctypes.c_char_p
    lib.bc_version.restype = i32
    for name in ("bc_group_params", "bc_quantize_codes", "bc_pack_int4",
                 "bc_matmul_q", "bc_matmul_q_batched", "bc_matmul_q_batched_ex"):
        getattr(lib, name).restype = i32
    return lib


lib = _load()


def status_string(status: int) -> str:
    return lib.bc_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != BC_OK:
        raise BCError(status, what)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


_DT = {torch.float32: BC_F32, torch.float16: BC_F16, torch.bfloat16: BC_BF16}


def group_params(W: torch.Tensor, bits: int, group: int, out_dtype=torch.float32,
                 scales: Optional[torch.Tensor] = None,
                 zeros: Optional[torch.Tensor] = None, stream=None):
    """Per-group scale/zero of fp16 W [N][K]; returns (scales, zeros)."""
    N, K = W.shape
    g = K if group in (0, K) else group
    if scales is None:
        scales = torch.empty((N, K // g), dtype=out_dtype, device=W.device)
    if zeros is None:
        zeros = torch.empty((N, K // g), dtype=out_dtype, device=W.device)
    _check(lib.bc_group_params(_ptr(W), N, K, bits, group, _DT[out_dtype],
                               _ptr(scales), _ptr(zeros), _stream(stream)),
           "bc_group_params")
    return scales, zeros


def group_minmax(W: torch.Tensor, group: int, ranges: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    """Per-group range of fp16 W [N][K] as int32 words [N][K/group] (fp16 min
    in the low half, fp16 max in the high half), for BC_MODE_RUNTIME_RANGE."""
    N, K = W.shape
    g = K if group in (0, K) else group
    if ranges is None:
        ranges = torch.empty((N, K // g), dtype=torch.int32, device=W.device)
    _check(lib.bc_group_minmax(_ptr(W), N, K, group, _ptr(ranges), _stream(stream)),
           "bc_group_minmax")
    return ranges


def quantize_codes(W: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
                   bits: int, group: int, codes: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    N, K = W.shape
    if codes is None:
        codes = torch.empty((N, K), dtype=torch.uint8, device=W.device)
    _check(lib.bc_quantize_codes(_ptr(W), _ptr(scales), _ptr(zeros),
                                 _DT[scales.dtype], N, K, bits, group,
                                 _ptr(codes), _stream(stream)),
           "bc_quantize_codes")
    return codes


def pack_int4(W: torch.Tensor, scales_f16: torch.Tensor, zeros_f16: torch.Tensor,
              packed: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    N, K = W.shape
    if packed is None:
        packed = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    _check(lib.bc_pack_int4(_ptr(W), _ptr(scales_f16), _ptr(zeros_f16), N, K,
                            _ptr(packed), _stream(stream)), "bc_pack_int4")
    return packed


def pack_codes(W: torch.Tensor, scales_f16: torch.Tensor, zeros_f16: torch.Tensor,
               bits: int, packed: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Packed codes of `bits` (2, 3, 4, 8) bits: uint8 [N][K*bits/8]."""
    N, K = W.shape
    if packed is None:
        packed = torch.empty((N, K * bits // 8), dtype=torch.uint8, device=W.device)
    _check(lib.bc_pack_codes(_ptr(W), _ptr(scales_f16), _ptr(zeros_f16), N, K, bits,
                             _ptr(packed), _stream(stream)), "bc_pack_codes")
    return packed


def workspace_size(M: int, N: int, K: int, mode: int) -> int:
    return int(lib.bc_workspace_size(M, N, K, mode))


def matmul_q(x: torch.Tensor, W: torch.Tensor, scales: Optional[torch.Tensor],
             zeros: Optional[torch.Tensor], bits: int, group: int, mode: int,
             y: Optional[torch.Tensor] = None,
             workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """y = x . deq(W)^T.  W is fp16 [N][K] (runtime) or packed uint8 [N][K/2]."""
    M, K = x.shape
    N = W.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=x.device)
    need = workspace_size(M, N, K, mode) if x.dtype == torch.float32 else 0
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    wsp = _ptr(workspace) if workspace is not None else None
    wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib.bc_matmul_q(_ptr(x), _DT[x.dtype], _ptr(W), _ptr(scales),
                           _ptr(zeros), M, N, K, bits, group, mode, _ptr(y),
                           wsp, wsb, _stream(stream)), "bc_matmul_q")
    return y


def make_descs(items: Sequence[tuple]) -> ctypes.Array:
    """items: (x, W_or_packed, scales, zeros, y) tensors per matrix."""
    arr = (MatmulDesc * len(items))()
    for i, (x, W, s, z, y) in enumerate(items):
        arr[i] = MatmulDesc(_ptr(x), _ptr(W), _ptr(s), _ptr(z), _ptr(y),
                            y.shape[1], x.shape[1])
    return arr


def workspace_size_batched(descs, M: int, mode: int, x_dtype: int) -> int:
    return int(lib.bc_workspace_size_batched(descs, len(descs), M, mode, x_dtype))


def matmul_q_batched(descs, M: int, bits: int, group: int, mode: int,
                     x_dtype: int = BC_F32, workspace: Optional[torch.Tensor] = None,
                     stream=None, static_weights: bool = False) -> None:
    """One grouped launch over the matrices in `descs` (from make_descs).
    Without `workspace`, split-K scratch (if any) is taken from torch.
    static_weights: BC_FLAG_STATIC_WEIGHTS (no pending work writes the
    weights, scales or zeros; the decode kernel may then start before the
    previous kernel on the stream has finished)."""
    if workspace is None:
        need = workspace_size_batched(descs, M, mode, x_dtype)
        if need:
            workspace = torch.empty(need, dtype=torch.uint8, device="cuda")
    wsp = _ptr(workspace) if workspace is not None else None
    wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    flags = BC_FLAG_STATIC_WEIGHTS if static_weights else 0
    _check(lib.bc_matmul_q_batched_ex(descs, len(descs), M, bits, group, mode,
                                      x_dtype, wsp, wsb, flags, _stream(stream)),
           "bc_matmul_q_batched_ex")


def device_timeouts() -> int:
    """Bounded in-kernel waits that ran out on this device (0 when healthy)."""
    c = ctypes.c_uint(0)
    _check(lib.bc_device_timeouts(ctypes.byref(c)), "bc_device_timeouts")
    return int(c.value)


def set_wait_limit(cycles: int) -> None:
    """bc_set_wait_limit: the in-kernel wait limit in cycles (0 = default)."""
    _check(lib.bc_set_wait_limit(int(cycles)), "bc_set_wait_limit")


def matmul_q_noalloc(x: torch.Tensor, W: torch.Tensor,
                     scales: Optional[torch.Tensor], zeros: Optional[torch.Tensor],
                     bits: int, group: int, mode: int, y: torch.Tensor,
                     stream=None) -> torch.Tensor:
    """bc_matmul_q_noalloc: the fp32-x decode matmul using the library's own
    fixed scratch instead of a workspace (for callers that cannot allocate).
    `y` must be supplied; nothing is allocated by this call."""
    M, K = x.shape
    N = W.shape[0]
    # The C call reads x as fp32 [M][K] and writes y as fp32 [M][N]: anything
    # else would be read or written out of bounds, so refuse it here.
    if x.dtype != torch.float32 or y.dtype != torch.float32:
        raise ValueError("matmul_q_noalloc: x and y must be float32")
    if tuple(y.shape) != (M, N):
        raise ValueError(f"matmul_q_noalloc: y must have shape {(M, N)}")
    devs = {t.device for t in (x, W, y, scales, zeros) if t is not None}
    if len(devs) != 1 or not next(iter(devs)).type == "cuda":
        raise ValueError("matmul_q_noalloc: all tensors must be on one CUDA device")
    _check(lib.bc_matmul_q_noalloc(_ptr(x), _ptr(W), _ptr(scales), _ptr(zeros),
                                   M, N, K, bits, group, mode, _ptr(y),
                                   _stream(stream)), "bc_matmul_q_noalloc")
    return y


def workspace_size_argmax(M: int, N: int, K: int, mode: int, x_dtype: int = BC_F32) -> int:
    return int(lib.bc_workspace_size_argmax(M, N, K, mode, x_dtype))


def matmul_q_argmax(x: torch.Tensor, W: torch.Tensor, scales: Optional[torch.Tensor],
                    zeros: Optional[torch.Tensor], bits: int, group: int, mode: int,
                    token: Optional[torch.Tensor] = None,
                    workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """bc_matmul_q_argmax: int32 [M], per row of x the index of the largest
    output of x . deq(W)^T (lowest index among equal values)."""
    M, K = x.shape
    N = W.shape[0]
    if token is None:
        token = torch.empty((M,), dtype=torch.int32, device=x.device)
    need = workspace_size_argmax(M, N, K, mode, _DT[x.dtype])
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=x.device)
    _check(lib.bc_matmul_q_argmax(_ptr(x), _DT[x.dtype], _ptr(W), _ptr(scales), _ptr(zeros),
                                  M, N, K, bits, group, mode, _ptr(token), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(),
                                  _stream(stream)), "bc_matmul_q_argmax")
    return token
