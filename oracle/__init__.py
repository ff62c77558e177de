"""fp64 CPU oracle for the fused group-wise quantize/dequantize matmul.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline / reference leg of ``bench.py`` may import this package.
The product path (``quantized_matmul_02_b200``) never imports it and shares
no code with it.

Each function restates one step of the method as the pages define it
(BITCRUSH BC-06, "Under the hood" and the NAIVE / SMART row of "The
machine"; Enargeia, "Four bits per weight"), with the spec RTN
convention scale=(max-min)/(2^b-1), zero=round(-min/scale),
q=clamp(round(w/scale)+zero, 0, 2^b-1), w'=(q-zero)*scale.  The arithmetic
itself lives in ``oracle.c`` as plain fp64 loops; this module only marshals
numpy arrays into it and composes the steps.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
(range, exact grids, hand-worked golden groups, error bound, per-group vs
per-channel MSE, one-hot / closed-form matmuls, byte ledger).  No function
is "parity unpinned".
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        i64, i32 = ctypes.c_int64, ctypes.c_int
        P = ctypes.c_void_p
        lib.oracle_group_params.argtypes = [P, i64, i64, i32, i64, i32, P, P]
        lib.oracle_codes.argtypes = [P, P, P, i64, i64, i32, i64, P]
        lib.oracle_group_range.argtypes = [P, i64, i64, i64, P, P]
        lib.oracle_dequant.argtypes = [P, P, P, i64, i64, i64, P]
        lib.oracle_pack_int4.argtypes = [P, i64, i64, P]
        lib.oracle_pack_codes.argtypes = [P, i64, i64, i32, P]
        lib.oracle_matmul.argtypes = [P, P, i64, i64, i64, P, P]
        lib.oracle_half_rows_to_double.argtypes = [P, i64, P]
        lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_half_to_double.restype = ctypes.c_double
        lib.oracle_double_to_half.argtypes = [ctypes.c_double]
        lib.oracle_double_to_half.restype = ctypes.c_uint16
        lib.oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _half_bits(W):
    W = np.ascontiguousarray(W)
    if W.dtype == np.float16:
        return W.view(np.uint16)
    if W.dtype == np.uint16:
        return W
    raise TypeError("W must be float16 (or its uint16 bit patterns)")


def threads() -> int:
    """OpenMP threads the oracle uses."""
    return int(_load().oracle_max_threads())


def group_params(W, bits: int, group: int, f16_storage: bool):
    """Per-group scale and zero, returned as float64 arrays [N][K/group].

    fp32 storage (runtime mode) -> values are exactly fp32-representable;
    fp16 storage (packed mode)  -> values are exactly fp16-representable.
    """
    Wb = _half_bits(W)
    N, K = Wb.shape
    if K % group:
        raise ValueError("K must be a multiple of group")
    G = K // group
    s = np.empty((N, G), np.float64)
    z = np.empty((N, G), np.float64)
    _load().oracle_group_params(_ptr(Wb), N, K, bits, group,
                                1 if f16_storage else 0, _ptr(s), _ptr(z))
    return s, z


def group_range(W, group: int):
    """Exact (min, max) of every group, float64 arrays [N][K/group]."""
    Wb = _half_bits(W)
    N, K = Wb.shape
    G = K // group
    lo = np.empty((N, G), np.float64)
    hi = np.empty((N, G), np.float64)
    _load().oracle_group_range(_ptr(Wb), N, K, group, _ptr(lo), _ptr(hi))
    return lo, hi


def codes(W, s, z, bits: int, group: int):
    """uint8 codes [N][K] = clamp(rne(w/s) + z, 0, 2^bits-1)."""
    Wb = _half_bits(W)
    N, K = Wb.shape
    s = np.ascontiguousarray(s, np.float64)
    z = np.ascontiguousarray(z, np.float64)
    q = np.empty((N, K), np.uint8)
    _load().oracle_codes(_ptr(Wb), _ptr(s), _ptr(z), N, K, bits, group, _ptr(q))
    return q


def dequant(q, s, z, group: int):
    """w' = (q - z) * s in fp64, [N][K]."""
    q = np.ascontiguousarray(q, np.uint8)
    N, K = q.shape
    s = np.ascontiguousarray(s, np.float64)
    z = np.ascontiguousarray(z, np.float64)
    wq = np.empty((N, K), np.float64)
    _load().oracle_dequant(_ptr(q), _ptr(s), _ptr(z), N, K, group, _ptr(wq))
    return wq


def pack_int4(q):
    """Packed bytes [N][K/2], low nibble = even k."""
    q = np.ascontiguousarray(q, np.uint8)
    N, K = q.shape
    out = np.empty((N, K // 2), np.uint8)
    _load().oracle_pack_int4(_ptr(q), N, K, _ptr(out))
    return out


def pack_codes(q, bits: int):
    """Packed bytes [N][K*bits/8]: each row a little-endian bit string, code
    k at bits [bits*k, bits*k + bits)."""
    q = np.ascontiguousarray(q, np.uint8)
    N, K = q.shape
    out = np.empty((N, K * bits // 8), np.uint8)
    _load().oracle_pack_codes(_ptr(q), N, K, bits, _ptr(out))
    return out


def half_to_f64(W):
    """Exact decode of fp16 weights (the bits=16 passthrough)."""
    Wb = _half_bits(W)
    out = np.empty(Wb.shape, np.float64)
    _load().oracle_half_rows_to_double(_ptr(Wb), Wb.size, _ptr(out))
    return out


def matmul(x, wq):
    """(y, A): y = x . wq^T and A = sum_k |x_k * wq_nk|, both fp64 [M][N]."""
    x = np.ascontiguousarray(x, np.float64)
    wq = np.ascontiguousarray(wq, np.float64)
    M, K = x.shape
    N, K2 = wq.shape
    if K != K2:
        raise ValueError("x and W disagree on K")
    y = np.empty((M, N), np.float64)
    a = np.empty((M, N), np.float64)
    _load().oracle_matmul(_ptr(x), _ptr(wq), M, N, K, _ptr(y), _ptr(a))
    return y, a


def f32_to_half_rne(v: float) -> float:
    """fp16 round-to-nearest-even of a double (oracle's own encoder)."""
    lib = _load()
    return lib.oracle_half_to_double(lib.oracle_double_to_half(float(v)))


def matmul_q(x, W, bits: int, group: int, mode: str):
    """End-to-end oracle of the fused matmul.

    mode 'runtime': fp32 scale/zero recomputed from fp16 W (bits 2..8, or 16
                    for the fp16 passthrough);
    mode 'packed' : packed codes (bits 2, 3, 4 or 8) with fp16 scale/zero per
                    64-block.
    Returns dict with y, A (tolerance scale), codes, s, z, packed (packed
    mode only).
    """
    out = {}
    if mode == "runtime" and bits == 16:
        wq = half_to_f64(W)
    else:
        f16 = mode == "packed"
        s, z = group_params(W, bits, group, f16)
        q = codes(W, s, z, bits, group)
        wq = dequant(q, s, z, group)
        out.update(s=s, z=z, codes=q)
        if f16:
            out["packed"] = pack_int4(q) if bits == 4 else pack_codes(q, bits)
    y, a = matmul(x, wq)
    out.update(y=y, A=a, wq=wq)
    return out
