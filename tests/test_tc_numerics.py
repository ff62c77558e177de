"""CPU model of the arithmetic of the tensor-core decode kernel (5..16 x rows),
checked against the oracle.

The kernel computes s * sum_k (q_k - z) x_k per 64-group from:
  * x split into two bf16 pieces, hi = bf16(x) and lo = bf16(x - hi), and
    x~ = hi + lo;
  * A = 1 + q/16 (packed codes) or A = q (runtime codes), exact in bf16;
  * D = sum_k A_k * piece_k in fp32 per piece, in steps of 16 k (one MMA);
  * X~ = the group's sum of x~, computed in fp64 and rounded once to fp32;
  * y += c1 * (D_hi + D_lo) + c2 * X~, with c1 = 16 s and c2 = -s (16 + z)
    (packed), or c1 = s and c2 = -s z (runtime).
This model has no blocking beyond that: one MMA step, a fp32 rounding per
step.  These tests pin the decomposition and the error budget, not the CUDA
code.  The bound asserted is 2e-5 * A, five times inside the 1e-4 * A
acceptance bar.  Mistakes in the decomposition fail it by orders of
magnitude: a single bf16 piece (2^-9 relative), a dropped zero term, or a
wrong scale of the zero term.
"""
import numpy as np
import pytest

import oracle
import workloads as wl

TIGHT = 2e-5


def bf16(v):
    return wl.bf16_to_f32(wl.bf16_bits(np.asarray(v, np.float32)))


def model(x, q, s, z, mode):
    M, K = x.shape
    N = q.shape[0]
    x32 = x.astype(np.float32)
    hi = bf16(x32)
    lo = bf16((x32 - hi).astype(np.float32))
    y = np.zeros((M, N), np.float32)
    for g in range(K // 64):
        sl = slice(64 * g, 64 * g + 64)
        qg = q[:, sl].astype(np.float64)
        A = 1.0 + qg / 16.0 if mode == "packed" else qg
        assert np.array_equal(bf16(A), A.astype(np.float32)), "A must be exact in bf16"
        D = np.zeros((2, N, M), np.float32)
        for p, piece in enumerate((hi, lo)):
            for kk in range(4):
                c = slice(16 * kk, 16 * kk + 16)
                step = A[:, c] @ piece[:, sl][:, c].T.astype(np.float64)   # exact products
                D[p] = (D[p] + step.astype(np.float32)).astype(np.float32)
        Xt = (hi[:, sl].astype(np.float64) + lo[:, sl].astype(np.float64)).sum(axis=1)
        Xt = Xt.astype(np.float32)                                          # [M]
        sc = s[:, g].astype(np.float32)
        zc = z[:, g].astype(np.float32)
        if mode == "packed":
            c1 = np.float32(16.0) * sc
            c2 = -sc * (np.float32(16.0) + zc)
        else:
            c1 = sc
            c2 = -sc * zc
        Dsum = (D[0] + D[1]).T                                              # [M][N]
        y = (c1[None, :] * Dsum + (c2[None, :] * Xt[:, None] + y)).astype(np.float32)
    return y


def case(mode, bits, x, W):
    ref = oracle.matmul_q(x, W, bits, 64, mode)
    y = model(x, ref["codes"], ref["s"], ref["z"], mode)
    err = np.abs(y.astype(np.float64) - ref["y"])
    return err, ref["A"]


@pytest.mark.parametrize("mode,bits", [("packed", 4), ("runtime", 3), ("runtime", 8)])
def test_tc_decomposition_within_tight_bound(mode, bits):
    rng = np.random.default_rng(7 + bits)
    N, K, M = 48, 320, 16
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    x = wl.activation(21, bits, "x", M, K)
    err, A = case(mode, bits, x, W)
    assert np.all(err <= TIGHT * A), float((err / A).max())


@pytest.mark.parametrize("mode,bits", [("packed", 4), ("runtime", 5)])
def test_tc_decomposition_activation_outliers(mode, bits):
    """Two-piece activations keep 16 bits of every element relative to its
    own magnitude: a 10^4 outlier per group and a 1e-30 value cost nothing."""
    rng = np.random.default_rng(30 + bits)
    N, K, M = 32, 256, 8
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    x = wl.activation(22, bits, "x", M, K).copy()
    x[:, ::64] *= 1.0e4
    x[:, 5::64] = 1.0e-30
    err, A = case(mode, bits, x, W)
    assert np.all(err <= TIGHT * A), float((err / A).max())


def test_tc_single_piece_would_fail():
    """The same decomposition with only hi = bf16(x) misses the bar: the
    second piece is needed."""
    rng = np.random.default_rng(99)
    N, K, M = 48, 320, 16
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    x = wl.activation(23, 0, "x", M, K)
    ref = oracle.matmul_q(x, W, 4, 64, "packed")
    y1 = model(bf16(x.astype(np.float32)), ref["codes"], ref["s"], ref["z"], "packed")
    err = np.abs(y1.astype(np.float64) - ref["y"])
    assert np.any(err > 1e-4 * ref["A"])


def test_tc_packed_a_encoding_bits():
    """A = 1 + q/16 in bf16 is 0x3F80 with the code in mantissa bits 3..6,
    which is what one shift and one LOP3 per output word produce."""
    for q in range(16):
        assert int(wl.bf16_bits(np.array([1.0 + q / 16.0], np.float32))[0]) == 0x3F80 | (q << 3)
