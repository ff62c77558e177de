"""GPU parity of the bit-width-independent precompute (BITCRUSH BC-06,
"Under the hood": a change of bit width costs one kernel argument).
bc_group_minmax stores each group's exact range once; BC_MODE_RUNTIME_RANGE
matmuls derive scale and zero for any bits inside the kernel.  Checked:
the ranges against the oracle's, the outputs bit-identical to the runtime
mode fed with bc_group_params' (scale, zero) (same codes, same arithmetic),
and against the oracle at the fp32 bar, over a lever sweep 8 -> 2 bits that
reuses one precompute."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from parity_util import TOL_FP32, assert_close, dev, host

pytestmark = pytest.mark.gpu


def _ranges_host(r):
    """int32 words -> (lo, hi) float64 (fp16 halves)."""
    w = host(r).astype(np.uint32)
    lo = (w & 0xFFFF).astype(np.uint16).view(np.float16).astype(np.float64)
    hi = (w >> 16).astype(np.uint16).view(np.float16).astype(np.float64)
    return lo, hi


@pytest.mark.parametrize("group", [64, 0])
def test_ranges_match_oracle(cuda_lib, group):
    from test_parity_quant import _edge_matrix
    for W in (_edge_matrix(3), wl.weight(0, 0, "single", 1024, 1024, 0.02)):
        g = W.shape[1] if group == 0 else group
        lo_ref, hi_ref = oracle.group_range(W, g)
        lo, hi = _ranges_host(cuda_lib.group_minmax(dev(W), group))
        assert np.array_equal(lo, lo_ref) and np.array_equal(hi, hi_ref)


def _items(qmm, Ws, xs, bits, group, range_form, M):
    items = []
    for W, x in zip(Ws, xs):
        Wd = dev(W)
        if range_form:
            s, z = qmm.group_minmax(Wd, group), None
        else:
            s, z = qmm.group_params(Wd, bits, group, torch.float32)
        items.append((x, Wd, s, z, torch.full((M, W.shape[0]), float("nan"), device="cuda")))
    return items


@pytest.mark.parametrize("M,count", [(1, 40), (3, 40), (8, 40), (1, 1), (16, 1)])
@pytest.mark.parametrize("group", [64, 0])
def test_range_mode_lever_sweep(cuda_lib, M, count, group):
    """One range precompute serves every bit width; count = 40 takes the
    streaming / tensor-core decode kernels, count = 1 the general GEMV."""
    qmm = cuda_lib
    rng = np.random.default_rng(200 + M + count)
    shapes = [(896, 896), (4864, 896), (896, 4864), (128, 896)]
    Ws = [(rng.standard_normal(shapes[i % 4]) * 0.02).astype(np.float16) for i in range(count)]
    xh = {K: wl.activation(201, K, "x", M, K) for K in (896, 4864)}
    xs = [dev(xh[W.shape[1]]) for W in Ws]
    ranged = _items(qmm, Ws, xs, 8, group, True, M)
    descs_r = qmm.make_descs(ranged)
    for bits in (8, 7, 6, 5, 4, 3, 2):
        qmm.matmul_q_batched(descs_r, M, bits, group, qmm.BC_MODE_RUNTIME_RANGE)
        plain = _items(qmm, Ws, xs, bits, group, False, M)
        qmm.matmul_q_batched(qmm.make_descs(plain), M, bits, group, qmm.BC_MODE_RUNTIME)
        torch.cuda.synchronize()
        for i in range(count):
            assert np.array_equal(host(ranged[i][4]), host(plain[i][4])), f"bits={bits} #{i}"
        for i in {0, count - 1}:
            W = Ws[i]
            g = W.shape[1] if group == 0 else group
            ref = oracle.matmul_q(xh[W.shape[1]], W, bits, g, "runtime")
            assert_close(host(ranged[i][4]), ref["y"], ref["A"], TOL_FP32,
                         f"range bits={bits} M={M} #{i}")
    assert qmm.device_timeouts() == 0


def test_range_mode_grid_ties(cuda_lib):
    """Weights on the quantization grid with exact half-way points: the zero
    derived in the kernel and the codes must still be the exact ones."""
    qmm = cuda_lib
    rng = np.random.default_rng(240)
    bits, L = 3, 7
    N, K = 256, 512
    G = K // 64
    e = rng.integers(4, 10, size=(N, G))
    z = rng.integers(1, L, size=(N, G))
    h = rng.integers(0, L, size=(N, K)) + 0.5 * rng.integers(0, 2, size=(N, K))
    h[:, 0::64] = 0
    h[:, 1::64] = L
    w = (h - np.repeat(z, 64, axis=1)) * np.repeat(np.ldexp(1.0, -e), 64, axis=1)
    W = w.astype(np.float16)
    x = wl.activation(241, 0, "x", 1, K)
    xd, Wd = dev(x), dev(W)
    r = qmm.group_minmax(Wd, 64)
    y = qmm.matmul_q(xd, Wd, r, None, bits, 64, qmm.BC_MODE_RUNTIME_RANGE)
    ref = oracle.matmul_q(x, W, bits, 64, "runtime")
    assert_close(host(y), ref["y"], ref["A"], TOL_FP32, "range ties")
