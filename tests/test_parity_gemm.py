"""GPU parity of the tcgen05 prefill GEMM (packed int4 W, bf16 x, M >= 64)
against the oracle: max |y - y_ref| <= 8e-3 * sum_k |x_k * w'_nk|.

Enargeia, "Four bits per weight" (int4 with scale/zero per 64-block,
unpacked on chip) and its benchmark table (prefill at 128 and 2048 tokens).
The oracle multiplies the exact bf16 x by the exact dequantized w'."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from parity_util import TOL_BF16, assert_close, dev, host

pytestmark = pytest.mark.gpu


def _bf16(x32):
    bits = wl.bf16_bits(x32)
    t = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    return t, wl.bf16_to_f32(bits).astype(np.float64)


def _prep(qmm, W):
    Wd = dev(W)
    s, z = qmm.group_params(Wd, 4, 64, torch.float16)
    p = qmm.pack_int4(Wd, s, z)
    ref = oracle.matmul_q(np.zeros((1, W.shape[1])), W, 4, 64, "packed")
    return p, s, z, ref["wq"]


@pytest.mark.parametrize("M", [64, 128, 129, 256, 300])
@pytest.mark.parametrize("NK", [(896, 896), (128, 896), (896, 4864), (200, 192)])
def test_gemm_shapes(cuda_lib, M, NK):
    N, K = NK
    W = wl.weight(20, M, "single", K, N, 0.02)
    xb, xf = _bf16(wl.activation(20, M, "x", M, K))
    p, s, z, wq = _prep(cuda_lib, W)
    y = cuda_lib.matmul_q(xb, p, s, z, 4, 64, cuda_lib.BC_MODE_PACKED_INT4)
    yr, A = oracle.matmul(xf, wq)
    assert_close(host(y), yr, A, TOL_BF16, f"gemm M={M} N={N} K={K}")
    assert cuda_lib.device_timeouts() == 0


def test_gemm_deterministic(cuda_lib):
    N, K, M = 896, 896, 256
    W = wl.weight(21, 0, "single", K, N, 0.02)
    xb, _ = _bf16(wl.activation(21, 0, "x", M, K))
    p, s, z, _ = _prep(cuda_lib, W)
    outs = [host(cuda_lib.matmul_q(xb, p, s, z, 4, 64, cuda_lib.BC_MODE_PACKED_INT4))
            for _ in range(4)]
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_gemm_wide_zero_blocks(cuda_lib):
    """Blocks whose zero point lies far outside [0, 15] (single-sign groups)
    take the fp32 dequant branch."""
    rng = np.random.default_rng(3)
    N, K, M = 128, 256, 128
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    W[:16] = (1.0 + rng.integers(0, 40, (16, K)) * 2.0 ** -10).astype(np.float16)
    W[16:32] = -(0.5 + rng.integers(0, 40, (16, K)) * 2.0 ** -11).astype(np.float16)
    xb, xf = _bf16(wl.activation(22, 0, "x", M, K))
    p, s, z, wq = _prep(cuda_lib, W)
    assert np.abs(host(z).astype(np.float64)).max() > 128
    y = cuda_lib.matmul_q(xb, p, s, z, 4, 64, cuda_lib.BC_MODE_PACKED_INT4)
    yr, A = oracle.matmul(xf, wq)
    assert_close(host(y), yr, A, TOL_BF16, "wide zero")


def _prefill_set(qmm, layers, M, sample_rows=None, seed=3):
    """Grouped prefill launch over `layers` of the Qwen2.5-0.5B set; checks
    every output, or a seeded sample of rows per matrix."""
    mats = wl.layer_set("qwen2.5-0.5b", layers)
    xs, items, refs = {}, [], []
    rng = np.random.default_rng(seed)
    for m in mats:
        key = (m.layer, m.x_tag)
        if key not in xs:
            xs[key] = _bf16(wl.activation(seed, m.layer, m.x_tag, M, m.K))
        xb, xf = xs[key]
        W = wl.weight(seed, m.layer, m.name, m.K, m.N, 0.02)
        p, s, z, wq = _prep(qmm, W)
        y = torch.full((M, m.N), float("nan"), device="cuda")
        items.append((xb, p, s, z, y))
        refs.append((m, xf, wq))
    descs = qmm.make_descs(items)
    qmm.matmul_q_batched(descs, M, 4, 64, qmm.BC_MODE_PACKED_INT4, qmm.BC_BF16)
    torch.cuda.synchronize()
    for (m, xf, wq), it in zip(refs, items):
        y = host(it[4])
        if sample_rows is None:
            yr, A = oracle.matmul(xf, wq)
            assert_close(y, yr, A, TOL_BF16, f"L{m.layer} {m.name}")
        else:
            rows = rng.choice(M, size=min(sample_rows, M), replace=False)
            cols = rng.choice(m.N, size=min(64, m.N), replace=False)
            yr, A = oracle.matmul(xf[rows], wq[cols])
            assert_close(y[np.ix_(rows, cols)], yr, A, TOL_BF16,
                         f"L{m.layer} {m.name} (sampled)")
    assert qmm.device_timeouts() == 0


def test_prefill_qwen25_one_layer_m128(cuda_lib):
    _prefill_set(cuda_lib, 1, 128)


def test_prefill_qwen25_full_set_m128_sampled(cuda_lib):
    """The full 24-layer set at M = 128, in the grouped launch the prefill
    benchmark times; sampled outputs against the oracle."""
    _prefill_set(cuda_lib, 24, 128, sample_rows=16)


def test_prefill_qwen25_two_layers_m2048_sampled(cuda_lib):
    _prefill_set(cuda_lib, 2, 2048, sample_rows=24)


def test_prefill_qwen25_full_set_m2048_sampled(cuda_lib):
    """The full 24-layer set at M = 2048: 168 matrices, three launches, the
    pairs dealing the x-block-major tile list in snake rounds."""
    _prefill_set(cuda_lib, 24, 2048, sample_rows=8)


# ---- runtime RTN prefill (fp16 W re-quantized inline in the dequant stage) --
# BITCRUSH BC-06, "Under the hood" (codes computed as the weights are read,
# at any lever position) and "The machine" (THE LEVER 16 -> 2).

def _rt_params(qmm, Wd, bits, group, range_form=False):
    if bits == 16:
        return None, None, qmm.BC_MODE_RUNTIME
    if range_form:
        return qmm.group_minmax(Wd, group), None, qmm.BC_MODE_RUNTIME_RANGE
    s, z = qmm.group_params(Wd, bits, group, torch.float32)
    return s, z, qmm.BC_MODE_RUNTIME


@pytest.mark.parametrize("bits", [2, 3, 4, 8, 16])
@pytest.mark.parametrize("group", [64, 0])
@pytest.mark.parametrize("M,N,K", [(64, 896, 896), (129, 200, 192), (300, 128, 4864)])
def test_runtime_gemm(cuda_lib, bits, group, M, N, K):
    W = wl.weight(23, M + bits, "single", K, N, 0.02)
    xb, xf = _bf16(wl.activation(23, M, "x", M, K))
    Wd = dev(W)
    s, z, mode = _rt_params(cuda_lib, Wd, bits, group)
    y = cuda_lib.matmul_q(xb, Wd, s, z, bits, group, mode)
    g = K if group == 0 else group
    ref = oracle.matmul_q(xf, W, bits, g, "runtime")
    assert_close(host(y), ref["y"], ref["A"], TOL_BF16, f"rt gemm bits={bits} M={M}")
    assert cuda_lib.device_timeouts() == 0


@pytest.mark.parametrize("bits", [3, 6])
def test_runtime_gemm_range_form_matches(cuda_lib, bits):
    """The range form (bc_group_minmax once, scale and zero derived in the
    kernel) gives the same output bits as the stored (scale, zero)."""
    M, N, K = 256, 384, 1024
    W = wl.weight(24, bits, "single", K, N, 0.02)
    xb, xf = _bf16(wl.activation(24, 0, "x", M, K))
    Wd = dev(W)
    s, z, mode = _rt_params(cuda_lib, Wd, bits, 64)
    r, _, rmode = _rt_params(cuda_lib, Wd, bits, 64, range_form=True)
    y1 = host(cuda_lib.matmul_q(xb, Wd, s, z, bits, 64, mode))
    y2 = host(cuda_lib.matmul_q(xb, Wd, r, None, bits, 64, rmode))
    assert np.array_equal(y1, y2)
    ref = oracle.matmul_q(xf, W, bits, 64, "runtime")
    assert_close(y2, ref["y"], ref["A"], TOL_BF16, "range form")


def test_runtime_gemm_grid_ties(cuda_lib):
    """Weights on the quantization grid with exact half-way points: the
    dequant stage must take the exact quotient for them."""
    rng = np.random.default_rng(250)
    bits, L = 3, 7
    N, K, M = 256, 512, 128
    G = K // 64
    e = rng.integers(4, 10, size=(N, G))
    zz = rng.integers(1, L, size=(N, G))
    h = rng.integers(0, L, size=(N, K)) + 0.5 * rng.integers(0, 2, size=(N, K))
    h[:, 0::64] = 0
    h[:, 1::64] = L
    w = (h - np.repeat(zz, 64, axis=1)) * np.repeat(np.ldexp(1.0, -e), 64, axis=1)
    W = w.astype(np.float16)
    xb, xf = _bf16(wl.activation(251, 0, "x", M, K))
    Wd = dev(W)
    s, z, mode = _rt_params(cuda_lib, Wd, bits, 64)
    y = cuda_lib.matmul_q(xb, Wd, s, z, bits, 64, mode)
    ref = oracle.matmul_q(xf, W, bits, 64, "runtime")
    assert_close(host(y), ref["y"], ref["A"], TOL_BF16, "rt ties")


def _rt_prefill_set(qmm, layers, M, bits, group, sample_rows, seed=3):
    mats = wl.layer_set("qwen2.5-0.5b", layers)
    xs, items, refs = {}, [], []
    rng = np.random.default_rng(seed + 100)
    for m in mats:
        key = (m.layer, m.x_tag)
        if key not in xs:
            xs[key] = _bf16(wl.activation(seed, m.layer, m.x_tag, M, m.K))
        xb, xf = xs[key]
        W = wl.weight(seed, m.layer, m.name, m.K, m.N, 0.02)
        Wd = dev(W)
        s, z, mode = _rt_params(qmm, Wd, bits, group)
        y = torch.full((M, m.N), float("nan"), device="cuda")
        items.append((xb, Wd, s, z, y))
        refs.append((m, xf, W))
    qmm.matmul_q_batched(qmm.make_descs(items), M, bits, group, mode, qmm.BC_BF16)
    torch.cuda.synchronize()
    for (m, xf, W), it in zip(refs, items):
        rows = rng.choice(M, size=min(sample_rows, M), replace=False)
        cols = np.sort(rng.choice(m.N, size=min(64, m.N), replace=False))
        g = m.K if group == 0 else group
        ref = oracle.matmul_q(xf[rows], W[cols], bits, g, "runtime")
        assert_close(host(it[4])[np.ix_(rows, cols)], ref["y"], ref["A"], TOL_BF16,
                     f"rt L{m.layer} {m.name} (sampled)")
    assert qmm.device_timeouts() == 0


def test_runtime_prefill_full_set_m128_3bit(cuda_lib):
    _rt_prefill_set(cuda_lib, 24, 128, 3, 64, sample_rows=16)


@pytest.mark.parametrize("bits,group", [(3, 64), (16, 64), (8, 0)])
def test_runtime_prefill_two_layers_m2048(cuda_lib, bits, group):
    _rt_prefill_set(cuda_lib, 2, 2048, bits, group, sample_rows=24)
