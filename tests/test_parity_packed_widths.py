"""GPU parity of the other packed widths (2, 3 and 8 bits; BITCRUSH BC-06,
"The machine", BRAIN SIZE at 2 bits; Enargeia, "Honestly", an int8 tied
embedding): packed bytes bit-exact against the oracle's bit-string packing,
and the decode GEMV over them within the fp32 bar of the oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from parity_util import TOL_FP32, assert_close, dev, host

pytestmark = pytest.mark.gpu


def _packed(qmm, W, bits):
    Wd = dev(W)
    s, z = qmm.group_params(Wd, bits, 64, torch.float16)
    return qmm.pack_codes(Wd, s, z, bits), s, z


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_pack_codes_bit_exact(cuda_lib, bits):
    from test_parity_quant import _edge_matrix
    for W in (_edge_matrix(4), wl.weight(25, bits, "single", 1024, 300, 0.02)):
        ref = oracle.matmul_q(np.zeros((1, W.shape[1])), W, bits, 64, "packed")
        p, s, z = _packed(cuda_lib, W, bits)
        np.testing.assert_array_equal(host(s).astype(np.float64), ref["s"])
        np.testing.assert_array_equal(host(z).astype(np.float64), ref["z"])
        np.testing.assert_array_equal(host(p), ref["packed"])


@pytest.mark.parametrize("bits", [2, 3, 8])
@pytest.mark.parametrize("M", [1, 5, 16, 21])
@pytest.mark.parametrize("N,K", [(300, 1024), (37, 192), (4864, 896)])
def test_packed_width_gemv(cuda_lib, bits, M, N, K):
    W = wl.weight(26, bits * 100 + M, "single", K, N, 0.02)
    x = wl.activation(26, M, "x", M, K)
    p, s, z = _packed(cuda_lib, W, bits)
    y = cuda_lib.matmul_q(dev(x), p, s, z, bits, 64, cuda_lib.BC_MODE_PACKED)
    ref = oracle.matmul_q(x, W, bits, 64, "packed")
    assert_close(host(y), ref["y"], ref["A"], TOL_FP32, f"packed{bits} M={M} N={N} K={K}")


@pytest.mark.parametrize("bits", [2, 3, 8])
def test_packed_width_layer_set(cuda_lib, bits):
    """One Qwen3-0.6B layer (7 matrices) in one grouped call, and the
    bytes of the packed weights falling with the width."""
    qmm = cuda_lib
    items, refs, nbytes = [], [], 0
    xs = {}
    for m in wl.layer_set("qwen3-0.6b", 1):
        if m.x_tag not in xs:
            xs[m.x_tag] = wl.activation(2, 0, m.x_tag, 1, m.K)
        W = wl.weight(2, 0, m.name, m.K, m.N, 0.02)
        p, s, z = _packed(qmm, W, bits)
        nbytes += p.numel()
        items.append((dev(xs[m.x_tag]), p, s, z, torch.full((1, m.N), float("nan"), device="cuda")))
        refs.append(oracle.matmul_q(xs[m.x_tag], W, bits, 64, "packed"))
    assert nbytes == wl.linear_params("qwen3-0.6b") // 28 * bits // 8
    qmm.matmul_q_batched(qmm.make_descs(items), 1, bits, 64, qmm.BC_MODE_PACKED)
    torch.cuda.synchronize()
    for it, ref in zip(items, refs):
        assert_close(host(it[4]), ref["y"], ref["A"], TOL_FP32, f"layer packed{bits}")


def test_packed_width_rejections(cuda_lib):
    qmm = cuda_lib
    FAKE = 0x10000
    # bf16 x (prefill) is int4 only; widths 5..7 are not packed
    assert qmm.lib.bc_matmul_q(FAKE, qmm.BC_BF16, FAKE, FAKE, FAKE, 128, 8, 64, 3, 64,
                               qmm.BC_MODE_PACKED, FAKE, None, 0, None) == qmm.BC_ERR_UNSUPPORTED
    assert qmm.lib.bc_pack_codes(FAKE, FAKE, FAKE, 8, 64, 5, FAKE, None) == qmm.BC_ERR_UNSUPPORTED
