"""The failure path of the bounded in-kernel waits, run on purpose without
faulting the GPU: bc_set_wait_limit shortens every pipeline wait to a few
hundred cycles, so the decode and prefill kernels' waits run out.  Each
kernel must then record the timeout, stop, wait (with the normal limit) for
its own copies and MMAs in flight, free its tensor memory and return -- no
hang, no fault, the context usable.  Restoring the limit gives correct
results again.  Collected late so that the timeouts it records do not meet
the other tests' checks for none."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from parity_util import TOL_BF16, TOL_FP32, assert_close, dev, host

pytestmark = pytest.mark.gpu


def _decode_set(qmm, M, count=40):
    rng = np.random.default_rng(300 + M)
    items, Ws = [], []
    x = wl.activation(300, M, "x", M, 896)
    xd = dev(x)
    for _ in range(count):
        W = (rng.standard_normal((896, 896)) * 0.02).astype(np.float16)
        Wd = dev(W)
        s, z = qmm.group_params(Wd, 4, 64, torch.float16)
        items.append((xd, qmm.pack_int4(Wd, s, z), s, z,
                      torch.full((M, 896), float("nan"), device="cuda")))
        Ws.append(W)
    return x, items, Ws


@pytest.mark.timeout(120)
def test_waits_run_out_and_kernels_recover(cuda_lib):
    qmm = cuda_lib
    t0 = qmm.device_timeouts()
    sets = {M: _decode_set(qmm, M) for M in (1, 8)}
    W = wl.weight(301, 0, "single", 896, 896, 0.02)
    bits = wl.bf16_bits(wl.activation(301, 0, "x", 128, 896))
    xb = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    xf = wl.bf16_to_f32(bits).astype(np.float64)
    Wd = dev(W)
    s, z = qmm.group_params(Wd, 4, 64, torch.float16)
    p = qmm.pack_int4(Wd, s, z)

    def run_all():
        for M, (_, items, _) in sets.items():
            qmm.matmul_q_batched(qmm.make_descs(items), M, 4, 64, qmm.BC_MODE_PACKED_INT4)
        return qmm.matmul_q(xb, p, s, z, 4, 64, qmm.BC_MODE_PACKED_INT4)

    qmm.set_wait_limit(300)
    try:
        run_all()
        torch.cuda.synchronize()
        t1 = qmm.device_timeouts()
    finally:
        qmm.set_wait_limit(0)
    assert t1 > t0, "no wait ran out under a 300-cycle limit"
    # the context is usable and the results right again
    y = run_all()
    torch.cuda.synchronize()
    assert qmm.device_timeouts() == t1
    for M, (x, items, Ws) in sets.items():
        ref = oracle.matmul_q(x, Ws[0], 4, 64, "packed")
        assert_close(host(items[0][4]), ref["y"], ref["A"], TOL_FP32, f"after reset M={M}")
    ref = oracle.matmul_q(xf, W, 4, 64, "packed")
    assert_close(host(y), ref["y"], ref["A"], TOL_BF16, "gemm after reset")
