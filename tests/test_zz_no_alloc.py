"""bc_matmul_q_noalloc: the decode matmul for callers that cannot allocate
device memory (no workspace to hand over), using the library's own fixed
scratch array.  Checked through the C ABI against bc_matmul_q, the entry
point that takes a caller workspace, on consecutive calls that share the
scratch.  This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from parity_util import TOL_FP32, assert_close, dev, host

pytestmark = pytest.mark.gpu


def _case(qmm, mode, M, N, K, bits, group, seed):
    W = wl.weight(30 + seed, 0, "single", K, N, 0.02)
    x = wl.activation(30 + seed, 0, "x", M, K)
    Wd, xd = dev(W), dev(x)
    g = K if group == 0 else group
    if mode == "packed":
        s, z = qmm.group_params(Wd, 4, 64, torch.float16)
        Wk = qmm.pack_int4(Wd, s, z)
        m = qmm.BC_MODE_PACKED_INT4
        ref = oracle.matmul_q(x, W, 4, 64, "packed")
    else:
        s, z = qmm.group_params(Wd, bits, group, torch.float32)
        Wk = Wd
        m = qmm.BC_MODE_RUNTIME
        ref = oracle.matmul_q(x, W, bits, g, "runtime")
    # these shapes split K, so the scratch is really used
    assert qmm.workspace_size(M, N, K, m) > 0
    return xd, Wk, s, z, bits, group, m, ref


def _noalloc_vs_workspace(qmm, c):
    xd, Wk, s, z, bits, group, m, ref = c
    y_ws = qmm.matmul_q(xd, Wk, s, z, bits, group, m)          # caller workspace
    y_na = torch.full_like(y_ws, float("nan"))
    qmm.matmul_q_noalloc(xd, Wk, s, z, bits, group, m, y_na)    # fixed scratch
    y_ws, y_na = host(y_ws), host(y_na)
    assert_close(y_na, y_ws.astype(np.float64), ref["A"], TOL_FP32, "noalloc")
    assert_close(y_na, ref["y"], ref["A"], TOL_FP32, "noalloc vs oracle")


def test_noalloc_matches_workspace_entry_two_calls_in_a_row(cuda_lib):
    t0 = cuda_lib.device_timeouts()
    a = _case(cuda_lib, "packed", 8, 128, 4864, 4, 64, 0)
    b = _case(cuda_lib, "runtime", 5, 256, 3072, 3, 64, 1)
    _noalloc_vs_workspace(cuda_lib, a)     # first call: sets the scratch up
    _noalloc_vs_workspace(cuda_lib, b)     # second call reuses the scratch
    _noalloc_vs_workspace(cuda_lib, a)
    assert cuda_lib.device_timeouts() == t0


def test_noalloc_rejects_bad_arguments_without_enqueueing(cuda_lib):
    lib = cuda_lib.lib
    assert lib.bc_matmul_q_noalloc(None, 16, 16, 16, 1, 8, 64, 4, 64, 1, 16,
                                   None) == cuda_lib.BC_ERR_INVALID_ARG
    assert lib.bc_matmul_q_noalloc(16, 16, 16, 16, 1, 8, 96, 4, 64, 1, 16,
                                   None) == cuda_lib.BC_ERR_INVALID_ARG


def test_noalloc_tensor_core_decode_path(cuda_lib):
    """A shape large enough for the tcgen05 decode kernel (packed int4, M = 8,
    96 row blocks of 128): its split activations go to the fixed array, and
    the prepared launch is reused on the second call."""
    qmm = cuda_lib
    t0 = qmm.device_timeouts()
    M, N, K = 8, 12288, 4096
    need = qmm.workspace_size(M, N, K, qmm.BC_MODE_PACKED_INT4)
    assert 0 < need < (4 << 20)
    W = wl.weight(33, 0, "single", K, N, 0.02)
    x = wl.activation(33, 0, "x", M, K)
    ref = oracle.matmul_q(x, W, 4, 64, "packed")
    Wd, xd = dev(W), dev(x)
    s, z = qmm.group_params(Wd, 4, 64, torch.float16)
    Wk = qmm.pack_int4(Wd, s, z)
    y_ws = host(qmm.matmul_q(xd, Wk, s, z, 4, 64, qmm.BC_MODE_PACKED_INT4))
    for _ in range(2):
        y_na = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        qmm.matmul_q_noalloc(xd, Wk, s, z, 4, 64, qmm.BC_MODE_PACKED_INT4, y_na)
        y_na = host(y_na)
        assert_close(y_na, y_ws.astype(np.float64), ref["A"], TOL_FP32, "noalloc tc")
        assert_close(y_na, ref["y"], ref["A"], TOL_FP32, "noalloc tc vs oracle")
    assert qmm.device_timeouts() == t0


def test_noalloc_rejects_scratch_beyond_the_fixed_array(cuda_lib):
    """M = 16 packed with K = 65536 over 74 row blocks needs more than the
    4 MiB array for its split activations: refused with BC_ERR_WORKSPACE,
    nothing enqueued, y untouched."""
    qmm = cuda_lib
    M, N, K = 16, 74 * 128, 65536
    assert qmm.workspace_size(M, N, K, qmm.BC_MODE_PACKED_INT4) > (4 << 20)
    Wk = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
    s = torch.empty((N, K // 64), dtype=torch.float16, device="cuda")
    z = torch.empty_like(s)
    xd = torch.zeros((M, K), dtype=torch.float32, device="cuda")
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    st = qmm.lib.bc_matmul_q_noalloc(xd.data_ptr(), Wk.data_ptr(), s.data_ptr(),
                                     z.data_ptr(), M, N, K, 4, 64,
                                     qmm.BC_MODE_PACKED_INT4, y.data_ptr(), None)
    assert st == qmm.BC_ERR_WORKSPACE
    assert torch.isnan(y).all().item()
    del Wk


def test_noalloc_wrapper_refuses_wrong_dtypes(cuda_lib):
    qmm = cuda_lib
    x = torch.zeros((1, 64), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((8, 32), dtype=torch.uint8, device="cuda")
    s = torch.ones((8, 1), dtype=torch.float16, device="cuda")
    y = torch.empty((1, 8), dtype=torch.float32, device="cuda")
    with pytest.raises(ValueError):
        qmm.matmul_q_noalloc(x, W, s, s, 4, 64, qmm.BC_MODE_PACKED_INT4, y)
    with pytest.raises(ValueError):
        qmm.matmul_q_noalloc(x.float(), W, s, s, 4, 64, qmm.BC_MODE_PACKED_INT4,
                             y[:, :4])
