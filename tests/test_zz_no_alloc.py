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
    a = _case(cuda_lib, "packed", 8, 128, 4864, 4, 64, 0)
    b = _case(cuda_lib, "runtime", 5, 256, 3072, 3, 64, 1)
    _noalloc_vs_workspace(cuda_lib, a)     # first call: sets the scratch up
    _noalloc_vs_workspace(cuda_lib, b)     # second call reuses the scratch
    _noalloc_vs_workspace(cuda_lib, a)
    assert cuda_lib.device_timeouts() == 0


def test_noalloc_rejects_bad_arguments_without_enqueueing(cuda_lib):
    lib = cuda_lib.lib
    assert lib.bc_matmul_q_noalloc(None, 16, 16, 16, 1, 8, 64, 4, 64, 1, 16,
                                   None) == cuda_lib.BC_ERR_INVALID_ARG
    assert lib.bc_matmul_q_noalloc(16, 16, 16, 16, 1, 8, 96, 4, 64, 1, 16,
                                   None) == cuda_lib.BC_ERR_INVALID_ARG
