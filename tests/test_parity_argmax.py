"""GPU parity of bc_matmul_q_argmax (greedy token selection after the LM
head) against the oracle's matmul: the GPU's index must be the oracle's
argmax of y, except where the oracle's best and the GPU's pick are within
the fp32 bar of each other, where either is a correct greedy choice (both
are within rounding of the maximum).  Ties in the exact result go to the
lowest index.  Enargeia, "One decode step" (one readback carrying a token
id); BITCRUSH BC-06, "Honest notes" (greedy decoding; tied LM head kept at
fp16)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from parity_util import TOL_FP32, dev, host

pytestmark = pytest.mark.gpu


def _check_tokens(tok, ref, what):
    y, A = ref["y"], ref["A"]
    for m, t in enumerate(tok):
        best = int(np.argmax(y[m]))                  # first index of the maximum
        if t == best:
            continue
        assert 0 <= t < y.shape[1], f"{what}: row {m} token {t} out of range"
        slack = TOL_FP32 * (A[m, t] + A[m, best])
        assert y[m, best] - y[m, t] <= slack, (
            f"{what}: row {m} picked {t} (y={y[m, t]!r}), best {best} (y={y[m, best]!r})")


def _case(qmm, W, x, mode, bits, group):
    g = W.shape[1] if group == 0 else group
    Wd, xd = dev(W), dev(x)
    if mode == "packed":
        s, z = qmm.group_params(Wd, 4, 64, torch.float16)
        Wk, mid = qmm.pack_int4(Wd, s, z), qmm.BC_MODE_PACKED_INT4
    elif bits == 16:
        s = z = None
        Wk, mid = Wd, qmm.BC_MODE_RUNTIME
    else:
        s, z = qmm.group_params(Wd, bits, group, torch.float32)
        Wk, mid = Wd, qmm.BC_MODE_RUNTIME
    tok = host(qmm.matmul_q_argmax(xd, Wk, s, z, bits, group, mid))
    ref = oracle.matmul_q(x, W, bits, g, mode)
    return tok, ref


@pytest.mark.parametrize("M", [1, 3])
def test_lm_head_fp16_argmax(cuda_lib, M):
    """Qwen3-0.6B's tied head, 1024 -> 151936, fp16 passthrough."""
    K, N = 1024, wl.VOCAB
    W = wl.weight(2, 0, "lm_head", K, N, 0.02)
    x = wl.activation(2, 28, "x", M, K)
    tok, ref = _case(cuda_lib, W, x, "runtime", 16, 64)
    _check_tokens(tok, ref, f"lm head M={M}")


@pytest.mark.parametrize("mode,bits,group", [("packed", 4, 64), ("runtime", 3, 64),
                                             ("runtime", 8, 0)])
@pytest.mark.parametrize("M,N,K", [(1, 5000, 512), (2, 20000, 1024), (5, 777, 192)])
def test_quantized_head_argmax(cuda_lib, mode, bits, group, M, N, K):
    W = wl.weight(17, M, "lm_head", K, N, 0.02)
    x = wl.activation(17, M, "x", M, K)
    tok, ref = _case(cuda_lib, W, x, mode, bits, group)
    _check_tokens(tok, ref, f"{mode} bits={bits} M={M} N={N}")


def test_ties_go_to_the_lowest_index(cuda_lib):
    """Identical weight rows give exactly equal logits: rows 3, 4100 and
    9000 are copies of one large row, so the maximum is reached three times
    (in different 4096-wide partials) and the token must be 3."""
    K, N = 256, 12000
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    big = (np.abs(rng.standard_normal(K)) * 0.5 + 0.1).astype(np.float16)
    for r in (9000, 4100, 3):
        W[r] = big
    x = np.abs(wl.activation(18, 0, "x", 1, K))
    tok, ref = _case(cuda_lib, W, x, "runtime", 16, 64)
    assert int(np.argmax(ref["y"][0])) == 3
    assert tok.tolist() == [3]


def test_argmax_rejects_small_workspace(cuda_lib):
    qmm = cuda_lib
    M, N, K = 1, 4096, 256
    W = dev(wl.weight(19, 0, "lm_head", K, N, 0.02))
    x = dev(wl.activation(19, 0, "x", M, K))
    tok = torch.full((M,), -1, dtype=torch.int32, device="cuda")
    need = qmm.workspace_size_argmax(M, N, K, qmm.BC_MODE_RUNTIME)
    assert need >= M * N * 4
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    st = qmm.lib.bc_matmul_q_argmax(x.data_ptr(), qmm.BC_F32, W.data_ptr(), None, None,
                                    M, N, K, 16, 64, qmm.BC_MODE_RUNTIME, tok.data_ptr(),
                                    ws.data_ptr(), need - 256, None)
    assert st == qmm.BC_ERR_WORKSPACE
    assert host(tok).tolist() == [-1]
