"""Guard bands around outputs and scratch (a stand-in for a memory checker,
which this pool does not offer): every y and every workspace is placed
between padding filled with a sentinel pattern, and the padding must be
untouched after the call -- no kernel writes past the end (or before the
start) of what it owns.  Covers each kernel family: streaming decode (M = 1,
packed and runtime), tensor-core decode (M = 16, with its workspace), the
general GEMV with split-K scratch, the prefill GEMM (packed and runtime),
the other packed widths and the argmax reduction."""
import numpy as np
import pytest
import torch

import workloads as wl
from parity_util import dev

pytestmark = pytest.mark.gpu

PAD = 1024                        # elements of padding on each side
SENTINEL = -0x2A4D2A4D            # int32 pattern (a NaN payload as fp32)


def _guarded(shape, dtype=torch.float32):
    """(view, buffer): a tensor of `shape` inside sentinel padding."""
    n = int(np.prod(shape))
    ebytes = torch.tensor([], dtype=dtype).element_size()
    buf = torch.empty(n * ebytes + 2 * PAD * 4, dtype=torch.uint8, device="cuda")
    buf.view(torch.int32).fill_(SENTINEL)
    inner = buf[PAD * 4: PAD * 4 + n * ebytes].view(dtype).view(*shape)
    return inner, buf


def _check(buf, nbytes, what):
    torch.cuda.synchronize()
    head = buf[:PAD * 4].view(torch.int32)
    tail = buf[PAD * 4 + nbytes:].view(torch.int32)
    assert bool((head == SENTINEL).all()), f"{what}: write before the start"
    assert bool((tail == SENTINEL).all()), f"{what}: write past the end"


def _ws(nbytes):
    return _guarded((max(nbytes, 256),), torch.uint8)


def _mats(qmm, M, count, mode, bits, shapes, seed):
    rng = np.random.default_rng(seed)
    items, bufs, xs = [], [], {}
    for i in range(count):
        N, K = shapes[i % len(shapes)]
        if K not in xs:
            xs[K] = dev(wl.activation(seed, K, "x", M, K))
        Wd = dev((rng.standard_normal((N, K)) * 0.02).astype(np.float16))
        if mode == "packed":
            s, z = qmm.group_params(Wd, bits, 64, torch.float16)
            Wk = qmm.pack_codes(Wd, s, z, bits)
        elif bits == 16:
            s = z = None
            Wk = Wd
        else:
            s, z = qmm.group_params(Wd, bits, 64, torch.float32)
            Wk = Wd
        y, buf = _guarded((M, N))
        items.append((xs[K], Wk, s, z, y))
        bufs.append((buf, M * N * 4))
    return items, bufs


@pytest.mark.parametrize("M,count,mode,bits", [
    (1, 40, "packed", 4), (1, 40, "runtime", 3), (2, 40, "packed", 4),
    (16, 40, "packed", 4), (16, 40, "runtime", 5),
    (1, 1, "packed", 4), (3, 2, "runtime", 16),
    (1, 3, "packed", 2), (5, 3, "packed", 3), (2, 3, "packed", 8)])
def test_decode_writes_stay_inside(cuda_lib, M, count, mode, bits):
    qmm = cuda_lib
    shapes = [(896, 896), (130, 4864), (4864, 896), (37, 192)]
    items, bufs = _mats(qmm, M, count, mode, bits, shapes, 310 + M)
    descs = qmm.make_descs(items)
    mid = qmm.BC_MODE_PACKED if mode == "packed" else qmm.BC_MODE_RUNTIME
    need = qmm.workspace_size_batched(descs, M, mid, qmm.BC_F32)
    ws, wbuf = _ws(need)
    qmm.matmul_q_batched(descs, M, bits, 64, mid, workspace=ws)
    for i, (buf, nb) in enumerate(bufs):
        _check(buf, nb, f"y of matrix {i}")
        assert not torch.isnan(items[i][4]).any(), f"matrix {i}: output not fully written"
    _check(wbuf, max(need, 256), "workspace")


@pytest.mark.parametrize("mode,bits,M", [("packed", 4, 129), ("runtime", 3, 300),
                                         ("runtime", 16, 64)])
def test_prefill_writes_stay_inside(cuda_lib, mode, bits, M):
    qmm = cuda_lib
    N, K = 200, 192
    rng = np.random.default_rng(320)
    Wd = dev((rng.standard_normal((N, K)) * 0.02).astype(np.float16))
    bits16 = wl.bf16_bits(wl.activation(320, M, "x", M, K))
    xb = torch.from_numpy(bits16.view(np.int16)).cuda().view(torch.bfloat16)
    if mode == "packed":
        s, z = qmm.group_params(Wd, 4, 64, torch.float16)
        Wk, mid = qmm.pack_int4(Wd, s, z), qmm.BC_MODE_PACKED
    elif bits == 16:
        s = z = None
        Wk, mid = Wd, qmm.BC_MODE_RUNTIME
    else:
        s, z = qmm.group_params(Wd, bits, 64, torch.float32)
        Wk, mid = Wd, qmm.BC_MODE_RUNTIME
    y, buf = _guarded((M, N))
    qmm.matmul_q(xb, Wk, s, z, bits, 64, mid, y=y)
    _check(buf, M * N * 4, "prefill y")
    assert not torch.isnan(y).any()


def test_argmax_writes_stay_inside(cuda_lib):
    qmm = cuda_lib
    M, N, K = 3, 20000, 512
    W = dev(wl.weight(330, 0, "lm_head", K, N, 0.02))
    x = dev(wl.activation(330, 0, "x", M, K))
    tok, tbuf = _guarded((M,), torch.int32)
    need = qmm.workspace_size_argmax(M, N, K, qmm.BC_MODE_RUNTIME)
    ws, wbuf = _ws(need)
    qmm.matmul_q_argmax(x, W, None, None, 16, 64, qmm.BC_MODE_RUNTIME, token=tok, workspace=ws)
    _check(tbuf, M * 4, "token")
    _check(wbuf, need, "argmax workspace")
