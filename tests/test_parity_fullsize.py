"""GPU parity at the benchmark's full sizes, in the launch configuration
bench.py times, on sampled output rows the oracle computes one by one
(each output row depends only on its own weight row, its group parameters
and x).

* the headline call: the 24-layer Qwen2.5-0.5B set (168 matrices), packed
  int4, M = 1, one grouped launch with BC_FLAG_STATIC_WEIGHTS, three steps
  back to back (Enargeia, "One decode step" and "Four bits per weight");
* the tied LM head of Qwen3-0.6B (1024 -> 151936, fp16 passthrough) and the
  28-layer Qwen3-0.6B set at 3 bits (BITCRUSH BC-06, "The machine": the
  lever sweep; "Honest notes": embeddings stay fp16);
* 200 back-to-back grouped calls of one Qwen3-8B layer at M = 16 through
  the tensor-core decode kernel, packed and runtime 3-bit: every call
  bit-identical to the first and within the fp32 bar of the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from parity_util import TOL_FP32, assert_close, dev, host

pytestmark = pytest.mark.gpu


def _sample_rows(rng, N, count=12):
    rows = set(rng.choice(N, size=min(count, N), replace=False).tolist())
    rows.update({0, N - 1})
    return np.array(sorted(rows))


def _build_set(qmm, mats, workload, sigma, mode, bits, group, M):
    xs, items, Ws = {}, [], []
    for m in mats:
        key = (m.layer, m.x_tag)
        if key not in xs:
            xs[key] = (wl.activation(workload, m.layer, m.x_tag, M, m.K), None)
            xs[key] = (xs[key][0], dev(xs[key][0]))
        W = wl.weight(workload, m.layer, m.name, m.K, m.N, sigma)
        Wd = dev(W)
        if mode == "packed":
            s, z = qmm.group_params(Wd, 4, 64, torch.float16)
            Wk = qmm.pack_int4(Wd, s, z)
            del Wd
        elif bits == 16:
            s = z = None
            Wk = Wd
        else:
            s, z = qmm.group_params(Wd, bits, group, torch.float32)
            Wk = Wd
        y = torch.full((M, m.N), float("nan"), device="cuda")
        items.append((xs[key][1], Wk, s, z, y))
        Ws.append(W)
    return xs, items, Ws


def _check_sampled(items, Ws, mats, xs, mode, bits, group, seed, what):
    rng = np.random.default_rng(seed)
    for i, (m, W, it) in enumerate(zip(mats, Ws, items)):
        rows = _sample_rows(rng, m.N)
        x = xs[(m.layer, m.x_tag)][0]
        g = m.K if group == 0 else group
        ref = oracle.matmul_q(x, W[rows], bits, g, mode)
        y = host(it[4])[:, rows]
        assert_close(y, ref["y"], ref["A"], TOL_FP32, f"{what} matrix {i} ({m.name})")


def test_headline_call_full_set_static_weights(cuda_lib):
    """The exact benchmark call: 168 matrices, one grouped launch per step,
    static weights (programmatic dependent launch), three steps in a row,
    with a different x each step written by a torch kernel in between."""
    qmm = cuda_lib
    mats = wl.layer_set("qwen2.5-0.5b", 24)
    xs, items, Ws = _build_set(qmm, mats, 1, wl.SIGMA["qwen2.5-0.5b"], "packed", 4, 64, 1)
    torch.cuda.synchronize()
    descs = qmm.make_descs(items)
    # three steps; x is rewritten (scaled copies of the seeded draw) before
    # each, the last step's x being the seeded draw itself
    keep = {k: v[1].clone() for k, v in xs.items()}
    for step, scale in enumerate((3.0, -0.5, 1.0)):
        for k, v in xs.items():
            torch.mul(keep[k], scale, out=v[1])
        qmm.matmul_q_batched(descs, 1, 4, 64, qmm.BC_MODE_PACKED_INT4, static_weights=True)
    torch.cuda.synchronize()
    _check_sampled(items, Ws, mats, xs, "packed", 4, 64, 101, "headline")
    assert qmm.device_timeouts() == 0


def test_lm_head_fp16_passthrough(cuda_lib):
    """Qwen3-0.6B's tied LM head, 1024 -> 151936 at 16 bits (one matrix of
    1,187 row blocks), alone and after the 28-layer set at 3 bits in one
    grouped call (197 matrices: two launches of the streaming kernel)."""
    qmm = cuda_lib
    K, N = 1024, wl.VOCAB
    W = wl.weight(2, 0, "lm_head", K, N, 0.02)
    x = wl.activation(2, 28, "x", 1, K)
    xd, Wd = dev(x), dev(W)
    y = torch.full((1, N), float("nan"), device="cuda")
    qmm.matmul_q(xd, Wd, None, None, 16, 64, qmm.BC_MODE_RUNTIME, y=y)
    rows = _sample_rows(np.random.default_rng(7), N, 64)
    ref = oracle.matmul_q(x, W[rows], 16, 64, "runtime")
    assert_close(host(y)[:, rows], ref["y"], ref["A"], TOL_FP32, "lm head")


def test_qwen3_06b_full_set_3bit(cuda_lib):
    """The 28-layer Qwen3-0.6B set at 3 bits, per-group: one grouped call
    over 196 matrices (two launches of the streaming kernel)."""
    qmm = cuda_lib
    mats = wl.layer_set("qwen3-0.6b", 28)
    xs, items, Ws = _build_set(qmm, mats, 2, 0.02, "runtime", 3, 64, 1)
    descs = qmm.make_descs(items)
    qmm.matmul_q_batched(descs, 1, 3, 64, qmm.BC_MODE_RUNTIME, static_weights=True)
    torch.cuda.synchronize()
    _check_sampled(items, Ws, mats, xs, "runtime", 3, 64, 102, "qwen3-0.6b rtn3")
    assert qmm.device_timeouts() == 0


@pytest.mark.parametrize("mode,bits", [("packed", 4), ("runtime", 3)])
def test_tc_decode_200_calls_bit_identical(cuda_lib, mode, bits):
    qmm = cuda_lib
    M = 16
    mats = wl.layer_set("qwen3-8b", 1)
    xs, items, Ws = _build_set(qmm, mats, 4, wl.SIGMA["qwen3-8b"], mode, bits, 64, M)
    descs = qmm.make_descs(items)
    mid = qmm.BC_MODE_PACKED_INT4 if mode == "packed" else qmm.BC_MODE_RUNTIME
    ws = torch.empty(max(1, qmm.workspace_size_batched(descs, M, mid, qmm.BC_F32)),
                     dtype=torch.uint8, device="cuda")
    qmm.matmul_q_batched(descs, M, bits, 64, mid, workspace=ws, static_weights=True)
    first = torch.cat([it[4].flatten() for it in items]).clone()
    bad = 0
    for _ in range(199):
        for it in items:
            it[4].fill_(float("nan"))
        qmm.matmul_q_batched(descs, M, bits, 64, mid, workspace=ws, static_weights=True)
        bad += int(not torch.equal(torch.cat([it[4].flatten() for it in items]), first))
    torch.cuda.synchronize()
    assert bad == 0, f"{bad} of 199 repeated calls differ from the first"
    _check_sampled(items, Ws, mats, xs, mode, bits, 64, 103, f"qwen3-8b m16 {mode}")
    assert qmm.device_timeouts() == 0
