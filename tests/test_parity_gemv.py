"""GPU parity of the fused dequant GEMV (decode shapes, fp32 x) against the
oracle: max |y - y_ref| <= 1e-4 * sum_k |x_k * w'_nk| per output element.

BITCRUSH BC-06 "Under the hood" (matmul_q: runtime RTN inline as weights
are read; NAIVE / SMART row: per-channel vs per-group) and Enargeia "Four
bits per weight" (packed int4 unpacked in registers)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from parity_util import TOL_FP32, assert_close, dev, host

pytestmark = pytest.mark.gpu


def _runtime_case(qmm, W, x, bits, group):
    N, K = W.shape
    g = K if group == 0 else group
    Wd, xd = dev(W), dev(x)
    if bits == 16:
        s = z = None
        ref = oracle.matmul_q(x, W, 16, g, "runtime")
    else:
        s, z = qmm.group_params(Wd, bits, group, torch.float32)
        ref = oracle.matmul_q(x, W, bits, g, "runtime")
        np.testing.assert_array_equal(host(s).astype(np.float64), ref["s"])
    y = qmm.matmul_q(xd, Wd, s, z, bits, group, qmm.BC_MODE_RUNTIME)
    return host(y), ref


def _packed_case(qmm, W, x):
    Wd, xd = dev(W), dev(x)
    s, z = qmm.group_params(Wd, 4, 64, torch.float16)
    p = qmm.pack_int4(Wd, s, z)
    ref = oracle.matmul_q(x, W, 4, 64, "packed")
    np.testing.assert_array_equal(host(p), ref["packed"])
    y = qmm.matmul_q(xd, p, s, z, 4, 64, qmm.BC_MODE_PACKED_INT4)
    return host(y), ref


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("group", [64, 0])
def test_single_layer_1024_runtime(cuda_lib, bits, group):
    """The 1024 x 1024 single-layer workload (seed 0), M = 1."""
    W = wl.weight(0, 0, "single", 1024, 1024, 0.02)
    x = wl.activation(0, 0, "x", 1, 1024)
    y, ref = _runtime_case(cuda_lib, W, x, bits, group)
    assert_close(y, ref["y"], ref["A"], TOL_FP32, f"bits={bits} group={group}")


def test_single_layer_1024_group_beats_channel_on_gpu(cuda_lib):
    """NAIVE / SMART on the GPU output: per-group output error against the
    fp16 reference matmul is smaller than per-channel at 3 bits."""
    W = wl.weight(0, 0, "single", 1024, 1024, 0.02)
    x = wl.activation(0, 0, "x", 1, 1024)
    y16, _ = _runtime_case(cuda_lib, W, x, 16, 64)
    err = {}
    for group in (64, 0):
        y, _ = _runtime_case(cuda_lib, W, x, 3, group)
        err[group] = np.mean((y.astype(np.float64) - y16) ** 2)
    assert err[64] < err[0]


@pytest.mark.parametrize("M", [2, 5, 16, 17, 40])
@pytest.mark.parametrize("bits,group", [(3, 64), (8, 0), (16, 64)])
def test_runtime_multi_row(cuda_lib, M, bits, group):
    W = wl.weight(11, 0, "single", 1024, 300, 0.02)
    x = wl.activation(11, 0, "x", M, 1024)
    y, ref = _runtime_case(cuda_lib, W, x, bits, group)
    assert_close(y, ref["y"], ref["A"], TOL_FP32, f"M={M} bits={bits}")


@pytest.mark.parametrize("M", [1, 3, 16, 21])
@pytest.mark.parametrize("NK", [(896, 896), (128, 896), (896, 4864), (37, 192),
                                (1, 64)])
def test_packed_shapes(cuda_lib, M, NK):
    N, K = NK
    W = wl.weight(12, M, "single", K, N, 0.02)
    x = wl.activation(12, M, "x", M, K)
    y, ref = _packed_case(cuda_lib, W, x)
    assert_close(y, ref["y"], ref["A"], TOL_FP32, f"packed M={M} N={N} K={K}")


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 7, 8])
def test_runtime_ties_take_exact_path(cuda_lib, bits):
    """Weights on the quantization grid with many exact half-way points:
    the fast reciprocal path must hand these to the exact quotient."""
    rng = np.random.default_rng(40 + bits)
    L = (1 << bits) - 1
    N, K = 64, 512
    G = K // 64
    e = rng.integers(4, 10, size=(N, G))
    z = rng.integers(1, L, size=(N, G))
    h = rng.integers(0, L, size=(N, K)) + 0.5 * rng.integers(0, 2, size=(N, K))
    h[:, 0::64] = 0
    h[:, 1::64] = L
    w = (h - np.repeat(z, 64, axis=1)) * np.repeat(np.ldexp(1.0, -e), 64, axis=1)
    W = w.astype(np.float16)
    assert np.array_equal(W.astype(np.float64), w)
    x = wl.activation(13, bits, "x", 1, K)
    y, ref = _runtime_case(cuda_lib, W, x, bits, 64)
    assert_close(y, ref["y"], ref["A"], TOL_FP32, f"ties bits={bits}")


def test_edge_rows_runtime_and_packed(cuda_lib):
    from test_parity_quant import _edge_matrix
    W = _edge_matrix(8)
    x = wl.activation(14, 0, "x", 3, W.shape[1])
    for bits, group in ((2, 64), (4, 0), (8, 64)):
        y, ref = _runtime_case(cuda_lib, W, x, bits, group)
        assert_close(y, ref["y"], ref["A"], TOL_FP32, f"edges bits={bits}")
    y, ref = _packed_case(cuda_lib, W, x)
    assert_close(y, ref["y"], ref["A"], TOL_FP32, "edges packed")


@pytest.mark.parametrize("mode", ["runtime", "packed"])
def test_split_k_small_n_is_deterministic(cuda_lib, mode):
    """A lone small-N matrix is split along K; the last CTA reduces the
    partials in split order, so repeated calls are bit-identical."""
    N, K = 128, 4864
    assert cuda_lib.workspace_size(1, N, K, int(mode == "packed")) > 0
    W = wl.weight(15, 0, "single", K, N, 0.02)
    x = wl.activation(15, 0, "x", 1, K)
    if mode == "runtime":
        y, ref = _runtime_case(cuda_lib, W, x, 4, 64)
    else:
        y, ref = _packed_case(cuda_lib, W, x)
    assert_close(y, ref["y"], ref["A"], TOL_FP32, f"split-K {mode}")
    Wd, xd = dev(W), dev(x)
    s, z = cuda_lib.group_params(Wd, 4, 64,
                                 torch.float32 if mode == "runtime" else torch.float16)
    Wk = Wd if mode == "runtime" else cuda_lib.pack_int4(Wd, s, z)
    m = cuda_lib.BC_MODE_RUNTIME if mode == "runtime" else cuda_lib.BC_MODE_PACKED_INT4
    outs = [host(cuda_lib.matmul_q(xd, Wk, s, z, 4, 64, m)) for _ in range(5)]
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def _layer_set_case(qmm, shape_set, layers, workload, mode, bits, group, M=1):
    mats = wl.layer_set(shape_set, layers)
    xs, items, refs = {}, [], []
    keep = []
    for m in mats:
        key = (m.layer, m.x_tag)
        if key not in xs:
            xs[key] = wl.activation(workload, m.layer, m.x_tag, M, m.K)
        x = xs[key]
        W = wl.weight(workload, m.layer, m.name, m.K, m.N, wl.SIGMA[shape_set])
        g = m.K if group == 0 else group
        Wd = dev(W)
        if mode == "packed":
            s, z = qmm.group_params(Wd, 4, 64, torch.float16)
            Wk = qmm.pack_int4(Wd, s, z)
            ref = oracle.matmul_q(x, W, 4, 64, "packed")
        elif bits == 16:
            s = z = None
            Wk = Wd
            ref = oracle.matmul_q(x, W, 16, g, "runtime")
        else:
            s, z = qmm.group_params(Wd, bits, group, torch.float32)
            Wk = Wd
            ref = oracle.matmul_q(x, W, bits, g, "runtime")
        y = torch.full((M, m.N), float("nan"), device="cuda")
        xd = dev(x)
        keep.append((xd, Wk, s, z, y))
        items.append((xd, Wk, s, z, y))
        refs.append((m, ref))
    descs = qmm.make_descs(items)
    mode_id = qmm.BC_MODE_PACKED_INT4 if mode == "packed" else qmm.BC_MODE_RUNTIME
    ws_bytes = qmm.workspace_size_batched(descs, M, mode_id, qmm.BC_F32)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device="cuda")
    qmm.matmul_q_batched(descs, M, bits, group, mode_id, workspace=ws)
    torch.cuda.synchronize()
    for (m, ref), it in zip(refs, items):
        assert_close(host(it[4]), ref["y"], ref["A"], TOL_FP32,
                     f"{shape_set} L{m.layer} {m.name}")


def test_batched_qwen25_packed_two_layers(cuda_lib):
    _layer_set_case(cuda_lib, "qwen2.5-0.5b", 2, 1, "packed", 4, 64)


@pytest.mark.parametrize("bits,group", [(3, 64), (3, 0), (16, 64), (2, 64)])
def test_batched_qwen3_runtime_one_layer(cuda_lib, bits, group):
    _layer_set_case(cuda_lib, "qwen3-0.6b", 1, 2, "runtime", bits, group)


def test_batched_qwen3_8b_one_layer_m16(cuda_lib):
    _layer_set_case(cuda_lib, "qwen3-8b", 1, 4, "packed", 4, 64, M=16)
    _layer_set_case(cuda_lib, "qwen3-8b", 1, 4, "runtime", 3, 64, M=1)


def test_determinism_batched(cuda_lib):
    """Enargeia: the output is identical every run (no float atomics)."""
    mats = wl.layer_set("qwen2.5-0.5b", 1)
    items = []
    for m in mats:
        W = dev(wl.weight(1, 0, m.name, m.K, m.N, 0.02))
        s, z = cuda_lib.group_params(W, 4, 64, torch.float16)
        items.append((dev(wl.activation(1, 0, m.x_tag, 1, m.K)),
                      cuda_lib.pack_int4(W, s, z), s, z,
                      torch.empty((1, m.N), device="cuda")))
    descs = cuda_lib.make_descs(items)
    outs = []
    for _ in range(10):
        cuda_lib.matmul_q_batched(descs, 1, 4, 64, cuda_lib.BC_MODE_PACKED_INT4)
        outs.append(torch.cat([it[4].flatten() for it in items]).cpu())
    for o in outs[1:]:
        assert torch.equal(o, outs[0])


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 13, 16])
@pytest.mark.parametrize("mode,bits,group", [("packed", 4, 64), ("runtime", 5, 64),
                                             ("runtime", 3, 0), ("runtime", 16, 64)])
def test_batched_mixed_shapes_stream(cuda_lib, M, mode, bits, group):
    """A grouped launch large enough for the streaming kernel, with ragged
    row blocks (N not a multiple of 128) and K tails (K not a multiple of
    the 256-byte stage chunk), several matrices sharing one x.  Packed codes
    at M = 5..16 take the chunked-activation form (rows padded to 8 or 16)."""
    rng = np.random.default_rng(M * 10 + bits)
    shapes = [(37, 192), (200, 896), (896, 1024), (130, 64), (256, 4864),
              (1000, 320)]
    items, refs = [], []
    xs = {}
    for i in range(36):
        N, K = shapes[i % len(shapes)]
        key = (K, i // 12)
        if key not in xs:
            xs[key] = wl.activation(50 + i // 12, K, "x", M, K)
        x = xs[key]
        W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
        g = K if group == 0 else group
        Wd = dev(W)
        if mode == "packed":
            s, z = cuda_lib.group_params(Wd, 4, 64, torch.float16)
            Wk = cuda_lib.pack_int4(Wd, s, z)
            ref = oracle.matmul_q(x, W, 4, 64, "packed")
        elif bits == 16:
            s = z = None
            Wk = Wd
            ref = oracle.matmul_q(x, W, 16, g, "runtime")
        else:
            s, z = cuda_lib.group_params(Wd, bits, group, torch.float32)
            Wk = Wd
            ref = oracle.matmul_q(x, W, bits, g, "runtime")
        y = torch.full((M, N), float("nan"), device="cuda")
        items.append((dev(x), Wk, s, z, y))
        refs.append(ref)
    descs = cuda_lib.make_descs(items)
    mid = cuda_lib.BC_MODE_PACKED_INT4 if mode == "packed" else cuda_lib.BC_MODE_RUNTIME
    cuda_lib.matmul_q_batched(descs, M, bits, group, mid)
    torch.cuda.synchronize()
    for i, (ref, it) in enumerate(zip(refs, items)):
        assert_close(host(it[4]), ref["y"], ref["A"], TOL_FP32, f"matrix {i}")
    assert cuda_lib.device_timeouts() == 0


def _stream_set(cuda_lib, M, seed, count=40):
    """A grouped packed-int4 launch large enough for the streaming kernel."""
    rng = np.random.default_rng(seed)
    shapes = [(896, 896), (128, 896), (4864, 896), (896, 4864)]
    items, Ws = [], []
    x_dev = {}
    for i in range(count):
        N, K = shapes[i % len(shapes)]
        if K not in x_dev:
            x_dev[K] = torch.zeros((M, K), device="cuda")
        W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
        Wd = dev(W)
        s, z = cuda_lib.group_params(Wd, 4, 64, torch.float16)
        Wk = cuda_lib.pack_int4(Wd, s, z)
        y = torch.full((M, N), float("nan"), device="cuda")
        items.append((x_dev[K], Wk, s, z, y))
        Ws.append(W)
    return items, Ws, x_dev


@pytest.mark.parametrize("M", [1, 2, 11])
def test_static_weights_early_start_sees_new_x(cuda_lib, M):
    """BC_FLAG_STATIC_WEIGHTS launches the decode kernel as a programmatic
    dependent launch.  Between back-to-back launches a torch kernel on the
    same stream rewrites x; each launch must still read the x written just
    before it (and write y after the previous launch is done)."""
    items, Ws, x_dev = _stream_set(cuda_lib, M, 91)
    torch.cuda.synchronize()           # weights are complete before the launches
    descs = cuda_lib.make_descs(items)
    xs_host = []
    staged = []
    for rep in range(3):
        xk = {K: wl.activation(60 + rep, K, "x", M, K) for K in x_dev}
        staged.append({K: dev(v) for K, v in xk.items()})
        xs_host.append(xk)
    torch.cuda.synchronize()
    for rep in range(3):
        for K, t in x_dev.items():      # an elementwise kernel rewrites x
            torch.mul(staged[rep][K], 1.0, out=t)
        cuda_lib.matmul_q_batched(descs, M, 4, 64, cuda_lib.BC_MODE_PACKED_INT4,
                                  static_weights=True)
    torch.cuda.synchronize()
    last = xs_host[-1]
    for i, ((_, _, _, _, y), W) in enumerate(zip(items, Ws)):
        ref = oracle.matmul_q(last[W.shape[1]], W, 4, 64, "packed")
        assert_close(host(y), ref["y"], ref["A"], TOL_FP32, f"matrix {i}")
    assert cuda_lib.device_timeouts() == 0


def test_static_weights_matches_default_launch(cuda_lib):
    items, Ws, x_dev = _stream_set(cuda_lib, 1, 92)
    for K, t in x_dev.items():
        t.copy_(torch.from_numpy(wl.activation(70, K, "x", 1, K)).to("cuda"))
    torch.cuda.synchronize()
    descs = cuda_lib.make_descs(items)
    cuda_lib.matmul_q_batched(descs, 1, 4, 64, cuda_lib.BC_MODE_PACKED_INT4)
    torch.cuda.synchronize()
    first = [host(it[4]).copy() for it in items]
    for it in items:
        it[4].fill_(float("nan"))
    cuda_lib.matmul_q_batched(descs, 1, 4, 64, cuda_lib.BC_MODE_PACKED_INT4,
                              static_weights=True)
    torch.cuda.synchronize()
    for i, it in enumerate(items):
        assert np.array_equal(host(it[4]), first[i]), f"matrix {i}"


def test_batched_ex_rejects_unknown_flags(cuda_lib):
    items, _, _ = _stream_set(cuda_lib, 1, 93, count=2)
    descs = cuda_lib.make_descs(items)
    st = cuda_lib.lib.bc_matmul_q_batched_ex(descs, len(descs), 1, 4, 64,
                                             cuda_lib.BC_MODE_PACKED_INT4,
                                             cuda_lib.BC_F32, None, 0, 0x80, None)
    assert st == cuda_lib.BC_ERR_INVALID_ARG


def test_stream_activation_outliers(cuda_lib):
    """Activations are staged as integers relative to their 64-group maximum;
    a group holding an outlier 10^4 times its neighbours must still meet the
    fp32 bar (the neighbours keep ~2^-13 relative precision or better)."""
    rng = np.random.default_rng(77)
    items, refs = [], []
    x = wl.activation(80, 896, "x", 1, 896).copy()
    x[0, ::64] *= 1.0e4                  # one outlier in every group
    x[0, 5::64] = 1.0e-30                # and a value far below everything
    xd = dev(x)
    for i in range(160):
        N, K = (896, 896)
        W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
        Wd = dev(W)
        s, z = cuda_lib.group_params(Wd, 4, 64, torch.float16)
        Wk = cuda_lib.pack_int4(Wd, s, z)
        y = torch.full((1, N), float("nan"), device="cuda")
        items.append((xd, Wk, s, z, y))
        if i < 3:
            refs.append(oracle.matmul_q(x, W, 4, 64, "packed"))
    cuda_lib.matmul_q_batched(cuda_lib.make_descs(items), 1, 4, 64,
                              cuda_lib.BC_MODE_PACKED_INT4)
    torch.cuda.synchronize()
    for i, ref in enumerate(refs):
        assert_close(host(items[i][4]), ref["y"], ref["A"], TOL_FP32, f"matrix {i}")
    assert cuda_lib.device_timeouts() == 0


def test_chunked_activation_workspace(cuda_lib):
    """Packed launches with M > 4 keep the activation digits in the caller's
    workspace: a size queried without x pointers covers the call, matrices
    sharing an x share space, and a short workspace is refused before any
    work is enqueued."""
    M = 16
    items, Ws, x_dev = _stream_set(cuda_lib, M, 94)
    descs = cuda_lib.make_descs(items)
    mode = cuda_lib.BC_MODE_PACKED_INT4
    need = cuda_lib.workspace_size_batched(descs, M, mode, cuda_lib.BC_F32)
    anon = cuda_lib.make_descs(items)
    for d in anon:
        d.x = None
    bound = cuda_lib.workspace_size_batched(anon, M, mode, cuda_lib.BC_F32)
    assert 0 < need < bound
    short = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    st = cuda_lib.lib.bc_matmul_q_batched_ex(descs, len(descs), M, 4, 64, mode,
                                             cuda_lib.BC_F32, cuda_lib._ptr(short),
                                             need - 256, 0, None)
    assert st == cuda_lib.BC_ERR_WORKSPACE
    xk = {K: wl.activation(70, K, "x", M, K) for K in x_dev}
    for K, t in x_dev.items():
        t.copy_(dev(xk[K]))
    ws = torch.empty(bound, dtype=torch.uint8, device="cuda")
    cuda_lib.matmul_q_batched(descs, M, 4, 64, mode, workspace=ws)
    torch.cuda.synchronize()
    for i in (0, 1, 2, 3, 38, 39):
        W = Ws[i]
        ref = oracle.matmul_q(xk[W.shape[1]], W, 4, 64, "packed")
        assert_close(host(items[i][4]), ref["y"], ref["A"], TOL_FP32, f"matrix {i}")
    assert cuda_lib.device_timeouts() == 0


@pytest.mark.parametrize("bits,M", [(3, 16), (5, 8), (8, 11)])
def test_tc_runtime_ties_take_exact_path(cuda_lib, bits, M):
    """The tensor-core decode kernel (runtime RTN, 5..16 x rows) on weights
    with exact half-way points: its transform warps must take the exact
    quotient for these, like the other decode kernels.  A grouped launch of
    copies of one grid-valued matrix, large enough for the streaming path."""
    rng = np.random.default_rng(140 + bits)
    L = (1 << bits) - 1
    N, K = 512, 512
    G = K // 64
    e = rng.integers(4, 10, size=(N, G))
    z = rng.integers(1, L, size=(N, G))
    h = rng.integers(0, L, size=(N, K)) + 0.5 * rng.integers(0, 2, size=(N, K))
    h[:, 0::64] = 0
    h[:, 1::64] = L
    w = (h - np.repeat(z, 64, axis=1)) * np.repeat(np.ldexp(1.0, -e), 64, axis=1)
    W = w.astype(np.float16)
    assert np.array_equal(W.astype(np.float64), w)
    x = wl.activation(14, bits, "x", M, K)
    xd, Wd = dev(x), dev(W)
    s, zz = cuda_lib.group_params(Wd, bits, 64, torch.float32)
    items = [(xd, Wd, s, zz, torch.full((M, N), float("nan"), device="cuda"))
             for _ in range(24)]
    cuda_lib.matmul_q_batched(cuda_lib.make_descs(items), M, bits, 64,
                              cuda_lib.BC_MODE_RUNTIME)
    torch.cuda.synchronize()
    ref = oracle.matmul_q(x, W, bits, 64, "runtime")
    for i in (0, 23):
        assert_close(host(items[i][4]), ref["y"], ref["A"], TOL_FP32, f"ties bits={bits} #{i}")
    assert cuda_lib.device_timeouts() == 0


def test_batched_qwen3_8b_one_layer_m16_runtime(cuda_lib):
    _layer_set_case(cuda_lib, "qwen3-8b", 1, 4, "runtime", 3, 64, M=16)


@pytest.mark.parametrize("mode,bits", [("packed", 4), ("runtime", 5)])
def test_tc_decode_more_matrices_than_one_launch(cuda_lib, mode, bits):
    """More matrices than one launch of the tensor-core decode kernel takes
    (168): the call runs in batches that reuse the activation workspace one
    after the other; every matrix, first and last batch, must be right."""
    rng = np.random.default_rng(160 + bits)
    M, count = 8, 200
    shapes = [(256, 512), (128, 448), (384, 256)]
    xs = {K: wl.activation(90, K, "x", M, K) for _, K in shapes}
    xd = {K: dev(v) for K, v in xs.items()}
    items, Ws = [], []
    for i in range(count):
        N, K = shapes[i % len(shapes)]
        W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
        Wd = dev(W)
        if mode == "packed":
            s, z = cuda_lib.group_params(Wd, 4, 64, torch.float16)
            Wk = cuda_lib.pack_int4(Wd, s, z)
        else:
            s, z = cuda_lib.group_params(Wd, bits, 64, torch.float32)
            Wk = Wd
        items.append((xd[K], Wk, s, z, torch.full((M, N), float("nan"), device="cuda")))
        Ws.append(W)
    mid = cuda_lib.BC_MODE_PACKED_INT4 if mode == "packed" else cuda_lib.BC_MODE_RUNTIME
    cuda_lib.matmul_q_batched(cuda_lib.make_descs(items), M, bits, 64, mid)
    torch.cuda.synchronize()
    for i in (0, 1, 2, 166, 167, 168, 169, 198, 199):
        W = Ws[i]
        ref = oracle.matmul_q(xs[W.shape[1]], W, bits, 64, mode)
        assert_close(host(items[i][4]), ref["y"], ref["A"], TOL_FP32, f"matrix {i}")
    assert cuda_lib.device_timeouts() == 0


@pytest.mark.parametrize("M", [1, 2, 4, 8])
@pytest.mark.parametrize("big", [3.0e3, 1.0e5, 1.0e6])
def test_stream_outliers_where_weights_are_zero(cuda_lib, M, big):
    """Activation outliers placed where every row's dequantized weight is 0
    (the weight column is zero, so its code equals the zero point): the
    outlier adds nothing to y or to A = sum |x w'|, but it sets the group's
    integer grid and enters the zero-point term.  Neighbours 3000, 10^5 and
    10^6 times smaller, and 1e-30 values, must still meet the fp32 bar.  A grouped launch of 160 matrices (large
    enough for the streaming kernels); M = 8 takes the tensor-core decode."""
    rng = np.random.default_rng(int(big) % 1000 + M)
    K, N = 896, 896
    G = K // 64
    x = wl.activation(81, M, "x", M, K).astype(np.float64)
    cols = set()
    for m in range(M):
        for g in range(G):
            k_big = 64 * g + (7 + 2 * m if g % 2 else 10 + 2 * m)   # odd, even k
            x[m, k_big] = big * (1 if (g + m) % 2 else -1)
            x[m, 64 * g + 21 + m] = 1.0e-30
            cols.add(k_big)
    x = x.astype(np.float32)
    items, refs = [], []
    xd = dev(x)
    for i in range(160):
        W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
        W[:, sorted(cols)] = 0.0
        Wd = dev(W)
        s, z = cuda_lib.group_params(Wd, 4, 64, torch.float16)
        Wk = cuda_lib.pack_int4(Wd, s, z)
        y = torch.full((M, N), float("nan"), device="cuda")
        items.append((xd, Wk, s, z, y))
        if i < 3 or i == 159:
            refs.append((i, oracle.matmul_q(x, W, 4, 64, "packed")))
    cuda_lib.matmul_q_batched(cuda_lib.make_descs(items), M, 4, 64,
                              cuda_lib.BC_MODE_PACKED_INT4)
    torch.cuda.synchronize()
    for i, ref in refs:
        # the outliers meet w' = 0 exactly: they must not show up in A
        assert np.all(ref["A"] < 1.0e3)
        assert_close(host(items[i][4]), ref["y"], ref["A"], TOL_FP32,
                     f"outlier {big:g} M={M} matrix {i}")
    assert cuda_lib.device_timeouts() == 0
