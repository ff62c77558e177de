"""GPU parity of the quantizer kernels against the oracle: scales, zeros,
codes and packed bytes must be bit-exact (BITCRUSH BC-06 "Under the hood":
per-group scale/zero precompute and RTN codes; Enargeia "Four bits per
weight": int4 packing)."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from parity_util import dev, host

pytestmark = pytest.mark.gpu


def _edge_matrix(seed=5):
    """Rows that hit every reading: constant, zero, subnormal, single-sign,
    ties on a grid, huge range, and plain Gaussian."""
    rng = np.random.default_rng(seed)
    K = 192
    rows = []
    rows.append(np.full(K, 0.75))                                  # constant
    rows.append(np.zeros(K))                                       # all zero
    rows.append(rng.integers(-40, 40, K) * 2.0 ** -24)             # subnormal
    rows.append(1.0 + rng.integers(0, 512, K) * 2.0 ** -10)        # positive only
    rows.append(-(1.0 + rng.integers(0, 512, K) * 2.0 ** -10))     # negative only
    g = (rng.integers(-3, 4, K) + 0.5 * rng.integers(0, 2, K)) * 2.0 ** -5
    g[0], g[1] = -4 * 2.0 ** -5, 3 * 2.0 ** -5
    rows.append(g)                                                 # ties (2-bit grid)
    rows.append(rng.standard_normal(K) * 300.0)                    # large range
    rows.append(np.concatenate([np.full(64, -2.0 ** -24), np.full(64, 65504.0),
                                rng.standard_normal(64)]))
    # group 0: fp16 scale below 2^-25, floored to 2^-24; group 1: single-sign
    # group near 1000 whose zero (|z| > 2048) is rounded to fp16
    r = np.zeros(K)
    r[0:4] = np.array([-2, 5, 0, -1]) * 2.0 ** -24
    r[64:128] = 1000.0 + 0.5 * rng.integers(0, 3, 64)
    r[64], r[65] = 1000.0, 1001.0
    r[128:] = rng.standard_normal(64) * 0.02
    rows.append(r)
    for _ in range(29):
        rows.append(rng.standard_normal(K) * 0.02)                 # 38 rows total
    return np.array(rows).astype(np.float16)


CASES = [("cfg1_1024", lambda: wl.weight(0, 0, "single", 1024, 1024, 0.02)),
         ("edges_38x192", _edge_matrix),
         ("tiny_1x64", lambda: wl.weight(9, 0, "single", 64, 1, 0.02))]


@pytest.mark.parametrize("name,make", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("bits", [2, 3, 4, 5, 8])
@pytest.mark.parametrize("group", [64, 0])
def test_group_params_and_codes_fp32(cuda_lib, name, make, bits, group):
    W = make()
    N, K = W.shape
    g = K if group == 0 else group
    s_ref, z_ref = oracle.group_params(W, bits, g, False)
    q_ref = oracle.codes(W, s_ref, z_ref, bits, g)
    Wd = dev(W)
    s, z = cuda_lib.group_params(Wd, bits, group, torch.float32)
    q = cuda_lib.quantize_codes(Wd, s, z, bits, group)
    np.testing.assert_array_equal(host(s).astype(np.float64), s_ref)
    np.testing.assert_array_equal(host(z).astype(np.float64), z_ref)
    np.testing.assert_array_equal(host(q), q_ref)


@pytest.mark.parametrize("name,make", CASES, ids=[c[0] for c in CASES])
def test_group_params_codes_pack_fp16(cuda_lib, name, make):
    W = make()
    s_ref, z_ref = oracle.group_params(W, 4, 64, True)
    q_ref = oracle.codes(W, s_ref, z_ref, 4, 64)
    p_ref = oracle.pack_int4(q_ref)
    Wd = dev(W)
    s, z = cuda_lib.group_params(Wd, 4, 64, torch.float16)
    q = cuda_lib.quantize_codes(Wd, s, z, 4, 64)
    p = cuda_lib.pack_int4(Wd, s, z)
    np.testing.assert_array_equal(host(s).astype(np.float64), s_ref)
    np.testing.assert_array_equal(host(z).astype(np.float64), z_ref)
    np.testing.assert_array_equal(host(q), q_ref)
    np.testing.assert_array_equal(host(p), p_ref)


def test_pack_full_qwen25_layer(cuda_lib):
    """One full Qwen2.5-0.5B layer (every shape of the decode set)."""
    for m in wl.layer_set("qwen2.5-0.5b", 1):
        W = wl.weight(1, m.layer, m.name, m.K, m.N, 0.02)
        s_ref, z_ref = oracle.group_params(W, 4, 64, True)
        p_ref = oracle.pack_int4(oracle.codes(W, s_ref, z_ref, 4, 64))
        Wd = dev(W)
        s, z = cuda_lib.group_params(Wd, 4, 64, torch.float16)
        np.testing.assert_array_equal(host(cuda_lib.pack_int4(Wd, s, z)), p_ref)


GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "rtn_worked_groups.json")
SINGLE = [c for c in json.load(open(GOLDEN))["cases"] if "w" in c]


@pytest.mark.parametrize("case", SINGLE, ids=lambda c: c["name"])
def test_golden_groups_on_gpu(cuda_lib, case):
    """The hand-worked groups straight through the GPU kernels (not via the
    oracle): stored scale and zero, codes and packed bytes as derived by
    hand from the definitions."""
    K = case["K"]
    w = np.full(K, case["fill"], np.float64)
    w[:len(case["w"])] = case["w"]
    Wd = dev(w.astype(np.float16)[None, :])
    packed = case["mode"] == "packed"
    s, z = cuda_lib.group_params(Wd, case["bits"], case["group"],
                                 torch.float16 if packed else torch.float32)
    assert host(s).astype(np.float64).ravel().tolist() == case["scales"]
    assert host(z).astype(np.float64).ravel().tolist() == case["zeros"]
    q = host(cuda_lib.quantize_codes(Wd, s, z, case["bits"], case["group"])).ravel()
    exp_q = np.full(K, case["codes_fill"])
    exp_q[:len(case["codes"])] = case["codes"]
    assert q.tolist() == exp_q.tolist()
    if packed:
        p = host(cuda_lib.pack_int4(Wd, s, z)).ravel()
        exp_p = np.full(K // 2, case["packed_fill"])
        exp_p[:len(case["packed"])] = case["packed"]
        assert p.tolist() == exp_p.tolist()
