"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each test checks the oracle against something the pages or plain
mathematics fix, chosen so that a plausible slip in the oracle (a dropped
term, a wrong sign, adding the zero before rounding, a transposed operand,
a wrong nibble order, round-half-up instead of half-even) fails at least one:

* hand-worked groups (tests/golden/rtn_worked_groups.json);
* exact reproduction of weights that already lie on a quantization grid,
  including exact half-way ties;
* the range of codes and the per-weight error bound |w - w'| <= s/2 (+slack);
* the NAIVE / SMART claim of BITCRUSH BC-06 ("The machine" table): per-group
  scales lose less than per-channel scales at the same bit budget;
* matmuls whose answers have closed forms (one-hot and all-ones inputs) and
  a brute-force rational matmul on tiny shapes;
* the byte ledger against the model sizes the pages print (BITCRUSH BC-06,
  BRAIN SIZE row: 1,192 MB at fp16, 421 MB at 2 bits, "596-million-
  parameter"; Enargeia: 494.0M parameters, 1884.6 MiB in fp32).
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden",
                      "rtn_worked_groups.json")


def _row(case):
    K = case["K"]
    w = np.full(K, case["fill"], np.float64)
    for i, v in enumerate(case["w"]):
        w[i] = v
    return w.astype(np.float16)[None, :]


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"][0:2]
                         + json.load(open(GOLDEN))["cases"][3:],
                         ids=lambda c: c["name"])
def test_golden_single_group(case):
    W = _row(case)
    f16 = case["mode"] == "packed"
    s, z = oracle.group_params(W, case["bits"], case["group"], f16)
    assert s.ravel().tolist() == case["scales"]
    assert z.ravel().tolist() == case["zeros"]
    q = oracle.codes(W, s, z, case["bits"], case["group"])
    exp_q = np.full(case["K"], case["codes_fill"])
    exp_q[:len(case["codes"])] = case["codes"]
    assert q.ravel().tolist() == exp_q.tolist()
    wq = oracle.dequant(q, s, z, case["group"])
    exp_w = np.full(case["K"], case["wq_fill"])
    exp_w[:len(case["wq"])] = case["wq"]
    assert wq.ravel().tolist() == exp_w.tolist()
    if "packed" in case:
        p = oracle.pack_int4(q)
        exp_p = np.full(case["K"] // 2, case["packed_fill"])
        exp_p[:len(case["packed"])] = case["packed"]
        assert p.ravel().tolist() == exp_p.tolist()


def test_golden_group_vs_channel():
    case = [c for c in json.load(open(GOLDEN))["cases"]
            if c["name"] == "runtime_3bit_per_group_vs_per_channel"][0]
    K = case["K"]
    w = np.where(np.arange(K) < 64, case["rows"]["fill_lo"],
                 case["rows"]["fill_hi"]).astype(np.float64)
    for k, v in case["rows"]["w"]:
        w[k] = v
    W = w.astype(np.float16)[None, :]
    for key, group in (("group64", 64), ("channel", K)):
        exp = case[key]
        s, z = oracle.group_params(W, case["bits"], group, False)
        assert s.ravel().tolist() == exp["scales"]
        assert z.ravel().tolist() == exp["zeros"]
        q = oracle.codes(W, s, z, case["bits"], group).ravel()
        wq = oracle.dequant(q[None, :], s, z, group).ravel()
        for k, v in exp["codes"]:
            assert q[k] == v, (key, k)
        for k, v in exp["wq"]:
            assert wq[k] == v, (key, k)
        assert q[10] == exp["codes_fill_lo"] and q[100] == exp["codes_fill_hi"]
        assert wq[10] == exp["wq_fill_lo"] and wq[100] == exp["wq_fill_hi"]


# ---- exact grids ---------------------------------------------------------

def _grid_matrix(rng, bits, N, K, e_lo=4, e_hi=12):
    """W = (q - z) * 2^-e with 0 and L present in every group: the method
    must give back exactly these s, z, q and w' = w."""
    L = (1 << bits) - 1
    G = K // 64
    e = rng.integers(e_lo, e_hi + 1, size=(N, G))
    z = rng.integers(1, L, size=(N, G))           # 0 < z < L: group spans 0
    q = rng.integers(0, L + 1, size=(N, K))
    q[:, 0::64] = 0
    q[:, 1::64] = L
    s = np.ldexp(1.0, -e)
    w = (q - np.repeat(z, 64, axis=1)) * np.repeat(s, 64, axis=1)
    W = w.astype(np.float16)
    assert np.array_equal(W.astype(np.float64), w)    # exact in fp16
    return W, s, z.astype(np.float64), q


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("f16", [False, True])
def test_grid_reproduces_exactly(bits, f16):
    if f16 and bits != 4:
        pytest.skip("fp16 storage is the packed int4 mode")
    rng = np.random.default_rng(100 + bits)
    W, s_true, z_true, q_true = _grid_matrix(rng, bits, 16, 256)
    s, z = oracle.group_params(W, bits, 64, f16)
    assert np.array_equal(s, s_true)
    assert np.array_equal(z, z_true)
    q = oracle.codes(W, s, z, bits, 64)
    assert np.array_equal(q, q_true)
    assert np.array_equal(oracle.dequant(q, s, z, 64), W.astype(np.float64))


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_exact_ties_round_half_even(bits):
    """Weights exactly half-way between grid points: the code is the even
    neighbour of w/s, then the zero is added (Python's round() is
    half-to-even, an implementation independent of the oracle's C rint)."""
    rng = np.random.default_rng(7 + bits)
    L = (1 << bits) - 1
    N, K = 8, 64
    s_true = 2.0 ** -6
    z_true = rng.integers(1, L, size=N)
    W = np.zeros((N, K))
    expect = np.zeros((N, K), np.int64)
    for n in range(N):
        z = int(z_true[n])
        W[n, 0] = -z * s_true
        W[n, 1] = (L - z) * s_true
        expect[n, 0], expect[n, 1] = 0, L
        for k in range(2, K):
            h = int(rng.integers(-z, L - z)) + 0.5      # half-integer in range
            W[n, k] = h * s_true
            expect[n, k] = min(max(round(h) + z, 0), L)
    Wh = W.astype(np.float16)
    assert np.array_equal(Wh.astype(np.float64), W)
    s, z = oracle.group_params(Wh, bits, 64, False)
    assert np.all(s == s_true) and np.array_equal(z[:, 0], z_true)
    assert np.array_equal(oracle.codes(Wh, s, z, bits, 64), expect)


# ---- invariants on Gaussian weights -------------------------------------

@pytest.mark.parametrize("bits", [2, 3, 4, 5, 8])
@pytest.mark.parametrize("group", [64, 512])
def test_range_and_error_bound_fp32(bits, group):
    W = wl.weight(0, 0, "single", 512, 64, 0.02)
    L = (1 << bits) - 1
    s, z = oracle.group_params(W, bits, group, False)
    assert np.all(np.isfinite(s)) and np.all(s > 0)
    assert np.all(z == np.round(z))
    assert np.array_equal(s.astype(np.float32).astype(np.float64), s)
    q = oracle.codes(W, s, z, bits, group)
    assert q.min() >= 0 and q.max() <= L
    wq = oracle.dequant(q, s, z, group)
    srep = np.repeat(s, group, axis=1)
    err = np.abs(W.astype(np.float64) - wq)
    assert np.all(err <= srep * (0.5 + 2.0 ** -14))
    # every group uses its two extreme codes (or L-1 after an exact tie)
    qg = q.reshape(q.shape[0], -1, group)
    assert np.all(qg.min(axis=2) == 0)
    assert np.all(qg.max(axis=2) >= L - 1)


def test_range_and_error_bound_fp16_packed():
    W = wl.weight(0, 1, "single", 1024, 128, 0.02)
    s, z = oracle.group_params(W, 4, 64, True)
    s16 = s.astype(np.float16).astype(np.float64)
    assert np.array_equal(s16, s) and np.array_equal(
        z.astype(np.float16).astype(np.float64), z)
    assert np.all(np.abs(z) <= 2048)
    q = oracle.codes(W, s, z, 4, 64)
    assert q.max() <= 15
    wq = oracle.dequant(q, s, z, 64)
    srep = np.repeat(s, 64, axis=1)
    err = np.abs(W.astype(np.float64) - wq)
    assert np.all(err <= srep * (0.5 + 15 * 2.0 ** -10))


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 7, 8])
def test_per_group_beats_per_channel(bits):
    """BITCRUSH BC-06, NAIVE / SMART: at the same bits, one scale per
    64-weight group loses less than one scale per output channel."""
    W = wl.weight(0, 2, "single", 1024, 256, 0.02)
    w = W.astype(np.float64)
    mse = {}
    for group in (64, 1024):
        s, z = oracle.group_params(W, bits, group, False)
        wq = oracle.dequant(oracle.codes(W, s, z, bits, group), s, z, group)
        mse[group] = np.mean((w - wq) ** 2)
    assert mse[64] < mse[1024]
    # range of 64 vs 1024 normal samples: the ratio is well above 1
    assert mse[1024] / mse[64] > 1.3


def test_subnormal_and_single_sign_groups():
    """Groups of tiny (fp16-subnormal) weights and groups that do not span
    zero: codes stay in range and the zero lands where -min/s puts it."""
    rng = np.random.default_rng(3)
    W = np.zeros((4, 64), np.float16)
    W[0] = (rng.integers(-40, 40, 64) * 2.0 ** -24).astype(np.float16)
    W[1] = (1.0 + rng.integers(0, 512, 64) * 2.0 ** -10).astype(np.float16)
    W[2] = -(1.0 + rng.integers(0, 512, 64) * 2.0 ** -10).astype(np.float16)
    W[3] = (rng.integers(1, 4, 64) * 2.0 ** -24).astype(np.float16)
    for f16, bits in ((False, 3), (False, 8), (True, 4)):
        s, z = oracle.group_params(W, bits, 64, f16)
        q = oracle.codes(W, s, z, bits, 64)
        assert q.max() <= (1 << bits) - 1
        assert np.all(s > 0)
        lo = W.astype(np.float64).min(axis=1)
        assert np.array_equal(z[:, 0], np.array(
            [float(round(-l / sc)) + 0.0 for l, sc in zip(lo, s[:, 0])]))
        if not f16:
            err = np.abs(W.astype(np.float64) - oracle.dequant(q, s, z, 64))
            assert np.all(err <= s * (0.5 + 2.0 ** -14))


# ---- matmul -------------------------------------------------------------

def test_matmul_one_hot_selects_a_column():
    """x = e_k picks column k of W' (catches a transposed operand)."""
    rng = np.random.default_rng(11)
    N, K = 48, 128
    wq = rng.standard_normal((N, K))
    x = np.zeros((3, K))
    x[0, 5] = 1.0
    x[1, 127] = 1.0
    x[2, 64] = -2.0
    y, a = oracle.matmul(x, wq)
    assert np.array_equal(y[0], wq[:, 5])
    assert np.array_equal(y[1], wq[:, 127])
    assert np.array_equal(y[2], -2.0 * wq[:, 64])
    assert np.array_equal(a[2], np.abs(2.0 * wq[:, 64]))


def test_matmul_all_ones_is_row_sum_and_passthrough():
    W = (np.arange(64 * 192).reshape(64, 192) % 13 - 6).astype(np.float16)
    w = oracle.half_to_f64(W)
    assert np.array_equal(w, W.astype(np.float64))
    y, _ = oracle.matmul(np.ones((1, 192)), w)
    assert np.array_equal(y[0], W.astype(np.float64).sum(axis=1))


@pytest.mark.parametrize("bits,group,mode", [(3, 64, "runtime"),
                                             (2, 192, "runtime"),
                                             (4, 64, "packed"),
                                             (16, 64, "runtime")])
def test_brute_force_rational(bits, group, mode):
    """Tiny shapes against exact rational arithmetic: a second, slower
    restatement that rounds Fractions, so the fp64 quotient shortcut of the
    oracle is checked against exact quotients and the fp64 dot product
    against an exact one."""
    rng = np.random.default_rng(bits * 100 + group)
    M, N, K = 3, 5, 192
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    x = rng.standard_normal((M, K)).astype(np.float32)
    r = oracle.matmul_q(x, W, bits, group, mode)
    L = (1 << bits) - 1

    def fl32(f):
        return Fraction(float(np.float32(float(f))))

    def rne(f):
        fl = f.numerator // f.denominator
        rem = f - fl
        if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2):
            fl += 1
        return fl

    wq = [[None] * K for _ in range(N)]
    for n in range(N):
        for j in range(K // group):
            g = [Fraction(float(W[n, k])) for k in range(j * group, (j + 1) * group)]
            if bits == 16:
                for i, v in enumerate(g):
                    wq[n][j * group + i] = v
                continue
            lo, hi = min(g), max(g)
            s = fl32(fl32(hi - lo) / L)
            if mode == "packed":
                s = Fraction(float(np.float16(float(s))))
            z = rne(-lo / s)
            if mode == "packed":
                z = Fraction(float(np.float16(float(z))))
            assert float(s) == r["s"][n, j] and float(z) == r["z"][n, j]
            for i, v in enumerate(g):
                q = min(max(rne(v / s) + z, 0), L)
                assert q == r["codes"][n, j * group + i]
                wq[n][j * group + i] = (q - z) * s
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(x[m, k])) * wq[n][k] for k in range(K))
            assert abs(float(exact) - r["y"][m, n]) <= 1e-12 * r["A"][m, n]


def test_pack_nibble_order():
    q = np.array([[1, 2, 3, 4, 15, 0, 7, 9]], np.uint8)
    assert oracle.pack_int4(q).ravel().tolist() == [0x21, 0x43, 0x0F, 0x97]


def test_half_encoder_rne():
    """The oracle's own fp16 encoder agrees with IEEE RNE at the edges."""
    cases = {1.0 + 2.0 ** -11: 1.0, 1.0 + 3 * 2.0 ** -11: 1.0 + 2 * 2.0 ** -10,
             65519.0: 65504.0, 2.0 ** -25: 0.0, 3 * 2.0 ** -25: 2.0 ** -23,
             0.1: 0.0999755859375}
    for v, e in cases.items():
        assert oracle.f32_to_half_rne(v) == e
    assert oracle.f32_to_half_rne(65520.0) == float("inf")


# ---- byte ledger against the pages' printed sizes -------------------------

def test_byte_ledger_qwen3_06b():
    total = wl.linear_params("qwen3-0.6b") + wl.other_params("qwen3-0.6b")
    assert round(total / 1e6) == 596                 # "596-million-parameter"
    assert round(wl.model_bytes("qwen3-0.6b", 16) / 1e6) == 1192   # 1,192 MB
    assert round(wl.model_bytes("qwen3-0.6b", 2) / 1e6) == 421     # 421 MB
    assert len(wl.layer_set("qwen3-0.6b")) == 196    # 196 weight matrices


def test_byte_ledger_qwen25_05b():
    total = wl.linear_params("qwen2.5-0.5b") + wl.other_params("qwen2.5-0.5b")
    assert round(total / 1e5) / 10 == 494.0          # 494.0M parameters
    assert round(total * 4 / 2 ** 20, 1) == 1884.6   # 1884.6 MiB fp32
    assert wl.linear_params("qwen2.5-0.5b") == 357826560


def test_algorithmic_bytes_qwen25_int4_set():
    tot = sum(wl.gemv_bytes(m.K, m.N, 1, "packed", 4, 64)
              for m in wl.layer_set("qwen2.5-0.5b"))
    assert tot == 203476992


def test_group_range_is_the_library_min_max():
    """The bit-width-independent precompute (BITCRUSH BC-06, "Under the
    hood") stores each group's exact range; numpy's own reductions over the
    fp16 groups must give the same values, per group and per channel."""
    rng = np.random.default_rng(12)
    W = (rng.standard_normal((9, 192)) * np.exp(rng.uniform(-8, 4, (9, 1)))).astype(np.float16)
    W[0] = 0.75
    W[1, :64] = -2.0 ** -24
    for group in (64, 192):
        lo, hi = oracle.group_range(W, group)
        g = W.astype(np.float64).reshape(9, 192 // group, group)
        assert np.array_equal(lo, g.min(axis=2))
        assert np.array_equal(hi, g.max(axis=2))


def test_pack_codes_hand_worked_bytes():
    """Other packed widths: each row is a little-endian bit string with code
    k at bits [bits*k, bits*k + bits).  Hand-worked bytes:
    3-bit codes 1,2,3,4,5,6,7,0: byte0 = 1 | 2<<3 | (3&3)<<6 = 209,
    byte1 = 3>>2 | 4<<1 | 5<<4 | (6&1)<<7 = 88, byte2 = 6>>1 | 7<<2 | 0<<5 = 31;
    2-bit codes 1,2,3,0,3,3,0,1: 1 | 2<<2 | 3<<4 | 0<<6 = 57 and
    3 | 3<<2 | 0<<4 | 1<<6 = 79."""
    q3 = np.zeros((1, 64), np.uint8)
    q3[0, :8] = [1, 2, 3, 4, 5, 6, 7, 0]
    assert oracle.pack_codes(q3, 3)[0, :4].tolist() == [209, 88, 31, 0]
    q2 = np.zeros((1, 64), np.uint8)
    q2[0, :8] = [1, 2, 3, 0, 3, 3, 0, 1]
    assert oracle.pack_codes(q2, 2)[0, :3].tolist() == [57, 79, 0]
    q8 = np.arange(64, dtype=np.uint8)[None, :] * 3
    assert np.array_equal(oracle.pack_codes(q8, 8), q8)


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_pack_codes_matches_numpy_bit_string(bits):
    """Against numpy's own bit packing of the row bit strings (little-endian
    bit order); for 4 bits it is also the int4 packing."""
    rng = np.random.default_rng(bits)
    q = rng.integers(0, 1 << bits, size=(5, 192)).astype(np.uint8)
    bitsarr = ((q[:, :, None] >> np.arange(bits)) & 1).astype(np.uint8).reshape(5, -1)
    expect = np.packbits(bitsarr, axis=1, bitorder="little")
    got = oracle.pack_codes(q, bits)
    assert np.array_equal(got, expect)
    if bits == 4:
        assert np.array_equal(got, oracle.pack_int4(q))
