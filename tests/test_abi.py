"""The C-ABI library loads, exports every symbol include/bc.h declares, and
rejects bad arguments on the host before touching the GPU (CPU only)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bc.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"BC_API\s+[\w\s\*]*?\b(bc_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def qmm():
    import quantized_matmul_02_b200 as q
    return q


def test_header_declares_the_calls():
    names = _declared()
    for n in ("bc_group_params", "bc_pack_int4", "bc_matmul_q",
              "bc_quantize_codes", "bc_matmul_q_batched"):
        assert n in names


def test_library_exports_every_declared_symbol(qmm):
    lib = ctypes.CDLL(qmm.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
    assert set(_declared()) == set(qmm.EXPORTS)


def test_status_strings_and_version(qmm):
    assert qmm.lib.bc_version() >= 100
    for st in range(6):
        assert qmm.status_string(st)
    assert qmm.status_string(0) == "ok"


FAKE = 0x10000  # 16-byte aligned non-null address: never dereferenced


@pytest.mark.parametrize("args,expect", [
    # x is NULL
    ((None, 0, FAKE, FAKE, FAKE, 1, 8, 64, 4, 64, 0, FAKE, None, 0, None), 1),
    # K not a multiple of 64
    ((FAKE, 0, FAKE, FAKE, FAKE, 1, 8, 96, 4, 64, 0, FAKE, None, 0, None), 1),
    # bits 9 (the lever goes 16 -> 2; 9..15 are not offered)
    ((FAKE, 0, FAKE, FAKE, FAKE, 1, 8, 64, 9, 64, 0, FAKE, None, 0, None), 2),
    # packed mode at a width that is not packed (2, 3, 4 and 8 are)
    ((FAKE, 0, FAKE, FAKE, FAKE, 1, 8, 64, 5, 64, 1, FAKE, None, 0, None), 2),
    # group 32 is not offered
    ((FAKE, 0, FAKE, FAKE, FAKE, 1, 8, 128, 4, 32, 0, FAKE, None, 0, None), 2),
    # bf16 x below M=64
    ((FAKE, 2, FAKE, FAKE, FAKE, 8, 8, 64, 4, 64, 1, FAKE, None, 0, None), 2),
    # fp16 x is not offered (fp32 decode, bf16 prefill)
    ((FAKE, 1, FAKE, FAKE, FAKE, 128, 8, 64, 4, 64, 0, FAKE, None, 0, None), 2),
    # bf16 x in runtime mode below M = 64
    ((FAKE, 2, FAKE, FAKE, FAKE, 32, 8, 64, 4, 64, 0, FAKE, None, 0, None), 2),
    # range mode without the ranges
    ((FAKE, 0, FAKE, None, None, 1, 8, 64, 4, 64, 2, FAKE, None, 0, None), 1),
    # no such mode
    ((FAKE, 0, FAKE, FAKE, FAKE, 1, 8, 64, 4, 64, 7, FAKE, None, 0, None), 2),
    # misaligned x
    ((FAKE + 4, 0, FAKE, FAKE, FAKE, 1, 8, 64, 4, 64, 0, FAKE, None, 0, None), 3),
    # misaligned fp32 scales
    ((FAKE, 0, FAKE, FAKE + 2, FAKE, 1, 8, 64, 4, 64, 0, FAKE, None, 0, None), 3),
    # scales NULL while bits < 16
    ((FAKE, 0, FAKE, None, FAKE, 1, 8, 64, 4, 64, 0, FAKE, None, 0, None), 1),
    # M = 0
    ((FAKE, 0, FAKE, FAKE, FAKE, 0, 8, 64, 4, 64, 0, FAKE, None, 0, None), 1),
])
def test_matmul_rejects_on_host(qmm, args, expect):
    assert qmm.lib.bc_matmul_q(*args) == expect


def test_other_calls_reject_on_host(qmm):
    L = qmm.lib
    assert L.bc_group_params(None, 8, 64, 4, 64, 0, FAKE, FAKE, None) == 1
    assert L.bc_group_params(FAKE, 8, 64, 1, 64, 0, FAKE, FAKE, None) == 2
    assert L.bc_group_params(FAKE, 8, 64, 4, 64, 2, FAKE, FAKE, None) == 2
    assert L.bc_group_params(FAKE + 8, 8, 64, 4, 64, 0, FAKE, FAKE, None) == 3
    assert L.bc_quantize_codes(FAKE, FAKE, FAKE, 0, 8, 100, 4, 64, FAKE, None) == 1
    assert L.bc_pack_int4(FAKE, FAKE, FAKE, 8, 64, None, None) == 1
    assert L.bc_pack_int4(FAKE, FAKE, FAKE, -1, 64, FAKE, None) == 1
    assert L.bc_matmul_q_batched(None, 1, 1, 4, 64, 1, 0, None, 0, None) == 1
    assert L.bc_group_minmax(None, 8, 64, 64, FAKE, None) == 1
    assert L.bc_group_minmax(FAKE, 8, 64, 32, FAKE, None) == 2
    assert L.bc_group_minmax(FAKE, 8, 64, 64, FAKE + 2, None) == 3
    # argmax: no token buffer; workspace smaller than the logits
    assert L.bc_matmul_q_argmax(FAKE, 0, FAKE, None, None, 1, 8, 64, 16, 64, 0, None,
                                FAKE, 4096, None) == 1
    assert L.bc_matmul_q_argmax(FAKE, 0, FAKE, None, None, 1, 1 << 20, 64, 16, 64, 0, FAKE,
                                FAKE, 4096, None) == 4
