"""The C ABI library: it loads without a GPU, exports every function the header
declares, and rejects bad arguments on the host before touching a device."""
import os
import re

import pytest

import fp8_linear_layers_b200 as ql
from fp8_linear_layers_b200 import build as qbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qlinear.h")


@pytest.fixture(scope="module")
def L():
    qbuild.build()
    return ql.lib()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qlinear_\w+)\s*\(", text)))


def test_header_declarations_match_binding():
    assert _declared() == sorted(ql.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    for name in _declared():
        assert hasattr(L, name), name


def test_status_strings(L):
    for code in range(8):
        assert L.qlinear_status_string(code)
    assert L.qlinear_status_string(99) == b"unknown status"


ALIGNED = 0x10000  # a fake, 16-byte aligned address: never dereferenced on these paths


def test_host_validation_rejects_before_launch(L):
    INV, SHAPE, MIS = 1, 2, 3
    # unknown scheme, null pointers, misaligned pointers
    assert L.qlinear_gemv(7, ALIGNED, ALIGNED, ALIGNED, 64, 64, ALIGNED, None, None) == INV
    assert L.qlinear_gemv(0, None, ALIGNED, ALIGNED, 64, 64, ALIGNED, None, None) == INV
    assert L.qlinear_gemv(0, ALIGNED + 2, ALIGNED, ALIGNED, 64, 64, ALIGNED, None, None) == MIS
    # K must be a multiple of 16; block scheme needs multiples of 128
    assert L.qlinear_gemv(0, ALIGNED, ALIGNED, ALIGNED, 64, 40, ALIGNED, None, None) == SHAPE
    assert L.qlinear_gemv(2, ALIGNED, ALIGNED, ALIGNED, 64, 256, ALIGNED, None, None) == SHAPE
    assert L.qlinear_gemv(2, ALIGNED, ALIGNED, ALIGNED, 128, 192, ALIGNED, None, None) == SHAPE
    assert L.qlinear_quantize_act(2, ALIGNED, 4, 200, ALIGNED, ALIGNED, None) == SHAPE
    assert L.qlinear_quantize_weight(2, ALIGNED, 100, 128, ALIGNED, ALIGNED, None) == SHAPE
    # int8 accumulators are int32: K * 127^2 must stay below 2^31
    assert L.qlinear_gemm(0, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 64, 64, 133152, ALIGNED, None, 0,
                          None, None) == SHAPE
    # negative sizes, and the small-M path's token limit
    assert L.qlinear_quantize_act(0, ALIGNED, -1, 64, ALIGNED, ALIGNED, None) == INV
    assert L.qlinear_gemm_small(0, ALIGNED, ALIGNED, ALIGNED, 33, 64, 64, ALIGNED, ALIGNED, 1 << 20,
                                None, None) == SHAPE
    # the weight-only GEMV: the same argument rules, and K at most 16384
    WO = L.qlinear_gemv_weight_only
    assert WO(7, ALIGNED, ALIGNED, ALIGNED, 64, 64, ALIGNED, None) == INV
    assert WO(1, None, ALIGNED, ALIGNED, 64, 64, ALIGNED, None) == INV
    assert WO(1, ALIGNED, ALIGNED + 8, ALIGNED, 64, 64, ALIGNED, None) == MIS
    assert WO(0, ALIGNED, ALIGNED, ALIGNED, 64, 40, ALIGNED, None) == SHAPE
    assert WO(2, ALIGNED, ALIGNED, ALIGNED, 100, 256, ALIGNED, None) == SHAPE
    assert WO(0, ALIGNED, ALIGNED, ALIGNED, 16, 16400, ALIGNED, None) == SHAPE
    # the grouped GEMV: 1 to QL_GEMV_MAX_GROUP products, each checked as qlinear_gemv
    import ctypes
    P = ql._GemvProblem
    table = (P * 2)(P(ALIGNED, 0, 0, ALIGNED, ALIGNED, ALIGNED, 64), P(ALIGNED, 0, 0, ALIGNED, ALIGNED, ALIGNED, 64))
    tp = ctypes.cast(table, ctypes.c_void_p)
    GR = L.qlinear_gemv_grouped
    assert GR(0, tp, 0, 64, None) == INV
    assert GR(0, tp, ql.GEMV_MAX_GROUP + 1, 64, None) == INV
    assert GR(0, None, 1, 64, None) == INV
    assert GR(7, tp, 2, 64, None) == INV
    assert GR(0, tp, 2, 40, None) == SHAPE
    assert GR(2, tp, 2, 256, None) == SHAPE      # N = 64: not a multiple of 128
    table[1].y = ALIGNED + 4
    assert GR(0, tp, 2, 64, None) == MIS
    table[1].y = 0
    assert GR(0, tp, 2, 64, None) == INV
    table[1].y, table[1].x = ALIGNED, 0   # no x and no pre-quantized input
    assert GR(0, tp, 2, 64, None) == INV
    table[1].qx = ALIGNED
    assert GR(0, tp, 2, 64, None) == INV  # codes without scales
    table[1].sx = ALIGNED + 4
    assert GR(0, tp, 2, 64, None) == MIS
    # the grouped GEMM: 1 to QL_GEMM_MAX_GROUP products on one quantized input
    G = ql._GemmProblem
    gt = (G * 2)(G(ALIGNED, ALIGNED, ALIGNED, 0, 0, 256), G(ALIGNED, ALIGNED, ALIGNED, 0, 0, 256))
    gp = ctypes.cast(gt, ctypes.c_void_p)
    GG = L.qlinear_gemm_grouped
    assert GG(0, ALIGNED, ALIGNED, gp, 0, 64, 256, None, 0, None) == INV
    assert GG(0, ALIGNED, ALIGNED, gp, ql.GEMM_MAX_GROUP + 1, 64, 256, None, 0, None) == INV
    assert GG(0, ALIGNED, ALIGNED, None, 1, 64, 256, None, 0, None) == INV
    assert GG(7, ALIGNED, ALIGNED, gp, 2, 64, 256, None, 0, None) == INV
    assert GG(0, ALIGNED, ALIGNED, gp, 2, 64, 40, None, 0, None) == SHAPE
    assert GG(0, None, ALIGNED, gp, 2, 64, 256, None, 0, None) == INV
    gt[1].N = 200
    assert GG(2, ALIGNED, ALIGNED, gp, 2, 64, 256, None, 0, None) == SHAPE  # N % 128 (block)
    gt[1].N, gt[1].y = 256, 0
    assert GG(0, ALIGNED, ALIGNED, gp, 2, 64, 256, None, 0, None) == INV
    assert GG(0, None, None, gp, 2, 0, 256, None, 0, None) == 0  # M = 0: nothing to do
    gt[1].y = ALIGNED
    gt[0].qy, gt[0].sy = ALIGNED, ALIGNED  # output codes asked of one product but not the other
    assert GG(2, ALIGNED, ALIGNED, gp, 2, 64, 256, None, 0, None) == INV
    gt[1].qy, gt[1].sy = ALIGNED, ALIGNED
    assert GG(0, ALIGNED, ALIGNED, gp, 2, 64, 256, None, 0, None) == SHAPE  # codes: block scheme only
    gt[1].sy = ALIGNED + 4
    assert GG(2, ALIGNED, ALIGNED, gp, 2, 64, 256, None, 0, None) == MIS
    # the grouped small-M path: 1 <= M <= 32, tokens bf16 or pre-quantized, no output codes
    gt[0].qy = gt[0].sy = gt[1].qy = gt[1].sy = 0
    gt[0].y = gt[1].y = ALIGNED
    gt[1].N = 256
    GS = L.qlinear_gemm_small_grouped
    assert GS(0, ALIGNED, None, None, gp, 0, 8, 256, ALIGNED, 1 << 20, None) == INV
    assert GS(0, ALIGNED, None, None, gp, ql.GEMM_MAX_GROUP + 1, 8, 256, ALIGNED, 1 << 20, None) == INV
    assert GS(0, ALIGNED, None, None, gp, 2, 33, 256, ALIGNED, 1 << 20, None) == SHAPE
    assert GS(0, None, None, None, gp, 2, 8, 256, ALIGNED, 1 << 20, None) == INV      # no tokens
    assert GS(0, None, ALIGNED, None, gp, 2, 8, 256, ALIGNED, 1 << 20, None) == INV   # codes without scales
    assert GS(0, ALIGNED + 8, None, None, gp, 2, 8, 256, ALIGNED, 1 << 20, None) == MIS
    gt[1].qy = ALIGNED
    assert GS(0, ALIGNED, None, None, gp, 2, 8, 256, ALIGNED, 1 << 20, None) == INV   # no output codes here
    gt[1].qy = 0
    assert GS(0, ALIGNED, None, None, gp, 2, 0, 256, None, 0, None) == 0             # M = 0
    PQ = L.qlinear_gemv_prequant
    assert PQ(0, None, ALIGNED, ALIGNED, ALIGNED, 64, 64, ALIGNED, None) == INV
    assert PQ(0, ALIGNED, None, ALIGNED, ALIGNED, 64, 64, ALIGNED, None) == INV
    assert PQ(0, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 64, 40, ALIGNED, None) == SHAPE
    # M = 0 is a no-op that succeeds without a device
    assert L.qlinear_quantize_act(0, None, 0, 64, None, None, None) == 0
    assert L.qlinear_forward(0, None, None, None, 0, 64, 64, None, None, 0, None) == 0


def test_no_code_shared_between_oracle_and_product():
    """The product never imports or links the oracle, and the oracle never
    includes the product's headers."""
    pkg = os.path.join(ROOT, "fp8_linear_layers_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", src, re.M), f
                assert "oracle" not in src or f.endswith(".py") and "oracle" not in re.sub(
                    r"(#.*|\"\"\"[\s\S]*?\"\"\")", "", src), f
    osrc = open(os.path.join(ROOT, "oracle", "oracle.c")).read()
    assert "#include \"" not in osrc and "qlinear" not in osrc.split("*/", 1)[1]
