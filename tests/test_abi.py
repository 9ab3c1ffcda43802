"""The C ABI without a GPU: the library builds and loads, exports every
function include/bwta.h declares, the header is valid C, and host-side
argument validation rejects bad calls before any launch."""
import ctypes as C
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bwta.h")


@pytest.fixture(scope="module")
def lib():
    from binarized_transformer_b200 import build as b
    b.build()
    import binarized_transformer_b200 as bt
    return bt.load_library()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^(?:int|const char \*)\s*(\w+)\(", text, re.M)))


def test_header_is_plain_c():
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-fsyntax-only", "-x", "c", HEADER])


def test_every_declared_function_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 7, names
    out = subprocess.check_output(["nm", "-D", "--defined-only",
                                   os.path.join(ROOT, "binarized_transformer_b200", "libbwta.so")],
                                  text=True)
    exported = set(re.findall(r" T (\w+)$", out, re.M))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert getattr(lib, n) is not None
    assert lib.bwta_version().decode().startswith("bwta")


FAKE = C.c_void_p(0x10000)         # 16-byte aligned, never dereferenced
MISALIGNED = C.c_void_p(0x10004)


def test_validation_rejects_before_launch(lib):
    import binarized_transformer_b200 as bt
    E = bt
    # bwta_pack_weights: K <= 0, ldW < K, bad group, misaligned planes
    assert lib.bwta_pack_weights(FAKE, 4, 0, 0, 0, FAKE, 4, FAKE, None, None) == E.BWTA_ERR_INVALID_ARG
    assert lib.bwta_pack_weights(FAKE, 4, 64, 32, 0, FAKE, 4, FAKE, None, None) == E.BWTA_ERR_INVALID_ARG
    assert lib.bwta_pack_weights(FAKE, 4, 256, 256, 100, FAKE, 8, FAKE, None, None) == E.BWTA_ERR_UNSUPPORTED
    assert lib.bwta_pack_weights(FAKE, 4, 256, 256, 0, MISALIGNED, 8, FAKE, None, None) == E.BWTA_ERR_ALIGNMENT
    assert lib.bwta_pack_weights(FAKE, 4, 256, 256, 0, FAKE, 10, FAKE, None, None) == E.BWTA_ERR_ALIGNMENT
    assert lib.bwta_pack_weights(FAKE, 4, 256, 256, 0, FAKE, 4, FAKE, None, None) == E.BWTA_ERR_INVALID_ARG
    # bwta_quantize_pack_acts: ratio, mode, plane alignment, K bound (fp16 rows of
    # any alignment are accepted, so no call here may pass validation)
    qa = lib.bwta_quantize_pack_acts
    assert qa(FAKE, 2, 64, 64, 0, 0.25, FAKE, FAKE, 4, FAKE, None, None) == E.BWTA_ERR_UNSUPPORTED
    assert qa(FAKE, 2, 64, 64, 7, 0.5, FAKE, FAKE, 4, FAKE, None, None) == E.BWTA_ERR_INVALID_ARG
    assert qa(FAKE, 2, 64, 60, 0, 0.5, FAKE, FAKE, 4, FAKE, None, None) == E.BWTA_ERR_INVALID_ARG
    assert qa(FAKE, 2, 64, 64, 0, 0.5, MISALIGNED, FAKE, 4, FAKE, None, None) == E.BWTA_ERR_ALIGNMENT
    assert qa(FAKE, 2, (1 << 22) + 1, 1 << 23, 0, 0.5, FAKE, FAKE, 1 << 18, FAKE, None, None) == \
        E.BWTA_ERR_UNSUPPORTED
    # bwta_gemm: no outputs, bad group, short ld
    g = lib.bwta_gemm
    assert g(FAKE, FAKE, FAKE, 4, 4, FAKE, FAKE, 4, 4, 64, 0, None, 4, None, 4, None, None) == \
        E.BWTA_ERR_INVALID_ARG
    assert g(FAKE, FAKE, FAKE, 4, 4, FAKE, FAKE, 4, 4, 64, 64, FAKE, 4, None, 4, None, None) == \
        E.BWTA_ERR_UNSUPPORTED
    assert g(FAKE, FAKE, FAKE, 4, 4, FAKE, FAKE, 4, 4, 256, 0, FAKE, 4, None, 4, None, None) == \
        E.BWTA_ERR_INVALID_ARG
    assert g(FAKE, FAKE, FAKE, 4, 4, FAKE, FAKE, 8, 4, 64, 0, FAKE, 4, None, 4, None, None) == \
        E.BWTA_ERR_INVALID_ARG
    assert g(MISALIGNED, FAKE, FAKE, 4, 4, FAKE, FAKE, 4, 4, 64, 0, FAKE, 4, None, 4, None, None) == \
        E.BWTA_ERR_ALIGNMENT
    gx = lib.bwta_gemm_ex
    assert gx(FAKE, FAKE, FAKE, 4, 4, FAKE, FAKE, 4, 4, 64, 0, FAKE, 4, None, 4, 2, None, None) == \
        E.BWTA_ERR_INVALID_ARG
    # bwta_attn_scores: no outputs, ld too large
    at = lib.bwta_attn_scores
    assert at(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 4, 4, 64, 4, None, None, None) == E.BWTA_ERR_INVALID_ARG
    assert at(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 4, 4, 64, 36, FAKE, None, None) == E.BWTA_ERR_UNSUPPORTED
    # BiLLM: block must be 128, n_sal <= 8, K % 128 == 0
    w = bt.BillmWeightsC(0x10000, 0x10000, 0x10000, 0x10000, 0x10000, 4, 256, 8, 64, 8)
    assert lib.billm_gemm(FAKE, 1, 256, C.byref(w), FAKE, 4, None, None) == E.BWTA_ERR_UNSUPPORTED
    w = bt.BillmWeightsC(0x10000, 0x10000, 0x10000, 0x10000, 0x10000, 4, 200, 8, 128, 8)
    assert lib.billm_gemm(FAKE, 1, 256, C.byref(w), FAKE, 4, None, None) == E.BWTA_ERR_UNSUPPORTED
    w = bt.BillmWeightsC(0x10000, 0x10000, 0x10000, 0x10000, 0x10000, 4, 256, 8, 128, 9)
    assert lib.billm_pack_weights(FAKE, 256, 1, C.byref(w), None, None) == E.BWTA_ERR_UNSUPPORTED
    w = bt.BillmWeightsC(0x10004, 0x10000, 0x10000, 0x10000, 0x10000, 4, 256, 8, 128, 8)
    assert lib.billm_gemm(FAKE, 1, 256, C.byref(w), FAKE, 4, None, None) == E.BWTA_ERR_ALIGNMENT
    assert lib.billm_gemm(FAKE, 1, 256, None, FAKE, 4, None, None) == E.BWTA_ERR_INVALID_ARG


def test_binding_has_no_cpu_fallback():
    import torch
    import binarized_transformer_b200 as bt
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(RuntimeError):
        bt.bwta_quantize_pack_acts(torch.zeros((2, 64), dtype=torch.float16))


def test_product_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "binarized_transformer_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "oracle/" not in text, f
