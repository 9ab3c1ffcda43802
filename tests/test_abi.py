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


def test_validation_of_the_fused_and_tensor_core_calls(lib):
    """The packer with E4M3 output, the tensor-core GEMM, the fused decode
    (single and batched) and the attention calls past the scores reject bad
    arguments, and accept empty problems, without any launch."""
    import binarized_transformer_b200 as bt
    E = bt
    nan = float("nan")
    # bwta_quantize_pack_acts_ex: half a plane pair, no output, short or
    # misaligned E4M3 rows, ratio, plane stride
    qx = lib.bwta_quantize_pack_acts_ex
    assert qx(FAKE, 2, 256, 256, 0, 0.5, FAKE, None, 8, None, 0, FAKE, None, None) == E.BWTA_ERR_INVALID_ARG
    assert qx(FAKE, 2, 256, 256, 0, 0.5, None, None, 8, None, 0, FAKE, None, None) == E.BWTA_ERR_INVALID_ARG
    assert qx(FAKE, 2, 256, 256, 0, 0.5, None, None, 8, FAKE, 128, FAKE, None, None) == E.BWTA_ERR_INVALID_ARG
    assert qx(FAKE, 2, 256, 256, 0, 0.5, None, None, 8, MISALIGNED, 256, FAKE, None, None) == \
        E.BWTA_ERR_ALIGNMENT
    assert qx(FAKE, 2, 256, 256, 0, 0.5, None, None, 8, FAKE, 264, FAKE, None, None) == E.BWTA_ERR_ALIGNMENT
    assert qx(FAKE, 2, 256, 256, 0, 0.3, None, None, 8, FAKE, 256, FAKE, None, None) == E.BWTA_ERR_UNSUPPORTED
    assert qx(FAKE, 2, 256, 256, 0, 0.5, FAKE, FAKE, 10, None, 0, FAKE, None, None) == E.BWTA_ERR_ALIGNMENT
    # bwta_gemm_tc: no outputs, group, K bound, E4M3 row stride and alignment,
    # weight-plane stride; an empty problem returns OK without a launch
    tc = lib.bwta_gemm_tc
    assert tc(FAKE, 256, FAKE, 4, FAKE, FAKE, 4, 8, 256, 0, None, 4, None, 4, None, None) == \
        E.BWTA_ERR_INVALID_ARG
    assert tc(FAKE, 256, FAKE, 4, FAKE, FAKE, 4, 8, 256, 100, FAKE, 4, None, 4, None, None) == \
        E.BWTA_ERR_UNSUPPORTED
    assert tc(FAKE, 256, FAKE, 4, FAKE, FAKE, 4, 8, (1 << 22) + 1, 0, FAKE, 4, None, 4, None, None) == \
        E.BWTA_ERR_UNSUPPORTED
    assert tc(FAKE, 128, FAKE, 4, FAKE, FAKE, 4, 8, 256, 0, FAKE, 4, None, 4, None, None) == \
        E.BWTA_ERR_INVALID_ARG
    assert tc(MISALIGNED, 256, FAKE, 4, FAKE, FAKE, 4, 8, 256, 0, FAKE, 4, None, 4, None, None) == \
        E.BWTA_ERR_ALIGNMENT
    assert tc(FAKE, 256, FAKE, 4, FAKE, FAKE, 4, 9, 256, 0, FAKE, 4, None, 4, None, None) == \
        E.BWTA_ERR_ALIGNMENT
    assert tc(None, 256, None, 0, FAKE, FAKE, 4, 8, 256, 0, FAKE, 4, None, 4, None, None) == E.BWTA_OK
    # bwta_linear_decode: M > 8, K beyond the decode kernel, ldX < K, flags,
    # ratio, mode, no outputs, misaligned weights
    dc = lib.bwta_linear_decode
    args = dict(X=FAKE, M=1, K=256, ldX=256, mode=0, r=0.5, wb=FAKE, ws=FAKE, N=4, ldw=8, g=128,
                Y=FAKE, ldY=4, D=None, ldD=4, fl=0)

    def dec(**kw):
        a = dict(args, **kw)
        return dc(a["X"], a["M"], a["K"], a["ldX"], a["mode"], a["r"], a["wb"], a["ws"], a["N"],
                  a["ldw"], a["g"], a["Y"], a["ldY"], a["D"], a["ldD"], a["fl"], None, None)
    assert dec(M=9) == E.BWTA_ERR_UNSUPPORTED
    assert dec(K=16385, ldX=16385, ldw=516, g=0) == E.BWTA_ERR_UNSUPPORTED
    assert dec(ldX=128) == E.BWTA_ERR_INVALID_ARG
    assert dec(fl=2) == E.BWTA_ERR_INVALID_ARG
    assert dec(r=0.25) == E.BWTA_ERR_UNSUPPORTED
    assert dec(mode=7) == E.BWTA_ERR_INVALID_ARG
    assert dec(Y=None) == E.BWTA_ERR_INVALID_ARG
    assert dec(wb=MISALIGNED) == E.BWTA_ERR_ALIGNMENT
    # bwta_linear_decode_batched: too many jobs, no descriptor array, the
    # jobs' activation planes beyond the kernel's shared memory; all-empty
    # jobs return OK without a launch
    db = lib.bwta_linear_decode_batched

    def jobs(*specs):
        arr = (bt.DecodeJobC * len(specs))()
        for i, (M, K, N) in enumerate(specs):
            arr[i] = bt.DecodeJobC(0x10000, M, K, K, 0x10000, 0x10000, N, (K + 127) // 128 * 4, 128,
                                   0x10000, N, None, N)
        return arr
    assert db(jobs(*[(1, 256, 4)] * 9), 9, 0, 0.5, 0, None, None) == E.BWTA_ERR_UNSUPPORTED
    assert db(None, 1, 0, 0.5, 0, None, None) == E.BWTA_ERR_INVALID_ARG
    assert db(jobs((8, 16384, 4), (8, 16384, 4)), 2, 0, 0.5, 0, None, None) == E.BWTA_ERR_UNSUPPORTED
    assert db(jobs((0, 256, 4), (1, 256, 0)), 2, 0, 0.5, 0, None, None) == E.BWTA_OK
    # bwta_attn_softmax_ternarize: no keys, wide rows, NaN scale, misaligned
    # probability plane, missing probability scales
    sm = lib.bwta_attn_softmax_ternarize

    def soft(Lk=64, ld=4, scale=0.125, pm=FAKE, ps=FAKE):
        return sm(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 8, Lk, 64, ld, scale, pm, FAKE, 4, ps, None)
    assert soft(Lk=0) == E.BWTA_ERR_INVALID_ARG
    assert soft(ld=36) == E.BWTA_ERR_UNSUPPORTED
    assert soft(scale=nan) == E.BWTA_ERR_UNSUPPORTED
    assert soft(pm=MISALIGNED) == E.BWTA_ERR_ALIGNMENT
    assert soft(ps=None) == E.BWTA_ERR_INVALID_ARG
    # bwta_attn_av: no output
    assert lib.bwta_attn_av(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, 8, 64, 64, 4, None, None, None) == \
        E.BWTA_ERR_INVALID_ARG


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
