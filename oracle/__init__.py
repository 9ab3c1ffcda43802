"""CPU oracle for the BWTA / BiLLM hot path -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg import this package. The product (``binarized_transformer_b200``) never
does, and the two share no code. The arithmetic lives in ``oracle.c`` (plain C,
loops over unpacked {-1, 0, +1} values, int64 / fp64 accumulation); this file
only compiles it with gcc and marshals numpy arrays.

Pins: ``tests/test_oracle_pins.py`` checks every function here against values
the pages and the mathematics fix (worked tie examples, dense fp64 matmul of
the dequantized operands, brute force on tiny inputs, invariants).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

OK, ERR_ARG, ERR_NONFINITE = 0, 1, 5


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc (no fast-math, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", "-Wall", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        i64, vp, ip = C.c_int64, C.c_void_p, C.c_int
        _lib.orc_quantize_acts.argtypes = [vp, i64, i64, i64, ip, vp, vp]
        _lib.orc_binarize_weights.argtypes = [vp, i64, i64, i64, i64, vp, vp]
        _lib.orc_pack_plane.argtypes = [vp, i64, i64, i64, ip, vp]
        _lib.orc_int_dots.argtypes = [vp, i64, vp, i64, i64, i64, vp]
        _lib.orc_linear_out.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, vp]
        _lib.orc_attn_scores.argtypes = [vp, vp, i64, i64, i64, i64, vp, vp, vp, vp, vp]
        _lib.orc_softmax_ternarize.argtypes = [vp, i64, i64, C.c_float, vp, vp, vp]
        _lib.orc_billm_salient.argtypes = [vp, i64, i64, i64, i64, i64, vp]
        _lib.orc_billm_quantize_rows.argtypes = [vp, i64, i64, i64, i64, i64, i64, ip, vp, vp, vp,
                                                 vp, vp]
        _lib.orc_billm_gemm.argtypes = [vp, i64, i64, i64, i64, i64, vp, vp, vp, vp, vp, vp]
        _lib.orc_billm_dequant.argtypes = [vp, i64, i64, vp, vp, vp, vp, vp]
        _lib.orc_billm_pack.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, i64, vp, vp, vp, vp]
        _lib.orc_set_threads.argtypes = [ip]
        _lib.orc_set_threads.restype = None
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _check(rc, what):
    if rc != OK:
        raise OracleError(f"{what}: status {rc}")


def num_threads() -> int:
    return lib().orc_num_threads()


def set_threads(n: int) -> None:
    lib().orc_set_threads(int(n))


def _half_bits(X):
    X = np.ascontiguousarray(X)
    if X.dtype == np.float16:
        return X.view(np.uint16)
    assert X.dtype == np.uint16
    return X


def quantize_acts(X, ternary=True):
    """fp16 X [M, K] -> (a int8 [M, K] in {-1,0,1}, scale fp32 [M])."""
    Xb = _half_bits(X)
    M, K = Xb.shape
    a = np.zeros((M, K), np.int8)
    s = np.zeros(M, np.float32)
    _check(lib().orc_quantize_acts(_p(Xb), M, K, K, int(bool(ternary)), _p(a), _p(s)),
           "quantize_acts")
    return a, s


def binarize_weights(W, group=0):
    """fp32 W [N, K] -> (b int8 [N, K] in {-1,1}, alpha fp32 [N, G])."""
    W = np.ascontiguousarray(W, np.float32)
    N, K = W.shape
    gs = group if group else K
    G = -(-K // gs)
    b = np.zeros((N, K), np.int8)
    alpha = np.zeros((N, G), np.float32)
    _check(lib().orc_binarize_weights(_p(W), N, K, K, int(group), _p(b), _p(alpha)),
           "binarize_weights")
    return b, alpha


def pack_plane(v, ld_words, plane):
    """int8 [R, K] -> uint32 [R, ld_words]; plane 'mask' (v != 0) or 'sign' (v < 0)."""
    v = np.ascontiguousarray(v, np.int8)
    R, K = v.shape
    out = np.zeros((R, ld_words), np.uint32)
    _check(lib().orc_pack_plane(_p(v), R, K, ld_words, {"mask": 0, "sign": 1}[plane], _p(out)),
           "pack_plane")
    return out


def int_dots(a, b, group=0):
    """int8 a [M, K], b [N, K] -> int64 d [M, N, G] (per-group dot products)."""
    a = np.ascontiguousarray(a, np.int8)
    b = np.ascontiguousarray(b, np.int8)
    M, K = a.shape
    N = b.shape[0]
    gs = group if group else K
    G = -(-K // gs)
    d = np.zeros((M, N, G), np.int64)
    _check(lib().orc_int_dots(_p(a), M, _p(b), N, K, int(group), _p(d)), "int_dots")
    return d


def linear_out(d, alpha, s):
    """d [M, N, G], alpha [N, G], s [M] -> (yref f64, mag f64, yrep f32), each [M, N]."""
    d = np.ascontiguousarray(d, np.int64)
    M, N, G = d.shape
    alpha = np.ascontiguousarray(alpha, np.float32).reshape(N, G)
    s = np.ascontiguousarray(s, np.float32)
    yref = np.zeros((M, N), np.float64)
    mag = np.zeros((M, N), np.float64)
    yrep = np.zeros((M, N), np.float32)
    _check(lib().orc_linear_out(_p(d), M, N, G, _p(alpha), _p(s), _p(yref), _p(mag), _p(yrep)),
           "linear_out")
    return yref, mag, yrep


def attn_scores(q, k, sq, sk):
    """q int8 [BH, Lq, D], k int8 [BH, Lk, D], sq [BH, Lq], sk [BH, Lk] ->
    (S int64, fref f64, frep f32), each [BH, Lq, Lk]."""
    q = np.ascontiguousarray(q, np.int8)
    k = np.ascontiguousarray(k, np.int8)
    BH, Lq, D = q.shape
    Lk = k.shape[1]
    sq = np.ascontiguousarray(sq, np.float32)
    sk = np.ascontiguousarray(sk, np.float32)
    S = np.zeros((BH, Lq, Lk), np.int64)
    fref = np.zeros((BH, Lq, Lk), np.float64)
    frep = np.zeros((BH, Lq, Lk), np.float32)
    _check(lib().orc_attn_scores(_p(q), _p(k), BH, Lq, Lk, D, _p(sq), _p(sk), _p(S), _p(fref),
                                 _p(frep)), "attn_scores")
    return S, fref, frep


def softmax_ternarize(f, c):
    """fp32 scores f [..., L], softmax factor c -> (a int8 {0,1} [..., L],
    scale fp32 [...], p fp64 [..., L]): softmax of f*c per row, kept where
    p > 1/(2L) (0.5 x the row mean), scale = mean of the kept p."""
    f = np.ascontiguousarray(f, np.float32)
    shape = f.shape
    L = shape[-1]
    R = f.size // L
    a = np.zeros(shape, np.int8)
    s = np.zeros(shape[:-1], np.float32)
    p = np.zeros(shape, np.float64)
    _check(lib().orc_softmax_ternarize(_p(f), R, L, C.c_float(c), _p(a), _p(s), _p(p)),
           "softmax_ternarize")
    return a, s, p


def attn_av(a_p, s_p, a_vt, s_vt):
    """A . V with ternary probabilities a_p [BH, Lq, L] (scales s_p [BH, Lq])
    and ternary V^T rows a_vt [BH, D, L] (scales s_vt [BH, D]) ->
    (O int64, O fp64, O fp32 replica), each [BH, Lq, D]."""
    return attn_scores(a_p, a_vt, s_p, s_vt)


def billm_salient(W, block=128, n_sal=8):
    W = np.ascontiguousarray(W, np.float32)
    N, K = W.shape
    sal = np.zeros((K // block, n_sal), np.int32)
    _check(lib().orc_billm_salient(_p(W), N, K, K, block, n_sal, _p(sal)), "billm_salient")
    return sal


def billm_quantize_rows(W, sal, n0, n1, block=128, split=True):
    """Quantize rows [n0, n1) -> dict(cat, b1, b2, scales) for those rows."""
    W = np.ascontiguousarray(W, np.float32)
    N, K = W.shape
    sal = np.ascontiguousarray(sal, np.int32)
    n_sal = sal.shape[1] if sal.ndim == 2 else 0
    R = n1 - n0
    cat = np.zeros((R, K), np.int8)
    b1 = np.zeros((R, K), np.int8)
    b2 = np.zeros((R, K), np.int8)
    scales = np.zeros((R, K // block, 4), np.float32)
    _check(lib().orc_billm_quantize_rows(_p(W), n0, n1, K, K, block, n_sal, int(split),
                                         _p(sal), _p(cat), _p(b1), _p(b2), _p(scales)),
           "billm_quantize_rows")
    return dict(cat=cat, b1=b1, b2=b2, scales=scales, sal=sal, block=block)


def billm_gemm(X, q):
    """fp16 X [M, K] x quantized rows q -> (yref f64 [M, R], mag f64 [M, R])."""
    Xb = _half_bits(X)
    M, K = Xb.shape
    R = q["cat"].shape[0]
    yref = np.zeros((M, R), np.float64)
    mag = np.zeros((M, R), np.float64)
    _check(lib().orc_billm_gemm(_p(Xb), M, K, K, R, q["block"], _p(q["cat"]), _p(q["b1"]),
                                _p(q["b2"]), _p(q["scales"]), _p(yref), _p(mag)), "billm_gemm")
    return yref, mag


def billm_dequant(q):
    R, K = q["cat"].shape
    what = np.zeros((R, K), np.float64)
    _check(lib().orc_billm_dequant(R, K, q["block"], _p(q["cat"]), _p(q["b1"]), _p(q["b2"]),
                                   _p(q["scales"]), _p(what)), "billm_dequant")
    return what


def billm_pack(q, ldw):
    """Packed BiLLM format of the quantized rows (see oracle.c)."""
    R, K = q["cat"].shape
    block = q["block"]
    sal = q["sal"]
    n_sal = sal.shape[1]
    nb = K // block
    sign = np.zeros((R, ldw), np.uint32)
    gmap = np.zeros((R, ldw), np.uint32)
    res = np.zeros((R, nb), np.uint8)
    sal8 = np.zeros((nb, n_sal), np.uint8)
    _check(lib().orc_billm_pack(R, K, block, n_sal, _p(sal), _p(q["cat"]), _p(q["b1"]),
                                _p(q["b2"]), ldw, _p(sign), _p(gmap), _p(res), _p(sal8)),
           "billm_pack")
    return dict(sign=sign, gmap=gmap, res=res, sal=sal8, bscale=q["scales"].copy())


# ------------------------------------------------------------- conveniences
def linear(X, W, group=0, ternary=True):
    """Whole linear layer on the CPU: returns a dict of every intermediate."""
    a, s = quantize_acts(X, ternary)
    b, alpha = binarize_weights(W, group)
    d = int_dots(a, b, group)
    yref, mag, yrep = linear_out(d, alpha, s)
    return dict(a=a, s=s, b=b, alpha=alpha, d=d, dots=d.sum(axis=2), yref=yref, mag=mag,
                yrep=yrep)
