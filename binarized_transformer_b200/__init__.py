"""Python binding of libbwta.so (include/bwta.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libbwta.so. PyTorch provides device memory and the current CUDA
stream. There is no CPU fallback: importing works anywhere, but every call
raises if the compiled library is missing or no CUDA device is present.

Bit planes are returned as int32 tensors holding the uint32 words
(bit i of word w is element 32*w + i).
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbwta.so")
MB_LIB_PATH = os.path.join(_HERE, "libbwta_microbench.so")

BWTA_OK, BWTA_ERR_INVALID_ARG, BWTA_ERR_UNSUPPORTED, BWTA_ERR_ALIGNMENT, BWTA_ERR_CUDA = range(5)
STATUS_NONFINITE, STATUS_TIMEOUT, STATUS_DRAIN = 0x1, 0x2, 0x4
TERNARY, BINARY = 0, 1
ERROR_NAMES = {1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "ALIGNMENT", 4: "CUDA"}

EXPORTS = ["bwta_pack_weights", "bwta_quantize_pack_acts", "bwta_quantize_pack_acts_ex",
           "bwta_gemm", "bwta_gemm_ex", "bwta_gemm_tc",
           "bwta_linear_decode", "bwta_attn_scores", "billm_pack_weights", "billm_gemm",
           "bwta_linear_decode_batched", "bwta_attn_softmax_ternarize", "bwta_attn_av",
           "bwta_selftest_gemm_timeout", "bwta_version"]
GEMM_WEIGHTS_READY = 0x1


class BwtaError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} returned {code} ({ERROR_NAMES.get(code, '?')})")
        self.code = code


class BillmWeightsC(C.Structure):
    _fields_ = [("sign", C.c_void_p), ("gmap", C.c_void_p), ("res", C.c_void_p),
                ("sal", C.c_void_p), ("bscale", C.c_void_p), ("N", C.c_int64),
                ("K", C.c_int64), ("ldw_words", C.c_int64), ("block", C.c_int64),
                ("n_sal", C.c_int64)]


class DecodeJobC(C.Structure):
    _fields_ = [("X", C.c_void_p), ("M", C.c_int64), ("K", C.c_int64), ("ldX", C.c_int64),
                ("wbits", C.c_void_p), ("wscale", C.c_void_p), ("N", C.c_int64),
                ("ldw_words", C.c_int64), ("group", C.c_int64), ("Y", C.c_void_p),
                ("ldY", C.c_int64), ("dots", C.c_void_p), ("ldD", C.c_int64)]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libbwta.so (raises FileNotFoundError if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise FileNotFoundError(f"{path} is missing: run `python -m binarized_transformer_b200.build`")
    lib = C.CDLL(path)
    vp, i64, ci, cf = C.c_void_p, C.c_int64, C.c_int, C.c_float
    lib.bwta_pack_weights.argtypes = [vp, i64, i64, i64, i64, vp, i64, vp, vp, vp]
    lib.bwta_quantize_pack_acts.argtypes = [vp, i64, i64, i64, ci, cf, vp, vp, i64, vp, vp, vp]
    lib.bwta_quantize_pack_acts_ex.argtypes = [vp, i64, i64, i64, ci, cf, vp, vp, i64, vp, i64, vp,
                                               vp, vp]
    lib.bwta_gemm_tc.argtypes = [vp, i64, vp, i64, vp, vp, i64, i64, i64, i64, vp, i64, vp, i64,
                                 vp, vp]
    lib.bwta_gemm.argtypes = [vp, vp, vp, i64, i64, vp, vp, i64, i64, i64, i64, vp, i64, vp, i64,
                              vp, vp]
    lib.bwta_gemm_ex.argtypes = [vp, vp, vp, i64, i64, vp, vp, i64, i64, i64, i64, vp, i64, vp,
                                 i64, C.c_uint32, vp, vp]
    lib.bwta_linear_decode.argtypes = [vp, i64, i64, i64, ci, cf, vp, vp, i64, i64, i64, vp, i64,
                                       vp, i64, C.c_uint32, vp, vp]
    lib.bwta_attn_scores.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, vp, vp, vp]
    lib.bwta_attn_softmax_ternarize.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64,
                                                cf, vp, vp, i64, vp, vp]
    lib.bwta_attn_av.argtypes = [vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, vp, vp, vp]
    lib.billm_pack_weights.argtypes = [vp, i64, ci, C.POINTER(BillmWeightsC), vp, vp]
    lib.billm_gemm.argtypes = [vp, i64, i64, C.POINTER(BillmWeightsC), vp, i64, vp, vp]
    lib.bwta_linear_decode_batched.argtypes = [C.POINTER(DecodeJobC), i64, ci, cf, C.c_uint32, vp,
                                               vp]
    lib.bwta_selftest_gemm_timeout.argtypes = [vp, vp, vp, i64, i64, vp, vp, i64, i64, i64, i64,
                                               vp, i64, vp, i64, i64, vp, vp]
    lib.bwta_version.restype = C.c_char_p
    for name in EXPORTS[:-1]:
        getattr(lib, name).restype = C.c_int
    _lib = lib
    return lib


def _L():
    if not torch.cuda.is_available():
        raise RuntimeError("libbwta needs a CUDA device; there is no CPU fallback")
    return load_library()


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream():
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check(fn, rc):
    if rc != BWTA_OK:
        raise BwtaError(fn, rc)


def _row_stride(t: torch.Tensor) -> int:
    """Leading dimension of a row-major 2-D tensor (a single row may carry any stride)."""
    return t.stride(0) if t.shape[0] > 1 else t.shape[1]


def ld_words_for(K: int) -> int:
    """Smallest legal row stride in words: ceil(K/32) rounded up to a multiple of 4."""
    return ((K + 31) // 32 + 3) // 4 * 4


def new_status(device=None):
    return torch.zeros(1, dtype=torch.int32, device=device or "cuda")


def version() -> str:
    return load_library().bwta_version().decode()


# ------------------------------------------------------------------ BWTA
def bwta_pack_weights(W: torch.Tensor, group: int = 0, ld_words: int | None = None,
                      status: torch.Tensor | None = None):
    """fp32 W [N, K] (cuda) -> (wbits int32 [N, ld_words], wscale fp32 [N, G])."""
    lib = _L()
    assert W.is_cuda and W.dtype == torch.float32 and W.dim() == 2 and W.stride(1) == 1
    N, K = W.shape
    ld = ld_words or ld_words_for(K)
    G = -(-K // group) if group else 1
    wbits = torch.empty((N, ld), dtype=torch.int32, device=W.device)
    wscale = torch.empty((N, G), dtype=torch.float32, device=W.device)
    _check("bwta_pack_weights", lib.bwta_pack_weights(
        _ptr(W), N, K, _row_stride(W), group, _ptr(wbits), ld, _ptr(wscale), _ptr(status), _stream()))
    return wbits, wscale


def bwta_quantize_pack_acts(X: torch.Tensor, mode: int = TERNARY, thresh_ratio: float = 0.5,
                            ld_words: int | None = None, status: torch.Tensor | None = None,
                            out=None):
    """fp16 X [M, K] (cuda) -> (mask int32 [M, ld], sign int32 [M, ld], scale fp32 [M])."""
    lib = _L()
    assert X.is_cuda and X.dtype == torch.float16 and X.dim() == 2 and X.stride(1) == 1
    M, K = X.shape
    ld = ld_words or ld_words_for(K)
    if out is None:
        mask = torch.empty((M, ld), dtype=torch.int32, device=X.device)
        sign = torch.empty((M, ld), dtype=torch.int32, device=X.device)
        scale = torch.empty((M,), dtype=torch.float32, device=X.device)
    else:
        mask, sign, scale = out
    _check("bwta_quantize_pack_acts", lib.bwta_quantize_pack_acts(
        _ptr(X), M, K, _row_stride(X), mode, thresh_ratio, _ptr(mask), _ptr(sign), ld, _ptr(scale),
        _ptr(status), _stream()))
    return mask, sign, scale


def e4m3_ld_for(K: int) -> int:
    """Row stride in bytes of E4M3 activations for the tensor-core GEMM."""
    return ld_words_for(K) * 32


def bwta_quantize_pack_acts_ex(X: torch.Tensor, mode: int = TERNARY, thresh_ratio: float = 0.5,
                               planes: bool = True, e4m3: bool = True, status=None, out=None):
    """fp16 X [M, K] -> (mask, sign or None, E4M3 uint8 [M, 32*ld] or None, scale [M])."""
    lib = _L()
    assert X.is_cuda and X.dtype == torch.float16 and X.dim() == 2 and X.stride(1) == 1
    M, K = X.shape
    ld = ld_words_for(K)
    if out is None:
        mask = torch.empty((M, ld), dtype=torch.int32, device=X.device) if planes else None
        sign = torch.empty((M, ld), dtype=torch.int32, device=X.device) if planes else None
        a8 = torch.empty((M, 32 * ld), dtype=torch.uint8, device=X.device) if e4m3 else None
        scale = torch.empty((M,), dtype=torch.float32, device=X.device)
    else:
        mask, sign, a8, scale = out
    _check("bwta_quantize_pack_acts_ex", lib.bwta_quantize_pack_acts_ex(
        _ptr(X), M, K, _row_stride(X), mode, thresh_ratio, _ptr(mask), _ptr(sign), ld, _ptr(a8),
        a8.shape[1] if a8 is not None else 0, _ptr(scale), _ptr(status), _stream()))
    return mask, sign, a8, scale


def bwta_gemm_tc(a_e4m3, a_scale, wbits, wscale, K: int, group: int = 0, want_y: bool = True,
                 want_dots: bool = False, status=None, out=None):
    """Tensor-core GEMM on E4M3 activations. Returns (Y fp32 [M, N] or None, dots or None)."""
    lib = _L()
    M, ld8 = a_e4m3.shape
    N, ldw = wbits.shape
    if out is None:
        Y = torch.empty((M, N), dtype=torch.float32, device=a_e4m3.device) if want_y else None
        D = torch.empty((M, N), dtype=torch.int32, device=a_e4m3.device) if want_dots else None
    else:
        Y, D = out
    _check("bwta_gemm_tc", lib.bwta_gemm_tc(
        _ptr(a_e4m3), ld8, _ptr(a_scale), M, _ptr(wbits), _ptr(wscale), N, ldw, K, group, _ptr(Y),
        _row_stride(Y) if Y is not None else N, _ptr(D), _row_stride(D) if D is not None else N,
        _ptr(status), _stream()))
    return Y, D


def bwta_gemm(a_mask, a_sign, a_scale, wbits, wscale, K: int, group: int = 0,
              want_y: bool = True, want_dots: bool = False, status=None, out=None,
              flags: int = 0):
    """Bit-packed GEMM. Returns (Y fp32 [M, N] or None, dots int32 [M, N] or None).
    flags=GEMM_WEIGHTS_READY (weights complete before the call) goes through
    bwta_gemm_ex; 0 through bwta_gemm."""
    lib = _L()
    M, lda = a_mask.shape
    N, ldw = wbits.shape
    if out is None:
        Y = torch.empty((M, N), dtype=torch.float32, device=a_mask.device) if want_y else None
        D = torch.empty((M, N), dtype=torch.int32, device=a_mask.device) if want_dots else None
    else:
        Y, D = out
    ldY = _row_stride(Y) if Y is not None else N
    ldD = _row_stride(D) if D is not None else N
    if flags:
        rc = lib.bwta_gemm_ex(_ptr(a_mask), _ptr(a_sign), _ptr(a_scale), M, lda, _ptr(wbits),
                              _ptr(wscale), N, ldw, K, group, _ptr(Y), ldY, _ptr(D), ldD, flags,
                              _ptr(status), _stream())
        _check("bwta_gemm_ex", rc)
    else:
        _check("bwta_gemm", lib.bwta_gemm(
            _ptr(a_mask), _ptr(a_sign), _ptr(a_scale), M, lda, _ptr(wbits), _ptr(wscale), N, ldw,
            K, group, _ptr(Y), ldY, _ptr(D), ldD, _ptr(status), _stream()))
    return Y, D


def bwta_selftest_gemm_timeout(a_mask, a_sign, a_scale, wbits, wscale, K: int, group: int = 0,
                               wait_limit_ns: int = 1_000_000, status=None, out=None):
    """Failure-path self-test: the tiled GEMM with a wait that is made to run
    out after wait_limit_ns. Returns the status tensor (BWTA_STATUS_TIMEOUT set)."""
    lib = _L()
    M, lda = a_mask.shape
    N, ldw = wbits.shape
    status = new_status(a_mask.device) if status is None else status
    if out is None:
        Y = torch.empty((M, N), dtype=torch.float32, device=a_mask.device)
        D = None
    else:
        Y, D = out
    _check("bwta_selftest_gemm_timeout", lib.bwta_selftest_gemm_timeout(
        _ptr(a_mask), _ptr(a_sign), _ptr(a_scale), M, lda, _ptr(wbits), _ptr(wscale), N, ldw, K,
        group, _ptr(Y), _row_stride(Y) if Y is not None else N, _ptr(D),
        _row_stride(D) if D is not None else N, wait_limit_ns, _ptr(status), _stream()))
    return status


def bwta_linear_decode(X, wbits, wscale, group: int = 0, mode: int = TERNARY,
                       thresh_ratio: float = 0.5, want_y: bool = True, want_dots: bool = False,
                       flags: int = 0, status=None, out=None):
    """Fused decode: fp16 X [M<=8, K] -> ternarize in-kernel -> x packed weights.
    Returns (Y fp32 [M, N] or None, dots int32 [M, N] or None)."""
    lib = _L()
    assert X.is_cuda and X.dtype == torch.float16 and X.dim() == 2 and X.stride(1) == 1
    M, K = X.shape
    N, ldw = wbits.shape
    if out is None:
        Y = torch.empty((M, N), dtype=torch.float32, device=X.device) if want_y else None
        D = torch.empty((M, N), dtype=torch.int32, device=X.device) if want_dots else None
    else:
        Y, D = out
    _check("bwta_linear_decode", lib.bwta_linear_decode(
        _ptr(X), M, K, _row_stride(X), mode, thresh_ratio, _ptr(wbits), _ptr(wscale), N, ldw, group,
        _ptr(Y), _row_stride(Y) if Y is not None else N, _ptr(D),
        _row_stride(D) if D is not None else N, flags, _ptr(status), _stream()))
    return Y, D


def decode_jobs(jobs, want_dots: bool = False):
    """C descriptors for bwta_linear_decode_batched. Each job is a tuple
    (X fp16 [M, K], wbits, wscale, group) or (X, wbits, wscale, group, Y, dots)
    with preallocated outputs (either may be None). Returns (array, outputs)."""
    arr = (DecodeJobC * max(1, len(jobs)))()
    outs = []
    for i, job in enumerate(jobs):
        X, wbits, wscale, group = job[:4]
        assert X.is_cuda and X.dtype == torch.float16 and X.dim() == 2 and X.stride(1) == 1
        M, K = X.shape
        N, ldw = wbits.shape
        if len(job) > 4:
            Y, D = job[4], job[5]
        else:
            Y = torch.empty((M, N), dtype=torch.float32, device=X.device)
            D = torch.empty((M, N), dtype=torch.int32, device=X.device) if want_dots else None
        arr[i] = DecodeJobC(X.data_ptr(), M, K, _row_stride(X), wbits.data_ptr(), wscale.data_ptr(),
                            N, ldw, group, Y.data_ptr() if Y is not None else None,
                            _row_stride(Y) if Y is not None else N,
                            D.data_ptr() if D is not None else None,
                            _row_stride(D) if D is not None else N)
        outs.append((Y, D))
    return arr, outs


def bwta_linear_decode_batched(jobs, mode: int = TERNARY, thresh_ratio: float = 0.5,
                               want_dots: bool = False, flags: int = 0, status=None,
                               descriptors=None):
    """Several fused decode projections in one launch. `jobs` as decode_jobs();
    or pass `descriptors` = decode_jobs(...) built once (the outputs they name).
    Returns [(Y, dots or None)] per job."""
    lib = _L()
    arr, outs = descriptors if descriptors is not None else decode_jobs(jobs, want_dots)
    n = len(outs)
    _check("bwta_linear_decode_batched", lib.bwta_linear_decode_batched(
        arr, n, mode, thresh_ratio, flags, _ptr(status), _stream()))
    return outs


def bwta_attn_scores(q_mask, q_sign, q_scale, k_mask, k_sign, k_scale, BH: int, Lq: int, Lk: int,
                     D: int, want_int: bool = True, want_float: bool = True, out=None):
    """Ternary Q.K^T scores. Returns (S int32 [BH, Lq, Lk] or None, S fp32 or None)."""
    lib = _L()
    ld = q_mask.shape[-1]
    dev = q_mask.device
    if out is None:
        Si = torch.empty((BH, Lq, Lk), dtype=torch.int32, device=dev) if want_int else None
        Sf = torch.empty((BH, Lq, Lk), dtype=torch.float32, device=dev) if want_float else None
    else:
        Si, Sf = out
    _check("bwta_attn_scores", lib.bwta_attn_scores(
        _ptr(q_mask), _ptr(q_sign), _ptr(q_scale), _ptr(k_mask), _ptr(k_sign), _ptr(k_scale),
        BH, Lq, Lk, D, ld, _ptr(Si), _ptr(Sf), _stream()))
    return Si, Sf


def bwta_attn_softmax_ternarize(q_mask, q_sign, q_scale, k_mask, k_sign, k_scale, BH: int,
                                Lq: int, Lk: int, D: int, softmax_scale: float, out=None):
    """Ternary attention probabilities from ternary Q, K planes (scores never
    stored). Returns (p_mask, p_sign, p_scale): [BH*Lq, ld_words_for(Lk)] x2, [BH*Lq]."""
    lib = _L()
    ld = q_mask.shape[-1]
    ldp = ld_words_for(Lk)
    dev = q_mask.device
    if out is None:
        pm = torch.empty((BH * Lq, ldp), dtype=torch.int32, device=dev)
        ps = torch.empty((BH * Lq, ldp), dtype=torch.int32, device=dev)
        sc = torch.empty((BH * Lq,), dtype=torch.float32, device=dev)
    else:
        pm, ps, sc = out
    _check("bwta_attn_softmax_ternarize", lib.bwta_attn_softmax_ternarize(
        _ptr(q_mask), _ptr(q_sign), _ptr(q_scale), _ptr(k_mask), _ptr(k_sign), _ptr(k_scale),
        BH, Lq, Lk, D, ld, softmax_scale, _ptr(pm), _ptr(ps), pm.shape[1], _ptr(sc), _stream()))
    return pm, ps, sc


def bwta_attn_av(p_mask, p_sign, p_scale, vt_mask, vt_sign, vt_scale, BH: int, Lq: int, D: int,
                 Lk: int, want_int: bool = False, want_float: bool = True, out=None):
    """A . V with ternary probabilities and V^T planes. Returns (O int32 or None,
    O fp32 or None), each [BH, Lq, D]."""
    lib = _L()
    ld = p_mask.shape[-1]
    dev = p_mask.device
    if out is None:
        Oi = torch.empty((BH, Lq, D), dtype=torch.int32, device=dev) if want_int else None
        Of = torch.empty((BH, Lq, D), dtype=torch.float32, device=dev) if want_float else None
    else:
        Oi, Of = out
    _check("bwta_attn_av", lib.bwta_attn_av(
        _ptr(p_mask), _ptr(p_sign), _ptr(p_scale), _ptr(vt_mask), _ptr(vt_sign), _ptr(vt_scale),
        BH, Lq, D, Lk, ld, _ptr(Oi), _ptr(Of), _stream()))
    return Oi, Of


# ------------------------------------------------------------------ BiLLM
@dataclass
class BillmWeights:
    sign: torch.Tensor     # int32 [N, ldw]
    gmap: torch.Tensor     # int32 [N, ldw]
    res: torch.Tensor      # uint8 [N, K/block]
    sal: torch.Tensor      # uint8 [K/block, n_sal]
    bscale: torch.Tensor   # fp32 [N, K/block, 4]
    N: int
    K: int
    block: int = 128
    n_sal: int = 8

    @property
    def ldw(self) -> int:
        return self.sign.shape[1]

    def cstruct(self) -> BillmWeightsC:
        return BillmWeightsC(self.sign.data_ptr(), self.gmap.data_ptr(), self.res.data_ptr(),
                             self.sal.data_ptr() if self.sal.numel() else None,
                             self.bscale.data_ptr(), self.N, self.K, self.ldw, self.block,
                             self.n_sal)

    @staticmethod
    def empty(N: int, K: int, n_sal: int = 8, block: int = 128, device="cuda"):
        ld = ld_words_for(K)
        nb = K // block
        return BillmWeights(
            sign=torch.empty((N, ld), dtype=torch.int32, device=device),
            gmap=torch.empty((N, ld), dtype=torch.int32, device=device),
            res=torch.empty((N, nb), dtype=torch.uint8, device=device),
            sal=torch.empty((nb, n_sal), dtype=torch.uint8, device=device),
            bscale=torch.empty((N, nb, 4), dtype=torch.float32, device=device),
            N=N, K=K, block=block, n_sal=n_sal)


def billm_pack_weights(W: torch.Tensor, n_sal: int = 8, split=True, block: int = 128,
                       status=None) -> BillmWeights:
    """Latent fp32 W [N, K] (cuda) -> packed BiLLM weights, built on the GPU.
    split: False/0 no split, True/1 break-point 0.5*max|w|, 2 searched break-point."""
    lib = _L()
    assert W.is_cuda and W.dtype == torch.float32 and W.dim() == 2 and W.stride(1) == 1
    N, K = W.shape
    out = BillmWeights.empty(N, K, n_sal, block, W.device)
    cs = out.cstruct()
    _check("billm_pack_weights", lib.billm_pack_weights(
        _ptr(W), _row_stride(W), int(split), C.byref(cs), _ptr(status), _stream()))
    return out


def billm_gemm(X: torch.Tensor, Wq: BillmWeights, status=None, out=None) -> torch.Tensor:
    """fp16 X [M, K] x BiLLM weights -> Y fp32 [M, N]."""
    lib = _L()
    assert X.is_cuda and X.dtype == torch.float16 and X.dim() == 2 and X.stride(1) == 1
    M = X.shape[0]
    Y = out if out is not None else torch.empty((M, Wq.N), dtype=torch.float32, device=X.device)
    cs = Wq.cstruct()
    _check("billm_gemm", lib.billm_gemm(_ptr(X), M, _row_stride(X), C.byref(cs), _ptr(Y),
                                        _row_stride(Y), _ptr(status), _stream()))
    return Y


# ------------------------------------------------------------------ helpers
def as_u32(t: torch.Tensor):
    """A bit-plane tensor (int32 on any device) as a numpy uint32 array."""
    return t.detach().cpu().numpy().view("uint32")


def half_from_numpy(x, device="cuda") -> torch.Tensor:
    return torch.from_numpy(x).to(device)
