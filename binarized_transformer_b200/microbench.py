"""Measured ceilings for the roofline of each kernel (libbwta_microbench.so).

* word-op rate: acc += popc(m & (a ^ w)) -- one LOP3, one POPC, one add; one
  word-op is 32 multiply-adds = 64 binary ops.
* popc4 rate: the bit GEMM's own inner mix per 4-word chunk (four LOP3s, a
  carry-save adder of two LOP3s, three POPCs, the adds), in word-ops: the
  ceiling the tiled GEMM is measured against.
* LOP3, POPC(+add), IMAD issue rates on their own.
* legacy warp MMA rates: b1 AND+POPC (bit products), s8, f16 (fp32 accumulate).
* HBM streaming read and write bandwidth over a 1 GiB buffer.
All rates are per second over the whole GPU, timed with CUDA events.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_lib = None

KINDS = {"wordop": 0, "lop3": 1, "popc": 2, "imad": 3, "mma_b1": 4, "mma_s8": 5, "mma_f16": 6,
         "popc4": 7}
# work per thread per loop iteration
_PER_THREAD_ITER = {"wordop": 16, "lop3": 16, "popc": 16, "imad": 16, "popc4": 32}
_MMA_WORK = {"mma_b1": 16 * 8 * 256, "mma_s8": 16 * 8 * 32, "mma_f16": 16 * 8 * 16}  # MACs / instr


def lib():
    global _lib
    if _lib is None:
        path = os.path.join(_HERE, "libbwta_microbench.so")
        if not os.path.exists(path):
            raise FileNotFoundError(path)
        _lib = C.CDLL(path)
        _lib.bwta_mb_launch.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int, C.c_void_p, C.c_void_p]
        _lib.bwta_mb_read.argtypes = [C.c_void_p, C.c_size_t, C.c_int, C.c_void_p, C.c_void_p]
        _lib.bwta_mb_write.argtypes = [C.c_void_p, C.c_size_t, C.c_int, C.c_void_p]
    return _lib


def _time(fn, reps=5):
    s = torch.cuda.current_stream()
    fn()
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s)
        fn()
        b.record(s)
        b.synchronize()
        best = min(best, a.elapsed_time(b) * 1e-3)
    return best


def rate(kind: str, iters: int = 2048) -> float:
    """Operations per second: word-ops / instructions-lanes for ALU kinds,
    multiply-accumulates for MMA kinds."""
    L = lib()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    blocks, threads = sms * 8, 256
    sink = torch.zeros(4, dtype=torch.int32, device="cuda")
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    k = KINDS[kind]

    def run():
        rc = L.bwta_mb_launch(k, blocks, threads, iters, C.c_void_p(sink.data_ptr()), stream)
        if rc != 0:
            raise RuntimeError(f"microbench {kind}: cuda error {rc}")

    t = _time(run)
    if kind in _MMA_WORK:
        instrs = blocks * (threads // 32) * iters * 4
        return instrs * _MMA_WORK[kind] / t
    return blocks * threads * iters * _PER_THREAD_ITER[kind] / t


def hbm(gib: float = 1.0):
    """(read GB/s, write GB/s) streaming over a buffer of `gib` GiB."""
    L = lib()
    nbytes = int(gib * (1 << 30))
    buf = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    sink = torch.zeros(4, dtype=torch.int32, device="cuda")
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    tw = _time(lambda: L.bwta_mb_write(C.c_void_p(buf.data_ptr()), nbytes, sms * 4, stream))
    tr = _time(lambda: L.bwta_mb_read(C.c_void_p(buf.data_ptr()), nbytes, sms * 4,
                                      C.c_void_p(sink.data_ptr()), stream))
    del buf
    return nbytes / tr / 1e9, nbytes / tw / 1e9


def ceilings() -> dict:
    out = {k: rate(k) for k in KINDS}
    out["hbm_read_gbs"], out["hbm_write_gbs"] = hbm()
    return out


if __name__ == "__main__":
    import json
    print(json.dumps(ceilings(), indent=1))
