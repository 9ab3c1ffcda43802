"""Shared helpers for the GPU parity tests (CUDA path vs the CPU oracle)."""
import numpy as np
import torch

import binarized_transformer_b200 as bt

REL_TOL = 1e-5          # fp32 outputs: |y - yref| <= 1e-5 * |yref| (or * mag, see below)
SENTINEL = -0x5A5A5A5B  # int32 fill of guard regions


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def u32(t):
    return t.detach().cpu().numpy().view(np.uint32)


def guarded(shape, dtype, guard_rows=2, guard_cols=4):
    """A tensor view inside a larger buffer filled with a sentinel.

    Returns (view, check) where check() asserts the guard cells are untouched."""
    R, Ccols = shape
    itemsize = torch.empty((), dtype=dtype).element_size()
    # keep rows 16-byte aligned: pad the row length to a multiple of 16 bytes
    per16 = 16 // itemsize
    ld = ((Ccols + guard_cols) + per16 - 1) // per16 * per16
    buf = torch.empty((R + 2 * guard_rows, ld), dtype=dtype, device="cuda")
    buf.view(torch.int32 if itemsize == 4 else torch.uint8).fill_(SENTINEL if itemsize == 4 else 0xA5)
    ref = buf.clone()
    view = buf[guard_rows:guard_rows + R, :Ccols]

    def check():
        cur = buf.cpu()
        r = ref.cpu()
        cur[guard_rows:guard_rows + R, :Ccols] = r[guard_rows:guard_rows + R, :Ccols]
        assert torch.equal(cur.view(torch.uint8) if itemsize != 4 else cur.view(torch.int32),
                           r.view(torch.uint8) if itemsize != 4 else r.view(torch.int32)), \
            "a kernel wrote outside its output"

    return view, check


def assert_close_rel(y, yref, mag=None, what=""):
    """fp32 y against the fp64 yref: |y-yref| <= 1e-5*|yref| everywhere, or
    <= 1e-5*mag where mag is given (group terms that cancel)."""
    y = np.asarray(y, np.float64)
    err = np.abs(y - yref)
    bound = REL_TOL * np.abs(yref)
    if mag is not None:
        bound = np.maximum(bound, REL_TOL * mag)
    bad = err > bound
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} elements out of tolerance, first at {tuple(i)}: "
                             f"y={y[tuple(i)]!r} yref={yref[tuple(i)]!r} bound={bound[tuple(i)]!r}")
    return int((err > REL_TOL * np.abs(yref)).sum())


def sample_rows(M, n=64):
    """A deterministic spread of row indices including the first and the last."""
    if M <= n:
        return np.arange(M)
    return np.unique(np.concatenate([[0, M - 1], np.linspace(0, M - 1, n - 2).round().astype(int)]))
