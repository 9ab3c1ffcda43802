"""The batched decode entry point (several projections, one launch): every job
must equal the oracle exactly -- planes and dots as integers, fp32 outputs bit
for bit with the oracle's serial fp32 replica (and within 1e-5 of its fp64
value) -- and equal the single-projection call."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_common import assert_close_rel, dev, guarded

pytestmark = pytest.mark.gpu

bt = pytest.importorskip("binarized_transformer_b200")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    bt.load_library()
    oracle.build()


def check_job(X, W, group, Y, D, ternary=True):
    ref = oracle.linear(X, W, group, ternary=ternary)
    np.testing.assert_array_equal(D, ref["dots"])
    np.testing.assert_array_equal(Y.view(np.uint32), ref["yrep"].view(np.uint32))
    assert_close_rel(Y, ref["yref"], ref["mag"] if group else None, what="decode job")


# (M, N, K, group): ragged N and K, several M, per-row and grouped scales, a
# group that does not divide 32 chunks, K of one chunk and of many slices
MIXED = [(1, 4096, 4096, 128), (1, 11008, 4096, 128), (1, 4096, 11008, 128),
         (3, 300, 1000, 0), (8, 77, 16384, 384), (2, 129, 256, 128), (5, 9, 64, 0),
         (1, 1000, 7000, 256)]


@pytest.mark.parametrize("ready", [False, True])
def test_batched_mixed_jobs_exact(ready):
    jobs, data, checks = [], [], []
    for i, (M, N, K, group) in enumerate(MIXED):
        X = workloads.edge_acts(M, K, "student", tag=100 + i)
        W = workloads.edge_weights(N, K, tag=100 + i)
        wb, ws = bt.bwta_pack_weights(dev(W), group)
        Yv, yc = guarded((M, N), torch.float32)
        Dv, dc = guarded((M, N), torch.int32)
        jobs.append((dev(X), wb, ws, group, Yv, Dv))
        data.append((X, W, group))
        checks += [yc, dc]
    torch.cuda.synchronize()
    st = bt.new_status()
    outs = bt.bwta_linear_decode_batched(jobs, status=st,
                                         flags=bt.GEMM_WEIGHTS_READY if ready else 0)
    torch.cuda.synchronize()
    assert st.item() == 0
    for c in checks:
        c()
    for (X, W, group), (Y, D) in zip(data, outs):
        check_job(X, W, group, Y.cpu().numpy(), D.cpu().numpy())


# at most two activation rows and K small enough for two 32-row tiles in the
# copy ring: the launch takes 32-row tiles; jobs end inside a tile (N = 1000,
# 77) and one job has per-row scales
TALL = [(1, 4096, 4096, 128), (2, 1000, 4096, 128), (1, 77, 2048, 0), (1, 11008, 4096, 128),
        (2, 33, 300, 128)]


@pytest.mark.parametrize("ready", [False, True])
def test_batched_tall_tiles_exact(ready):
    jobs, data = [], []
    for i, (M, N, K, group) in enumerate(TALL):
        X = workloads.edge_acts(M, K, "student", tag=200 + i)
        W = workloads.edge_weights(N, K, tag=200 + i)
        wb, ws = bt.bwta_pack_weights(dev(W), group)
        jobs.append((dev(X), wb, ws, group))
        data.append((X, W, group))
    torch.cuda.synchronize()
    st = bt.new_status()
    outs = bt.bwta_linear_decode_batched(jobs, status=st, want_dots=True,
                                         flags=bt.GEMM_WEIGHTS_READY if ready else 0)
    torch.cuda.synchronize()
    assert st.item() == 0
    for (X, W, group), (Y, D) in zip(data, outs):
        check_job(X, W, group, Y.cpu().numpy(), D.cpu().numpy())


def test_batched_equals_single_calls():
    jobs, singles = [], []
    for i, (K, N) in enumerate(workloads.LLAMA_SHAPES):
        t = workloads.llama(i, 1)
        wb, ws = bt.bwta_pack_weights(dev(t["W"]), 128)
        Xd = dev(t["X"])
        jobs.append((Xd, wb, ws, 128))
        singles.append(bt.bwta_linear_decode(Xd, wb, ws, 128, want_dots=True))
        # the two-call path: packer, then the GEMV on bit planes
        m, s, sc = bt.bwta_quantize_pack_acts(Xd)
        singles.append(bt.bwta_gemm(m, s, sc, wb, ws, K, 128, want_dots=True))
    outs = bt.bwta_linear_decode_batched(jobs, want_dots=True)
    torch.cuda.synchronize()
    for i, (Y, D) in enumerate(outs):
        for Ys, Ds in singles[2 * i:2 * i + 2]:
            assert torch.equal(Y.view(torch.int32), Ys.view(torch.int32))
            assert torch.equal(D, Ds)
        t = workloads.llama(i, 1)
        check_job(t["X"], t["W"], 128, Y.cpu().numpy(), D.cpu().numpy())


def test_batched_binary_mode_zero_rows_and_empty_jobs():
    K, N = 512, 64
    W = workloads.edge_weights(N, K, tag=5)
    wb, ws = bt.bwta_pack_weights(dev(W), 128)
    X = workloads.edge_acts(4, K, "normal", tag=5)
    X[1] = 0
    Xe = torch.empty((0, K), dtype=torch.float16, device="cuda")
    for mode, ternary in ((bt.BINARY, False), (bt.TERNARY, True)):
        outs = bt.bwta_linear_decode_batched([(dev(X), wb, ws, 128), (Xe, wb, ws, 128)],
                                             mode=mode, want_dots=True)
        torch.cuda.synchronize()
        Y, D = outs[0]
        check_job(X, W, 128, Y.cpu().numpy(), D.cpu().numpy(), ternary=ternary)
        assert (Y[1] == 0).all() if ternary else True
    assert bt.bwta_linear_decode_batched([]) == []


def test_batched_dots_only_and_unaligned_rows():
    M, N, K = 3, 200, 1000
    X = workloads.edge_acts(M, K + 3, "student", tag=9)
    W = workloads.edge_weights(N, K, tag=9)
    wb, ws = bt.bwta_pack_weights(dev(W), 0)
    Xd = dev(X)[:, 1:K + 1]        # rows start 2 bytes off a 16-byte boundary, ld = K + 3
    D = torch.empty((M, N), dtype=torch.int32, device="cuda")
    bt.bwta_linear_decode_batched([(Xd, wb, ws, 0, None, D)])
    torch.cuda.synchronize()
    ref = oracle.linear(X[:, 1:K + 1], W, 0)
    np.testing.assert_array_equal(D.cpu().numpy(), ref["dots"])


def test_batched_nonfinite_flag():
    K, N = 256, 32
    W = workloads.edge_weights(N, K, tag=3)
    wb, ws = bt.bwta_pack_weights(dev(W), 0)
    X = workloads.edge_acts(1, K, "normal", tag=3)
    X[0, 7] = np.inf
    st = bt.new_status()
    bt.bwta_linear_decode_batched([(dev(X), wb, ws, 0)], status=st)
    torch.cuda.synchronize()
    assert st.item() & bt.STATUS_NONFINITE


def test_batched_validation():
    lib = bt.load_library()
    W = workloads.edge_weights(16, 256, tag=1)
    wb, ws = bt.bwta_pack_weights(dev(W), 0)
    X = dev(workloads.edge_acts(1, 256, "normal", tag=1))
    arr, _ = bt.decode_jobs([(X, wb, ws, 0)] * 9)
    assert lib.bwta_linear_decode_batched(arr, 9, 0, 0.5, 0, None, None) == bt.BWTA_ERR_UNSUPPORTED
    assert lib.bwta_linear_decode_batched(arr, 1, 0, 0.25, 0, None, None) == bt.BWTA_ERR_UNSUPPORTED
    assert lib.bwta_linear_decode_batched(arr, 1, 0, 0.5, 2, None, None) == bt.BWTA_ERR_INVALID_ARG
    assert lib.bwta_linear_decode_batched(None, 1, 0, 0.5, 0, None, None) == bt.BWTA_ERR_INVALID_ARG
    big = dev(workloads.edge_acts(9, 256, "normal", tag=2))
    arr, _ = bt.decode_jobs([(big, wb, ws, 0)])
    assert lib.bwta_linear_decode_batched(arr, 1, 0, 0.5, 0, None, None) == bt.BWTA_ERR_UNSUPPORTED
