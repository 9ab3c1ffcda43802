"""Failure detection on the GPU without a fault: a bounded wait is made to
run out (a barrier that nothing completes), the kernel reports
BWTA_STATUS_TIMEOUT through the device status word and returns, and the
context stays usable -- the next call computes the oracle's result."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_common import assert_close_rel, dev

pytestmark = pytest.mark.gpu

bt = pytest.importorskip("binarized_transformer_b200")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    bt.load_library()
    oracle.build()


@pytest.mark.parametrize("group", [0, 128])
def test_tiled_gemm_wait_runs_out_then_next_call_is_correct(group):
    M, N, K = 200, 300, 1024
    X = workloads.edge_acts(M, K, "student", tag=11)
    W = workloads.edge_weights(N, K, tag=11)
    wb, ws = bt.bwta_pack_weights(dev(W), group)
    m, s, sc = bt.bwta_quantize_pack_acts(dev(X))
    torch.cuda.synchronize()
    status = bt.bwta_selftest_gemm_timeout(m, s, sc, wb, ws, K, group, wait_limit_ns=1_000_000)
    torch.cuda.synchronize()                      # no fault: the kernel returned
    assert status.item() == bt.STATUS_TIMEOUT     # timed out, and its loads drained
    # the context is still good: the same product through the normal call
    st = bt.new_status()
    Y, D = bt.bwta_gemm(m, s, sc, wb, ws, K, group, want_dots=True, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    ref = oracle.linear(X, W, group)
    np.testing.assert_array_equal(D.cpu().numpy(), ref["dots"])
    np.testing.assert_array_equal(Y.cpu().numpy().view(np.uint32), ref["yrep"].view(np.uint32))
    assert_close_rel(Y.cpu().numpy(), ref["yref"], ref["mag"] if group else None, what="after")


def test_selftest_rejects_bad_arguments():
    m = torch.zeros((4, 4), dtype=torch.int32, device="cuda")
    sc = torch.zeros(4, dtype=torch.float32, device="cuda")
    with pytest.raises(bt.BwtaError):   # M <= 8 is the GEMV, which has no such wait
        bt.bwta_selftest_gemm_timeout(m, m, sc, m, sc, 64, 0)
    m = torch.zeros((16, 4), dtype=torch.int32, device="cuda")
    sc = torch.zeros(16, dtype=torch.float32, device="cuda")
    with pytest.raises(bt.BwtaError):
        bt.bwta_selftest_gemm_timeout(m, m, sc, m, sc, 64, 0, wait_limit_ns=0)
