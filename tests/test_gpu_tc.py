"""Parity of the tensor-core path (E4M3 activations + tcgen05 GEMM) with the
CPU oracle. The E4M3 bytes and the integer dots must match exactly; the fp32
outputs follow the same evaluation order as the oracle's fp32 replica, so they
must match it bit for bit (and the fp64 value within 1e-5)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_common import assert_close_rel, dev, guarded, sample_rows, u32

pytestmark = pytest.mark.gpu

bt = pytest.importorskip("binarized_transformer_b200")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    bt.load_library()
    oracle.build()


def e4m3_of(a, width):
    """Expected E4M3 bytes of ternary values a [M, K], zero padded to width, in
    the tensor-core order of the header: within each 32-element block, byte
    4k + j holds element 8j + k."""
    nat = np.zeros((a.shape[0], width), np.uint8)
    nat[:, :a.shape[1]] = np.where(a == 1, 0x38, np.where(a == -1, 0xB8, 0)).astype(np.uint8)
    pos = np.arange(32)
    elem = 8 * (pos % 4) + pos // 4          # element held by byte position pos
    blocks = nat.reshape(a.shape[0], width // 32, 32)
    return blocks[:, :, elem].reshape(a.shape[0], width)


def test_e4m3_order_is_a_permutation():
    elem = 8 * (np.arange(32) % 4) + np.arange(32) // 4
    assert sorted(elem.tolist()) == list(range(32))
    assert elem[4 * 3 + 2] == 8 * 2 + 3      # byte 4k + j <- element 8j + k


@pytest.mark.parametrize("M,K,kind", [(16, 256, "normal"), (9, 33, "student"), (129, 1000, "student"),
                                      (3, 11008, "student"), (4, 128, "zeros")])
def test_quantize_pack_acts_ex_e4m3(M, K, kind):
    X = workloads.edge_acts(M, K, kind, tag=3)
    st = bt.new_status()
    m, s, a8, sc = bt.bwta_quantize_pack_acts_ex(dev(X), status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    a, s_ref = oracle.quantize_acts(X)
    np.testing.assert_array_equal(a8.cpu().numpy(), e4m3_of(a, a8.shape[1]))
    np.testing.assert_array_equal(u32(m), oracle.pack_plane(a, m.shape[1], "mask"))
    np.testing.assert_array_equal(u32(s), oracle.pack_plane(a, s.shape[1], "sign"))
    np.testing.assert_array_equal(sc.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    # E4M3 only
    _, _, a8b, sc2 = bt.bwta_quantize_pack_acts_ex(dev(X), planes=False)
    assert torch.equal(a8b, a8) and torch.equal(sc2, sc)


def run_tc(X, W, group, rows=None, check_rep=True):
    wb, ws = bt.bwta_pack_weights(dev(W), group)
    _, _, a8, sc = bt.bwta_quantize_pack_acts_ex(dev(X), planes=False)
    M, K = X.shape
    N = W.shape[0]
    Yv, ycheck = guarded((M, N), torch.float32)
    Dv, dcheck = guarded((M, N), torch.int32)
    st = bt.new_status()
    bt.bwta_gemm_tc(a8, sc, wb, ws, K, group, want_dots=True, status=st, out=(Yv, Dv))
    torch.cuda.synchronize()
    assert st.item() == 0, st.item()
    ycheck()
    dcheck()
    rows = np.arange(M) if rows is None else rows
    a, s_ref = oracle.quantize_acts(X[rows])
    b, alpha = oracle.binarize_weights(W, group)
    d = oracle.int_dots(a, b, group)
    yref, mag, yrep = oracle.linear_out(d, alpha, s_ref)
    Y = Yv.cpu().numpy()[rows]
    np.testing.assert_array_equal(Dv.cpu().numpy()[rows], d.sum(axis=2))
    assert_close_rel(Y, yref, mag if group else None, what=f"tc M={M} N={N} K={K} g={group}")
    if check_rep:
        np.testing.assert_array_equal(Y.view(np.uint32), yrep.view(np.uint32))
    return Yv


@pytest.mark.parametrize("M,N,K,group", [
    (16, 128, 256, 0), (129, 130, 300, 128), (9, 7, 64, 0), (200, 300, 1000, 0),
    (256, 256, 4096, 128), (130, 70, 11008, 128), (300, 129, 768, 384), (1, 40, 512, 128)])
def test_gemm_tc_small(M, N, K, group):
    X = workloads.edge_acts(M, K, "student", tag=K + 1)
    W = workloads.edge_weights(N, K, tag=K + 1)
    run_tc(X, W, group)


@pytest.mark.parametrize("shape", [0, 1, 2])
def test_gemm_tc_llama_full(shape):
    t = workloads.llama(shape, 2048)
    run_tc(t["X"], t["W"], t["group"], rows=sample_rows(2048, 48))


@pytest.mark.parametrize("shape", [0, 1])
def test_gemm_tc_bert_full(shape):
    t = workloads.bert(shape)
    run_tc(t["X"], t["W"], 0, rows=sample_rows(t["M"], 48))


def test_gemm_tc_equals_popcount_path():
    t = workloads.llama(0, 512)
    X, W = dev(t["X"]), dev(t["W"])
    wb, ws = bt.bwta_pack_weights(W, 128)
    m, s, a8, sc = bt.bwta_quantize_pack_acts_ex(X)
    Y1, D1 = bt.bwta_gemm(m, s, sc, wb, ws, t["K"], 128, want_dots=True)
    Y2, D2 = bt.bwta_gemm_tc(a8, sc, wb, ws, t["K"], 128, want_dots=True)
    torch.cuda.synchronize()
    assert torch.equal(D1, D2)
    assert torch.equal(Y1.view(torch.int32), Y2.view(torch.int32))


@pytest.mark.parametrize("K", [4096, 11008, 1000])
def test_quantize_pack_acts_ex_many_rows(K):
    """Many rows take the packer's narrow-team path (at most QA_NREG chunk steps
    per thread); planes, E4M3 bytes and scales must match the oracle exactly."""
    M = 1100
    X = workloads.edge_acts(M, K, "student", tag=K + 7)
    st = bt.new_status()
    m, s, a8, sc = bt.bwta_quantize_pack_acts_ex(dev(X), status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    a, s_ref = oracle.quantize_acts(X)
    np.testing.assert_array_equal(u32(m), oracle.pack_plane(a, m.shape[1], "mask"))
    np.testing.assert_array_equal(u32(s), oracle.pack_plane(a, s.shape[1], "sign"))
    np.testing.assert_array_equal(a8.cpu().numpy(), e4m3_of(a, a8.shape[1]))
    np.testing.assert_array_equal(sc.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
