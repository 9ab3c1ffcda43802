"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bit planes, salient indices and integer dots must match exactly; fp32 outputs
must be within 1e-5 relative of the oracle's fp64 value (per-group outputs,
whose group terms can cancel, may instead be within 1e-5 of the magnitude
sum_g |alpha_g d_g|). Full-size workloads are checked on sampled rows.
"""
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


# ------------------------------------------------------------------ helpers
def gpu_pack_weights(W, group):
    status = bt.new_status()
    wb, ws = bt.bwta_pack_weights(dev(W), group, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    return wb, ws


def gpu_pack_acts(X, mode=bt.TERNARY):
    status = bt.new_status()
    m, s, sc = bt.bwta_quantize_pack_acts(dev(X), mode, status=status)
    torch.cuda.synchronize()
    return m, s, sc, status.item()


def check_acts(X, mode=bt.TERNARY):
    m, s, sc, st = gpu_pack_acts(X, mode)
    assert st == 0
    a, s_ref = oracle.quantize_acts(X, ternary=(mode == bt.TERNARY))
    ld = m.shape[1]
    np.testing.assert_array_equal(u32(m), oracle.pack_plane(a, ld, "mask"))
    np.testing.assert_array_equal(u32(s), oracle.pack_plane(a, ld, "sign"))
    np.testing.assert_array_equal(sc.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    return m, s, sc, a, s_ref


# ------------------------------------------------------------------ K0
@pytest.mark.parametrize("N,K,group", [
    (128, 256, 0), (130, 300, 128), (7, 33, 0), (64, 1024, 384), (33, 4096, 128)])
def test_pack_weights_small(N, K, group):
    W = workloads.edge_weights(N, K, tag=group)
    W[0, :3] = [0.0, -0.0, -1e-30]
    wb, ws = gpu_pack_weights(W, group)
    b, alpha = oracle.binarize_weights(W, group)
    np.testing.assert_array_equal(u32(wb), oracle.pack_plane(b, wb.shape[1], "sign"))
    np.testing.assert_array_equal(ws.cpu().numpy().view(np.uint32), alpha.view(np.uint32))


@pytest.mark.parametrize("which", ["bert0", "bert1", "llama0", "llama1", "llama2"])
def test_pack_weights_full(which):
    if which.startswith("bert"):
        W, group = workloads.bert(int(which[-1]), M=1)["W"], 0
    else:
        W, group = workloads.llama_weights(int(which[-1])), workloads.LLAMA_GROUP
    wb, ws = gpu_pack_weights(W, group)
    b, alpha = oracle.binarize_weights(W, group)
    np.testing.assert_array_equal(u32(wb), oracle.pack_plane(b, wb.shape[1], "sign"))
    np.testing.assert_array_equal(ws.cpu().numpy().view(np.uint32), alpha.view(np.uint32))


# ------------------------------------------------------------------ K1
@pytest.mark.parametrize("M,K,kind", [
    (16, 256, "normal"), (9, 33, "student"), (129, 100, "student"), (7, 1000, "normal"),
    (5, 64, "normal"), (3, 5000, "student"), (4, 128, "zeros"), (4, 96, "negzero"),
    (6, 300, "subnormal"), (6, 2048, "big"), (2, 20000, "student"), (1, 11008, "student")])
def test_quantize_pack_acts_edges(M, K, kind):
    check_acts(workloads.edge_acts(M, K, kind))


def test_quantize_pack_acts_golden_tie_rows():
    from conftest import read_golden
    for xs, _, _ in read_golden("ternary_rows.txt"):
        x = np.array([float(v) for v in xs.split()], np.float64).astype(np.float16)[None, :]
        check_acts(x)


def test_quantize_pack_acts_binary_mode():
    check_acts(workloads.edge_acts(33, 700, "student"), mode=bt.BINARY)
    X = workloads.edge_acts(4, 64, "normal")
    X[0, :2] = np.array([0.0, -0.0], np.float16)
    check_acts(X, mode=bt.BINARY)


def test_quantize_pack_acts_nonfinite_flag():
    X = workloads.edge_acts(4, 256, "normal")
    X[2, 17] = np.float16(np.inf)
    *_, st = gpu_pack_acts(X)
    assert st & bt.STATUS_NONFINITE


@pytest.mark.parametrize("which", ["tiny", "bert0", "bert1", "llama0", "llama2", "llama_m1", "attn"])
def test_quantize_pack_acts_workloads(which):
    if which == "tiny":
        X = workloads.tiny()["X"]
    elif which.startswith("bert"):
        X = workloads.bert(int(which[-1]))["X"]
    elif which == "llama_m1":
        X = workloads.llama_acts(2, 1)
    elif which.startswith("llama"):
        X = workloads.llama_acts(int(which[-1]), 2048)
    else:
        X = workloads.attn()["Q"].reshape(-1, 64)
    check_acts(X)


# ------------------------------------------------------------------ K2 / K3
def run_linear(X, W, group, rows=None, want_rep=True):
    """GPU quantize + pack + gemm vs the oracle, on all rows or sampled ones."""
    wb, ws = gpu_pack_weights(W, group)
    m, s, sc, st = gpu_pack_acts(X)
    assert st == 0
    K = X.shape[1]
    M, N = X.shape[0], W.shape[0]
    Yv, ycheck = guarded((M, N), torch.float32)
    Dv, dcheck = guarded((M, N), torch.int32)
    status = bt.new_status()
    bt.bwta_gemm(m, s, sc, wb, ws, K, group, status=status, out=(Yv, Dv))
    torch.cuda.synchronize()
    assert status.item() == 0
    ycheck()
    dcheck()
    rows = np.arange(M) if rows is None else rows
    a, s_ref = oracle.quantize_acts(X[rows])
    b, alpha = oracle.binarize_weights(W, group)
    d = oracle.int_dots(a, b, group)
    yref, mag, yrep = oracle.linear_out(d, alpha, s_ref)
    Y = Yv.cpu().numpy()[rows]
    D = Dv.cpu().numpy()[rows]
    np.testing.assert_array_equal(D, d.sum(axis=2))
    assert_close_rel(Y, yref, mag if group else None, what=f"Y M={M} N={N} K={K} g={group}")
    return Y, yrep


@pytest.mark.parametrize("M,N,K,group", [
    (16, 128, 256, 0),          # tiny
    (129, 130, 300, 128),       # ragged M, N, K and a short last group
    (9, 7, 64, 0),              # one chunk
    (200, 300, 1000, 0),        # K not a multiple of 32
    (256, 256, 4096, 128),
    (130, 70, 11008, 128),
    (300, 129, 768, 384)])
def test_gemm_tiled_small(M, N, K, group):
    X = workloads.edge_acts(M, K, "student", tag=K)
    W = workloads.edge_weights(N, K, tag=K)
    Y, yrep = run_linear(X, W, group)
    # the tiled kernel evaluates the fp32 epilogue in the oracle's order
    np.testing.assert_array_equal(Y.view(np.uint32), yrep.view(np.uint32))


@pytest.mark.parametrize("M", [1, 2, 7, 8])
@pytest.mark.parametrize("N,K,group", [(100, 256, 0), (64, 4096, 128), (50, 11008, 128),
                                       (33, 300, 128)])
def test_gemv_small(M, N, K, group):
    X = workloads.edge_acts(M, K, "student", tag=M)
    W = workloads.edge_weights(N, K, tag=M)
    Y, yrep = run_linear(X, W, group)
    # the decode GEMV folds the groups in the oracle's serial fp32 order
    np.testing.assert_array_equal(Y.view(np.uint32), yrep.view(np.uint32))


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (1, 300, 11008), (3, 1000, 4096)])
def test_gemv_weights_ready_flag(M, N, K):
    """bwta_gemm_ex(WEIGHTS_READY): weights packed and synchronized first, then
    the GEMV streams them before waiting on the activation packer."""
    X = workloads.edge_acts(M, K, "student", tag=N)
    W = workloads.edge_weights(N, K, tag=N)
    wb, ws = gpu_pack_weights(W, 128)
    torch.cuda.synchronize()
    ref = oracle.linear(X, W, 128)
    Xd = dev(X)
    for _ in range(2):
        m, s, sc = bt.bwta_quantize_pack_acts(Xd)
        Y, D = bt.bwta_gemm(m, s, sc, wb, ws, K, 128, want_dots=True, flags=bt.GEMM_WEIGHTS_READY)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(D.cpu().numpy(), ref["dots"])
        assert_close_rel(Y.cpu().numpy(), ref["yref"], ref["mag"], what="gemv ready")
        np.testing.assert_array_equal(Y.cpu().numpy().view(np.uint32), ref["yrep"].view(np.uint32))


@pytest.mark.parametrize("ready", [False, True])
@pytest.mark.parametrize("M", [1, 3, 8])
@pytest.mark.parametrize("N,K,group", [(100, 256, 0), (64, 4096, 128), (50, 11008, 128),
                                       (33, 300, 128), (40, 16384, 0)])
def test_linear_decode_fused(M, N, K, group, ready):
    """bwta_linear_decode ternarizes inside the kernel: same dots as the
    two-call path (exact), fp32 within tolerance."""
    X = workloads.edge_acts(M, K, "student", tag=7 * N + M)
    W = workloads.edge_weights(N, K, tag=N + M)
    wb, ws = gpu_pack_weights(W, group)
    torch.cuda.synchronize()
    ref = oracle.linear(X, W, group)
    Yv, ycheck = guarded((M, N), torch.float32)
    Dv, dcheck = guarded((M, N), torch.int32)
    st = bt.new_status()
    bt.bwta_linear_decode(dev(X), wb, ws, group, want_dots=True, status=st, out=(Yv, Dv),
                          flags=bt.GEMM_WEIGHTS_READY if ready else 0)
    torch.cuda.synchronize()
    assert st.item() == 0
    ycheck()
    dcheck()
    np.testing.assert_array_equal(Dv.cpu().numpy(), ref["dots"])
    assert_close_rel(Yv.cpu().numpy(), ref["yref"], ref["mag"] if group else None, what="decode")
    np.testing.assert_array_equal(Yv.cpu().numpy().view(np.uint32), ref["yrep"].view(np.uint32))


def test_linear_decode_binary_and_zero_rows():
    K, N = 512, 64
    W = workloads.edge_weights(N, K, tag=5)
    wb, ws = gpu_pack_weights(W, 128)
    X = workloads.edge_acts(4, K, "normal", tag=5)
    X[1] = 0
    for mode, ternary in ((bt.BINARY, False), (bt.TERNARY, True)):
        Y, D = bt.bwta_linear_decode(dev(X), wb, ws, 128, mode=mode, want_dots=True)
        a, sc = oracle.quantize_acts(X, ternary=ternary)
        b, alpha = oracle.binarize_weights(W, 128)
        d = oracle.int_dots(a, b, 128)
        yref, mag, _ = oracle.linear_out(d, alpha, sc)
        np.testing.assert_array_equal(D.cpu().numpy(), d.sum(axis=2))
        assert_close_rel(Y.cpu().numpy(), yref, mag, what="decode binary")


def test_gemm_tiny_workload():
    t = workloads.tiny()
    Y, yrep = run_linear(t["X"], t["W"], 0)
    np.testing.assert_array_equal(Y.view(np.uint32), yrep.view(np.uint32))


@pytest.mark.parametrize("shape", [0, 1])
def test_gemm_bert_full(shape):
    t = workloads.bert(shape)
    run_linear(t["X"], t["W"], 0, rows=sample_rows(t["M"]))


@pytest.mark.parametrize("shape", [0, 1, 2])
@pytest.mark.parametrize("M", [2048, 1])
def test_gemm_llama_full(shape, M):
    t = workloads.llama(shape, M)
    run_linear(t["X"], t["W"], t["group"], rows=sample_rows(M, 48))


def test_gemm_zero_activations_give_zero():
    W = workloads.edge_weights(64, 512)
    for M in (1, 40):
        X = np.zeros((M, 512), np.float16)
        wb, ws = gpu_pack_weights(W, 128)
        m, s, sc, _ = gpu_pack_acts(X)
        Y, D = bt.bwta_gemm(m, s, sc, wb, ws, 512, 128, want_dots=True)
        assert (Y == 0).all() and (D == 0).all() and not torch.isnan(Y).any()


def test_gemm_negated_weight_bits_negate_output():
    X = workloads.edge_acts(40, 512, "normal")
    W = workloads.edge_weights(64, 512)
    wb, ws = gpu_pack_weights(W, 0)
    m, s, sc, _ = gpu_pack_acts(X)
    ld_valid = 512 // 32
    wneg = wb.clone()
    wneg[:, :ld_valid] = ~wneg[:, :ld_valid]
    Y1, D1 = bt.bwta_gemm(m, s, sc, wb, ws, 512, 0, want_dots=True)
    Y2, D2 = bt.bwta_gemm(m, s, sc, wneg, ws, 512, 0, want_dots=True)
    assert torch.equal(D2, -D1) and torch.equal(Y2, -Y1)


# ------------------------------------------------------------------ K4
def run_attn(Q, Kt, heads=None):
    B, H, L, D = Q.shape
    BH = B * H
    qm, qs, qsc, _ = gpu_pack_acts(Q.reshape(-1, D))
    km, ks, ksc, _ = gpu_pack_acts(Kt.reshape(-1, D))
    Lk = Kt.shape[2]
    Si, Sf = bt.bwta_attn_scores(qm, qs, qsc, km, ks, ksc, BH, L, Lk, D)
    torch.cuda.synchronize()
    heads = np.arange(BH) if heads is None else heads
    aq, sq = oracle.quantize_acts(Q.reshape(BH, L, D)[heads].reshape(-1, D))
    ak, sk = oracle.quantize_acts(Kt.reshape(BH, Lk, D)[heads].reshape(-1, D))
    S, fref, frep = oracle.attn_scores(aq.reshape(len(heads), L, D), ak.reshape(len(heads), Lk, D),
                                       sq.reshape(len(heads), L), sk.reshape(len(heads), Lk))
    np.testing.assert_array_equal(Si.cpu().numpy()[heads], S)
    Sfh = Sf.cpu().numpy()[heads]
    assert_close_rel(Sfh, fref, what="attn fp32")
    np.testing.assert_array_equal(Sfh.view(np.uint32), frep.view(np.uint32))
    return Si, Sf


def test_attn_full_config_sampled_heads():
    t = workloads.attn()
    run_attn(t["Q"], t["K"], heads=np.array([0, 1, 47, 95]))


@pytest.mark.parametrize("Lq,Lk,D", [(70, 130, 64), (64, 128, 96), (33, 17, 200), (1, 5, 32)])
def test_attn_ragged(Lq, Lk, D):
    Q = workloads.edge_acts(2 * Lq, D, "normal", tag=1).reshape(1, 2, Lq, D)
    Kt = workloads.edge_acts(2 * Lk, D, "normal", tag=2).reshape(1, 2, Lk, D)
    run_attn(Q, Kt)


def test_attn_single_output_variants():
    t = workloads.attn((1, 2, 128, 64))
    Si, Sf = run_attn(t["Q"], t["K"])
    qm, qs, qsc, _ = gpu_pack_acts(t["Q"].reshape(-1, 64))
    km, ks, ksc, _ = gpu_pack_acts(t["K"].reshape(-1, 64))
    Si2, none = bt.bwta_attn_scores(qm, qs, qsc, km, ks, ksc, 2, 128, 128, 64, want_float=False)
    none2, Sf2 = bt.bwta_attn_scores(qm, qs, qsc, km, ks, ksc, 2, 128, 128, 64, want_int=False)
    assert none is None and none2 is None
    assert torch.equal(Si2, Si) and torch.equal(Sf2, Sf)


# ------------------------------------------------------------------ K5
def check_billm_pack(W, Wq, rows, n_sal=8, split=True):
    sal = oracle.billm_salient(W, 128, n_sal) if n_sal else np.zeros((W.shape[1] // 128, 0), np.int32)
    if n_sal:
        np.testing.assert_array_equal(Wq.sal.cpu().numpy(), sal)
    ref_rows = {}
    for n in rows:
        q = oracle.billm_quantize_rows(W, sal, int(n), int(n) + 1, 128, split=split)
        p = oracle.billm_pack(q, Wq.ldw)
        np.testing.assert_array_equal(u32(Wq.sign[n:n + 1]), p["sign"])
        np.testing.assert_array_equal(u32(Wq.gmap[n:n + 1]), p["gmap"])
        np.testing.assert_array_equal(Wq.res[n:n + 1].cpu().numpy(), p["res"])
        np.testing.assert_array_equal(Wq.bscale[n:n + 1].cpu().numpy().view(np.uint32),
                                      p["bscale"].view(np.uint32))
        ref_rows[int(n)] = q
    return sal, ref_rows


def billm_rows_ref(X, W, sal, rows, split=True):
    q = oracle.billm_quantize_rows(W, sal, 0, W.shape[0], 128, split=split) if rows is None else None
    if q is not None:
        return oracle.billm_gemm(X, q)
    outs, mags = [], []
    for n in rows:
        qn = oracle.billm_quantize_rows(W, sal, int(n), int(n) + 1, 128, split=split)
        y, mg = oracle.billm_gemm(X, qn)
        outs.append(y)
        mags.append(mg)
    return np.concatenate(outs, axis=1), np.concatenate(mags, axis=1)


@pytest.mark.parametrize("N,K,M,n_sal,split", [
    (40, 384, 3, 8, True), (33, 256, 17, 8, True), (70, 512, 1, 0, False), (64, 1024, 5, 3, True),
    (100, 128, 40, 8, False), (40, 384, 1, 8, 2), (50, 256, 20, 0, 2), (33, 512, 3, 3, 2)])
def test_billm_small(N, K, M, n_sal, split):
    W = workloads.latent_laplace((N, K), 0.01, 7, N, K)
    X = workloads.edge_acts(M, K, "normal", tag=N)
    Wq = bt.billm_pack_weights(dev(W), n_sal=n_sal, split=split)
    torch.cuda.synchronize()
    sal, _ = check_billm_pack(W, Wq, range(N), n_sal, split)
    Y = bt.billm_gemm(dev(X), Wq).cpu().numpy()
    yref, mag = billm_rows_ref(X, W, sal, None, split)
    assert_close_rel(Y, yref, mag, what="billm small")


@pytest.fixture(scope="module")
def billm_full():
    W = workloads.billm_weights()
    Wq = bt.billm_pack_weights(dev(W))
    torch.cuda.synchronize()
    rows = sample_rows(W.shape[0], 24)
    sal, _ = check_billm_pack(W, Wq, rows)
    return W, Wq, sal, rows


@pytest.mark.parametrize("M", [1, 16, 512])
def test_billm_full_config(billm_full, M):
    W, Wq, sal, rows = billm_full
    X = workloads.billm_acts(M)
    Y = bt.billm_gemm(dev(X), Wq).cpu().numpy()
    yref, mag = billm_rows_ref(X, W, sal, rows)
    assert_close_rel(Y[:, rows], yref, mag, what=f"billm M={M}")


def test_billm_searched_split_full_config_rows():
    """The searched break-point (split = 2) on the BiLLM configuration: packed
    planes, residual bits and scales equal the oracle's bit for bit on sampled
    rows, and the GEMM on those weights matches the oracle."""
    W = workloads.billm_weights()
    Wq = bt.billm_pack_weights(dev(W), split=2)
    torch.cuda.synchronize()
    rows = sample_rows(W.shape[0], 16)
    sal, _ = check_billm_pack(W, Wq, rows, 8, 2)
    X = workloads.billm_acts(1)
    Y = bt.billm_gemm(dev(X), Wq).cpu().numpy()
    yref, mag = billm_rows_ref(X, W, sal, rows, split=2)
    assert_close_rel(Y[:, rows], yref, mag, what="billm searched split")


@pytest.mark.parametrize("N,K,M", [(200, 384, 300), (129, 128, 70), (64, 1024, 9), (300, 256, 257),
                                   (64, 1024, 2), (130, 384, 3), (33, 256, 4), (200, 384, 7), (65, 512, 8)])
def test_billm_tc_shapes(N, K, M):
    """Tensor-core BiLLM path (M > 8): ragged token tiles (64 and 256), ragged
    weight-row tiles, odd block counts; M = 2..8 take the CUDA-core kernel
    (512 threads for M > 4)."""
    W = workloads.latent_laplace((N, K), 0.01, 11, N, K)
    X = workloads.edge_acts(M, K, "student", tag=N + K)
    Wq = bt.billm_pack_weights(dev(W), n_sal=8, split=True)
    torch.cuda.synchronize()
    sal, _ = check_billm_pack(W, Wq, range(N), 8, True)
    Y = bt.billm_gemm(dev(X), Wq).cpu().numpy()
    yref, mag = billm_rows_ref(X, W, sal, None, True)
    assert_close_rel(Y, yref, mag, what=f"billm tc {N}x{K} M={M}")


def test_billm_tc_scale_spread():
    """Rows whose scales differ by many powers of ten, and an all-zero row: the
    per-row power-of-two exponent keeps every row's hi/lo split in range."""
    N, K, M = 48, 512, 33
    W = workloads.latent_laplace((N, K), 0.01, 13, N, K)
    W = W * (10.0 ** (np.arange(N) % 10 - 6.0))[:, None].astype(np.float32)
    W[5] = 0.0
    X = workloads.edge_acts(M, K, "normal", tag=99)
    Wq = bt.billm_pack_weights(dev(W), n_sal=8, split=True)
    torch.cuda.synchronize()
    sal, _ = check_billm_pack(W, Wq, range(N), 8, True)
    Y = bt.billm_gemm(dev(X), Wq).cpu().numpy()
    yref, mag = billm_rows_ref(X, W, sal, None, True)
    assert_close_rel(Y, yref, mag, what="billm tc scale spread")
    assert np.all(Y[:, 5] == 0.0)


def test_billm_unaligned_x_takes_cuda_core_path():
    """X with a row stride that breaks the TMA rule (ldX % 8 != 0) runs on the
    CUDA-core kernel; both paths agree with the oracle."""
    N, K, M = 64, 256, 20
    W = workloads.latent_laplace((N, K), 0.01, 17, N, K)
    X = workloads.edge_acts(M, K, "normal", tag=5)
    Wq = bt.billm_pack_weights(dev(W), n_sal=8, split=True)
    torch.cuda.synchronize()
    sal, _ = check_billm_pack(W, Wq, range(N), 8, True)
    wide = torch.zeros((M, K + 3), dtype=torch.float16, device="cuda")
    wide[:, :K] = dev(X)
    Y_core = bt.billm_gemm(wide[:, :K], Wq).cpu().numpy()
    Y_tc = bt.billm_gemm(dev(X), Wq).cpu().numpy()
    yref, mag = billm_rows_ref(X, W, sal, None, True)
    assert_close_rel(Y_core, yref, mag, what="billm cuda-core path")
    assert_close_rel(Y_tc, yref, mag, what="billm tensor-core path")
