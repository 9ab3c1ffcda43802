"""The attention path past the scores: ternary probabilities straight from the
ternary Q, K planes (softmax, then the ternary threshold 0.5 * mean(p) =
1/(2L)), and the ternary A . V product, against the CPU oracle.

The probabilities come out of exp (fp32 on the GPU, fp64 in the oracle) and a
sum, so a probability whose exact value lies within a hair of the threshold may
be kept on one side and not on the other; positions within 1e-5 (relative) of
1/(2L) in the oracle's fp64 values are ambiguous and checked only for being
valid (0 or 1). Everything else must
match: mask words exactly, scales to one fp32 rounding, A . V integer sums
exactly and fp32 outputs within 1e-5 relative of the oracle's fp64 value."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_common import assert_close_rel, dev, u32

pytestmark = pytest.mark.gpu

bt = pytest.importorskip("binarized_transformer_b200")

AMBIG = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    bt.load_library()
    oracle.build()


def run_path(Q, Kt, V, heads, c):
    B, H, L, D = Q.shape
    Lk = Kt.shape[2]
    BH = B * H
    qm, qs, qsc = bt.bwta_quantize_pack_acts(dev(Q.reshape(-1, D)))
    km, ks, ksc = bt.bwta_quantize_pack_acts(dev(Kt.reshape(-1, D)))
    pm, ps, psc = bt.bwta_attn_softmax_ternarize(qm, qs, qsc, km, ks, ksc, BH, L, Lk, D, c)
    Vt = np.ascontiguousarray(V.reshape(BH, Lk, D).transpose(0, 2, 1)).reshape(-1, Lk)
    vm, vs, vsc = bt.bwta_quantize_pack_acts(dev(Vt))
    Oi, Of = bt.bwta_attn_av(pm, ps, psc, vm, vs, vsc, BH, L, D, Lk, want_int=True)
    torch.cuda.synchronize()

    # oracle on the sampled heads
    nh = len(heads)
    aq, sq = oracle.quantize_acts(Q.reshape(BH, L, D)[heads].reshape(-1, D))
    ak, sk = oracle.quantize_acts(Kt.reshape(BH, Lk, D)[heads].reshape(-1, D))
    _, _, frep = oracle.attn_scores(aq.reshape(nh, L, D), ak.reshape(nh, Lk, D),
                                    sq.reshape(nh, L), sk.reshape(nh, Lk))
    ap, sp, p = oracle.softmax_ternarize(frep, c)
    av, sv = oracle.quantize_acts(Vt.reshape(BH, D, Lk)[heads].reshape(-1, Lk))
    O, Oref, _ = oracle.attn_av(ap, sp, av.reshape(nh, D, Lk), sv.reshape(nh, D))

    # probabilities: mask words where unambiguous, scales, zero sign plane
    thr = 0.5 / Lk
    ambig = np.abs(p - thr) <= AMBIG * thr
    ldp = pm.shape[1]
    gm = u32(pm).reshape(BH, L, ldp)[heads]
    bits = np.unpackbits(gm.view(np.uint8), axis=-1, bitorder="little")[..., :Lk].astype(np.int8)
    assert (u32(ps) == 0).all()
    assert (gm.reshape(nh, L, ldp)[..., (Lk + 31) // 32:] == 0).all()
    np.testing.assert_array_equal(np.where(ambig, 0, bits), np.where(ambig, 0, ap))
    clean = ~ambig.any(axis=-1)                                   # rows with no ambiguous key
    gsc = psc.cpu().numpy().reshape(BH, L)[heads]
    # e in fp32 (a few ulp): the mean of the kept p to ~1e-6
    np.testing.assert_allclose(gsc[clean], sp[clean], rtol=2e-6, atol=0)
    # A . V on those rows
    Oi_h = Oi.cpu().numpy()[heads]
    Of_h = Of.cpu().numpy()[heads]
    np.testing.assert_array_equal(Oi_h[clean], O[clean])
    assert_close_rel(Of_h[clean], Oref[clean], what="A.V fp32")
    return clean.mean()


def test_attn_av_full_config_sampled_heads():
    a = workloads.attn()
    V = workloads.attn_v()
    B, H, L, D = workloads.ATTN_SHAPE
    frac = run_path(a["Q"], a["K"], V, heads=[0, 17, 50, 95], c=1.0 / np.sqrt(D))
    assert frac > 0.99


@pytest.mark.parametrize("shape,c", [((1, 2, 100, 64), 0.125), ((2, 1, 33, 32), 0.5),
                                     ((1, 1, 64, 128), 0.0884), ((1, 3, 300, 96), 0.1)])
def test_attn_av_ragged(shape, c):
    a = workloads.attn(shape)
    V = workloads.attn_v(shape)
    B, H, L, D = shape
    frac = run_path(a["Q"], a["K"], V, heads=list(range(B * H)), c=c)
    assert frac > 0.9


def test_attn_softmax_uniform_row_keeps_everything():
    # all-zero Q: every score is 0, every p = 1/L > 1/(2L): all kept, scale 1/L
    B, H, L, D = 1, 1, 96, 64
    Q = np.zeros((L, D), np.float16)
    Kt = workloads.attn((B, H, L, D))["K"].reshape(-1, D)
    qm, qs, qsc = bt.bwta_quantize_pack_acts(dev(Q))
    km, ks, ksc = bt.bwta_quantize_pack_acts(dev(Kt))
    pm, ps, psc = bt.bwta_attn_softmax_ternarize(qm, qs, qsc, km, ks, ksc, 1, L, L, D, 0.125)
    torch.cuda.synchronize()
    w = u32(pm)
    assert (w[:, :3] == 0xFFFFFFFF).all() and (w[:, 3:] == 0).all()
    np.testing.assert_array_equal(psc.cpu().numpy(), np.float32(1.0 / L))
