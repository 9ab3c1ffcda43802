"""Pins for the CPU oracle, checked against things other than the oracle.

Each test ties one oracle function to something the pages or the mathematics
fix: hand-worked rows (tests/golden), a library routine computing the same
quantity another way (numpy fp64 matmul, numpy packbits, stable argsort),
closed-form identities, and invariants (scaling, negation, zero inputs).
The pages print no numeric worked example, so the golden rows are worked by
hand from the stated rules.
"""
import itertools

import numpy as np
import pytest

import workloads
from conftest import read_golden

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def f16(vals):
    return np.array(vals, np.float64).astype(np.float16)


# ------------------------------------------------------------- ternarization
def test_ternary_golden_rows(orc):
    for xs, as_, s in read_golden("ternary_rows.txt"):
        x = f16([float(v) for v in xs.split()])[None, :]
        a, sc = orc.quantize_acts(x, ternary=True)
        assert a[0].tolist() == [int(v) for v in as_.split()], xs
        assert sc[0] == np.float32(float(s)), (xs, sc[0], s)


def test_ternary_matches_fp64_numpy_rule(orc):
    """|x| > 0.5*mean|x| evaluated in fp64 by numpy (exact for fp16 inputs at
    these sizes) gives the same kept set and the same scale."""
    for kind, K in [("normal", 256), ("student", 768), ("normal", 4096), ("student", 33)]:
        X = workloads.edge_acts(32, K, kind)
        a, s = orc.quantize_acts(X)
        x = X.astype(np.float64)
        mean = np.abs(x).sum(axis=1, keepdims=True) / K
        keep = np.abs(x) > 0.5 * mean
        np.testing.assert_array_equal(a, np.where(keep, np.sign(x), 0).astype(np.int8))
        for m in range(X.shape[0]):
            ref = np.float32(np.abs(x[m][keep[m]]).sum() / keep[m].sum()) if keep[m].any() else 0
            assert s[m] == ref


def test_ternary_scale_and_sign_invariance(orc):
    X = workloads.edge_acts(16, 512, "normal", tag=3)
    X[np.abs(X) < 2.0 ** -8] = 0  # keep every scaled value a normal fp16
    a, s = orc.quantize_acts(X)
    for e in (-6, -2, 3):
        Xs = (X.astype(np.float64) * 2.0 ** e).astype(np.float16)
        assert np.array_equal(Xs.astype(np.float64), X.astype(np.float64) * 2.0 ** e)
        a2, s2 = orc.quantize_acts(Xs)
        np.testing.assert_array_equal(a2, a)
        np.testing.assert_array_equal(s2, (s.astype(np.float64) * 2.0 ** e).astype(np.float32))
    a3, s3 = orc.quantize_acts(-X)
    np.testing.assert_array_equal(a3, -a)
    np.testing.assert_array_equal(s3, s)


def test_ternary_zero_negzero_and_subnormal_rows(orc):
    a, s = orc.quantize_acts(workloads.edge_acts(4, 64, "zeros"))
    assert not a.any() and not s.any()
    a, s = orc.quantize_acts(workloads.edge_acts(4, 64, "negzero"))
    assert not a.any() and not s.any()
    X = workloads.edge_acts(8, 128, "subnormal")
    a, s = orc.quantize_acts(X)
    x = X.astype(np.float64)
    keep = np.abs(x) > 0.5 * np.abs(x).mean(axis=1, keepdims=True)
    np.testing.assert_array_equal(a != 0, keep)


def test_binary_mode(orc):
    X = workloads.edge_acts(8, 100, "student")
    X[0, :4] = f16([0.0, -0.0, 1.0, -1.0])
    a, s = orc.quantize_acts(X, ternary=False)
    x = X.astype(np.float64)
    np.testing.assert_array_equal(a, np.where(x < 0, -1, 1))
    np.testing.assert_array_equal(s, (np.abs(x).sum(1) / x.shape[1]).astype(np.float32))


def test_nonfinite_is_an_error(orc):
    X = workloads.edge_acts(2, 32, "normal")
    X[1, 5] = np.inf
    with pytest.raises(orc.OracleError):
        orc.quantize_acts(X)


# -------------------------------------------------------------- weights
def test_binary_weight_golden(orc):
    for g, ws, bs, als in read_golden("binary_weights.txt"):
        W = np.array([float(v) for v in ws.split()], np.float32)[None, :]
        W[0][np.array([v == "-0" for v in ws.split()])] = -0.0
        b, alpha = orc.binarize_weights(W, int(g))
        assert b[0].tolist() == [int(v) for v in bs.split()]
        assert alpha[0].tolist() == [np.float32(float(v)) for v in als.split()]


def test_weight_scale_is_l2_optimal_and_matches_numpy(orc):
    W = workloads.edge_weights(64, 512)
    for group in (0, 128, 96):
        b, alpha = orc.binarize_weights(W, group)
        np.testing.assert_array_equal(b, np.where(W < 0, -1, 1))
        gs = group or 512
        G = -(-512 // gs)
        for g in range(G):
            blk = W[:, g * gs:(g + 1) * gs].astype(np.float64)
            ref = np.abs(blk).mean(axis=1)
            np.testing.assert_allclose(alpha[:, g], ref, rtol=2 ** -23)
            # mean|w| minimises ||w - alpha*sign(w)||^2 over alpha
            sgn = np.where(blk < 0, -1.0, 1.0)
            err = lambda al: ((blk - al[:, None] * sgn) ** 2).sum(axis=1)
            a0 = alpha[:, g].astype(np.float64)
            assert (err(a0) <= err(a0 * 1.01)).all() and (err(a0) <= err(a0 * 0.99)).all()


# -------------------------------------------------------------- packing
def test_pack_matches_numpy_packbits(orc):
    g = workloads.rng(99, 1)
    for K, ld in [(256, 8), (100, 4), (33, 4), (4096, 128)]:
        v = g.integers(-1, 2, (5, K)).astype(np.int8)
        for plane, bits in (("mask", v != 0), ("sign", v < 0)):
            padded = np.zeros((5, ld * 32), bool)
            padded[:, :K] = bits
            ref = np.packbits(padded, axis=1, bitorder="little").view("<u4")
            np.testing.assert_array_equal(orc.pack_plane(v, ld, plane), ref)


def test_linear_golden_example(orc):
    rows = dict((r[0].split(":")[0], r[0].split(":")[1]) for r in read_golden("linear_example.txt"))
    x = f16([float(v) for v in rows["x"].split()])[None, :]
    w = np.array([[float(v) for v in rows["w"].split()]], np.float32)
    r = orc.linear(x, w)
    assert r["dots"][0, 0] == int(rows["dot"])
    assert r["yref"][0, 0] == float(rows["y"]) and r["yrep"][0, 0] == np.float32(float(rows["y"]))
    assert orc.pack_plane(r["a"], 4, "mask")[0, 0] == int(rows["mask_word"])
    assert orc.pack_plane(r["a"], 4, "sign")[0, 0] == int(rows["act_sign_word"])
    assert orc.pack_plane(r["b"], 4, "sign")[0, 0] == int(rows["w_sign_word"])


# -------------------------------------------------------------- dots
def test_int_dots_match_dense_fp64_matmul(orc):
    g = workloads.rng(99, 2)
    for M, N, K, group in [(7, 9, 256, 0), (5, 3, 512, 128), (4, 6, 300, 128), (3, 2, 11008, 128)]:
        a = g.integers(-1, 2, (M, K)).astype(np.int8)
        b = np.where(g.random((N, K)) < 0.5, -1, 1).astype(np.int8)
        d = orc.int_dots(a, b, group)
        np.testing.assert_array_equal(d.sum(axis=2), a.astype(np.float64) @ b.T.astype(np.float64))
        gs = group or K
        for gi in range(d.shape[2]):
            sl = slice(gi * gs, (gi + 1) * gs)
            np.testing.assert_array_equal(d[:, :, gi], a[:, sl].astype(np.float64) @ b[:, sl].T)


def test_int_dots_brute_force_all_patterns(orc):
    """Every {-1,0,1}^3 activation against every {-1,1}^3 weight vector."""
    acts = np.array(list(itertools.product([-1, 0, 1], repeat=3)), np.int8)
    wts = np.array(list(itertools.product([-1, 1], repeat=3)), np.int8)
    d = orc.int_dots(acts, wts)[:, :, 0]
    for i, av in enumerate(acts):
        for j, wv in enumerate(wts):
            assert d[i, j] == sum(int(p) * int(q) for p, q in zip(av, wv))


def test_popcount_identities(orc):
    """The packed-bit forms of the dot product equal the oracle's dot:
    popc(m) - 2*popc(m & (sa ^ sw)) and the AND-popc form used with b1 MMAs."""
    g = workloads.rng(99, 3)
    M, N, K = 6, 5, 320
    ld = 12
    a = g.integers(-1, 2, (M, K)).astype(np.int8)
    b = np.where(g.random((N, K)) < 0.5, -1, 1).astype(np.int8)
    m, sa, sw = orc.pack_plane(a, ld, "mask"), orc.pack_plane(a, ld, "sign"), orc.pack_plane(b, ld, "sign")
    d = orc.int_dots(a, b)[:, :, 0]
    pc = lambda x: np.bitwise_count(x).astype(np.int64).sum(axis=-1)
    form1 = pc(m)[:, None] - 2 * pc(m[:, None, :] & (sa[:, None, :] ^ sw[None, :, :]))
    np.testing.assert_array_equal(form1, d)
    A0, A1 = m & ~sa, m & sa
    form2 = (pc(A0) - pc(A1))[:, None] - 2 * (pc(A0[:, None] & sw[None]) - pc(A1[:, None] & sw[None]))
    np.testing.assert_array_equal(form2, d)
    # binary activations: K - 2 * Hamming distance
    ab, _ = orc.quantize_acts(workloads.edge_acts(M, K, "normal"), ternary=False)
    sab = orc.pack_plane(ab, ld, "sign")
    np.testing.assert_array_equal(orc.int_dots(ab, b)[:, :, 0],
                                  K - 2 * pc(sab[:, None, :] ^ sw[None, :, :]))


# -------------------------------------------------------------- outputs
def test_linear_out_matches_dequantized_dense_product(orc):
    for group in (0, 128):
        M, N, K = 9, 11, 512
        X = workloads.edge_acts(M, K, "student", tag=group)
        W = workloads.edge_weights(N, K, tag=group)
        r = orc.linear(X, W, group)
        gs = group or K
        alpha_full = np.repeat(r["alpha"].astype(np.float64), gs, axis=1)[:, :K]
        dense = (r["s"].astype(np.float64)[:, None] * r["a"]) @ (alpha_full * r["b"]).T
        np.testing.assert_allclose(r["yref"], dense, rtol=0, atol=1e-12 * r["mag"].max())
        assert (np.abs(r["yrep"] - r["yref"]) <= 1e-5 * r["mag"] + 1e-30).all()


def test_linear_invariants(orc):
    M, N, K = 4, 8, 256
    X = workloads.edge_acts(M, K, "normal", tag=7)
    W = workloads.edge_weights(N, K, tag=7)
    r = orc.linear(X, W, 128)
    # unit scales reproduce the integer dot exactly
    yref, _, yrep = orc.linear_out(r["d"], np.ones_like(r["alpha"]), np.ones_like(r["s"]))
    np.testing.assert_array_equal(yref, r["dots"].astype(np.float64))
    np.testing.assert_array_equal(yrep, r["dots"].astype(np.float32))
    # flipping every weight sign negates the output (done on the binarized signs)
    d_neg = orc.int_dots(r["a"], -r["b"], 128)
    yneg, _, yneg_rep = orc.linear_out(d_neg, r["alpha"], r["s"])
    np.testing.assert_array_equal(yneg, -r["yref"])
    np.testing.assert_array_equal(yneg_rep, -r["yrep"])
    # all-zero activations give exactly 0 (not NaN)
    z = orc.linear(np.zeros((M, K), np.float16), W, 128)
    assert (z["yref"] == 0).all() and (z["yrep"] == 0).all() and not np.isnan(z["yrep"]).any()


# -------------------------------------------------------------- attention
def test_attn_scores_match_einsum(orc):
    q = workloads.edge_acts(2 * 5, 64, "normal", tag=1)
    k = workloads.edge_acts(2 * 7, 64, "normal", tag=2)
    aq, sq = orc.quantize_acts(q)
    ak, sk = orc.quantize_acts(k)
    aq, ak = aq.reshape(2, 5, 64), ak.reshape(2, 7, 64)
    S, fref, frep = orc.attn_scores(aq, ak, sq.reshape(2, 5), sk.reshape(2, 7))
    dense = np.einsum("hid,hjd->hij", aq.astype(np.float64), ak.astype(np.float64))
    np.testing.assert_array_equal(S, dense)
    outer = sq.reshape(2, 5, 1).astype(np.float64) * sk.reshape(2, 1, 7)
    np.testing.assert_allclose(fref, dense * outer, rtol=1e-15)
    np.testing.assert_allclose(frep, fref, rtol=1e-6)


# -------------------------------------------------------------- BiLLM
def test_billm_salient_matches_stable_argsort(orc):
    W = workloads.latent_laplace((40, 512), 0.01, 99, 4)
    W[:, 5] = W[:, 6]  # an exact tie between two columns of block 0
    sal = orc.billm_salient(W, 128, 8)
    metric = (W.astype(np.float64) ** 2).sum(axis=0)
    for j in range(4):
        order = np.argsort(-metric[j * 128:(j + 1) * 128], kind="stable")[:8]
        np.testing.assert_array_equal(sal[j], np.sort(order))


def test_billm_reduces_to_blockwise_binarization(orc):
    """No salient columns and no split: BiLLM is per-block binarization."""
    W = workloads.latent_laplace((16, 512), 0.01, 99, 5)
    q = orc.billm_quantize_rows(W, np.zeros((4, 0), np.int32), 0, 16, 128, split=False)
    b, alpha = orc.binarize_weights(W, 128)
    np.testing.assert_array_equal(q["b1"], b)
    np.testing.assert_array_equal(q["scales"][:, :, 0], alpha)
    assert not q["scales"][:, :, 1:].any() and not q["cat"].any()


def test_billm_structure_and_error_invariants(orc):
    N, K = 24, 512
    W = workloads.latent_laplace((N, K), 0.01, 99, 6)
    sal = orc.billm_salient(W, 128, 8)
    q = orc.billm_quantize_rows(W, sal, 0, N, 128, split=True)
    cat, sc = q["cat"], q["scales"]
    W64 = W.astype(np.float64)
    for j in range(4):
        blk = slice(j * 128, (j + 1) * 128)
        c = cat[:, blk]
        w = W64[:, blk]
        assert ((c == 2).sum(axis=1) == 8).all()
        assert (np.where(c[0] == 2)[0] == sal[j]).all()
        for n in range(N):
            ns = c[n] != 2
            mx = np.abs(w[n][ns]).max()
            np.testing.assert_array_equal(c[n][ns] == 1, np.abs(w[n][ns]) > 0.5 * mx)
            for gi, grp in ((0, c[n] == 0), (1, c[n] == 1)):
                ref = np.abs(w[n][grp]).mean() if grp.any() else 0.0
                assert abs(sc[n, j, gi] - ref) <= 2 ** -23 * ref
            s_ = c[n] == 2
            a1 = np.abs(w[n][s_]).mean()
            assert abs(sc[n, j, 2] - a1) <= 2 ** -23 * a1
            r1 = w[n][s_] - np.float64(sc[n, j, 2]) * np.where(w[n][s_] < 0, -1, 1)
            assert abs(sc[n, j, 3] - np.abs(r1).mean()) <= 2 ** -23 * np.abs(r1).mean()
    what = orc.billm_dequant(q)
    # the residual plane and the split each lower the reconstruction error
    plain = orc.billm_quantize_rows(W, np.zeros((4, 0), np.int32), 0, N, 128, split=False)
    err = lambda wh: ((W64 - wh) ** 2).sum()
    assert err(what) < err(orc.billm_dequant(plain))
    nores = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in q.items()}
    nores["scales"][:, :, 3] = 0
    assert err(what) < err(orc.billm_dequant(nores))


def test_billm_gemm_matches_dense_product(orc):
    N, K, M = 20, 384, 6
    W = workloads.latent_laplace((N, K), 0.01, 99, 7)
    X = workloads.edge_acts(M, K, "normal", tag=8)
    sal = orc.billm_salient(W, 128, 8)
    q = orc.billm_quantize_rows(W, sal, 0, N, 128)
    yref, mag = orc.billm_gemm(X, q)
    dense = X.astype(np.float64) @ orc.billm_dequant(q).T
    np.testing.assert_allclose(yref, dense, rtol=0, atol=1e-13 * mag.max())
    np.testing.assert_allclose(mag, np.abs(X.astype(np.float64)) @ np.abs(orc.billm_dequant(q)).T,
                               rtol=1e-13)
    # negating the binarized planes negates the output
    qn = dict(q, b1=-q["b1"], b2=-q["b2"])
    np.testing.assert_array_equal(orc.billm_gemm(X, qn)[0], -yref)


def test_billm_pack_matches_numpy_packbits(orc):
    N, K = 10, 256
    W = workloads.latent_laplace((N, K), 0.01, 99, 9)
    sal = orc.billm_salient(W, 128, 8)
    q = orc.billm_quantize_rows(W, sal, 0, N, 128)
    p = orc.billm_pack(q, 8)
    pk = lambda bits: np.packbits(bits, axis=1, bitorder="little").view("<u4")
    np.testing.assert_array_equal(p["sign"], pk(q["b1"] < 0))
    np.testing.assert_array_equal(p["gmap"], pk(q["cat"] == 1))
    for j in range(2):
        b2s = q["b2"][:, j * 128 + sal[j]] < 0
        np.testing.assert_array_equal(p["res"][:, j], np.packbits(b2s, axis=1, bitorder="little")[:, 0])
        np.testing.assert_array_equal(p["sal"][j], sal[j])


# ------------------------------------------------ attention probabilities, A.V
def _golden_scores(tok):
    return float(np.log(float(tok[2:]))) if tok.startswith("ln") else float(tok)


def test_softmax_ternarize_golden_rows(orc):
    for scores, c, keep, scale in read_golden("softmax_rows.txt"):
        f = np.array([[_golden_scores(t) for t in scores.split()]], np.float32)
        a, s, p = orc.softmax_ternarize(f, float(c))
        assert a[0].tolist() == [int(t) for t in keep.split()], scores
        assert abs(float(s[0]) - float(scale)) <= 1e-6 * float(scale), (scores, s)
        assert abs(p.sum() - 1.0) < 1e-12


def test_softmax_ternarize_matches_numpy(orc):
    g = np.random.default_rng(42)
    f = (g.standard_normal((64, 300)) * 3).astype(np.float32)
    c = 0.125
    a, s, p = orc.softmax_ternarize(f, c)
    x = (f * np.float32(c)).astype(np.float64)       # the product in fp32, as the definition
    e = np.exp(x - x.max(axis=1, keepdims=True))
    pn = e / e.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(p, pn, rtol=1e-13, atol=0)
    keep = pn > 0.5 / f.shape[1]
    np.testing.assert_array_equal(a.astype(bool), keep)
    mean_kept = np.array([pn[r, keep[r]].mean() if keep[r].any() else 0.0 for r in range(64)])
    np.testing.assert_array_equal(s, mean_kept.astype(np.float32))


def test_softmax_ternarize_invariants(orc):
    g = np.random.default_rng(7)
    f = g.integers(-20, 20, (16, 128)).astype(np.float32)
    a, s, p = orc.softmax_ternarize(f, 0.5)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    a2, s2, p2 = orc.softmax_ternarize(f + 6.0, 0.5)   # a shift of the row (exact in fp32)
    np.testing.assert_array_equal(a, a2)
    np.testing.assert_allclose(p2, p, rtol=1e-12)
    assert ((a == 0) | (a == 1)).all() and (a.sum(axis=1) >= 1).all()   # the max is always kept


def test_attn_av_matches_dense_dequantized_product(orc):
    g = np.random.default_rng(3)
    BH, Lq, L, D = 2, 5, 96, 7
    f = (g.standard_normal((BH, Lq, L)) * 4).astype(np.float32)
    ap, sp, _ = orc.softmax_ternarize(f, 0.25)
    V = g.standard_normal((BH, L, D)).astype(np.float16)
    vt = np.ascontiguousarray(V.transpose(0, 2, 1)).reshape(-1, L)
    av, sv = orc.quantize_acts(vt)
    O, Oref, Orep = orc.attn_av(ap, sp, av.reshape(BH, D, L), sv.reshape(BH, D))
    Pd = ap.astype(np.float64) * sp[..., None].astype(np.float64)
    Vd = av.reshape(BH, D, L).astype(np.float64) * sv.reshape(BH, D)[..., None].astype(np.float64)
    dense = np.einsum("hql,hdl->hqd", Pd, Vd)
    np.testing.assert_allclose(Oref, dense, rtol=1e-12, atol=1e-300)
    np.testing.assert_array_equal(O, np.einsum("hql,hdl->hqd", ap.astype(np.int64),
                                               av.reshape(BH, D, L).astype(np.int64)))


# ------------------------------------------------ BiLLM break-point search
def _frac(t):
    a, b = t.split("/")
    return float(a) / float(b)


def test_billm_split_golden(orc):
    for ws, mode, cats, ac, asp in read_golden("billm_split.txt"):
        W = (np.array([float(v) for v in ws.split()], np.float32) / np.float32(128))[None, :]
        sal = np.zeros((1, 0), np.int32)
        q = orc.billm_quantize_rows(W, sal, 0, 1, block=8, split=int(mode))
        assert q["cat"][0].tolist() == [int(v) for v in cats.split()], (ws, mode)
        assert q["scales"][0, 0, 0] == np.float32(_frac(ac)), (ws, mode, q["scales"])
        assert q["scales"][0, 0, 1] == np.float32(_frac(asp)), (ws, mode, q["scales"])


def _np_split_error(v, p):
    e = 0.0
    for grp in (v[v <= p], v[v > p]):
        if grp.size:
            e += float(((grp - grp.mean()) ** 2).sum())
    return e


def test_billm_split_search_matches_numpy_brute_force(orc):
    W = workloads.latent_laplace((12, 384), 0.01, 99, 12, 384)
    sal = orc.billm_salient(W, 128, 8)
    q = orc.billm_quantize_rows(W, sal, 0, 12, 128, split=2)
    qf = orc.billm_quantize_rows(W, sal, 0, 12, 128, split=1)
    for n in range(12):
        for j in range(3):
            cols = np.setdiff1d(np.arange(128), sal[j]) + 128 * j
            v = np.abs(W[n, cols].astype(np.float64))
            errs = [(_np_split_error(v, p), p) for p in np.unique(v)]
            e_best, p_best = min(errs)      # ties: the smaller p
            sparse = v > p_best
            np.testing.assert_array_equal(q["cat"][n, cols] == 1, sparse)
            ac = np.float32(v[~sparse].mean())
            asp = np.float32(v[sparse].mean()) if sparse.any() else np.float32(0)
            np.testing.assert_allclose(q["scales"][n, j, :2], [ac, asp], rtol=2 ** -23)
            # the search never does worse than the fixed 0.5 * max break-point
            fixed = v > 0.5 * v.max()
            assert e_best <= _np_split_error(v, v[~fixed].max()) + 1e-18
            assert (qf["cat"][n, cols] == 1).tolist() == fixed.tolist()


def test_billm_split_search_lowers_reconstruction_error(orc):
    W = workloads.latent_laplace((16, 256), 0.01, 98, 16, 256)
    sal = orc.billm_salient(W, 128, 8)
    e = {}
    for mode in (0, 1, 2):
        q = orc.billm_quantize_rows(W, sal, 0, 16, 128, split=mode)
        e[mode] = float(((W.astype(np.float64) - orc.billm_dequant(q)) ** 2).sum())
    assert e[2] <= e[1] <= e[0]
