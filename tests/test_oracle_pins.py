"""Pins of the CPU oracle against what the pages and mathematics fix.

Every check here compares the oracle with something other than itself:
published values (golden fixtures), closed forms, library routines for
special cases (Hadamard matrices, Beta laws, dense attention), brute force
on small inputs, and invariants.  No GPU is used.
"""
import math

import numpy as np
import pytest
import scipy.integrate
import scipy.linalg
import scipy.stats
import torch

import oracle
from tests.conftest import read_golden

D, M, B = 128, 8, 16


def _signs(seed=0):
    return oracle.srht_signs(seed, D)


# ------------------------------------------------------------------ SRHT
def test_splitmix64_published_vector():
    want = [int(x, 16) for x in read_golden("splitmix64_seed0.txt")]
    gamma = 0x9E3779B97F4A7C15
    got = [oracle.splitmix64((i * gamma) % 2**64) for i in range(4)]
    assert got == want


def test_srht_signs_follow_splitmix64_bit63():
    s = oracle.srht_signs(7, D)
    for j in (0, 1, 77, 127):
        bit = oracle.splitmix64(7 * D + j) >> 63
        assert s[j] == (-1 if bit else 1)
    assert set(np.unique(s)) <= {-1, 1}


def test_rotation_equals_explicit_srht_matrix():
    """R = H_D diag(s) / sqrt(D) (slides, Eq. 5; H from scipy's Sylvester
    construction).  R e_j is column j of R."""
    s = _signs(3)
    R = scipy.linalg.hadamard(D).astype(np.float64) @ np.diag(s.astype(np.float64)) / math.sqrt(D)
    cols = np.stack([oracle.rotate(np.eye(D, dtype=np.float32)[j], s)[0] for j in range(D)], 1)
    np.testing.assert_allclose(cols, R, rtol=0, atol=1e-7)
    np.testing.assert_allclose(cols.T.astype(np.float64) @ cols, np.eye(D), atol=2e-6)


def test_rotation_preserves_normalised_inner_products():
    rng = np.random.default_rng(1)
    s = _signs(0)
    X = rng.standard_normal((64, D)).astype(np.float32) * rng.lognormal(0, 0.5, D).astype(np.float32)
    T = np.stack([oracle.rotate(x, s)[0] for x in X]).astype(np.float64)
    Xh = X.astype(np.float64) / np.linalg.norm(X.astype(np.float64), axis=1, keepdims=True)
    np.testing.assert_allclose(T @ T.T, Xh @ Xh.T, atol=2e-6)
    np.testing.assert_allclose(np.linalg.norm(T, axis=1), 1.0, atol=1e-6)
    nrm = np.array([oracle.rotate(x, s)[1] for x in X], np.float64)
    np.testing.assert_allclose(nrm, np.linalg.norm(X.astype(np.float64), axis=1), rtol=1e-6)


def test_rotation_of_zero_vector_is_zero():
    t, n = oracle.rotate(np.zeros(D, np.float32), _signs())
    assert n == 0.0 and not t.any()


def test_block_energy_and_direction_follow_beta_laws():
    """Slides, Prop. 4.1 / App. B.1: with a Haar rotation (and exactly, for
    Gaussian keys and any orthogonal R), r_b^2 ~ Beta(m/2, (D-m)/2) and
    (u_b)_j^2 ~ Beta(1/2, (m-1)/2)."""
    rng = np.random.default_rng(2)
    K = rng.standard_normal((20000, D)).astype(np.float32)
    enc = oracle.encode_keys(K, _signs(), debug=True)
    for b in (0, 7, 15):
        p = scipy.stats.kstest(enc["rb"][:, b].astype(np.float64) ** 2, "beta",
                               args=(M / 2, (D - M) / 2)).pvalue
        assert p > 1e-3, (b, p)
        for j in (0, 5):
            p = scipy.stats.kstest(enc["u"][:, b * M + j].astype(np.float64) ** 2, "beta",
                                   args=(0.5, (M - 1) / 2)).pvalue
            assert p > 1e-3, (b, j, p)


# ---------------------------------------------------------- Lloyd-Max
def _F0_m8(y):
    th = np.arcsin(np.clip(y, 0.0, 1.0))
    return 5 * th / 16 + 15 * np.sin(2 * th) / 64 + 3 * np.sin(4 * th) / 64 + np.sin(6 * th) / 192


def _F1_m8(y):
    return (1.0 - (1.0 - np.clip(y, 0.0, 1.0) ** 2) ** 3.5) / 7.0


def test_magnitude_density_closed_form_m8():
    """For m = 8: f(y) = 2(1-y^2)^{5/2} / B(1/2, 7/2) = 32/(5 pi) (1-y^2)^{5/2}."""
    for y in (0.0, 0.1, 0.37, 0.8, 0.999, 1.0):
        want = 32.0 / (5.0 * math.pi) * (1 - y * y) ** 2.5
        assert oracle.magnitude_density(8, y) == pytest.approx(want, rel=1e-13, abs=1e-15)


@pytest.mark.parametrize("m", [3, 4, 8, 16])
def test_magnitude_density_integrates_to_one(m):
    val, err = scipy.integrate.quad(lambda y: oracle.magnitude_density(m, y), 0, 1,
                                    epsabs=1e-13, epsrel=1e-13, limit=200)
    assert val == pytest.approx(1.0, abs=1e-9)


def test_lloyd_max_m3_is_uniform_quantiser():
    """m = 3: the density is uniform on [0,1], whose Lloyd-Max levels are
    (2t+1)/(2L)."""
    lev, thr, it = oracle.lloyd_max(3, 8)
    np.testing.assert_allclose(lev, (2 * np.arange(8) + 1) / 16.0, atol=1e-15)
    np.testing.assert_allclose(thr, np.arange(1, 8) / 8.0, atol=1e-15)


def test_lloyd_max_m8_centroid_and_midpoint_conditions_closed_form():
    lev, thr, it = oracle.lloyd_max(8, 8)
    assert it > 0
    edges = np.concatenate([[0.0], thr, [1.0]])
    cent = (_F1_m8(edges[1:]) - _F1_m8(edges[:-1])) / (_F0_m8(edges[1:]) - _F0_m8(edges[:-1]))
    np.testing.assert_allclose(lev, cent, atol=1e-12)
    np.testing.assert_allclose(thr, 0.5 * (lev[:-1] + lev[1:]), atol=1e-15)
    assert np.all(np.diff(lev) > 0) and 0 < lev[0] and lev[-1] < 1
    assert _F0_m8(1.0) == pytest.approx(5 * math.pi / 32, rel=1e-14)


def test_lloyd_max_m8_agrees_with_monte_carlo():
    """Conditional means of |u_j| for Gaussian-direction samples (the readme's
    Monte-Carlo generator) inside the oracle's cells match its levels."""
    rng = np.random.default_rng(5)
    g = rng.standard_normal((1_000_000, M))
    y = np.abs(g / np.linalg.norm(g, axis=1, keepdims=True)).ravel()
    lev, thr, _ = oracle.lloyd_max(8, 8)
    cell = np.searchsorted(thr, y, side="left")
    mc = np.bincount(cell, weights=y, minlength=8) / np.bincount(cell, minlength=8)
    np.testing.assert_allclose(mc, lev, atol=1.5e-3)


def test_levels_f32_are_rounded_fp64_levels():
    lev32, thr32 = oracle.levels_f32(8, 8)
    lev, thr, _ = oracle.lloyd_max(8, 8)
    assert np.array_equal(lev32, lev.astype(np.float32))
    assert np.array_equal(thr32, thr.astype(np.float32))


# -------------------------------------------------------------- encoding
@pytest.fixture(scope="module")
def enc_random():
    rng = np.random.default_rng(11)
    K = (rng.standard_normal((3000, D)) * rng.lognormal(0, 0.5, D)).astype(np.float32)
    K[5] = 0.0                       # a zero key
    K[6] = 0.0                       # e_0 + e_8: Walsh rows cancel on whole
    K[6, 0] = K[6, 8] = 1.0          # aligned blocks, so some rotated blocks are 0
    enc = oracle.encode_keys(K, _signs(), debug=True)
    enc["K"] = K
    return enc


def test_codes_are_brute_force_nearest_sign_pattern(enc_random):
    """c_b = argmax_{w in {+-1/sqrt m}^m} <u_b, w> (slides, Eq. 6), by brute
    force over all 256 centres, lowest id on ties."""
    u = enc_random["u"].astype(np.float64).reshape(-1, B, M)
    omega = np.array([[(-1.0 if (c >> j) & 1 else 1.0) / math.sqrt(M) for j in range(M)]
                      for c in range(256)])
    scores = u @ omega.T                                   # [n][B][256]
    bf = scores.argmax(-1)
    ties = (np.abs(u) < 1e-6).any(-1) & (np.linalg.norm(u, axis=-1) > 0)
    assert ties.sum() == 0
    assert np.array_equal(bf, enc_random["codes"].astype(np.int64))


def test_zero_key_and_zero_block_encode_to_zero(enc_random):
    assert not enc_random["codes"][5].any() and not enc_random["w"][5].any()
    zero = enc_random["rb"][6] == 0
    assert zero.sum() == B // 2
    assert not enc_random["codes"][6][zero].any() and not enc_random["w"][6][zero].any()
    assert not enc_random["tidx"][6].reshape(B, M)[zero].any()
    assert (enc_random["w"][6][~zero] > 0).all()


def test_level_index_is_nearest_level(enc_random):
    lev, thr = enc_random["lev"], enc_random["thr"]
    y = np.abs(enc_random["u"].astype(np.float64))
    near = np.abs(y[..., None] - lev.astype(np.float64)).argmin(-1)
    close = (np.abs(y[..., None] - thr.astype(np.float64)) < 1e-6).any(-1)
    ok = (near == enc_random["tidx"]) | close
    assert ok.all()
    assert close.sum() < 20


def test_weights_match_definition(enc_random):
    """w_b = ||k|| r_b / alpha_b with alpha_b = <v_b, u_b> (slides, Eqs. 7-8)."""
    lev = enc_random["lev"].astype(np.float64)
    u = enc_random["u"].astype(np.float64).reshape(-1, B, M)
    v = lev[enc_random["tidx"].reshape(-1, B, M)] * np.sign(u)
    alpha = (v * u).sum(-1)
    knorm = np.linalg.norm(enc_random["K"].astype(np.float64), axis=1)
    rb = enc_random["rb"].astype(np.float64)
    live = rb > 0
    w = np.zeros_like(rb)
    w[live] = (knorm[:, None] * rb)[live] / alpha[live]
    np.testing.assert_allclose(enc_random["w"], w, rtol=2e-6, atol=0)
    assert (alpha[live] > 0).all()
    assert (alpha[live] <= np.sqrt((v ** 2).sum(-1))[live] + 1e-6).all()


def test_occupancy_counts(enc_random):
    n = enc_random["codes"].shape[0]
    occ = enc_random["occ"]
    assert (occ.sum(1) == n).all()
    for b in range(B):
        assert np.array_equal(np.bincount(enc_random["codes"][:, b], minlength=256), occ[b])


def test_encoding_is_append_consistent():
    """Encoding keys one at a time equals encoding them together; new keys
    need no retraining (slides, Prop. 4.1: the codebook does not depend on
    the data)."""
    rng = np.random.default_rng(3)
    K = rng.standard_normal((200, D)).astype(np.float32)
    full = oracle.encode_keys(K, _signs())
    a = oracle.encode_keys(K[:150], _signs())
    b = oracle.encode_keys(K[150:], _signs())
    assert np.array_equal(full["codes"], np.concatenate([a["codes"], b["codes"]]))
    assert np.array_equal(full["tidx"], np.concatenate([a["tidx"], b["tidx"]]))
    assert np.array_equal(full["w"], np.concatenate([a["w"], b["w"]]))
    assert np.array_equal(full["occ"], a["occ"] + b["occ"])


# --------------------------------------------------------------- Stage I
def test_tiers_hand_example(golden):
    rows = {ln.split()[0]: ln.split()[1:] for ln in golden("tiers_hand.txt")}
    m = int(rows["m"][0])
    R = int(rows["R"][0])
    qt = np.array(rows["qt"], np.float32)
    occ = np.array(rows["occ"], np.uint32).reshape(-1, 1 << m)
    lut, bonus = oracle.bonus_from_qt(qt, occ, R, m=m)
    assert np.array_equal(lut.ravel(), np.array(rows["lut"], np.float32))
    assert np.array_equal(bonus.ravel(), np.array(rows["bonus"], np.uint8))


def test_tier_bonuses_golden(golden):
    """Buckets of 100 keys each starting at P = 0,100,..,500 with R = 600 get
    the six printed bonuses; the next bucket (P = R) gets none."""
    want = [int(ln.split()[1]) for ln in golden("tier_bonuses.txt")]
    qt = np.zeros(D, np.float32)
    qt[:M] = -(np.float32(2.0) ** (np.arange(M, dtype=np.float32) - 8))  # L(c) increases with c
    occ = np.zeros((B, 256), np.uint32)
    occ[:, 248:] = 1000 // 8
    occ[0, :] = 0
    order = np.arange(255, 248, -1)                        # highest L first
    occ[0, order] = 100
    occ[0, 0] = 1000 - 700
    lut, bonus = oracle.bonus_from_qt(qt, occ, 600)
    assert list(np.argsort(-lut[0], kind="stable")[:7]) == list(order)
    assert [int(bonus[0, c]) for c in order[:6]] == want
    assert bonus[0, order[6]] == 0


def test_bonus_closed_form_for_centroid_aligned_query():
    """If q~_b is a sign-pattern centre w*, L_b(c) is proportional to
    m - 2 Hamming(c, c*): the bucket ranking is by Hamming distance (ties by
    id), so the tiers can be computed without any bucket scores."""
    rng = np.random.default_rng(4)
    cstar = rng.integers(0, 256, B)
    qt = np.array([(-0.125 if (cstar[b] >> j) & 1 else 0.125) for b in range(B) for j in range(M)],
                  np.float32)
    occ = rng.integers(0, 40, (B, 256)).astype(np.uint32)
    occ[:, 0] += (5000 - occ.sum(1)).clip(0).astype(np.uint32)
    n = int(occ[0].sum())
    occ[1:, 0] += (n - occ[1:].sum(1)).astype(np.uint32)
    R = math.ceil(0.2 * n)
    _, bonus = oracle.bonus_from_qt(qt, occ, R)
    for b in range(B):
        ham = np.array([bin(c ^ int(cstar[b])).count("1") for c in range(256)])
        order = np.lexsort((np.arange(256), ham))
        P = np.concatenate([[0], np.cumsum(occ[b, order].astype(np.int64))[:-1]])
        want = np.zeros(256, np.uint8)
        want[order] = np.where(P < R, 6 - (6 * P) // R, 0)
        assert np.array_equal(bonus[b], want), b


def test_lut_matches_fp64_centre_scores():
    rng = np.random.default_rng(8)
    qt = rng.standard_normal(D).astype(np.float32) / np.float32(11.3)
    lut, _ = oracle.bonus_from_qt(qt, np.ones((B, 256), np.uint32), 1000)
    sgn = np.array([[(-1.0 if (c >> j) & 1 else 1.0) for j in range(M)] for c in range(256)])
    want = qt.astype(np.float64).reshape(B, M) @ sgn.T
    np.testing.assert_allclose(lut, want, atol=1e-6)


def test_collision_counts_brute_force_over_keys(enc_random):
    """S_i by a key-level brute force: per block, order keys by the score of
    their centre (then centre id), a key is in T_b(rho) when the first key of
    its bucket sits before position R, its tier is floor(6 pos / R)."""
    rng = np.random.default_rng(9)
    qt, _ = oracle.rotate(rng.standard_normal(D).astype(np.float32), _signs())
    codes = enc_random["codes"].astype(np.int64)
    n = codes.shape[0]
    R = math.ceil(0.25 * n)
    lut, bonus = oracle.bonus_from_qt(qt, enc_random["occ"], R)
    S = oracle.collision(enc_random["codes"], bonus)
    want = np.zeros(n, np.int64)
    for b in range(B):
        c = codes[:, b]
        order = np.lexsort((np.arange(n), c, -lut[b][c].astype(np.float64)))
        pos = np.empty(n, np.int64)
        pos[order] = np.arange(n)
        first = np.full(256, n, np.int64)
        np.minimum.at(first, c, pos)
        p = first[c]
        want += np.where(p < R, 6 - (6 * p) // R, 0)
    assert np.array_equal(S.astype(np.int64), want)
    assert int(S.astype(np.int64).sum()) == int((bonus.astype(np.int64) * enc_random["occ"]).sum())


def test_candidates_hand_example(golden):
    lines = golden("candidates_hand.txt")
    S = np.array(lines[0].split()[1:], np.uint8)
    for ln in lines[1:]:
        lhs, rhs = ln.split("->")
        C = int(lhs.split()[1])
        assert list(oracle.candidates(S, C)) == [int(x) for x in rhs.split()]


def test_candidates_brute_force_random():
    rng = np.random.default_rng(10)
    S = rng.integers(0, 30, 5000).astype(np.uint8)
    for C in (1, 100, 777, 4999, 5000):
        order = np.lexsort((np.arange(5000), -S.astype(np.int64)))
        assert np.array_equal(oracle.candidates(S, C), np.sort(order[:C]))


# -------------------------------------------------------------- Stage II
def _exact_mode_search(K, q, signs):
    enc = oracle.encode_keys(K, signs, quantize=False, debug=True)
    v = enc["u"].astype(np.float64)
    qt, qn = oracle.rotate(q, signs)
    cand = np.arange(K.shape[0], dtype=np.int32)
    return oracle.rerank(cand, v, enc["w"], qt, qn), cand


def test_estimator_is_exact_without_quantisation():
    """With v = u (no quantisation) alpha = 1 and the estimate equals <k, q>
    (slides, Eqs. 7-10)."""
    rng = np.random.default_rng(12)
    K = (rng.standard_normal((500, D)) * rng.lognormal(0, 0.5, D)).astype(np.float32)
    q = rng.standard_normal(D).astype(np.float32)
    est, _ = _exact_mode_search(K, q, _signs())
    true = K.astype(np.float64) @ q.astype(np.float64)
    scale = np.linalg.norm(K.astype(np.float64), axis=1) * np.linalg.norm(q.astype(np.float64))
    assert (np.abs(est - true) <= 3e-6 * scale).all()


def test_estimator_error_shrinks_as_quantisation_is_removed():
    rng = np.random.default_rng(13)
    K = (rng.standard_normal((2000, D)) * rng.lognormal(0, 0.5, D)).astype(np.float32)
    q = K[:8].sum(0) + rng.standard_normal(D).astype(np.float32)
    true = K.astype(np.float64) @ q.astype(np.float64)
    signs = _signs()
    qt, qn = oracle.rotate(q, signs)
    cand = np.arange(K.shape[0], dtype=np.int32)
    errs = []
    for L in (2, 4, 8, 16, 32):
        lev = oracle.levels_f32(8, L)
        enc = oracle.encode_keys(K, signs, L=L, levels=lev)
        v = oracle.dequantize(enc["codes"], enc["tidx"], lev[0])
        est = oracle.rerank(cand, v, enc["w"], qt, qn)
        errs.append(np.mean(np.abs(est - true)))
    # each extra bit roughly halves the error (quantisation step ~ 1/L)
    assert all(b < 0.75 * a for a, b in zip(errs, errs[1:])), errs
    assert errs[-1] < 0.1 * errs[0]


def test_topk_with_full_budget_is_exact_topk():
    """With C = n and no quantisation the path returns the exact Top-k of
    <k_i, q> (except at gaps below the fp32 rounding of the inputs)."""
    rng = np.random.default_rng(14)
    K = (rng.standard_normal((3000, D)) * rng.lognormal(0, 0.5, D)).astype(np.float32)
    q = rng.standard_normal(D).astype(np.float32)
    est, cand = _exact_mode_search(K, q, _signs())
    idx, _ = oracle.topk(cand, est, 100)
    true = K.astype(np.float64) @ q.astype(np.float64)
    ref = np.lexsort((np.arange(len(true)), -true))[:100]
    kth = true[ref[-1]]
    diff = set(idx.tolist()) ^ set(ref.tolist())
    assert all(abs(true[i] - kth) < 1e-4 for i in diff)
    assert len(diff) <= 2


def test_topk_tie_rule():
    cand = np.array([9, 3, 7, 1, 5], np.int32)
    est = np.array([1.0, 2.0, 2.0, 0.5, 2.0])
    idx, score = oracle.topk(cand, est, 4)
    assert list(idx) == [3, 5, 7, 9] and list(score) == [2.0, 2.0, 2.0, 1.0]


def test_full_pipeline_full_budget_covers_all_keys():
    rng = np.random.default_rng(15)
    K = rng.standard_normal((600, D)).astype(np.float32)
    enc = oracle.build_index(K)
    out = oracle.search(enc, rng.standard_normal((1, D)).astype(np.float32), topk_k=50,
                        cand_budget=600)
    assert np.array_equal(out["cand"], np.arange(600))
    est_all = oracle.rerank(np.arange(600, dtype=np.int32), enc["v"], enc["w"], out["qt"],
                            out["qnorm"])
    ref = np.lexsort((np.arange(600), -est_all))[:50]
    assert np.array_equal(out["idx"], ref)


def test_gqa_group_of_one_is_the_single_query():
    rng = np.random.default_rng(16)
    q = rng.standard_normal((1, D)).astype(np.float32)
    occ = np.full((B, 256), 10, np.uint32)
    a = oracle.query_prep(q, _signs(), occ, 500)
    qt, qn = oracle.rotate(q[0], _signs())
    assert np.array_equal(a[0], qt) and a[1] == qn
    q4 = rng.standard_normal((4, D)).astype(np.float32)
    b = oracle.query_prep(q4, _signs(), occ, 500)
    agg = ((q4[0] + q4[1]) + q4[2]) + q4[3]
    assert np.array_equal(b[0], oracle.rotate(agg, _signs())[0])


# ------------------------------------------------------------- attention
def test_attention_full_selection_equals_dense_attention():
    """k = n selects every row, so the result is dense softmax attention
    (torch's scaled_dot_product_attention in fp64)."""
    rng = np.random.default_rng(17)
    n = 300
    K = rng.standard_normal((n, D)).astype(np.float32)
    V = rng.standard_normal((n, D)).astype(np.float32)
    q = rng.standard_normal((4, D)).astype(np.float32)
    idx = rng.permutation(n).astype(np.int32)
    o = oracle.attend(q, K, V, idx, 1.0 / math.sqrt(D))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).double()[None, :, None, :],
        torch.from_numpy(K).double()[None, None].expand(1, 4, n, D),
        torch.from_numpy(V).double()[None, None].expand(1, 4, n, D))[0, :, 0, :].numpy()
    np.testing.assert_allclose(o, ref, atol=1e-12)


def test_attention_over_selected_and_dense_rows():
    """Sink/local rows kept outside the index join the retrieved rows under
    one softmax: with no dense rows it is the selected-row attention, with no
    selected rows it is attention over the dense rows, moving a row between
    the two sets changes nothing, and the result is torch's attention over
    the union of rows (fp64)."""
    rng = np.random.default_rng(23)
    n, m, k = 500, 40, 60
    K = rng.standard_normal((n, D)).astype(np.float32)
    V = rng.standard_normal((n, D)).astype(np.float32)
    Kd = rng.standard_normal((m, D)).astype(np.float32)
    Vd = rng.standard_normal((m, D)).astype(np.float32)
    q = rng.standard_normal((4, D)).astype(np.float32)
    idx = rng.choice(n, k, replace=False).astype(np.int32)
    sc = 1.0 / math.sqrt(D)
    o = oracle.attend_union(q, K, V, idx, Kd, Vd, sc)
    np.testing.assert_array_equal(oracle.attend_union(q, K, V, idx, Kd[:0], Vd[:0], sc),
                                  oracle.attend(q, K, V, idx, sc))
    np.testing.assert_allclose(oracle.attend_union(q, K, V, idx[:0], Kd, Vd, sc),
                               oracle.attend(q, Kd, Vd, np.arange(m), sc), atol=1e-14)
    # move selected row idx[0] into the dense set
    o2 = oracle.attend_union(q, K, V, idx[1:], np.concatenate([Kd, K[idx[:1]]]),
                             np.concatenate([Vd, V[idx[:1]]]), sc)
    np.testing.assert_allclose(o, o2, atol=1e-14)
    Ku = np.concatenate([K[idx], Kd])
    Vu = np.concatenate([V[idx], Vd])
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).double()[None, :, None, :],
        torch.from_numpy(Ku).double()[None, None].expand(1, 4, k + m, D),
        torch.from_numpy(Vu).double()[None, None].expand(1, 4, k + m, D))[0, :, 0, :].numpy()
    np.testing.assert_allclose(o, ref, atol=1e-12)


# ------------------------------------------------------------ parameters
def test_ratio_table_golden(golden):
    for ln in golden("ratio_table.txt"):
        lo, hi, beta, rho = ln.split()
        lo, hi = int(lo), int(hi)
        probes = [lo, lo + 1] + ([hi - 1] if hi > 0 else [lo + 10**6])
        for n in probes:
            assert oracle.ratio_table(n) == (float(beta), float(rho)), n


def test_resolve_budget_and_ratio():
    assert oracle.resolve(131072) == (math.ceil(0.1 * 131072), math.ceil(0.2 * 131072))
    assert oracle.resolve(4096, cand_budget=512) == (512, 2048)
    assert oracle.resolve(32768, cand_budget=2048, collision_ratio=0.2) == (2048, 6554)
    assert oracle.resolve(150, cand_budget=10, topk=100) == (100, 75)
    assert oracle.resolve(80, topk=100) == (80, 40)
