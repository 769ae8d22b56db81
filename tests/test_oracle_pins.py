"""Pins for the CPU oracle: each test checks the oracle against something other than itself
(a library routine, a closed form, an invariant the mathematics fixes, or brute force on tiny
inputs). Sources: "Technical Summary: ParisKV" (gist.science/paper/2602.07721), Methodology,
Core Algorithmic Innovations 1-2."""
import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from long_context_kv_srht_b200 import workload

D, M = 128, 8
B = D // M


def _signs(d, seed=0):
    return np.where(np.random.default_rng(seed).integers(0, 2, d) == 1, -1, 1).astype(np.int8)


def _rotation_matrix(d, signs):
    """R built by applying the oracle to basis vectors (column j = R e_j)."""
    cols = [oracle.rotate_f64(np.eye(d)[j], signs) for j in range(d)]
    return np.stack(cols, axis=1)


# ----------------------------------------------------------------------------- rotation
@pytest.mark.parametrize("d", [4, 16, 128])
def test_rotation_is_orthogonal(d):
    R = _rotation_matrix(d, _signs(d, d))
    np.testing.assert_allclose(R @ R.T, np.eye(d), atol=1e-12)


@pytest.mark.parametrize("d", [8, 128])
def test_rotation_is_sylvester_hadamard_times_signs(d):
    s = _signs(d, 7)
    R = _rotation_matrix(d, s)
    ref = scipy.linalg.hadamard(d).astype(np.float64) * s[None, :].astype(np.float64) / np.sqrt(d)
    np.testing.assert_allclose(R, ref, atol=1e-12)


def test_rotation_closed_form_d4():
    s = np.array([1, 1, 1, 1], np.int8)
    np.testing.assert_allclose(oracle.rotate_f64(np.array([1.0, 0, 0, 0]), s), [0.5] * 4)
    np.testing.assert_allclose(oracle.rotate_f64(np.array([0, 1.0, 0, 0]), s),
                               [0.5, -0.5, 0.5, -0.5])
    s2 = np.array([1, -1, 1, 1], np.int8)
    np.testing.assert_allclose(oracle.rotate_f64(np.array([0, 1.0, 0, 0]), s2),
                               [-0.5, 0.5, -0.5, 0.5])


def test_normalized_rotation_unit_norm_and_norms():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((10000, D)) * rng.uniform(0.1, 30, (10000, 1))).astype(np.float32)
    y, nr = oracle.normalize_rotate(x, _signs(D))
    ny = np.linalg.norm(y.astype(np.float64), axis=1)
    assert np.max(np.abs(ny - 1.0)) <= 1e-5
    np.testing.assert_allclose(nr, np.linalg.norm(x.astype(np.float64), axis=1), rtol=1e-6)


def test_normalized_rotation_zero_row():
    x = np.zeros((2, D), np.float32)
    x[1, 3] = 2.0
    y, nr = oracle.normalize_rotate(x, _signs(D))
    assert np.all(y[0] == 0) and nr[0] == 0
    assert nr[1] == 2.0


def test_rotation_preserves_inner_products():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((64, D)).astype(np.float32)
    y, nr = oracle.normalize_rotate(x, _signs(D, 3))
    xh = x.astype(np.float64) / np.linalg.norm(x.astype(np.float64), axis=1, keepdims=True)
    np.testing.assert_allclose(y.astype(np.float64) @ y.T.astype(np.float64), xh @ xh.T, atol=2e-6)


# ----------------------------------------------------------------------------- bucket ids
def _centroids(m):
    c = np.arange(1 << m)[:, None]
    bits = (c >> np.arange(m)[None, :]) & 1
    return np.where(bits == 1, -1.0, 1.0) / np.sqrt(m)   # [2^m, m], centroid id c


@pytest.mark.parametrize("m", [2, 4, 8])
def test_bucket_id_is_nearest_analytic_centroid(m):
    rng = np.random.default_rng(4)
    d = 16 * m if m < 8 else D
    y = rng.standard_normal((300, d)).astype(np.float32)
    y[::3, ::5] = 0.0          # exact zeros: ties between centroids -> lower id
    y[1::7, 2] = -0.0
    nr = np.ones(300, np.float32)
    enc = oracle.encode_rotated(y, nr, m)
    C = _centroids(m)
    for i in range(y.shape[0]):
        for b in range(d // m):
            yb = y[i, b * m:(b + 1) * m].astype(np.float64)
            ip = C @ yb
            dist = np.sum((C - yb[None, :]) ** 2, axis=1)
            best_ip = int(np.flatnonzero(ip == ip.max())[0])       # lowest id among ties
            best_dist = int(np.flatnonzero(dist == dist.min())[0])
            assert enc.ids[i, b] == best_ip == best_dist


# ----------------------------------------------------------------------------- RSQ codes
def test_codes_uniform_levels_exact_values():
    mx = 0.5
    yb = np.array([mx, -mx, mx * 3 / 7, -mx * 2.49 / 7, mx * 2.51 / 7, 0.0, -0.0, -mx * 0.4 / 7],
                  np.float32)
    y = np.zeros((1, D), np.float32)
    y[0, :8] = yb
    enc = oracle.encode_rotated(y, np.ones(1, np.float32), M)
    assert list(enc.mag[0, :8]) == [7, 7, 3, 2, 3, 0, 0, 0]
    assert list(enc.neg[0, :8]) == [0, 1, 0, 1, 0, 0, 0, 1]
    assert list(enc.codes[0, :8]) == [7, 15, 3, 10, 3, 0, 0, 8]
    # all-zero subspaces: codes 0, factor 0
    assert np.all(enc.mag[0, 8:] == 0) and np.all(enc.factor[0, 1:] == 0)


def test_codes_nearest_uniform_level():
    rng = np.random.default_rng(5)
    y = rng.standard_normal((2000, D)).astype(np.float32)
    enc = oracle.encode_rotated(y, np.ones(2000, np.float32), M)
    yb = np.abs(y.reshape(2000, B, M)).astype(np.float64)
    mx = yb.max(axis=2, keepdims=True)
    lvl = enc.mag.reshape(2000, B, M) * mx / 7.0
    assert np.all(np.abs(yb - lvl) <= mx / 14.0 * (1 + 1e-6))       # nearest of 8 levels
    assert np.all(enc.mag.reshape(2000, B, M).max(axis=2) == 7)      # the max maps to level 7
    np.testing.assert_array_equal(enc.neg, (y < 0).astype(np.uint8))


# ----------------------------------------------------------------------------- estimator
def _literal_terms(enc, y, knorm, qt):
    """The page's estimator written literally in fp64: w = ||k|| ||y_b|| / <u_b, v_b>,
    term_b = w * <v_b, q~_b> with v_b the normalised dequantised direction."""
    n = y.shape[0]
    yb = y.reshape(n, B, M).astype(np.float64)
    vt = enc.vt.reshape(n, B, M)
    nyb = np.linalg.norm(yb, axis=2)
    nvt = np.linalg.norm(vt, axis=2)
    with np.errstate(invalid="ignore", divide="ignore"):
        u = yb / nyb[..., None]
        v = vt / nvt[..., None]
        w = knorm.astype(np.float64)[:, None] * nyb / np.sum(u * v, axis=2)
        terms = w * np.sum(v * qt.reshape(B, M).astype(np.float64)[None], axis=2)
    return np.nan_to_num(terms)


def test_folded_factor_equals_literal_page_form():
    rng = np.random.default_rng(6)
    sg = _signs(D, 9)
    k = (rng.standard_normal((500, D)) * 3 + 1).astype(np.float32)
    q = rng.standard_normal((1, D)).astype(np.float32)
    y, kn = oracle.normalize_rotate(k, sg)
    qt, qn = oracle.normalize_rotate(q, sg)
    enc = oracle.encode_rotated(y, kn, M)
    lit = _literal_terms(enc, y, kn, qt[0])
    folded = enc.factor.astype(np.float64) * np.sum(
        enc.vt.reshape(500, B, M) * qt[0].reshape(B, M).astype(np.float64)[None], axis=2)
    scale = kn.astype(np.float64)[:, None]
    assert np.max(np.abs(folded - lit) / scale) <= 1e-5
    # full estimate from the fp32 rerank vs the literal fp64 sum
    cand = np.arange(500, dtype=np.int32)
    S = oracle.rerank(enc, cand, qt[0], M).astype(np.float64)
    est = float(qn[0]) * S
    est_lit = float(qn[0]) * lit.sum(axis=1)
    assert np.max(np.abs(est - est_lit) / (kn * qn[0])) <= 1e-5


def test_estimate_of_key_with_itself_is_squared_norm():
    rng = np.random.default_rng(7)
    sg = _signs(D, 11)
    k = (rng.standard_normal((200, D)) * rng.uniform(0.5, 5, (200, 1))).astype(np.float32)
    y, kn = oracle.normalize_rotate(k, sg)
    enc = oracle.encode_rotated(y, kn, M)
    for i in range(0, 200, 20):
        one = oracle.Encoded(enc.ids[i:i + 1], enc.mag[i:i + 1], enc.neg[i:i + 1],
                             enc.factor[i:i + 1])
        lit = _literal_terms(one, y[i:i + 1], kn[i:i + 1], y[i])
        k2 = float(kn[i]) ** 2
        # in real arithmetic the estimate of <k,k> is ||k||^2 ||y||^2 exactly (||y|| = 1 up to
        # the fp32 rounding of y)
        y2 = float(np.sum(y[i].astype(np.float64) ** 2))
        assert abs(float(kn[i]) * lit.sum() - k2 * y2) <= 1e-12 * k2
        assert abs(y2 - 1.0) <= 1e-6
        S = oracle.rerank(enc, np.array([i], np.int32), y[i], M)[0]
        assert abs(float(kn[i]) * float(S) - k2) <= 2e-6 * k2


def test_exact_subspaces_single_coordinate_and_equal_magnitudes():
    rng = np.random.default_rng(8)
    y = np.zeros((1, D), np.float32)
    y[0, 3] = 0.6                                  # subspace 0: one non-zero coordinate
    y[0, 8:16] = 0.2 * np.array([1, -1, 1, 1, -1, -1, 1, -1])   # subspace 1: equal magnitudes
    y[0, 16:] = rng.standard_normal(D - 16).astype(np.float32) * 0.05
    kn = np.array([3.0], np.float32)
    enc = oracle.encode_rotated(y, kn, M)
    qt = rng.standard_normal(D).astype(np.float32)
    lit = _literal_terms(enc, y, kn, qt)[0]
    exact = 3.0 * np.array([np.dot(y[0, 0:8].astype(np.float64), qt[0:8]),
                            np.dot(y[0, 8:16].astype(np.float64), qt[8:16])])
    np.testing.assert_allclose(lit[:2], exact, rtol=1e-6, atol=1e-7)


def test_estimate_converges_as_levels_refine():
    rng = np.random.default_rng(9)
    sg = _signs(D, 13)
    k = (rng.standard_normal((400, D)) + 0.3).astype(np.float32)
    q = rng.standard_normal((1, D)).astype(np.float32)
    y, kn = oracle.normalize_rotate(k, sg)
    qt, qn = oracle.normalize_rotate(q, sg)
    exact = k.astype(np.float64) @ q[0].astype(np.float64)
    denom = np.linalg.norm(k.astype(np.float64), axis=1) * np.linalg.norm(q[0].astype(np.float64))
    errs = []
    for bits in range(3, 21):
        L = (1 << bits) - 1
        enc = oracle.encode_rotated(y, kn, M, levels=L)
        lit = _literal_terms(enc, y, kn, qt[0])
        est = float(qn[0]) * lit.sum(axis=1)
        errs.append(float(np.mean(np.abs(est - exact) / denom)))
    for a, b in zip(errs[:-1], errs[1:]):
        assert b <= a * 1.05, errs             # non-increasing up to sampling noise
    assert errs[-1] <= 1e-4 and errs[0] > 10 * errs[-1]


# ----------------------------------------------------------------------------- query LUT
@pytest.mark.parametrize("rho", [1, 2, 4, 16, 256])
def test_query_top_rho_is_brute_force(rho):
    rng = np.random.default_rng(10 + rho)
    C = _centroids(M)
    checked = 0
    for trial in range(20):
        qt = rng.standard_normal(D).astype(np.float32)
        lut = oracle.query_lut(qt, M, rho, 2, 1)
        for b in range(B):
            ip = C @ qt[b * M:(b + 1) * M].astype(np.float64)
            order = np.argsort(-ip, kind="stable")   # descending, ties -> lower id
            if rho < 256 and ip[order[rho - 1]] - ip[order[rho]] <= 1e-6:
                continue
            sel = set(np.flatnonzero(lut[b]).tolist())
            assert sel == set(order[:rho].tolist())
            assert lut[b, order[0]] == 2
            assert all(lut[b, c] == 1 for c in order[1:rho])
            c1 = sum(1 << j for j in range(M) if qt[b * M + j] < 0)
            assert order[0] == c1
            checked += 1
    assert checked > 200


# ----------------------------------------------------------------------------- vote
def test_vote_invariants():
    rng = np.random.default_rng(11)
    sg = _signs(D, 5)
    q = rng.standard_normal((1, D)).astype(np.float32)
    qt, _ = oracle.normalize_rotate(q, sg)
    lut = oracle.query_lut(qt[0], M, 4, 2, 1)
    # keys: the query itself at several positive scales, random keys, and a key whose every
    # subspace sits in the rank-2 bucket
    keys = np.concatenate([q * 0.5, q * 7.0, rng.standard_normal((200, D)).astype(np.float32)])
    y, kn = oracle.normalize_rotate(keys, sg)
    enc = oracle.encode_rotated(y, kn, M)
    rank2 = np.array([[int(np.flatnonzero(lut[b] == 1)[0]) for b in range(B)]], np.uint8)
    ids = np.concatenate([enc.ids, rank2])
    sc = oracle.vote(ids, lut, M)
    assert sc[0] == sc[1] == 2 * B
    assert sc[-1] == B
    assert np.all((sc >= 0) & (sc <= 2 * B))
    assert np.bincount(sc, minlength=2 * B + 1).sum() == ids.shape[0]


# ----------------------------------------------------------------------------- selections
@pytest.mark.parametrize("n,k,bp,want", [(4096, 64, 1000, 410), (131072, 2048, 500, 6554),
                                          (1 << 20, 4096, 500, 52429), (100, 64, 500, 64),
                                          (50, 50, 500, 50), (33, 1, 10000, 33)])
def test_candidate_count(n, k, bp, want):
    assert oracle.candidate_count(n, k, bp) == want


@pytest.mark.parametrize("n,C", [(1, 1), (31, 7), (4096, 410), (5000, 5000)])
def test_select_candidates_is_stable_sort(n, C):
    rng = np.random.default_rng(n)
    sc = rng.integers(0, 6, n).astype(np.int32)        # many ties
    got = oracle.select_candidates(sc, C)
    order = np.argsort(-sc, kind="stable")[:C]
    np.testing.assert_array_equal(got, np.sort(order))


@pytest.mark.parametrize("C,k", [(1, 1), (410, 64), (3000, 3000), (6554, 2048)])
def test_topk_is_stable_sort(C, k):
    rng = np.random.default_rng(C + k)
    S = rng.standard_normal(C).astype(np.float32)
    S[::5] = S[0]                                       # ties -> lower key index wins
    cand = np.sort(rng.choice(10 * C + 10, C, replace=False)).astype(np.int32)
    idx, so = oracle.topk(S, cand, k)
    order = np.lexsort((cand, -S.astype(np.float64)))[:k]
    keep = np.sort(cand[order])
    np.testing.assert_array_equal(idx, keep)
    np.testing.assert_array_equal(so, S[np.searchsorted(cand, keep)])


# ----------------------------------------------------------------------------- attention
def test_attend_dense_equals_sdpa():
    rng = np.random.default_rng(12)
    n = 300
    q = rng.standard_normal(D).astype(np.float32)
    K = rng.standard_normal((n, D)).astype(np.float32)
    V = rng.standard_normal((n, D)).astype(np.float32)
    out = oracle.attend(q, K, V, np.arange(n, dtype=np.int32), 1 / np.sqrt(D))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).double()[None, None, None], torch.from_numpy(K).double()[None, None],
        torch.from_numpy(V).double()[None, None])[0, 0, 0].numpy()
    np.testing.assert_allclose(out, ref, atol=1e-12)
    # a subset equals dense attention over the gathered rows
    idx = np.sort(rng.choice(n, 40, replace=False)).astype(np.int32)
    sub = oracle.attend(q, K, V, idx, 0.1)
    ref2 = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).double()[None, None, None],
        torch.from_numpy(K[idx]).double()[None, None], torch.from_numpy(V[idx]).double()[None, None],
        scale=0.1)[0, 0, 0].numpy()
    np.testing.assert_allclose(sub, ref2, atol=1e-12)


def test_attend_equal_logits_is_mean():
    rng = np.random.default_rng(13)
    K = np.tile(rng.standard_normal(D).astype(np.float32), (50, 1))
    V = rng.standard_normal((50, D)).astype(np.float32)
    out = oracle.attend(rng.standard_normal(D).astype(np.float32), K, V,
                        np.arange(50, dtype=np.int32), 0.3)
    np.testing.assert_allclose(out, V.astype(np.float64).mean(axis=0), atol=1e-12)


# ----------------------------------------------------------------------------- end to end
def test_tiny_workload_retrieves_planted_keys():
    """Informational check of the method on the tiny workload: the planted near-duplicates of
    the query are retrieved, and top-k recall against the exact <k,q> top-k is high."""
    sp = workload.SPECS["tiny"]
    w = workload.generate(sp)
    p = oracle.SearchParams(m=sp.m, rho=sp.rho, cand_bp=sp.cand_bp)
    enc = oracle.build_unit(w.keys[0, 0], w.signs, sp.m)
    idx, s, est, cand, sc = oracle.search(enc, w.queries[0, 0], w.signs, sp.k, p)
    planted = set(w.planted[0, 0].tolist())
    assert len(planted & set(idx.tolist())) / len(planted) >= 0.9
    exact = w.keys[0, 0].astype(np.float64) @ w.queries[0, 0].astype(np.float64)
    true_top = set(np.argsort(-exact, kind="stable")[:sp.k].tolist())
    recall = len(true_top & set(idx.tolist())) / sp.k
    assert recall >= 0.5, recall


# ----------------------------------------------------------------------------- four-region cache
def test_cache_regions_worked_example():
    """Hand-traced against the Sliding-Window Update Mechanism ("Technical Summary: ParisKV",
    System-Level Innovations 2): n_sink=2, n_local=4, n_buffer=2, prefill of 9 tokens."""
    r = oracle.CacheRegions(2, 4, 2)
    r.prefill(9)
    assert (r.sink, r.local, r.buffer, r.retrieval) == ([0, 1], [5, 6, 7, 8], [], [2, 3, 4])
    r.append()                                    # token 9 waits in the buffer
    assert (r.local, r.buffer, r.retrieval) == ([5, 6, 7, 8], [9], [2, 3, 4])
    r.append()                                    # buffer full: 5, 6 evicted, 9, 10 join Local
    assert (r.local, r.buffer, r.retrieval) == ([7, 8, 9, 10], [], [2, 3, 4, 5, 6])
    short = oracle.CacheRegions(3, 4, 2)          # a short prefill leaves Sink to fill first
    short.prefill(1)
    short.append(); short.append()
    assert (short.sink, short.local, short.buffer) == ([0, 1, 2], [], [])
    short.append(); short.append()                # Local not yet full: nothing evicted
    assert (short.local, short.buffer, short.retrieval) == ([3, 4], [], [])


@pytest.mark.parametrize("cfg", [(0, 8, 8, 0), (4, 16, 4, 100), (4, 16, 16, 3), (1, 5, 2, 40)])
def test_cache_regions_invariants(cfg):
    """Over a long run: the regions partition the tokens seen so far, each region keeps token
    order, Retrieval row r holds token n_sink + r, Local never exceeds n_local and the buffer
    stays below n_buffer, and the newest token is always in a dense region."""
    n_sink, n_local, n_buffer, n0 = cfg
    r = oracle.CacheRegions(n_sink, n_local, n_buffer)
    r.prefill(n0)
    for _ in range(300):
        r.append()
        allt = r.sink + r.retrieval + r.local + r.buffer
        assert allt == list(range(r.total))
        assert len(r.local) <= n_local and len(r.buffer) < n_buffer
        assert r.retrieval == list(range(n_sink, n_sink + len(r.retrieval)))
        assert r.total - 1 in r.dense()
        if r.retrieval:                            # Local is full once anything was evicted
            assert len(r.local) + len(r.buffer) >= n_local


def test_cache_step_attend_is_dense_softmax_when_k_covers_retrieval():
    """With k at least the Retrieval size every token is attended: the result equals plain
    softmax attention over all tokens (numpy, fp64)."""
    rng = np.random.default_rng(5)
    s = _signs(D, 3)
    r = oracle.CacheRegions(2, 8, 4)
    r.prefill(30)
    for _ in range(7):
        r.append()
    K = rng.standard_normal((r.total, D)).astype(np.float32)
    V = rng.standard_normal((r.total, D)).astype(np.float32)
    q = rng.standard_normal(D).astype(np.float32)
    enc = oracle.build_unit(K[r.retrieval], s, M)
    out, rows = oracle.cache_step_attend(q, K, V, r, enc, s, 64, 0.09,
                                         oracle.SearchParams(m=M, cand_bp=10000))
    assert sorted(rows.tolist()) == list(range(len(r.retrieval)))
    z = K.astype(np.float64) @ q.astype(np.float64) * 0.09
    w = np.exp(z - z.max())
    np.testing.assert_allclose(out, (w / w.sum()) @ V.astype(np.float64), rtol=1e-10, atol=1e-12)


# ----------------------------------------------------------------------------- prior-derived levels
def _gaussian_ratios(n, seed):
    """r = |g_j| / max_i |g_i| over n i.i.d. Gaussian 8-vectors (all 8 coordinates)."""
    g = np.abs(np.random.default_rng(seed).standard_normal((n, M)))
    return (g / g.max(axis=1, keepdims=True)).ravel()


def test_ratio_law_matches_rotated_directions():
    """The density of r = |y_j| / max|y| (plus its mass 1/m at 1) integrates to one and its
    CDF matches r measured on rotated random keys (the oracle's own rotation of
    non-Gaussian keys, so the test also checks that the rotation makes subspace directions
    uniform)."""
    x = (np.arange(8192) + 0.5) / 8192
    f = oracle.ratio_density(x)
    assert abs(f.sum() / 8192 + 1 / M - 1.0) < 1e-6
    rng = np.random.default_rng(21)
    keys = rng.uniform(-1, 1, (20000, D)).astype(np.float32) ** 3      # far from Gaussian
    y, _ = oracle.normalize_rotate(keys, _signs(D, 4))
    a = np.abs(y.reshape(-1, M)).astype(np.float64)
    r = np.sort((a / a.max(axis=1, keepdims=True)).ravel())
    cdf_model = np.cumsum(f) / 8192                                     # P(r <= x), x < 1
    cdf_emp = np.searchsorted(r, x, side="right") / r.size
    assert np.max(np.abs(cdf_model - cdf_emp)) < 4e-3


def test_ratio_levels_are_lloyd_max():
    """Each level is the conditional mean of r over its nearest-level cell (independent
    quadrature by scipy on the same law), and the table equals a Lloyd-Max fit to sampled
    Gaussian ratios."""
    from scipy.integrate import quad
    lv = oracle.ratio_levels().astype(np.float64)
    assert np.all(np.diff(lv) > 0) and 0 < lv[0] and lv[-1] < 1
    th = np.concatenate([[0.0], 0.5 * (lv[:-1] + lv[1:]), [1.0]])
    for i in range(8):
        f = lambda x: float(oracle.ratio_density(np.array([x]))[0])
        m0 = quad(f, th[i], th[i + 1], limit=200)[0]
        m1 = quad(lambda x: x * f(x), th[i], th[i + 1], limit=200)[0]
        if i == 7:
            m0, m1 = m0 + 1 / M, m1 + 1 / M
        assert abs(m1 / m0 - lv[i]) < 2e-5, (i, m1 / m0, lv[i])
    r = _gaussian_ratios(400000, 3)
    emp = (np.arange(8) + 0.5) / 8
    for _ in range(300):
        c = np.searchsorted(0.5 * (emp[:-1] + emp[1:]), r, side="right")
        emp = np.bincount(c, r, 8) / np.bincount(c, None, 8)
    np.testing.assert_allclose(lv, emp, atol=3e-3)


def test_ratio_law_closed_forms_for_two_and_three_dims():
    """For m = 2, r = |g_j| / max|g| is 1 with probability 1/2 and otherwise the ratio of
    two half-normals, whose density on [0, 1) is 2 / (pi (1 + x^2)) (the half-Cauchy law
    of |g_1 / g_2|). For m = 3 the t-integral has the closed form
    integral_0^inf t exp(-a t^2) erf(b t) dt = b / (2 a sqrt(a + b^2)), which gives
    f(x) = 4 / (pi (1 + x^2) sqrt(2 + x^2)), of mass 2/3 on [0, 1). Both pin the density
    formula (the factor m - 1, the two half-normal densities and the Psi^(m - 2) term)
    without the oracle's own quadrature."""
    x = (np.arange(2000) + 0.5) / 2000
    np.testing.assert_allclose(oracle.ratio_density(x, m=2), 2 / (np.pi * (1 + x * x)),
                               atol=5e-7)
    np.testing.assert_allclose(oracle.ratio_density(x, m=3),
                               4 / (np.pi * (1 + x * x) * np.sqrt(2 + x * x)), atol=1e-9)
    assert abs(4 / np.pi * np.arctan(1 / np.sqrt(3)) - 2 / 3) < 1e-15   # the m = 3 mass


def test_ratio_levels_two_dims_by_closed_form_lloyd():
    """The level recipe (cell masses and moments from cumulative integrals, interpolated at
    the thresholds; the point mass at 1 in the top cell; Lloyd to convergence) against the
    same fixed point computed from the m = 2 law's closed-form integrals
    F0(x) = (2 / pi) atan x and F1(x) = ln(1 + x^2) / pi."""
    lv = oracle.ratio_levels(m=2).astype(np.float64)
    F0 = lambda t: 2 / np.pi * np.arctan(t)
    F1 = lambda t: np.log1p(t * t) / np.pi
    ref = (np.arange(8) + 0.5) / 8
    for _ in range(5000):
        e = np.concatenate([[0.0], 0.5 * (ref[:-1] + ref[1:]), [1.0]])
        s0, s1 = np.diff(F0(e)), np.diff(F1(e))
        s0[7] += 0.5
        s1[7] += 0.5
        ref = s1 / s0
    np.testing.assert_allclose(lv, ref, atol=1e-6)


def test_table_codes_nearest_level():
    """Table-coded magnitudes are the nearest table level to r = |y_j| / max|y| (fp32 ratio,
    fp32 midpoint thresholds), the signs are the coordinate signs, and the maximal coordinate
    takes the top level."""
    lv = oracle.ratio_levels()
    rng = np.random.default_rng(22)
    y = rng.standard_normal((3000, D)).astype(np.float32)
    enc = oracle.encode_rotated(y, np.ones(3000, np.float32), M, table=lv)
    a = np.abs(y.reshape(3000, B, M))
    r = a / a.max(axis=2, keepdims=True)                       # fp32 IEEE division
    th = (0.5 * (lv[:-1].astype(np.float64) + lv[1:].astype(np.float64))).astype(np.float32)
    want = (r[..., None] >= th).sum(axis=-1)
    np.testing.assert_array_equal(enc.mag.reshape(3000, B, M), want)
    dist = np.abs(r[..., None].astype(np.float64) - lv.astype(np.float64))
    np.testing.assert_array_equal(want, np.argmin(dist, axis=-1))   # nearest level
    assert np.all(enc.mag.reshape(3000, B, M).max(axis=2) == 7)
    np.testing.assert_array_equal(enc.neg, (y < 0).astype(np.uint8))


def test_table_estimator_equals_literal_page_form_and_self_estimate():
    """With table levels the folded factor still equals the literal w_{i,b} <v_b, q~_b>
    (1e-5), and the estimate of <k, k> is ||k||^2 (2e-6)."""
    lv = oracle.ratio_levels()
    rng = np.random.default_rng(23)
    sg = _signs(D, 13)
    k = (rng.standard_normal((400, D)) * 2 + 0.5).astype(np.float32)
    q = rng.standard_normal((1, D)).astype(np.float32)
    y, kn = oracle.normalize_rotate(k, sg)
    qt, qn = oracle.normalize_rotate(q, sg)
    enc = oracle.encode_rotated(y, kn, M, table=lv)
    lit = _literal_terms(enc, y, kn, qt[0])
    cand = np.arange(400, dtype=np.int32)
    S = oracle.rerank(enc, cand, qt[0], M).astype(np.float64)
    assert np.max(np.abs(float(qn[0]) * S - float(qn[0]) * lit.sum(axis=1)) /
                  (kn * qn[0])) <= 1e-5
    for i in range(0, 400, 40):
        S_ii = oracle.rerank(enc, np.array([i], np.int32), y[i], M)[0]
        k2 = float(kn[i]) ** 2
        assert abs(float(kn[i]) * float(S_ii) - k2) <= 2e-6 * k2


def test_ratio_levels_quantise_directions_better_than_uniform():
    """Over rotated random keys the table levels lose less of each subspace direction
    (mean 1 - cos(y_b, v_b)) than the uniform levels: the point of deriving them from the
    prior."""
    lv = oracle.ratio_levels()
    rng = np.random.default_rng(24)
    y, kn = oracle.normalize_rotate(rng.standard_normal((20000, D)).astype(np.float32),
                                    _signs(D, 5))
    yb = y.reshape(-1, B, M).astype(np.float64)

    def loss(enc):
        v = enc.vt.reshape(-1, B, M)
        cos = np.sum(v * yb, axis=2) / (np.linalg.norm(v, axis=2) * np.linalg.norm(yb, axis=2))
        return float(np.mean(1 - cos))
    uni, tab = loss(oracle.encode_rotated(y, kn, M)), loss(oracle.encode_rotated(y, kn, M, table=lv))
    assert tab < 0.85 * uni, (tab, uni)


# ----------------------------------------------------------------------------- learned centroids
def test_learned_path_with_sign_centroids_is_the_analytic_path():
    """With the 256 sign patterns / sqrt(m) as 'learned' centroids the comparator's ids, vote
    tables and whole search equal the analytic ones (zero coordinates included: both break
    ties toward the lower id)."""
    rng = np.random.default_rng(31)
    y = rng.standard_normal((3000, D)).astype(np.float32)
    y[:50, ::5] = 0.0
    sc = oracle.sign_centroids(M)
    enc = oracle.encode_rotated(y, np.ones(3000, np.float32), M)
    np.testing.assert_array_equal(oracle.learned_ids(y, sc, M), enc.ids)
    for s in range(5):
        qt = rng.standard_normal(D).astype(np.float32)
        for rho in (1, 4, 16):
            np.testing.assert_array_equal(oracle.learned_lut(qt, sc, M, rho),
                                          oracle.query_lut(qt, M, rho))
    qt = rng.standard_normal(D).astype(np.float32)
    a = oracle.search_rotated(enc, qt, 1.0, 64, oracle.SearchParams(m=M))
    b = oracle.search_rotated(enc, qt, 1.0, 64, oracle.SearchParams(m=M, centroids=sc))
    for x, z in zip(a, b):
        np.testing.assert_array_equal(x, z)


def test_learned_ids_and_lut_brute_force():
    """argmax / top-rho of fp64 inner products with arbitrary centroids (entries within 1e-6
    of a tie excluded)."""
    rng = np.random.default_rng(32)
    cent = rng.standard_normal((B, 256, M)).astype(np.float32)
    y = rng.standard_normal((500, D)).astype(np.float32)
    ids = oracle.learned_ids(y, cent, M)
    dots = np.einsum("nbj,bcj->nbc", y.reshape(500, B, M).astype(np.float64),
                     cent.astype(np.float64))
    srt = np.sort(dots, axis=2)
    clear = srt[..., -1] - srt[..., -2] > 1e-6
    assert clear.mean() > 0.99
    np.testing.assert_array_equal(ids[clear], dots.argmax(axis=2)[clear])
    qt = rng.standard_normal(D).astype(np.float32)
    lut = oracle.learned_lut(qt, cent, M, rho=4, w_rank1=2, w_rest=1)
    qd = np.einsum("bj,bcj->bc", qt.reshape(B, M).astype(np.float64), cent.astype(np.float64))
    for b in range(B):
        top = np.argsort(-qd[b], kind="stable")[:4]
        want = np.zeros(256, np.uint8)
        want[top[0]] = 2
        want[top[1:]] = 1
        np.testing.assert_array_equal(lut[b], want)


def test_train_centroids_recovers_directions_and_improves_fit():
    """Keys drawn as 4 copies each of 256 distinct directions per subspace (key i on
    direction i // 4) are recovered exactly: the start picks one key of each direction and
    every key then joins its own; on Gaussian keys the mean cosine to the assigned centroid
    never decreases over iterations, and centroids stay unit vectors."""
    rng = np.random.default_rng(33)
    dirs = rng.standard_normal((B, 256, M))
    dirs /= np.linalg.norm(dirs, axis=2, keepdims=True)
    scale = rng.uniform(0.5, 2.0, (1024, B, 1))
    y = (dirs[:, np.arange(1024) // 4].transpose(1, 0, 2) * scale).reshape(1024, D)
    cent = oracle.train_centroids(y.astype(np.float32), 3, M)
    np.testing.assert_allclose(cent, dirs.astype(np.float32), atol=1e-6)
    g = rng.standard_normal((4000, D)).astype(np.float32)
    u = g.reshape(4000, B, M) / np.linalg.norm(g.reshape(4000, B, M), axis=2, keepdims=True)
    prev = -1.0
    for it in range(0, 6):
        c = oracle.train_centroids(g, it, M)
        ids = oracle.learned_ids(g, c, M)
        fit = float(np.mean(np.take_along_axis(
            np.einsum("nbj,bcj->nbc", u, c.astype(np.float64)), ids[..., None].astype(np.int64),
            axis=2)))
        assert fit >= prev - 1e-12, (it, fit, prev)
        prev = fit
        np.testing.assert_allclose(np.linalg.norm(c, axis=2), 1.0, atol=1e-6)


def test_table_levels_i_over_7_reproduce_uniform_codes():
    """The table path with levels c_i = i / 7 is the uniform rule written another way: the
    midpoints (2i - 1) / 14 give mag = floor(7 r + 1/2), so the codes agree (barring ratios
    that land exactly on a midpoint), and since vt_table = vt_uniform / 7 the factor fold
    absorbs the scale: S agrees to fp32 rounding. Two independent code paths in the oracle
    checked against each other."""
    rng = np.random.default_rng(34)
    sg = _signs(D, 17)
    k = (rng.standard_normal((2000, D)) * 2 + 0.3).astype(np.float32)
    y, kn = oracle.normalize_rotate(k, sg)
    uni = oracle.encode_rotated(y, kn, M)
    tab = oracle.encode_rotated(y, kn, M, table=(np.arange(8) / 7).astype(np.float32))
    a = np.abs(y.reshape(-1, B, M))
    r = (a / a.max(axis=2, keepdims=True)).ravel()
    on_mid = np.any(np.abs(r[:, None] * 14 - (2 * np.arange(1, 8) - 1)) < 1e-5, axis=1)
    assert on_mid.mean() < 1e-3
    same = ~on_mid.reshape(-1, B * M)
    np.testing.assert_array_equal(uni.mag[same], tab.mag[same])
    np.testing.assert_array_equal(uni.ids, tab.ids)
    qt, _ = oracle.normalize_rotate(rng.standard_normal((1, D)).astype(np.float32), sg)
    rows = np.where(same.all(axis=1))[0].astype(np.int32)
    Su = oracle.rerank(uni, rows, qt[0], M).astype(np.float64)
    St = oracle.rerank(tab, rows, qt[0], M).astype(np.float64)
    np.testing.assert_allclose(St, Su, rtol=2e-5, atol=2e-6 * np.abs(Su).max())


def test_golden_basis_key():
    """A hand-derived worked example (tests/golden/basis_key_e5.json, derivation and citation
    inside): key 3 e_5 and query e_5 with all SRHT signs +1 -- ids, codes, factor, the
    rho = 4 vote table and the estimate."""
    import json
    import os
    fx = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "basis_key_e5.json")))
    k = np.zeros((1, D), np.float32)
    k[0, fx["basis_index"]] = fx["key_scale"]
    q = np.zeros((1, D), np.float32)
    q[0, fx["basis_index"]] = 1.0
    s = np.ones(D, np.int8)
    y, kn = oracle.normalize_rotate(k, s)
    enc = oracle.encode_rotated(y, kn, M)
    np.testing.assert_array_equal(enc.ids[0], fx["ids"])
    np.testing.assert_array_equal(enc.mag[0], fx["magnitude"])
    neg = np.zeros(M, np.uint8)
    neg[fx["negative_dims_in_subspace"]] = 1
    np.testing.assert_array_equal(enc.neg[0], np.tile(neg, B))
    np.testing.assert_allclose(enc.factor[0], fx["factor"], rtol=1e-6)
    qt, qn = oracle.normalize_rotate(q, s)
    lut = oracle.query_lut(qt[0], M, 4)
    want = np.zeros(256, np.uint8)
    for c, wgt in fx["lut_rho4"].items():
        want[int(c)] = wgt
    for b in range(B):
        np.testing.assert_array_equal(lut[b], want)
    S = oracle.rerank(enc, np.array([0], np.int32), qt[0], M)[0]
    assert abs(float(qn[0]) * float(S) - fx["estimate"]) <= 1e-5


def test_attend_saturated_logits_pick_the_best_row():
    """Logits hundreds apart (scale 50 on unit-scale rows): the softmax is one-hot to fp64
    precision, so the output is the value row of the largest logit, with no overflow."""
    rng = np.random.default_rng(35)
    K = rng.standard_normal((300, D)).astype(np.float32)
    V = rng.standard_normal((300, D)).astype(np.float32)
    q = K[123] * 4.0
    idx = np.arange(0, 300, 3, dtype=np.int32)          # row 123 is among them
    out = oracle.attend(q, K, V, idx, 50.0)
    np.testing.assert_allclose(out, V[123].astype(np.float64), atol=1e-12)
