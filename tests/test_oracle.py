"""Pins for the CPU oracle, checked against things other than the oracle itself:
closed forms, a hand-worked example, other library routines, Monte-Carlo
moments, brute force on tiny inputs and exact identities from the pages.
CPU only (no GPU marker)."""

import itertools
import json
import math
import os
import statistics

import numpy as np
import pytest
import torch

import oracle as O


RNG = np.random.default_rng(1234)


def _x(shape, rng=RNG, scale=1.0):
    return rng.standard_normal(shape) * scale


# ---------------------------------------------------------------- block stats

def test_block_stats_arithmetic_sequence_closed_form():
    # rows x_r = a + r*delta: mean a + delta (n-1)/2, population variance delta^2 (n^2-1)/12
    b, N, d = 8, 21, 3            # blocks of 8, 8, 5 rows (ragged tail)
    a = np.array([0.5, -2.0, 7.0])
    delta = np.array([1.0, 0.25, -3.0])
    X = np.zeros((1, 1, 24, d))
    for i in range(3):
        for r in range(8):
            X[0, 0, i * b + r] = a + r * delta
    X[0, 0, N:] = 1e30                       # padding must never be read
    mean, var, counts = O.block_stats(X, N, b)
    assert counts.tolist() == [8, 8, 5]
    for i, n in enumerate([8, 8, 5]):
        np.testing.assert_allclose(mean[0, 0, i], a + delta * (n - 1) / 2, rtol=1e-14)
        np.testing.assert_allclose(var[0, 0, i], delta ** 2 * (n * n - 1) / 12, rtol=1e-12)


def test_block_stats_vs_statistics_module():
    X = _x((2, 3, 40, 4))
    mean, var, _ = O.block_stats(X, 37, 16)
    for bb, h, i, m in itertools.product(range(2), range(3), range(3), range(4)):
        col = X[bb, h, i * 16: min(37, (i + 1) * 16), m].tolist()
        assert math.isclose(mean[bb, h, i, m], statistics.fmean(col), rel_tol=1e-12, abs_tol=1e-14)
        assert math.isclose(var[bb, h, i, m], statistics.pvariance(col), rel_tol=1e-10, abs_tol=1e-14)


def test_block_stats_shift_invariance_and_nonnegative():
    X = _x((1, 2, 64, 8))
    c = _x((8,)) * 100
    m1, v1, _ = O.block_stats(X, 64, 16)
    m2, v2, _ = O.block_stats(X + c, 64, 16)
    np.testing.assert_allclose(m2, m1 + c, rtol=1e-12, atol=1e-10)
    np.testing.assert_allclose(v2, v1, rtol=1e-8, atol=1e-9)
    assert (v1 >= 0).all()


# ------------------------------------------------------------ hand-worked case

def _golden():
    here = os.path.join(os.path.dirname(__file__), "golden", "hand_worked_tiny.json")
    with open(here) as f:
        return json.load(f)


def test_hand_worked_stats_scores_selection():
    g = _golden()
    Q = np.array(g["Q"], dtype=float)[None, None]
    K = np.array(g["K"], dtype=float)[None, None]
    qm, qv, qc = O.block_stats(Q, 4, g["block"])
    km, kv, kc = O.block_stats(K, 4, g["block"])
    np.testing.assert_array_equal(qm[0, 0], g["q_mean"])
    np.testing.assert_array_equal(qv[0, 0], g["q_var"])
    np.testing.assert_array_equal(km[0, 0], g["k_mean"])
    np.testing.assert_array_equal(kv[0, 0], g["k_var"])
    S = O.corrected_scores(qm, qv, km, kv, kc, g["sm_scale"])
    P = O.pooled_scores(qm, km, kc, g["sm_scale"])
    np.testing.assert_allclose(S[0, 0] - math.log(2), g["scores_minus_ln2"], atol=1e-14)
    np.testing.assert_allclose(P[0, 0] - math.log(2), g["pooled_minus_ln2"], atol=1e-14)
    k = O.keep_count(g["keep"], 2)
    idx, cnt = O.select_topk(S, k)
    assert idx[0, 0].tolist() == g["kept_corrected"]
    idx, cnt = O.select_topk(P, k)
    assert idx[0, 0].tolist() == g["kept_pooled"]


def test_hand_worked_merge():
    m = _golden()["merge"]
    Om, Lm = O.merge_lse(np.array(m["O1"]), np.array(m["L1"]), np.array(m["O2"]),
                         np.array(math.log(m["L2_is_ln"])))
    np.testing.assert_allclose(Om, m["O"], atol=1e-15)
    assert math.isclose(float(Lm), math.log(m["L_is_ln"]), rel_tol=1e-15)


# ------------------------------------------------------------ corrected score

def _rand_stats(nq=5, nk=7, d=6, Hq=4, Hkv=2, rng=RNG):
    qm = rng.standard_normal((1, Hq, nq, d))
    qv = rng.uniform(0.1, 2.0, (1, Hq, nq, d))
    km = rng.standard_normal((1, Hkv, nk, d))
    kv = rng.uniform(0.1, 2.0, (1, Hkv, nk, d))
    counts = rng.integers(1, 64, nk)
    return qm, qv, km, kv, counts


def test_zero_variance_reduces_to_pooled():
    # check (3): with zero within-block variance the correction vanishes
    qm, _, km, _, counts = _rand_stats()
    S = O.corrected_scores(qm, np.zeros_like(qm), km, np.zeros_like(km), counts, 0.37)
    P = O.pooled_scores(qm, km, counts, 0.37)
    np.testing.assert_array_equal(S, P)


def test_jensen_correction_is_nonnegative():
    qm, qv, km, kv, counts = _rand_stats()
    S = O.corrected_scores(qm, qv, km, kv, counts, 0.37)
    P = O.pooled_scores(qm, km, counts, 0.37)
    assert (S >= P).all()
    assert (S > P).mean() > 0.99


def test_identical_token_blocks_pre_equals_post():
    # every token in a block equal to its block mean: the pre-downsample map
    # equals the exact post-downsample map (closed form of both)
    rng = np.random.default_rng(7)
    b, nb, d = 4, 6, 8
    N = b * nb - 2                               # ragged last block of 2
    qb = rng.standard_normal((1, 2, nb, d))
    kb = rng.standard_normal((1, 1, nb, d)) * 1.5
    Q = np.repeat(qb, b, axis=2)
    K = np.repeat(kb, b, axis=2)
    s = d ** -0.5
    qm, qv, qc = O.block_stats(Q, N, b)
    km, kv, kc = O.block_stats(K, N, b)
    assert np.abs(qv).max() < 1e-24 and np.abs(kv).max() < 1e-24
    A_pre = O.pre_downsample_map(O.corrected_scores(qm, qv, km, kv, kc, s))
    A_post = O.post_downsample_map(Q, K, N, b, s)
    np.testing.assert_allclose(A_pre, A_post, rtol=1e-12, atol=1e-15)


def test_mc_variance_of_block_logit():
    # Var[s q.k] for independent diagonal Gaussians equals s^2 V_ij; each of the
    # three terms of V carries about a third of the total here, so dropping one
    # or mis-scaling s fails by far more than the Monte-Carlo error.
    rng = np.random.default_rng(11)
    d, n = 6, 1 << 19
    s = 0.4
    qbar = rng.uniform(0.8, 1.2, d) * rng.choice([-1, 1], d)
    kbar = rng.uniform(0.8, 1.2, d) * rng.choice([-1, 1], d)
    vq = rng.uniform(0.8, 1.2, d)
    vk = rng.uniform(0.8, 1.2, d)
    q = qbar + rng.standard_normal((n, d)) * np.sqrt(vq)
    k = kbar + rng.standard_normal((n, d)) * np.sqrt(vk)
    x = s * np.einsum("nd,nd->n", q, k)
    S = O.corrected_scores(qbar[None, None, None], vq[None, None, None],
                           kbar[None, None, None], vk[None, None, None], [1], s)[0, 0, 0, 0]
    mean_term = s * qbar @ kbar
    var_oracle = 2.0 * (S - mean_term)                 # ln m = 0
    var_mc = x.var()
    se = var_mc * math.sqrt(2.0 / n) * 3                # generous for the product's kurtosis
    assert abs(var_mc - var_oracle) < 5 * se, (var_mc, var_oracle, se)
    assert abs(x.mean() - mean_term) < 5 * math.sqrt(var_mc / n)


def test_mc_mgf_single_query_row():
    # one query row (zero query variance), m keys from N(kbar, diag vk): the
    # log-mean-exp of the logits converges to s q.kbar + (s^2/2) sum q^2 vk,
    # which is S~ - ln m. Pins the factor 1/2 and the s^2.
    rng = np.random.default_rng(5)
    d, m = 8, 1 << 18
    s = d ** -0.5
    q = rng.uniform(0.5, 1.0, d) * rng.choice([-1, 1], d)
    kbar = rng.standard_normal(d) * 0.5
    vk = rng.uniform(0.5, 1.5, d)
    k = kbar + rng.standard_normal((m, d)) * np.sqrt(vk)
    x = s * (k @ q)
    lme = np.log(np.mean(np.exp(x - x.max()))) + x.max()
    S = O.corrected_scores(q[None, None, None], np.zeros((1, 1, 1, d)), kbar[None, None, None],
                           vk[None, None, None], [m], s)[0, 0, 0, 0]
    target = S - math.log(m)
    var_x = float(s * s * (q * q) @ vk)
    se = math.sqrt((math.exp(var_x) - 1) / m)          # relative s.e. of a lognormal mean
    assert 0.2 < var_x < 1.5
    assert abs(lme - target) < 6 * se, (lme, target, se)


# ------------------------------------------------------------------ selection

def test_keep_count_values():
    assert O.keep_count(0.5, 16) == 8
    assert O.keep_count(0.5, 128) == 64
    assert [O.keep_count(k, 256) for k in (1.0, 0.5, 0.25)] == [256, 128, 64]
    assert O.keep_count(0.5, 1024) == 512
    assert O.keep_count(1e-6, 16) == 1
    assert O.keep_count(1.0 / 3.0, 3) == 1
    with pytest.raises(ValueError):
        O.keep_count(0.0, 4)


def test_topk_bruteforce_max_sum_subset():
    # with distinct scores, the kept set is the size-k subset of maximum total score
    rng = np.random.default_rng(3)
    for _ in range(20):
        nk = 8
        k = int(rng.integers(1, nk + 1))
        row = rng.standard_normal(nk)
        best = max(itertools.combinations(range(nk), k), key=lambda c: sum(row[j] for j in c))
        idx, cnt = O.select_topk(row[None], k)
        assert cnt[0] == k
        assert idx[0].tolist() == sorted(best)


def test_topk_ties_prefer_lower_index_and_ascending():
    row = np.array([[1.0, 2.0, 2.0, 2.0, 0.0, 2.0]])
    idx, _ = O.select_topk(row, 2, kmax=4)
    assert idx[0].tolist() == [1, 2, -1, -1]
    idx, _ = O.select_topk(row, 5)
    assert idx[0].tolist() == [0, 1, 2, 3, 5]


def test_topk_permutation_equivariance_and_keep_all():
    rng = np.random.default_rng(4)
    S = rng.standard_normal((3, 12))
    perm = rng.permutation(12)
    idx, _ = O.select_topk(S, 5)
    idx_p, _ = O.select_topk(S[:, perm], 5)
    for r in range(3):
        assert sorted(perm[idx_p[r]].tolist()) == idx[r].tolist()
    idx, cnt = O.select_topk(S, 12)
    assert (idx == np.arange(12)).all() and (cnt == 12).all()


def test_near_tie_band():
    row = np.array([[0.0, 1.0, 1.0005, 2.0, 1.0 + 2e-3]])
    # k=3: ranking 3 (2.0), 4 (1.002), 2 (1.0005) -> threshold 1.0005
    nt = O.near_tie_mask(row, 3)
    assert nt[0].tolist() == [False, True, True, False, False]
    # the band is the narrower of the score-relative and the map-relative one:
    # near a small threshold the score band decides (0.1005 is 5e-4 above 0.1,
    # inside the map band but outside 1e-3 * 0.1) ...
    row = np.array([[3.0, 0.1, 0.1005, 0.10005, -1.0]])      # k = 4: threshold 0.1
    assert O.near_tie_mask(row, 4)[0].tolist() == [False, True, False, True, False]
    # ... and near a large one the map band does (100.05 is within 1e-3 * 100
    # of 100 but exp(0.05) - 1 = 0.051 on the map)
    row = np.array([[200.0, 100.0, 100.05, 100.0004, 0.0]])   # k = 4: threshold 100
    assert O.near_tie_mask(row, 4)[0].tolist() == [False, True, False, True, False]


# ------------------------------------------------------------------ attention

def _qkv(B=1, Hq=4, Hkv=2, N=200, Na=208, d=16, rng=RNG):
    Q = rng.standard_normal((B, Hq, Na, d))
    K = rng.standard_normal((B, Hkv, Na, d))
    V = rng.standard_normal((B, Hkv, Na, d))
    Q[:, :, N:] = K[:, :, N:] = V[:, :, N:] = 1e30        # padding must never be read
    return Q, K, V


def test_dense_matches_torch_sdpa():
    Q, K, V = _qkv()
    N, s = 200, 16 ** -0.5
    Od, Ld = O.dense_attention(Q, K, V, N, s)
    q = torch.from_numpy(Q[:, :, :N])
    k = torch.from_numpy(np.repeat(K[:, :, :N], 2, axis=1))
    v = torch.from_numpy(np.repeat(V[:, :, :N], 2, axis=1))
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=s).numpy()
    np.testing.assert_allclose(Od, ref, rtol=1e-10, atol=1e-12)
    lse = torch.logsumexp(s * q @ k.transpose(-1, -2), dim=-1).numpy()
    np.testing.assert_allclose(Ld, lse, rtol=1e-12, atol=1e-12)


def test_dense_closed_forms():
    # identical keys: uniform weights, output = mean of values, LSE = s q.k + ln N
    rng = np.random.default_rng(9)
    N, d, s = 50, 8, 0.3
    Q = rng.standard_normal((1, 1, N, d))
    K = np.repeat(rng.standard_normal((1, 1, 1, d)), N, axis=2)
    V = rng.standard_normal((1, 1, N, d))
    Od, Ld = O.dense_attention(Q, K, V, N, s)
    np.testing.assert_allclose(Od[0, 0], np.repeat(V[0, 0].mean(0, keepdims=True), N, 0), atol=1e-13)
    np.testing.assert_allclose(Ld[0, 0], s * Q[0, 0] @ K[0, 0, 0] + math.log(N), atol=1e-12)


def test_masked_keep_all_equals_dense():
    # check (1): keeping every block is dense attention (ragged last block)
    Q, K, V = _qkv()
    N, b, s = 200, 32, 16 ** -0.5
    nb = O.num_blocks(N, b)
    idx = np.tile(np.arange(nb, dtype=np.int32), (1, 4, nb, 1))
    cnt = np.full((1, 4, nb), nb, dtype=np.int32)
    Om, Lm = O.masked_attention(Q, K, V, idx, cnt, N, b, s)
    Od, Ld = O.dense_attention(Q, K, V, N, s)
    np.testing.assert_allclose(Om[:, :, :N], Od, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(Lm[:, :, :N], Ld, rtol=1e-12, atol=1e-12)
    assert np.isnan(Om[:, :, N:]).all()                  # padding rows untouched


def test_merge_of_disjoint_spans_equals_union():
    # check (2): merging (O, L) over X and over Y equals attention over X u Y
    Q, K, V = _qkv()
    N, b, s = 200, 32, 16 ** -0.5
    nb = O.num_blocks(N, b)
    rng = np.random.default_rng(2)
    S = rng.standard_normal((1, 4, nb, nb))
    idx, cnt = O.select_topk(S, 4, kmax=nb)
    for split in (1, 3, nb - 1, nb):
        lo_i, lo_c, hi_i, hi_c = O.split_lists(idx, cnt, split)
        assert ((lo_c + hi_c) == cnt).all()
        O1, L1 = O.masked_attention(Q, K, V, lo_i, lo_c, N, b, s)
        O2, L2 = O.masked_attention(Q, K, V, hi_i, hi_c, N, b, s)
        Ou, Lu = O.masked_attention(Q, K, V, idx, cnt, N, b, s)
        Om, Lm = O.merge_lse(O1[:, :, :N], L1[:, :, :N], O2[:, :, :N], L2[:, :, :N])
        np.testing.assert_allclose(Om, Ou[:, :, :N], rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(Lm, Lu[:, :, :N], rtol=1e-12, atol=1e-12)


def test_block_rows_attention_cached_external_plus_internal_is_dense():
    # FlashBlock's block-external caching: the current block's rows attend the
    # prefix (cached as one partial) and the block itself (recomputed); the
    # merge equals textbook dense attention of those rows over every key
    rng = np.random.default_rng(21)
    B, Hq, Hkv, d, b, s = 1, 4, 2, 16, 16, 16 ** -0.5
    for r0, R, bk in ((64, 37, 16), (32, 48, 32), (0, 20, 16), (96, 16, 16)):
        N = r0 + R                                      # tokens so far: prefix + current block
        Q = rng.standard_normal((B, Hq, N + 5, d))
        K = rng.standard_normal((B, Hkv, N + 5, d))
        V = rng.standard_normal((B, Hkv, N + 5, d))
        rows = np.arange(r0, N)
        Qr = np.zeros((B, Hq, R + 3, d))                # compact range buffer with a few spare rows
        Qr[:, :, :R] = Q[:, :, rows]
        if r0 > 0:
            Oe, Le = O.dense_attention(Q, K, V, r0, s, rows=rows)          # external: keys [0, r0)
        else:
            Oe, Le = np.zeros((B, Hq, R, d)), np.full((B, Hq, R), -np.inf)
        Oc = np.zeros((B, Hq, R + 3, d))
        Lc = np.zeros((B, Hq, R + 3))
        Oc[:, :, :R], Lc[:, :, :R] = Oe, Le
        # internal: the key blocks of [r0, N) (r0 is a multiple of the key block size)
        internal = np.arange(r0 // bk, -(-N // bk), dtype=np.int32)
        nqr = O.num_blocks(R, b)
        idx = np.tile(internal, (B, Hq, nqr, 1))
        cnt = np.full((B, Hq, nqr), internal.size, dtype=np.int32)
        Og, Lg = O.block_rows_attention(Qr, K, V, idx, cnt, R, N, b, s, O_prev=Oc, L_prev=Lc, b_k=bk)
        Od, Ld = O.dense_attention(Q, K, V, N, s, rows=rows)
        np.testing.assert_allclose(Og[:, :, :R], Od, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(Lg[:, :, :R], Ld, rtol=1e-12, atol=1e-12)
        assert np.isnan(Og[:, :, R:]).all() and np.isnan(Lg[:, :, R:]).all()


def test_block_rows_attention_without_cache_is_masked_attention_on_those_rows():
    Q, K, V = _qkv()
    N, b, s = 200, 32, 16 ** -0.5
    nb = O.num_blocks(N, b)
    S = np.random.default_rng(8).standard_normal((1, 4, nb, nb))
    idx, cnt = O.select_topk(S, 3, kmax=5)
    cnt[0, 1, 2] = 0                                    # an empty list: O = 0, LSE = -inf
    Om, Lm = O.masked_attention(Q, K, V, idx, cnt, N, b, s)
    i0, R = 2, 200 - 64                                 # query blocks 2.. of the sequence, ragged at N
    rows = slice(i0 * b, i0 * b + R)
    Og, Lg = O.block_rows_attention(Q[:, :, rows], K, V, idx[:, :, i0:], cnt[:, :, i0:], R, N, b, s)
    np.testing.assert_array_equal(Og, Om[:, :, rows])
    np.testing.assert_array_equal(Lg, Lm[:, :, rows])
    assert (Og[0, 1, 0:32] == 0).all() and np.isneginf(Lg[0, 1, 0:32]).all()
    # an empty list with a cached partial passes the partial through
    Oc = np.random.default_rng(9).standard_normal(Og.shape)
    Lc = np.random.default_rng(10).standard_normal(Lg.shape)
    Ox, Lx = O.block_rows_attention(Q[:, :, rows], K, V, idx[:, :, i0:], cnt[:, :, i0:], R, N, b, s, Oc, Lc)
    np.testing.assert_allclose(Ox[0, 1, 0:32], Oc[0, 1, 0:32], rtol=1e-15)
    np.testing.assert_array_equal(Lx[0, 1, 0:32], Lc[0, 1, 0:32])


def test_complement_lists_partition_and_kept_plus_rest_is_dense():
    # the complement is the exact set difference (ascending, -1 padded), and
    # merging attention over the kept blocks with attention over the rest
    # gives dense attention (the "cached residual" identity)
    Q, K, V = _qkv()
    N, b, s = 200, 32, 16 ** -0.5
    nb = O.num_blocks(N, b)
    rng = np.random.default_rng(5)
    S = rng.standard_normal((1, 4, nb, nb))
    for k in (1, 3, nb):
        idx, cnt = O.select_topk(S, k, kmax=nb)
        cidx, ccnt = O.complement_lists(idx, cnt, nb)
        assert ((cnt + ccnt) == nb).all()
        for pos in np.ndindex(cnt.shape):
            kept = list(idx[pos][: cnt[pos]])
            rest = list(cidx[pos][: ccnt[pos]])
            assert sorted(kept + rest) == list(range(nb)) and rest == sorted(rest)
            assert (cidx[pos][ccnt[pos]:] == -1).all()
        O1, L1 = O.masked_attention(Q, K, V, idx, cnt, N, b, s)
        O2, L2 = O.masked_attention(Q, K, V, cidx, ccnt, N, b, s)
        Od, Ld = O.dense_attention(Q, K, V, N, s)
        Om, Lm = O.merge_lse(O1[:, :, :N], L1[:, :, :N], O2[:, :, :N], L2[:, :, :N])
        np.testing.assert_allclose(Om, Od, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(Lm, Ld, rtol=1e-12, atol=1e-12)
    # entries outside [0, nb) are ignored; a narrower stride truncates nothing that fits
    idx = np.array([[[[0, 7, -1, 99]]]], dtype=np.int32)
    cidx, ccnt = O.complement_lists(idx, np.array([[[4]]]), 8)
    assert ccnt[0, 0, 0] == 6 and list(cidx[0, 0, 0]) == [1, 2, 3, 4, 5, 6, -1, -1]


def test_selection_variants():
    rng = np.random.default_rng(11)
    B, Hq, Hkv, nb, d = 2, 4, 2, 9, 8
    qm, qv = rng.standard_normal((B, Hq, nb, d)), rng.random((B, Hq, nb, d))
    km, kv = rng.standard_normal((B, Hkv, nb, d)), rng.random((B, Hkv, nb, d))
    counts = np.full(nb, 16.0)
    s = 0.3
    full = O.corrected_scores(qm, qv, km, kv, counts, s)
    novar = O.corrected_scores(qm, qv, km, kv, counts, s, var_product=False)
    # the dropped term is (s^2/2) var_q . var_k, a plain matrix product per head
    G = Hq // Hkv
    for h in range(Hq):
        np.testing.assert_allclose(full[:, h] - novar[:, h],
                                   0.5 * s * s * np.einsum("bid,bjd->bij", qv[:, h], kv[:, h // G]), rtol=1e-12)
    assert (full >= novar - 1e-12).all()
    np.testing.assert_allclose(O.corrected_scores(qm, qv, km, 0 * kv, counts, s),
                               O.corrected_scores(qm, qv, km, 0 * kv, counts, s, var_product=False), rtol=0)
    k = 3
    # forced diagonal: block i always kept, plus the best k-1 of the others
    idx, cnt = O.select_topk(O.selection_scores(full, Hkv, force_diagonal=True), k)
    for pos in np.ndindex(cnt.shape):
        i = pos[-1]
        row = full[pos]
        others = sorted((j for j in range(nb) if j != i), key=lambda j: (-row[j], j))[: k - 1]
        assert sorted(idx[pos][:k]) == sorted(others + [i])
    # shared GQA selection: one list per KV group, the top k of the group mean
    idx, cnt = O.select_topk(O.selection_scores(full, Hkv, shared_gqa=True), k)
    for b in range(B):
        for g in range(Hkv):
            mean = full[b, g * G:(g + 1) * G].mean(axis=0)
            for i in range(nb):
                best = sorted(range(nb), key=lambda j: (-mean[i, j], j))[:k]
                for hh in range(G):
                    assert list(idx[b, g * G + hh, i, :k]) == sorted(best)


def test_select_by_mass():
    rng = np.random.default_rng(13)
    R = rng.standard_normal((2, 3, 5, 11)) * 2
    for tau in (1e-9, 0.3, 0.5, 0.9, 0.999, 1.0):
        idx, cnt = O.select_by_mass(R, tau)
        lo, hi = O.mass_share_before(R, idx, cnt)
        for pos in np.ndindex(cnt.shape):
            m = int(cnt[pos])
            row = R[pos]
            # brute force: the shortest prefix of the ranking whose softmax share reaches tau
            order = sorted(range(row.size), key=lambda j: (-row[j], j))
            p = np.exp(row - row.max()) / np.exp(row - row.max()).sum()
            shares = np.cumsum([p[j] for j in order])
            want = next((i + 1 for i, v in enumerate(shares) if v >= tau - 1e-15), row.size)
            assert m == max(1, want), (tau, pos, m, want)
            assert list(idx[pos][:m]) == sorted(order[:m]) and (idx[pos][m:] == -1).all()
            assert hi[pos] >= min(tau, 1.0) - 1e-12 and (m == 1 or lo[pos] < tau)
    # tau -> 0 keeps the single best block; tau = 1 keeps every block
    idx, cnt = O.select_by_mass(R, 1e-12)
    assert (cnt == 1).all() and (idx[..., 0] == R.argmax(-1)).all()
    assert (O.select_by_mass(R, 1.0)[1] == R.shape[-1]).all()


def test_select_by_mass_hand_worked_row():
    # scores ln 1, ln 4, ln 1, ln 2 (+ any constant): the normalised map is
    # exp(S) / sum = 1/8, 1/2, 1/8, 1/4, so the ranking is 1, 3, 0, 2 (the
    # two 1/8 shares tie and go to the lower index) with running shares
    # 1/2, 3/4, 7/8, 1
    for shift in (0.0, 7.3, -40.0):
        R = np.log(np.array([[[1.0, 4.0, 1.0, 2.0]]])) + shift
        for tau, want in ((0.4, [1]), (0.6, [1, 3]), (0.8, [0, 1, 3]), (0.95, [0, 1, 2, 3])):
            idx, cnt = O.select_by_mass(R, tau)
            assert int(cnt[0, 0]) == len(want), (shift, tau)
            assert idx[0, 0, : len(want)].tolist() == want and (idx[0, 0, len(want):] == -1).all()


def test_merge_edge_cases():
    o1 = np.array([[1.0, 2.0], [3.0, 4.0]])
    o2 = np.array([[5.0, 6.0], [7.0, 8.0]])
    ninf = -np.inf
    Om, Lm = O.merge_lse(o1, np.array([0.3, ninf]), o2, np.array([ninf, ninf]))
    np.testing.assert_array_equal(Om, [[1.0, 2.0], [0.0, 0.0]])
    assert Lm[0] == 0.3 and np.isneginf(Lm[1])
    # very different magnitudes stay finite
    Om, Lm = O.merge_lse(o1[:1], np.array([1000.0]), o2[:1], np.array([-1000.0]))
    np.testing.assert_allclose(Om, o1[:1], rtol=1e-15)


def test_empty_list_gives_zero_and_neginf():
    Q, K, V = _qkv(N=64, Na=64)
    idx = np.full((1, 4, 2, 2), -1, dtype=np.int32)
    cnt = np.zeros((1, 4, 2), dtype=np.int32)
    Om, Lm = O.masked_attention(Q, K, V, idx, cnt, 64, 32, 0.25)
    assert (Om == 0).all() and np.isneginf(Lm).all()


# ------------------------------------------------- post-downsample (check 4)

def test_post_downsample_two_routes_agree():
    # brute force over the full probability matrix vs per-block log-normalisers
    rng = np.random.default_rng(12)
    N, b, d = 90, 16, 8                       # 6 blocks, ragged last of 10
    Q = rng.standard_normal((1, 1, N, d))
    K = rng.standard_normal((1, 1, N, d))
    V = rng.standard_normal((1, 1, N, d))
    s = d ** -0.5
    nb = O.num_blocks(N, b)
    A = O.post_downsample_map(Q, K, N, b, s)
    np.testing.assert_allclose(A.sum(-1), 1.0, rtol=1e-13)
    _, L_full = O.dense_attention(Q, K, V, N, s)
    L_single = np.empty((nb, N))
    for j in range(nb):
        idx = np.full((1, 1, nb, 1), j, dtype=np.int32)
        cnt = np.ones((1, 1, nb), dtype=np.int32)
        _, L = O.masked_attention(Q, K, V, idx, cnt, N, b, s)
        L_single[j] = L[0, 0, :N]
    A2 = O.block_mass_via_lse(L_single, L_full[0, 0], O.block_counts(N, b))
    np.testing.assert_allclose(A2, A[0, 0], rtol=1e-11, atol=1e-14)


def test_correction_improves_rank_agreement_on_planted_blocks():
    # diagnostic, not a parity pin: on a planted case the corrected score tracks
    # the exact map at least as well as the plain pooled score.
    from block_sparse_attention_ba_b200.workloads import make_inputs
    Q, K, V, meta = make_inputs("tiny_fp32", N=512)
    w = meta["workload"]
    s = w.d ** -0.5
    qm, qv, _ = O.block_stats(Q, w.N, w.block)
    km, kv, kc = O.block_stats(K, w.N, w.block)
    S = O.corrected_scores(qm, qv, km, kv, kc, s)
    P = O.pooled_scores(qm, km, kc, s)
    A = O.post_downsample_map(Q, K, w.N, w.block, s)
    assert O.spearman_vs_post(S, A) >= O.spearman_vs_post(P, A) - 1e-9
    assert 0.0 <= O.topk_recall_vs_post(S, A, 4) <= 1.0


# ------------------------------------------------- asymmetric blocks (query block b, key block b_k)

def test_asymmetric_keep_all_equals_dense():
    # every key block kept is dense attention whatever the two block sizes
    Q, K, V = _qkv()
    N, s = 200, 16 ** -0.5
    for b, bk in ((32, 16), (16, 64), (64, 24)):
        nq, nk = O.num_blocks(N, b), O.num_blocks(N, bk)
        idx = np.tile(np.arange(nk, dtype=np.int32), (1, 4, nq, 1))
        cnt = np.full((1, 4, nq), nk, dtype=np.int32)
        Om, Lm = O.masked_attention(Q, K, V, idx, cnt, N, b, s, b_k=bk)
        Od, Ld = O.dense_attention(Q, K, V, N, s)
        np.testing.assert_allclose(Om[:, :, :N], Od, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(Lm[:, :, :N], Ld, rtol=1e-12, atol=1e-12)


def test_asymmetric_lists_equal_their_refinement():
    # a key block of 2c rows is the union of two blocks of c rows: lists over
    # b_k = 32 equal, row by row, lists over b_k = 16 naming both halves
    Q, K, V = _qkv()
    N, b, s = 200, 32, 16 ** -0.5                 # ragged last blocks: 200 = 6*32 + 8
    nq, nk = O.num_blocks(N, b), O.num_blocks(N, 32)
    rng = np.random.default_rng(7)
    idx = np.full((1, 4, nq, nk), -1, dtype=np.int32)
    cnt = np.zeros((1, 4, nq), dtype=np.int32)
    fine_idx = np.full((1, 4, nq, 2 * nk), -1, dtype=np.int32)
    fine_cnt = np.zeros((1, 4, nq), dtype=np.int32)
    for h in range(4):
        for i in range(nq):
            sel = np.sort(rng.choice(nk, size=int(rng.integers(1, nk + 1)), replace=False))
            idx[0, h, i, : len(sel)] = sel
            cnt[0, h, i] = len(sel)
            fine = [f for j in sel for f in (2 * j, 2 * j + 1) if f < O.num_blocks(N, 16)]
            fine_idx[0, h, i, : len(fine)] = fine
            fine_cnt[0, h, i] = len(fine)
    Oa, La = O.masked_attention(Q, K, V, idx, cnt, N, b, s, b_k=32)
    Of, Lf = O.masked_attention(Q, K, V, fine_idx, fine_cnt, N, b, s, b_k=16)
    np.testing.assert_allclose(Oa[:, :, :N], Of[:, :, :N], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(La[:, :, :N], Lf[:, :, :N], rtol=1e-13, atol=1e-13)


def test_asymmetric_post_downsample_map():
    # rows sum to 1; merging adjacent key columns gives the map at twice the key block
    rng = np.random.default_rng(13)
    N, d = 90, 8
    Q = rng.standard_normal((1, 2, N, d))
    K = rng.standard_normal((1, 1, N, d))
    s = d ** -0.5
    A16 = O.post_downsample_map(Q, K, N, 32, s, b_k=16)       # 3 query blocks x 6 key blocks
    A32 = O.post_downsample_map(Q, K, N, 32, s)
    assert A16.shape == (1, 2, 3, 6) and A32.shape == (1, 2, 3, 3)
    np.testing.assert_allclose(A16.sum(-1), 1.0, rtol=1e-13)
    np.testing.assert_allclose(A16[..., 0::2] + A16[..., 1::2], A32, rtol=1e-12, atol=1e-15)


# ------------------------------------------------- diagnostics: rank agreement and top-k recall

def test_spearman_vs_post_matches_library_and_closed_form():
    # tie-free rows: the mean of scipy's per-row Spearman rho, and the closed
    # form rho = 1 - 6 sum d^2 / (n (n^2 - 1)) on the ranks
    import scipy.stats
    rng = np.random.default_rng(11)
    S = rng.standard_normal((3, 4, 37))
    A = S + 0.7 * rng.standard_normal(S.shape)
    got = O.spearman_vs_post(S, A)
    rows_s, rows_a = S.reshape(-1, 37), A.reshape(-1, 37)
    lib = np.mean([scipy.stats.spearmanr(a, b).statistic for a, b in zip(rows_s, rows_a)])
    np.testing.assert_allclose(got, lib, rtol=0, atol=1e-12)
    n = 37
    closed = []
    for a, b in zip(rows_s, rows_a):
        ra = np.argsort(np.argsort(a))
        rb = np.argsort(np.argsort(b))
        closed.append(1.0 - 6.0 * float(((ra - rb) ** 2).sum()) / (n * (n * n - 1)))
    np.testing.assert_allclose(got, np.mean(closed), rtol=0, atol=1e-12)


def test_spearman_vs_post_special_cases():
    rng = np.random.default_rng(12)
    A = rng.random((2, 5, 16))
    assert O.spearman_vs_post(A, A) == pytest.approx(1.0, abs=1e-12)
    assert O.spearman_vs_post(-A, A) == pytest.approx(-1.0, abs=1e-12)
    # any strictly increasing transform of the score leaves the ranks alone
    assert O.spearman_vs_post(np.exp(3.0 * A) - 2.0, A) == pytest.approx(1.0, abs=1e-12)


def test_topk_recall_vs_post_hand_worked_and_limits():
    # top-2 of A is {0, 1}; top-2 of S is {0, 2}: one of two kept -> 0.5
    A = np.array([[[5.0, 4.0, 3.0, 2.0, 1.0]]])
    S = np.array([[[5.0, 1.0, 4.0, 2.0, 3.0]]])
    assert O.topk_recall_vs_post(S, A, 2) == pytest.approx(0.5)
    rng = np.random.default_rng(13)
    A = rng.random((2, 3, 20))
    assert O.topk_recall_vs_post(A, A, 7) == pytest.approx(1.0)
    # the top 7 of -A are the bottom 7 of A: disjoint from its top 7 (no ties)
    assert O.topk_recall_vs_post(-A, A, 7) == pytest.approx(0.0)
    # brute force over rows: |top_k(S) & top_k(A)| / k by full sorts
    S = A + 0.3 * rng.standard_normal(A.shape)
    k = 5
    hits = 0
    for a, s in zip(A.reshape(-1, 20), S.reshape(-1, 20)):
        hits += len(set(np.argsort(-a, kind="stable")[:k]) & set(np.argsort(-s, kind="stable")[:k]))
    assert O.topk_recall_vs_post(S, A, k) == pytest.approx(hits / (k * 6))
