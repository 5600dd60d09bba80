"""Pins of the CPU oracle to things other than itself (CPU only).

Each test ties one oracle function to a hand-worked example, a closed form, an
invariant, a brute-force or library computation, or a special case in which
the method reduces to a textbook operation. Method source: "ClusterKV:
Manipulating LLM KV Cache in Semantic Space for Recallable Compression"
(arXiv 2412.03213v2), paperlayer.ai section summaries.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def _golden():
    with open(os.path.join(HERE, "golden", "hand_example.json")) as f:
        return json.load(f)


# ---- number formats -----------------------------------------------------------

def test_bf16_rounding_matches_torch_on_fp32_values():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
                        [0.0, -0.0, 1.0, -1.0, 3.0e38, 1e-40, -1e-41]]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.bf16_bits(x.astype(np.float64))
    assert np.array_equal(got, ref)


def test_bf16_rounding_ties_to_even_and_hand_values():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: even mantissa wins (1.0)
    assert oracle.lib().ckvo_bf16_bits(1 + 2.0 ** -8) == 0x3F80
    # 1 + 3*2^-8 is halfway between 1 + 2^-7 and 1 + 2^-6: rounds to 1 + 2^-6
    assert oracle.lib().ckvo_bf16_bits(1 + 3 * 2.0 ** -8) == 0x3F82
    assert oracle.lib().ckvo_bf16_bits(1 / 3) == 0x3EAB
    assert oracle.bf16_value([0x3EAB])[0] == 0.333984375
    assert oracle.lib().ckvo_bf16_bits(-2.0) == 0xC000


# ---- hand-worked example ----------------------------------------------------------

def test_golden_hand_example_clustering_selection_attention():
    g = _golden()
    e = g["expect"]
    keys = np.array(g["keys"], np.float32)
    vals = np.array(g["values"], np.float32)
    S, Wn, L = g["sink"], g["window"], g["L"]
    clustered = keys[S:L - Wn]
    for mode in ("bf16", "f32", "none"):
        r = oracle.kmeans(clustered, g["C"], g["T"], mode, tok_begin=S)
        assert r["labels"].tolist() == e["labels"]
        assert r["sizes"].tolist() == e["sizes"]
        assert r["offsets"].tolist() == e["offsets"]
        assert r["perm"].tolist() == e["perm"]
        np.testing.assert_allclose(r["mu"], e["mu"], rtol=0, atol=1e-15)
    mu_lp = oracle.round_to(r["mu"], "bf16")
    assert mu_lp.tolist() == e["mu_lp_bf16"]
    for case in e["cases"]:
        s = oracle.score(np.array(case["q"], np.float32), mu_lp)
        assert s.tolist() == case["scores"]
        sel, cnt = oracle.select(s, r["offsets"], r["perm"], case["budget"])
        assert sel.tolist() == case["sel_idx"] and cnt == case["sel_cnt"]
    a = e["attention_budget0"]
    rows = oracle.attended_rows(S, [], L - Wn, L)
    assert rows.tolist() == a["rows"]
    out = oracle.attend(np.array(a["q"], np.float32), keys, vals, rows, 1 / np.sqrt(2))
    np.testing.assert_allclose(out, a["out"], rtol=0, atol=1e-15)


# ---- P1: assignment = exhaustive argmax ----------------------------------------------

@pytest.mark.parametrize("n,C,d", [(257, 13, 128), (64, 64, 32), (50, 1, 8)])
def test_assign_is_brute_force_argmax(n, C, d):
    rng = np.random.default_rng(n * C)
    keys = rng.standard_normal((n, d)).astype(np.float32)
    muhat = rng.standard_normal((C, d))
    muhat /= np.linalg.norm(muhat, axis=1, keepdims=True)
    labels, gap = oracle.assign(keys, muhat)
    sims = keys.astype(np.float64) @ muhat.T
    assert np.array_equal(labels, np.argmax(sims, axis=1))
    if C > 1:
        top2 = np.sort(sims, axis=1)[:, -2:]
        ref_gap = (top2[:, 1] - top2[:, 0]) / np.linalg.norm(keys.astype(np.float64), axis=1)
        np.testing.assert_allclose(gap, ref_gap, rtol=1e-9, atol=1e-12)
    else:
        assert np.all(np.isinf(gap))


def test_assign_is_cosine_argmax_and_ties_go_to_lowest_id():
    rng = np.random.default_rng(7)
    keys = rng.standard_normal((100, 16)).astype(np.float32)
    mu = rng.standard_normal((9, 16))
    muhat = mu / np.linalg.norm(mu, axis=1, keepdims=True)
    # cosine similarity with explicitly normalised keys picks the same winners
    kn = keys / np.linalg.norm(keys, axis=1, keepdims=True)
    labels, _ = oracle.assign(keys, muhat)
    assert np.array_equal(labels, np.argmax(kn.astype(np.float64) @ muhat.T, axis=1))
    # duplicated centroids: every winner must be the first copy
    dup = np.concatenate([muhat, muhat])
    labels2, gap2 = oracle.assign(keys, dup)
    assert np.array_equal(labels2, labels) and np.all(gap2 == 0)


# ---- update and index against independent numpy formulations --------------------------

def test_update_is_mean_of_assigned_raw_keys_and_keeps_empty_clusters():
    rng = np.random.default_rng(3)
    n, C, d = 500, 12, 64
    keys = (rng.standard_normal((n, d)) * rng.uniform(0.5, 2, (n, 1))).astype(np.float32)
    labels = rng.integers(0, C - 2, n).astype(np.int32)  # clusters C-2, C-1 stay empty
    mu0 = rng.standard_normal((C, d))
    mh0 = rng.standard_normal((C, d))
    mu, muhat, sizes = oracle.update(keys, labels, mu0, mh0, "none")
    cnt = np.bincount(labels, minlength=C)
    assert sizes.tolist() == cnt.tolist()
    sums = np.zeros((C, d))
    np.add.at(sums, labels, keys.astype(np.float64))
    for c in range(C - 2):
        np.testing.assert_allclose(mu[c], sums[c] / cnt[c], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(muhat[c], mu[c] / np.linalg.norm(mu[c]), rtol=1e-12,
                                   atol=1e-15)
    assert np.array_equal(mu[C - 2:], mu0[C - 2:]) and np.array_equal(muhat[C - 2:], mh0[C - 2:])
    # storage rounding of the unit copy
    _, mh_bf, _ = oracle.update(keys, labels, mu0, mh0, "bf16")
    ref = torch.from_numpy((mu[:C - 2] / np.linalg.norm(mu[:C - 2], axis=1, keepdims=True)))
    # round-to-nearest directly from double equals torch's fp32->bf16 except
    # where the fp32 step itself moved the value across a bf16 midpoint
    tb = ref.to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.mean(mh_bf[:C - 2] == tb) > 0.999
    np.testing.assert_allclose(mh_bf[:C - 2], ref.numpy(), rtol=2.0 ** -8, atol=0)


def test_update_zero_mean_keeps_previous():
    keys = np.array([[1, 2], [-1, -2], [3, 0]], np.float32)
    labels = np.array([0, 0, 1], np.int32)
    mu0 = np.array([[5.0, 5.0], [1.0, 1.0]])
    mh0 = np.array([[0.6, 0.8], [0.0, 1.0]])
    mu, muhat, sizes = oracle.update(keys, labels, mu0, mh0, "none")
    assert sizes.tolist() == [2, 1]
    assert mu[0].tolist() == [5.0, 5.0] and muhat[0].tolist() == [0.6, 0.8]
    assert mu[1].tolist() == [3.0, 0.0] and muhat[1].tolist() == [1.0, 0.0]


@pytest.mark.parametrize("n,C", [(1000, 17), (33, 40), (1, 1), (4096, 400)])
def test_index_is_stable_sort_by_cluster(n, C):
    rng = np.random.default_rng(n + C)
    labels = rng.integers(0, C, n).astype(np.int32)
    tok_begin, perm_base = 16, 1000
    offsets, perm = oracle.index(labels, C, tok_begin, perm_base)
    cnt = np.bincount(labels, minlength=C)
    assert offsets.tolist() == (perm_base + np.concatenate([[0], np.cumsum(cnt)])).tolist()
    order = np.argsort(labels, kind="stable")
    assert perm.tolist() == (tok_begin + order).tolist()


# ---- P2: invariants of a full clustering ----------------------------------------------

@pytest.mark.parametrize("mode", ["bf16", "f32"])
def test_kmeans_invariants(mode):
    rng = np.random.default_rng(11)
    n, C, d, tb = 3000, 37, 128, 16
    keys = rng.standard_normal((n, d)).astype(np.float32)
    if mode == "bf16":
        keys = oracle.round_to(keys, "bf16").astype(np.float32)
    r = oracle.kmeans(keys, C, 6, mode, tok_begin=tb, history=True)
    lab, sizes, off, perm = r["labels"], r["sizes"], r["offsets"], r["perm"]
    assert lab.min() >= 0 and lab.max() < C
    assert sizes.sum() == n and np.array_equal(np.bincount(lab, minlength=C), sizes)
    assert off[0] == 0 and off[-1] == n and np.all(np.diff(off) == sizes)
    assert sorted(perm.tolist()) == list(range(tb, tb + n))
    for c in range(C):
        seg = perm[off[c]:off[c + 1]]
        assert np.all(np.diff(seg) > 0) and np.all(lab[seg - tb] == c)
    # the returned labels are those of the last round, and the centroids the
    # means of exactly those clusters (empty clusters keep their old centroid)
    assert np.array_equal(r["labels_hist"][-1], lab)
    for c in range(C):
        if sizes[c]:
            np.testing.assert_allclose(r["mu"][c], keys[lab == c].astype(np.float64).mean(0),
                                       rtol=1e-10, atol=1e-12)
    # round t assigned with the unit centroids of round t-1, rounded to storage
    lab0, _ = oracle.assign(keys, r["muhat_hist"][0])
    assert np.array_equal(lab0, r["labels_hist"][0])
    assert np.array_equal(r["muhat_hist"][-1], r["muhat"])
    mh = r["muhat"]
    assert np.array_equal(mh, oracle.round_to(mh, mode))


def test_strided_init_seeds():
    rng = np.random.default_rng(5)
    keys = rng.standard_normal((103, 8)).astype(np.float32)
    mu, muhat = oracle.init(keys, 10, "none")
    stride = 103 // 10
    for c in range(10):
        assert np.array_equal(mu[c], keys[c * stride].astype(np.float64))
        np.testing.assert_allclose(muhat[c], mu[c] / np.linalg.norm(mu[c]), rtol=1e-15)


# ---- P3: planted partition (closed form) -----------------------------------------------

def test_planted_partition_recovers_blocks_and_block_means():
    rng = np.random.default_rng(2)
    C, per, d = 16, 25, 128
    dirs = rng.standard_normal((C, d))
    dirs /= np.linalg.norm(dirs, axis=1, keepdims=True)
    s = rng.uniform(0.5, 2.0, C * per)
    keys = (np.repeat(dirs, per, axis=0) * s[:, None]).astype(np.float32)
    r = oracle.kmeans(keys, C, 4, "none", history=True)
    blocks = np.repeat(np.arange(C), per)
    for t in range(4):
        assert np.array_equal(r["labels_hist"][t], blocks)
    kd = keys.astype(np.float64)
    for c in range(C):
        np.testing.assert_allclose(r["mu"][c], kd[c * per:(c + 1) * per].mean(0), rtol=1e-12)
        # closed form: the mean of s_i u_c is mean(s) u_c (up to the fp32 keys)
        np.testing.assert_allclose(r["mu"][c], s[c * per:(c + 1) * per].mean() * dirs[c],
                                   rtol=1e-6, atol=1e-7)


# ---- P7: Lloyd monotonicity --------------------------------------------------------------

def test_lloyd_objective_is_monotone():
    # J = sum_i k_i . muhat_{a_i}: assignment maximises it for fixed centroids,
    # and muhat_c = mean/||mean|| maximises it for fixed labels, so it never
    # decreases when the unit centroids are kept in double.
    rng = np.random.default_rng(9)
    n, C, d = 2000, 20, 32
    keys = rng.standard_normal((n, d)).astype(np.float32)
    r = oracle.kmeans(keys, C, 12, "none", history=True)
    kd = keys.astype(np.float64)
    J = []
    for t in range(12):
        lab = r["labels_hist"][t]
        J.append(np.sum(kd * r["muhat_hist"][t][lab]))       # after assignment t
        J.append(np.sum(kd * r["muhat_hist"][t + 1][lab]))   # after update t
    assert np.all(np.diff(J) >= -1e-9 * abs(J[-1]))
    assert J[-1] > J[0]


# ---- selection -------------------------------------------------------------------------------

def test_score_exact_on_integer_inputs_and_close_on_floats():
    rng = np.random.default_rng(4)
    G, C, d = 4, 50, 128
    q = rng.integers(-3, 4, (G, d)).astype(np.float32)
    mu = rng.integers(-3, 4, (C, d)).astype(np.float32)
    s = oracle.score(q, mu)
    ref = (q.astype(np.int64).sum(0) @ mu.astype(np.int64).T)
    assert np.array_equal(s.astype(np.int64), ref)
    qf = rng.standard_normal((G, d)).astype(np.float32)
    mf = rng.standard_normal((C, d)).astype(np.float32)
    sf = oracle.score(qf, mf)
    np.testing.assert_allclose(sf, qf.astype(np.float64).sum(0) @ mf.astype(np.float64).T,
                               rtol=1e-5, atol=1e-4)


@pytest.mark.parametrize("budget", [0, 1, 37, 500, 1999, 2000, 5000])
def test_select_is_prefix_of_clusters_in_rank_order(budget):
    # Independent formulation of "take clusters by score until the budget is
    # met, trimming the last one": concatenate each cluster's positions in rank
    # order and keep the first `budget`.
    rng = np.random.default_rng(budget + 1)
    C, n = 60, 2000
    labels = rng.integers(0, C - 5, n).astype(np.int32)   # a few empty clusters
    offsets, perm = oracle.index(labels, C, 16, 0)
    s = np.round(rng.standard_normal(C), 1).astype(np.float32)  # many exact ties
    sel, cnt = oracle.select(s, offsets, perm, budget)
    order = np.lexsort((np.arange(C), -s.astype(np.float64)))
    cat = np.concatenate([perm[offsets[c]:offsets[c + 1]] for c in order])
    assert cnt == min(budget, n)
    assert sel.tolist() == cat[:budget].tolist()


def test_select_with_one_token_per_cluster_is_top_b_of_token_logits():
    # P4: with C = N every token is its own centroid, so cluster recall is
    # exactly the top-B objective over q.k (ties to the lower position).
    rng = np.random.default_rng(6)
    n, d, B, S = 300, 128, 40, 4
    keys = rng.integers(-2, 3, (n, d)).astype(np.float32)
    q = rng.integers(-2, 3, (1, d)).astype(np.float32)
    r = oracle.kmeans(keys, n, 3, "bf16", tok_begin=S)
    assert np.array_equal(r["labels"], np.arange(n))
    mu_lp = oracle.round_to(r["mu"], "bf16").astype(np.float32)
    assert np.array_equal(mu_lp, keys)
    s = oracle.score(q, mu_lp)
    sel, cnt = oracle.select(s, r["offsets"], r["perm"], B)
    logits = keys.astype(np.int64) @ q[0].astype(np.int64)
    top = np.lexsort((np.arange(n), -logits))[:B]
    assert cnt == B and sel.tolist() == (S + top).tolist()


# ---- attention ---------------------------------------------------------------------------------

def test_attention_matches_torch_sdpa_float64():
    rng = np.random.default_rng(8)
    G, d, L = 4, 128, 700
    q = rng.standard_normal((G, d)).astype(np.float32) * 3
    K = rng.standard_normal((L, d)).astype(np.float32)
    V = rng.standard_normal((L, d)).astype(np.float32)
    rows = np.sort(rng.choice(L, 333, replace=False)).astype(np.int32)
    out = oracle.attend(q, K, V, rows, 1 / np.sqrt(d))
    tq = torch.from_numpy(q.astype(np.float64))[None, :, None, :]
    tk = torch.from_numpy(K[rows].astype(np.float64))[None, None].expand(1, G, -1, -1)
    tv = torch.from_numpy(V[rows].astype(np.float64))[None, None].expand(1, G, -1, -1)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)[0, :, 0].numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


def test_full_budget_reproduces_dense_attention_exactly():
    # P5: with B >= N every clustered token is recalled, the attended set is
    # all of [0, L), and the output equals dense attention bit for bit.
    rng = np.random.default_rng(10)
    L, d, S, Wn, C = 600, 128, 16, 64, 20
    K = rng.standard_normal((L, d)).astype(np.float32)
    V = rng.standard_normal((L, d)).astype(np.float32)
    q = rng.standard_normal((2, d)).astype(np.float32)
    r = oracle.kmeans(K[S:L - Wn], C, 3, "f32", tok_begin=S)
    s = oracle.score(q, oracle.round_to(r["mu"], "f32"))
    sel, cnt = oracle.select(s, r["offsets"], r["perm"], 10_000)
    assert cnt == L - S - Wn
    rows = oracle.attended_rows(S, sel, L - Wn, L)
    assert rows.tolist() == list(range(L))
    sparse = oracle.attend(q, K, V, rows, 1 / np.sqrt(d))
    dense = oracle.attend(q, K, V, np.arange(L, dtype=np.int32), 1 / np.sqrt(d))
    assert np.array_equal(sparse, dense)


def test_zero_budget_attends_sinks_and_window_and_equal_keys_average_values():
    # P6: budget 0 leaves the sinks and the recent window (a StreamingLLM-like
    # set); with all keys equal the weights are uniform, so out = mean of V.
    rng = np.random.default_rng(12)
    L, d, S, Wn = 200, 128, 4, 32
    K = np.tile(rng.standard_normal((1, d)).astype(np.float32), (L, 1))
    V = rng.standard_normal((L, d)).astype(np.float32)
    q = rng.standard_normal((3, d)).astype(np.float32)
    rows = oracle.attended_rows(S, np.zeros(0, np.int32), L - Wn, L)
    assert rows.tolist() == list(range(S)) + list(range(L - Wn, L))
    out = oracle.attend(q, K, V, rows, 1 / np.sqrt(d))
    ref = V[rows].astype(np.float64).mean(0)
    for g in range(3):
        np.testing.assert_allclose(out[g], ref, rtol=1e-12, atol=1e-14)


def test_attended_rows_sorts_recalled_positions():
    rows = oracle.attended_rows(2, [9, 4, 7, 5], 12, 15)
    assert rows.tolist() == [0, 1, 4, 5, 7, 9, 12, 13, 14]


# ---- incremental clustering of generated tokens ---------------------------------------------

def test_incremental_index_appends_after_prefill():
    # "III.B Clustering in the Semantic Space": generated tokens are clustered
    # on their own into 4 new centroids; their metadata is appended after the
    # prompt's (cluster ids and perm slots continue from the prompt's).
    rng = np.random.default_rng(13)
    keys = rng.standard_normal((400, 16)).astype(np.float32)
    pre = oracle.kmeans(keys[8:300], 10, 3, "none", tok_begin=8, perm_base=0)
    inc = oracle.kmeans(keys[300:364], 4, 3, "none", tok_begin=300, perm_base=292)
    assert pre["offsets"][-1] == 292 == inc["offsets"][0]
    assert inc["offsets"][-1] == 292 + 64
    assert sorted(inc["perm"].tolist()) == list(range(300, 364))


# ---- similarity variants: L2 and inner product (the paper's ablation) -----------------------

def _no_near_ties(gap, eps=1e-6):
    return gap >= eps


@pytest.mark.parametrize("n,C,d", [(300, 17, 16), (257, 40, 128)])
def test_l2_assign_is_scipy_sqeuclidean_argmin(n, C, d):
    from scipy.spatial.distance import cdist
    rng = np.random.default_rng(n + C)
    keys = rng.standard_normal((n, d)).astype(np.float32)
    mu = rng.standard_normal((C, d)) * rng.uniform(0.2, 2.0, (C, 1))
    lab, gap = oracle.assign(keys, mu, metric="l2")
    ref = cdist(keys.astype(np.float64), mu, "sqeuclidean").argmin(axis=1)
    ok = _no_near_ties(gap)
    assert ok.mean() > 0.99
    assert np.array_equal(lab[ok], ref[ok])
    # the gap is half the squared-distance margin over ||k||
    dist = cdist(keys.astype(np.float64), mu, "sqeuclidean")
    srt = np.sort(dist, axis=1)
    np.testing.assert_allclose(gap, 0.5 * (srt[:, 1] - srt[:, 0]) /
                               np.linalg.norm(keys.astype(np.float64), axis=1), rtol=1e-9,
                               atol=1e-12)


def test_inner_product_assign_is_matmul_argmax_and_differs_from_cosine():
    rng = np.random.default_rng(31)
    n, C, d = 400, 24, 64
    keys = rng.standard_normal((n, d)).astype(np.float32)
    mu = rng.standard_normal((C, d)) * rng.uniform(0.1, 3.0, (C, 1))  # unequal norms
    lab, gap = oracle.assign(keys, mu, metric="ip")
    ref = np.argmax(keys.astype(np.float64) @ mu.T, axis=1)
    ok = _no_near_ties(gap)
    assert np.array_equal(lab[ok], ref[ok])
    # with unequal centroid norms the inner product and the cosine disagree
    unit = mu / np.linalg.norm(mu, axis=1, keepdims=True)
    lab_cos, _ = oracle.assign(keys, unit)
    assert (lab != lab_cos).mean() > 0.05


def test_metric_cosine_entry_points_equal_the_cosine_functions():
    rng = np.random.default_rng(5)
    n, C, d = 500, 12, 128
    keys = oracle.round_to(rng.standard_normal((n, d)), "bf16").astype(np.float32)
    L = oracle.lib()
    for mode in ("none", "bf16"):
        mu, mh = oracle.init(keys, C, mode)
        mu2, mh2 = np.zeros_like(mu), np.zeros_like(mh)
        L.ckvo_init_m(keys, n, d, C, oracle.ROUND[mode], 0, mu2, mh2)
        assert np.array_equal(mu, mu2) and np.array_equal(mh, mh2)
        lab, gap = oracle.assign(keys, mh)
        lab2 = np.zeros(n, np.int32)
        gap2 = np.zeros(n)
        L.ckvo_assign_m(keys, n, d, mh, C, 0, lab2, gap2.ctypes.data_as(oracle.ctypes.c_void_p))
        assert np.array_equal(lab, lab2) and np.array_equal(gap, gap2)
        r = oracle.update(keys, lab, mu, mh, mode)
        mu3, mh3, sz3 = mu.copy(), mh.copy(), np.zeros(C, np.int32)
        L.ckvo_update_m(keys, n, d, lab, C, oracle.ROUND[mode], 0, mu3, mh3, sz3)
        assert np.array_equal(r[0], mu3) and np.array_equal(r[1], mh3)
        assert np.array_equal(r[2], sz3)


@pytest.mark.parametrize("metric", ["ip", "l2"])
def test_variant_init_and_update_keep_the_raw_mean(metric):
    rng = np.random.default_rng(8)
    n, C, d = 103, 10, 128
    keys = oracle.round_to(rng.standard_normal((n, d)), "bf16").astype(np.float32)
    mu, mh = oracle.init(keys, C, "bf16", metric=metric)
    stride = n // C
    for c in range(C):
        assert np.array_equal(mu[c], keys[c * stride].astype(np.float64))
        assert np.array_equal(mh[c], mu[c])  # a bf16 key is its own rounding
    lab = rng.integers(0, C - 1, n).astype(np.int32)  # cluster C-1 stays empty
    lab[:3] = 0  # and cluster 0 is never empty
    mu2, mh2, sz = oracle.update(keys, lab, mu, mh, "bf16", metric=metric)
    kd = keys.astype(np.float64)
    for c in range(C - 1):
        m = kd[lab == c].mean(0)
        np.testing.assert_allclose(mu2[c], m, rtol=1e-12, atol=1e-15)
        assert np.array_equal(mh2[c], oracle.round_to(mu2[c], "bf16"))
    assert sz[C - 1] == 0 and np.array_equal(mu2[C - 1], mu[C - 1])
    assert np.array_equal(mh2[C - 1], mh[C - 1])


def test_l2_lloyd_objective_is_monotone():
    # J = sum_i ||k_i - mu_{a_i}||^2: assignment minimises it for fixed
    # centroids and the mean minimises it for fixed labels
    rng = np.random.default_rng(12)
    n, C, d = 1500, 18, 24
    keys = rng.standard_normal((n, d)).astype(np.float32)
    r = oracle.kmeans(keys, C, 10, "none", history=True, metric="l2")
    kd = keys.astype(np.float64)
    J = []
    for t in range(10):
        lab = r["labels_hist"][t]
        J.append(np.sum((kd - r["muhat_hist"][t][lab]) ** 2))
        J.append(np.sum((kd - r["muhat_hist"][t + 1][lab]) ** 2))
    assert np.all(np.diff(J) <= 1e-9 * abs(J[0]))
    assert J[-1] < J[0]


def test_l2_kmeans_fixed_point_equals_sklearn_lloyd():
    from sklearn.cluster import KMeans
    rng = np.random.default_rng(21)
    C, per, d = 8, 60, 16
    centers = rng.standard_normal((C, d)) * 4.0
    keys = (np.repeat(centers, per, axis=0) +
            rng.standard_normal((C * per, d))).astype(np.float32)
    keys = keys[rng.permutation(C * per)]
    n = keys.shape[0]
    r = oracle.kmeans(keys, C, 60, "none", metric="l2")
    seeds = keys[np.arange(C) * (n // C)].astype(np.float64)
    km = KMeans(n_clusters=C, init=seeds, n_init=1, max_iter=300, tol=0.0,
                algorithm="lloyd").fit(keys.astype(np.float64))
    assert np.array_equal(r["labels"], km.labels_)
    np.testing.assert_allclose(r["mu"], km.cluster_centers_, rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("metric", ["ip", "l2"])
def test_variant_planted_partition_recovers_blocks(metric):
    # blocks along distinct unit directions with one common norm: every
    # similarity sends each key to its block's centroid
    rng = np.random.default_rng(3)
    C, per, d = 12, 20, 128
    dirs = rng.standard_normal((C, d))
    dirs /= np.linalg.norm(dirs, axis=1, keepdims=True)
    keys = (np.repeat(dirs, per, axis=0) * 1.5).astype(np.float32)
    r = oracle.kmeans(keys, C, 3, "none", history=True, metric=metric)
    blocks = np.repeat(np.arange(C), per)
    for t in range(3):
        assert np.array_equal(r["labels_hist"][t], blocks)
    np.testing.assert_allclose(r["mu"], keys[::per].astype(np.float64), rtol=1e-12)


@pytest.mark.parametrize("metric", ["ip", "l2"])
def test_variant_zero_mean_is_a_valid_centroid(metric):
    # a cluster of k and -k has mean zero: without a direction it is kept
    # under cosine, but it is an ordinary centroid for L2 and inner product
    rng = np.random.default_rng(14)
    d = 128
    k = oracle.round_to(rng.standard_normal(d), "bf16")
    keys = np.stack([k, -k, k * 2.0]).astype(np.float32)
    lab = np.array([0, 0, 1], np.int32)
    mu0 = rng.standard_normal((2, d))
    mu, mh, sz = oracle.update(keys, lab, mu0, mu0, "bf16", metric=metric)
    assert np.array_equal(mu[0], np.zeros(d)) and np.array_equal(mh[0], np.zeros(d))
    mu_c, mh_c, _ = oracle.update(keys, lab, mu0, mu0, "bf16")
    assert np.array_equal(mu_c[0], mu0[0])


# ---- the cache of the last R steps' clusters ("D. Caching KV of Selected Tokens") ----------

@pytest.mark.parametrize("budget", [0, 1, 50, 400, 10_000])
def test_selected_clusters_spell_out_the_token_selection(budget):
    rng = np.random.default_rng(budget + 3)
    C, n = 60, 2000
    lab = rng.integers(0, C, n).astype(np.int32)
    lab[lab == 7] = 8  # an empty cluster
    offsets, perm = oracle.index(lab, C, 16)
    s = rng.standard_normal(C).astype(np.float32)
    s[10] = s[11]  # a score tie
    sel, cnt = oracle.select(s, offsets, perm, budget)
    cl, taken = oracle.selected_clusters(s, offsets, budget)
    assert taken.sum() == cnt and np.all(taken > 0)
    rebuilt = np.concatenate([perm[offsets[c]:offsets[c] + t] for c, t in zip(cl, taken)]
                             or [np.zeros(0, np.int32)])
    assert np.array_equal(rebuilt, sel)
    sizes = np.diff(offsets)
    assert np.all(taken[:-1] == sizes[cl[:-1]]) if cl.size else True
    assert 7 not in cl


def test_cache_step_matches_a_window_of_sets():
    rng = np.random.default_rng(17)
    C = 40
    for R in (0, 1, 2, 5):
        last = np.full(C, oracle.NEVER, np.int32)
        history = []
        for step in range(30):
            m = int(rng.integers(1, 12))
            cl = rng.choice(C, m, replace=False).astype(np.int32)
            taken = rng.integers(1, 9, m).astype(np.int32)
            hits, ht, misses = oracle.cache_step(cl, taken, step, R, last)
            window = set().union(*history[-R:]) if R > 0 and history else set()
            ref_hit = np.array([c in window for c in cl])
            assert hits == ref_hit.sum() and ht == taken[ref_hit].sum()
            assert np.array_equal(misses, cl[~ref_hit])  # rank order kept
            history.append(set(cl.tolist()))
            assert np.all(last[cl] == step)


def test_cache_closed_forms():
    C = 10
    cl = np.array([3, 1, 4], np.int32)
    taken = np.array([5, 5, 2], np.int32)
    # the same selection every step: all hits from the second step on, for any R >= 1
    last = np.full(C, oracle.NEVER, np.int32)
    assert oracle.cache_step(cl, taken, 0, 1, last)[0] == 0
    for step in range(1, 5):
        hits, ht, misses = oracle.cache_step(cl, taken, step, 1, last)
        assert hits == 3 and ht == 12 and misses.size == 0
    # R = 0 keeps nothing
    last = np.full(C, oracle.NEVER, np.int32)
    for step in range(4):
        assert oracle.cache_step(cl, taken, step, 0, last)[0] == 0
    # a cluster selected R + 1 steps ago has left the cache
    last = np.full(C, oracle.NEVER, np.int32)
    oracle.cache_step(np.array([2], np.int32), np.array([4], np.int32), 0, 2, last)
    assert oracle.cache_step(np.array([2], np.int32), np.array([4], np.int32), 3, 2, last)[0] == 0
    assert oracle.cache_step(np.array([2], np.int32), np.array([4], np.int32), 5, 2, last)[0] == 1
