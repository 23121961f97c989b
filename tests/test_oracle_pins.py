"""Pins for the CPU oracle: what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: numbers
the pages print (tests/golden, with citations), closed forms, brute force on
tiny inputs, library routines, and invariants the pages state.  None of them
retypes the oracle's own formulas.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
from scipy.special import logsumexp

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (inputs only)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def _dense_reference(q, K, V, mask, scale):
    """Textbook masked softmax attention in fp64 (numpy), one head."""
    logits = (K.astype(np.float64) @ q.astype(np.float64)) * scale
    logits = np.where(mask, logits, -np.inf)
    w = np.exp(logits - logits.max())
    w /= w.sum()
    return w @ V.astype(np.float64), logsumexp(logits)


# ----------------------------------------------------------------- KV sizes

def test_kv_bytes_matches_printed_examples():
    g = _golden("kv_cache_examples.json")["cases"]
    c = g[0]
    assert oracle.kv_bytes_per_token(c["layers"], c["kv_heads"], c["head_dim"],
                                     c["elem_bytes"]) == c["printed_per_token_bytes"] == 327680
    c = g[1]
    per = oracle.kv_bytes_per_token(c["layers"], c["kv_heads"], c["head_dim"], c["elem_bytes"])
    tot = per * c["context"]
    assert abs(tot / 1e9 - c["printed_total_gb"]) / c["printed_total_gb"] <= c["rel_tol"]
    btot = tot * c["batch"]
    err = min(abs(btot / 1e9 - c["printed_batch_total_gb"]),
              abs(btot / 2**30 - c["printed_batch_total_gb"])) / c["printed_batch_total_gb"]
    assert err <= c["rel_tol"]
    c = g[2]
    per = oracle.kv_bytes_per_token(c["layers"], c["kv_heads"], c["head_dim"], c["elem_bytes"])
    assert per == c["printed_per_token_kib"] * 1024
    for n, gib in zip(c["contexts"], c["printed_total_gib"]):
        assert abs(per * n / 2**30 - gib) / gib <= c["rel_tol"]
    c = g[3]
    for h, gib in zip(c["kv_heads"], c["printed_total_gib"]):
        per = oracle.kv_bytes_per_token(c["layers"], h, c["head_dim"], c["elem_bytes"])
        assert per * c["context"] == gib * 2**30
    c = g[4]
    ms = c["bytes_gib"] * 2**30 / (c["bandwidth_tb_s"] * 1e12) * 1e3
    assert abs(ms - c["printed_ms"]) / c["printed_ms"] <= c["rel_tol"]


# --------------------------------------------------------------- summaries

def test_centroid_equals_mean_and_is_exact_on_integers():
    rng = np.random.default_rng(1)
    K = rng.standard_normal((300, 16)).astype(np.float32)
    beg = np.array([0, 64, 100, 299]); end = np.array([64, 100, 299, 300])
    C = oracle.block_summaries(K, beg, end, oracle.CENTROID)
    for b in range(4):
        ref = K[beg[b]:end[b]].astype(np.float64).mean(0)
        np.testing.assert_allclose(C[b], ref, rtol=0, atol=1e-5)
    # integer-valued keys: every partial sum is exact, so the mean is the
    # correctly rounded quotient
    Ki = rng.integers(-50, 50, (128, 8)).astype(np.float32)
    C = oracle.block_summaries(Ki, np.array([0, 64]), np.array([64, 128]), oracle.CENTROID)
    ref = np.stack([Ki[:64].sum(0) / 64, Ki[64:].sum(0) / 64]).astype(np.float32)
    assert np.array_equal(C, ref)


def test_centroid_reads_bf16_bits_exactly():
    rng = np.random.default_rng(2)
    K = rng.standard_normal((64, 8)).astype(np.float32)
    Kb = _bf16_bits(K)
    Kw = oracle.bf16_bits_to_f32(Kb)
    a = oracle.block_summaries(Kb, np.array([0]), np.array([64]), oracle.CENTROID)
    b = oracle.block_summaries(Kw, np.array([0]), np.array([64]), oracle.CENTROID)
    assert np.array_equal(a, b)


def test_minmax_equals_numpy():
    rng = np.random.default_rng(3)
    K = _bf16_bits(rng.standard_normal((96, 32)).astype(np.float32))
    beg = np.arange(6) * 16
    mn, mx = oracle.block_summaries(K, beg, beg + 16, oracle.MINMAX)
    Kf = oracle.bf16_bits_to_f32(K).reshape(6, 16, 32)
    assert np.array_equal(mn, Kf.min(1)) and np.array_equal(mx, Kf.max(1))


def test_semantic_centroid_is_unit_and_matches_definition():
    rng = np.random.default_rng(4)
    K = rng.standard_normal((200, 32)).astype(np.float32) + 2.0
    beg, end = np.array([0, 50]), np.array([50, 200])
    C = oracle.block_summaries(K, beg, end, oracle.CENTROID_NORM)
    for b in range(2):
        x = K[beg[b]:end[b]].astype(np.float64)
        u = x / np.linalg.norm(x, axis=1, keepdims=True)
        m = u.mean(0)
        np.testing.assert_allclose(C[b], m / np.linalg.norm(m), atol=2e-6)
        assert abs(np.linalg.norm(C[b].astype(np.float64)) - 1) < 1e-6
    # a block of one repeated key has that key's direction as its centre
    k = rng.standard_normal(32).astype(np.float32)
    Krep = np.tile(k, (10, 1))
    C = oracle.block_summaries(Krep, np.array([0]), np.array([10]), oracle.CENTROID_NORM)
    np.testing.assert_allclose(C[0], k / np.linalg.norm(k.astype(np.float64)), atol=1e-6)


# ------------------------------------------------------------------ scores

def test_quest_bound_is_an_upper_bound_and_tight_for_single_tokens():
    """sum_i max(q_i mn_i, q_i mx_i) >= q.k for every key of the page, with
    equality when the page holds one token."""
    rng = np.random.default_rng(5)
    D = 32
    K = rng.standard_normal((16 * 20, D)).astype(np.float32)
    q = rng.standard_normal((1, D)).astype(np.float32)
    beg = np.arange(20) * 16
    mn, mx = oracle.block_summaries(K, beg, beg + 16, oracle.MINMAX)
    s32, s64 = oracle.block_scores(q, (mn, mx), oracle.MINMAX)
    dots = (K.astype(np.float64) @ q[0].astype(np.float64)).reshape(20, 16)
    assert np.all(s64 >= dots.max(1) - 1e-12)
    assert np.all(s32 >= dots.max(1) - 1e-4)
    mn1, mx1 = oracle.block_summaries(K, np.arange(40), np.arange(40) + 1, oracle.MINMAX)
    s32, s64 = oracle.block_scores(q, (mn1, mx1), oracle.MINMAX)
    np.testing.assert_allclose(s64, dots.reshape(-1)[:40], rtol=0, atol=1e-12)


def test_group_score_is_sum_of_head_scores_and_close_to_fp64():
    rng = np.random.default_rng(6)
    G, D = 4, 64
    C = rng.standard_normal((30, D)).astype(np.float32)
    q = rng.standard_normal((G, D)).astype(np.float32)
    s32, s64 = oracle.block_scores(q, C, oracle.CENTROID)
    ref = (C.astype(np.float64) @ q.astype(np.float64).T).sum(1)
    np.testing.assert_allclose(s64, ref, rtol=1e-12, atol=1e-12)
    bound = G * D * 2.0**-23 * (np.abs(C) @ np.abs(q).T).sum(1)
    assert np.all(np.abs(s32 - ref) <= bound)


# --------------------------------------------------------------- selection

def test_topk_matches_rank_counting_brute_force():
    rng = np.random.default_rng(7)
    for trial in range(50):
        n_blocks, S = 12, 4
        n = n_blocks * S + int(rng.integers(0, S))
        s32 = rng.integers(-3, 3, n_blocks).astype(np.float32)     # many ties
        s64 = s32.astype(np.float64)
        k = int(rng.integers(0, 8))
        sel, ranges, _ = oracle.select_fixed(s32, s64, n, S, k, 0, sink=4, window=6,
                                             keep_current=False)
        forced = {t for t in range(4)} | set(range(n - 6, n))
        cands = [j for j in range(n // S) if not set(range(j * S, j * S + S)) <= forced]
        expect = []
        for j in cands:
            beats = sum(1 for i in cands if s32[i] > s32[j] or (s32[i] == s32[j] and i < j))
            if beats < k:
                expect.append(j)
        assert sel == expect


def test_forced_set_always_selected_and_ranges_disjoint():
    rng = np.random.default_rng(8)
    for trial in range(40):
        S = int(rng.choice([4, 8, 16]))
        n = int(rng.integers(1, 400))
        sink, window = int(rng.integers(0, 40)), int(rng.integers(0, 60))
        keep = bool(rng.integers(0, 2))
        nb = n // S
        s = rng.standard_normal(max(nb, 1)).astype(np.float32)
        k = int(rng.integers(0, 10))
        sel, ranges, _ = oracle.select_fixed(s, s.astype(np.float64), n, S, k, 0, sink,
                                             window, keep)
        toks = set(oracle.ranges_to_rows(ranges).tolist())
        assert set(range(min(sink, n))) <= toks                        # sink never dropped
        assert set(range(max(0, n - window), n)) <= toks               # window kept
        if keep:
            assert set(range(((n - 1) // S) * S, n)) <= toks           # current block
        for j in sel:
            assert set(range(j * S, (j + 1) * S)) <= toks
        assert max(toks, default=-1) < n                               # nothing from the future
        for (a, b), (c, d) in zip(ranges, ranges[1:]):
            assert b < c                                               # disjoint, maximal
        forced = oracle.forced_ranges(n, sink, window, S, keep)
        n_cands = sum(1 for j in range(nb)
                      if not any(a <= j * S and (j + 1) * S <= b for a, b in forced))
        assert len(sel) == min(k, n_cands)


def test_selected_token_counts_match_printed_sizes():
    g = _golden("block_sparse_examples.json")
    f = g["flop_ratio"]
    n, S, k = f["n_ctx"], f["block"], f["topk"]
    s = np.arange(n // S, dtype=np.float32)
    sel, ranges, _ = oracle.select_fixed(s, s.astype(np.float64), n, S, k, 0, 0, 0, False)
    rows = oracle.ranges_to_rows(ranges)
    pairs_sparse, pairs_full = len(rows) * n, n * n       # every query row alike
    ratio = oracle.attention_flops(pairs_sparse, 128) / oracle.attention_flops(pairs_full, 128)
    assert ratio == pytest.approx(f["printed_ratio"]) == k * S / n
    m = g["msa_tokens"]
    nb = 64
    s = np.random.default_rng(9).standard_normal(nb).astype(np.float32)
    sel, ranges, _ = oracle.select_fixed(s, s.astype(np.float64), nb * m["block"], m["block"],
                                         m["topk"], 0, 0, 0, False)
    assert len(oracle.ranges_to_rows(ranges)) == m["printed_tokens"]
    w = g["sliding_window"]
    r = oracle.forced_ranges(w["position"] + 1, 0, w["w"], 64, False)
    assert r == [(w["position"] - w["w"] + 1, w["position"] + 1)]
    assert r[0][1] - 1 == w["printed_last"]
    assert r[0][0] == w["printed_first"] + 1          # the recorded off-by-one


def test_tiny_config_token_count():
    """Tiny config: sink 64 + window 128 + 8 blocks of 64, no overlap = 704."""
    s = np.random.default_rng(10).standard_normal(64).astype(np.float32)
    sel, ranges, _ = oracle.select_fixed(s, s.astype(np.float64), 4096, 64, 8, 0, 64, 128, False)
    assert len(sel) == 8 and all(1 <= j <= 61 for j in sel)
    assert len(oracle.ranges_to_rows(ranges)) == 64 + 128 + 8 * 64


def test_budget_greedy_properties():
    rng = np.random.default_rng(11)
    for trial in range(40):
        nb = 20
        vis = rng.integers(0, 30, nb)
        s = rng.standard_normal(nb).astype(np.float32)
        budget = int(rng.integers(0, 150))
        sel, _ = oracle.select_budget_greedy(s, s.astype(np.float64), vis, budget)
        assert sum(vis[j] for j in sel) <= budget
        assert all(vis[j] > 0 for j in sel)
        # every skipped visible block did not fit in what its higher-ranked
        # selected blocks left over
        rank = sorted(range(nb), key=lambda j: (-s[j], j))
        used = 0
        for j in rank:
            if vis[j] == 0:
                continue
            if j in sel:
                used += vis[j]
            else:
                assert vis[j] > budget - used


# --------------------------------------------------------------- attention

def _random_case(rng, n, D, G, dtype):
    K = rng.standard_normal((n, D)).astype(np.float32)
    V = rng.standard_normal((n, D)).astype(np.float32)
    q = rng.standard_normal((G, D)).astype(np.float32)
    if dtype == "bf16":
        return q, _bf16_bits(K), _bf16_bits(V)
    return q, K, V


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_all_blocks_admitted_is_dense_causal(dtype):
    """Module 14 §14.3: when the gate admits every block the result is full
    attention.  Brute force: numpy softmax over every token up to the current
    one; rows after it (the future) must not matter."""
    rng = np.random.default_rng(12)
    D, G, S = 32, 4, 16
    n = 16 * 13 + 5
    q, K, V = _random_case(rng, n + 40, D, G, dtype)
    res = oracle.decode_fixed_segment(q, K, V, n, n, oracle.CENTROID, S, 10**6, 0, 0, 0,
                                      True, 1 / math.sqrt(D))
    Kf = oracle.bf16_bits_to_f32(K) if dtype == "bf16" else K
    Vf = oracle.bf16_bits_to_f32(V) if dtype == "bf16" else V
    mask = np.arange(n + 40) < n
    for h in range(G):
        o, l = _dense_reference(q[h], Kf, Vf, mask, 1 / math.sqrt(D))
        np.testing.assert_allclose(res["out"][h], o, rtol=0, atol=1e-12)
        assert res["lse"][h] == pytest.approx(l, abs=1e-12)


def test_budget_zero_is_sink_plus_window():
    rng = np.random.default_rng(13)
    D, G, S, n = 32, 2, 8, 300
    q, K, V = _random_case(rng, n, D, G, "f32")
    res = oracle.decode_fixed_segment(q, K, V, n, n, oracle.MINMAX, S, 0, 0, 24, 40, False,
                                      1 / math.sqrt(D))
    pos = np.arange(n)
    mask = (pos < 24) | (pos >= n - 40)
    for h in range(G):
        o, _ = _dense_reference(q[h], K, V, mask, 1 / math.sqrt(D))
        np.testing.assert_allclose(res["out"][h], o, atol=1e-12)


def test_weights_sum_to_one_and_single_token():
    rng = np.random.default_rng(14)
    D, G, n = 16, 3, 50
    q, K, V = _random_case(rng, n, D, G, "f32")
    ones = np.ones_like(V)
    out, lse = oracle.attend(q, K, ones, np.arange(7, 40), 0.25)
    np.testing.assert_allclose(out, 1.0, atol=1e-14)
    out, lse = oracle.attend(q, K, V, np.array([17]), 0.25)
    np.testing.assert_allclose(out, np.tile(V[17], (G, 1)), atol=0)
    np.testing.assert_allclose(lse, 0.25 * (K[17].astype(np.float64) @ q.T.astype(np.float64)),
                               atol=1e-12)
    out, lse = oracle.attend(q, K, V, np.zeros(0, np.int64), 0.25)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_refresh_extends_window():
    """'Sparse attention in hybrid LLMs': selection is refreshed every 32
    steps and the window grows in between, so new tokens stay visible."""
    rng = np.random.default_rng(15)
    D, G, S = 16, 2, 8
    q, K, V = _random_case(rng, 400, D, G, "f32")
    a = oracle.decode_fixed_segment(q, K, V, 300, 317, oracle.MINMAX, S, 3, 0, 8, 16, False, 0.25)
    rows = set(oracle.ranges_to_rows(a["ranges"]).tolist())
    assert set(range(300 - 16, 317)) <= rows and max(rows) == 316
    b = oracle.decode_fixed_segment(q, K, V, 300, 300, oracle.MINMAX, S, 3, 0, 8, 16, False, 0.25)
    assert a["sel"] == b["sel"]
    # between refreshes the pages are the ones the refresh step's queries
    # picked, whatever the current queries would pick
    q2 = -q
    c = oracle.decode_fixed_segment(q2, K, V, 300, 317, oracle.MINMAX, S, 3, 0, 8, 16, False,
                                    0.25, q_sel=q)
    d = oracle.decode_fixed_segment(q2, K, V, 300, 317, oracle.MINMAX, S, 3, 0, 8, 16, False, 0.25)
    assert c["sel"] == a["sel"] and c["ranges"] == a["ranges"]
    assert d["sel"] != a["sel"]
    rows = oracle.ranges_to_rows(c["ranges"])
    ref, _ = _dense_reference(q2[0], K, V, np.isin(np.arange(400), rows), 0.25)
    np.testing.assert_allclose(c["out"][0], ref, atol=1e-12)


def test_needle_blocks_are_recalled():
    """MoBA-style gating with mean-pooled keys finds blocks planted along the
    query direction (16 needle blocks among 64)."""
    rng = np.random.default_rng(16)
    D, G, S, nb = 64, 8, 64, 64
    n = nb * S
    u = rng.standard_normal(D); u /= np.linalg.norm(u)
    K = rng.standard_normal((n, D)).astype(np.float32)
    needles = sorted(rng.choice(nb - 1, 16, replace=False).tolist())
    for j in needles:
        K[j * S:(j + 1) * S] += (math.sqrt(D) * u).astype(np.float32)
    q = (math.sqrt(D) * u + rng.standard_normal((G, D))).astype(np.float32)
    res = oracle.decode_fixed_segment(q, _bf16_bits(K), _bf16_bits(K), n, n, oracle.CENTROID,
                                      S, 16, 0, 0, 0, True, 1 / math.sqrt(D))
    assert res["sel"] == needles


def test_semantic_selection_reads_only_visible_positions():
    rng = np.random.default_rng(17)
    D, G, nb, L = 16, 2, 12, 600
    lab = rng.integers(0, nb, L)
    K = rng.standard_normal((L, D)).astype(np.float32)
    q = rng.standard_normal((G, D)).astype(np.float32)
    sel, pos, _, C = oracle.semantic_select_positions(q, K, lab, nb, 400, 60)
    assert len(pos) <= 60 and np.all(pos < 400)
    assert set(lab[pos].tolist()) <= set(sel)
    for j in sel:
        members = np.nonzero(lab[:400] == j)[0]
        assert set(members.tolist()) <= set(pos.tolist())
    # the centres are computed from the blocks' keys in position order
    order = np.argsort(lab, kind="stable")
    for j in range(nb):
        m = K[order][lab[order] == j].astype(np.float64)
        if len(m):
            u = m / np.linalg.norm(m, axis=1, keepdims=True)
            c = u.mean(0)
            np.testing.assert_allclose(C[j], c / np.linalg.norm(c), atol=2e-6)


def test_near_ties_are_listed():
    s32 = np.array([1.0, 2.0, 2.0000001, 0.5], np.float32)
    s64 = np.array([1.0, 2.0, 2.0000001, 0.5])
    sel, ranges, ties = oracle.select_fixed(s32, s64, 16, 4, 1, 0, 0, 0, False)
    # 2.0000001 rounds to 2.0 in fp32: the fp32 tie goes to the lower index,
    # and the fp64 scores flag the pair as a near-tie across the cut
    assert s32[1] == s32[2]
    assert sel == [1] and ties == [(1, 2)]


# --------------------------------------------------------------------------
# Semantic index: spherical k-means ("Semantic blocks for sparse attention")
# --------------------------------------------------------------------------

def _planted(rng, L, k, D, noise):
    cent = rng.standard_normal((k, D))
    cent /= np.linalg.norm(cent, axis=1, keepdims=True)
    lab = rng.integers(0, k, L)
    X = (cent[lab] + noise * rng.standard_normal((L, D))).astype(np.float32)
    return X, lab


def test_kmeans_recovers_well_separated_clusters_and_stores_them_stably():
    rng = np.random.default_rng(11)
    L, k, D = 3000, 12, 64
    X, lab = _planted(rng, L, k, D, 0.05)
    init = np.array([np.flatnonzero(lab == j)[3] for j in range(k)])
    C, labels, off, order = oracle.spherical_kmeans(X, k, 6, init)
    assert (labels == lab).all()
    # block-ordered store: a stable sort by cluster, CSR offsets from the counts
    assert (order == np.argsort(labels, kind="stable")).all()
    assert (off == np.concatenate([[0], np.cumsum(np.bincount(labels, minlength=k))])).all()
    # centres are unit vectors near the planted directions
    assert np.allclose(np.linalg.norm(C.astype(np.float64), axis=1), 1.0, atol=1e-6)
    U = X / np.linalg.norm(X, axis=1, keepdims=True)
    for j in range(k):
        m = U[labels == j].mean(axis=0)
        assert np.abs(C[j] - m / np.linalg.norm(m)).max() < 1e-5


def _kmeans_fp64(X, k, iters, init):
    """Independent restatement in fp64 with numpy (no fixed order)."""
    U = X.astype(np.float64)
    nr = np.linalg.norm(U, axis=1, keepdims=True)
    U = np.where(nr > 0, U / np.where(nr > 0, nr, 1), 0)
    C = U[init].copy()
    margins = []
    for it in range(iters):
        dots = U @ C.T
        lab = np.argmax(dots, axis=1)
        srt = np.sort(dots, axis=1)
        margins.append(srt[:, -1] - srt[:, -2])
        if it == iters - 1:
            break
        for j in range(k):
            if (lab == j).any():
                m = U[lab == j].mean(axis=0)
                C[j] = m / np.linalg.norm(m)
    return C, lab, min(x.min() for x in margins)


def test_kmeans_matches_an_fp64_restatement_without_near_ties():
    rng = np.random.default_rng(5)
    L, k, D, iters = 400, 5, 16, 4
    X = rng.standard_normal((L, D)).astype(np.float32)
    init = rng.choice(L, k, replace=False)
    C64, lab64, margin = _kmeans_fp64(X, k, iters, init)
    assert margin > 1e-5, "seed gives a near tie; the fp32 result could differ legitimately"
    C, labels, _, _ = oracle.spherical_kmeans(X, k, iters, init)
    assert (labels == lab64).all()
    assert np.abs(C - C64).max() < 1e-5


def test_kmeans_empty_cluster_keeps_its_centre_and_ties_go_low():
    rng = np.random.default_rng(2)
    L, D = 300, 32
    X = rng.standard_normal((L, D)).astype(np.float32)
    X[1] = X[0]            # two identical starting centres: every tie goes to 0
    X[7] = 0.0             # a zero key: every dot is 0, so it goes to centre 0
    init = np.array([0, 1, 2, 3])
    # one assignment: centre 1 ties with centre 0 everywhere and loses
    _, lab1, off1, _ = oracle.spherical_kmeans(X, 4, 1, init)
    assert (lab1 != 1).all() and off1[2] - off1[1] == 0 and lab1[7] == 0
    # the update in between leaves the empty centre where it was (it may win
    # keys again once centre 0 has moved)
    C, labels, _, _ = oracle.spherical_kmeans(X, 4, 2, init)
    u1 = X[1] / np.float32(np.sqrt(np.sum(X[1].astype(np.float64) ** 2)))
    assert np.abs(C[1] - u1).max() < 1e-6
    assert np.abs(C[0] - u1).max() > 1e-3
    # the assignment helper agrees with the last assignment
    assert (oracle.kmeans_assign(X, np.arange(L), C) == labels).all()


def test_paged_cache_gathers_to_the_contiguous_cache():
    """A cache cut into pages and scattered over a pool by a random page table
    reads back as the original cache, and attention over it is unchanged."""
    rng = np.random.default_rng(4)
    H, D, P, n = 2, 16, 16, 16 * 7 + 5
    K = rng.standard_normal((H, n, D)).astype(np.float32)
    n_pages = -(-n // P)
    pool = np.zeros((n_pages + 3, H, P, D), np.float32)
    table = rng.permutation(n_pages + 3)[:n_pages]
    for i in range(n_pages):
        rows = K[:, i * P:min((i + 1) * P, n)]
        pool[table[i], :, :rows.shape[1]] = rows
    back = oracle.paged_to_contiguous(pool, table, P, n)
    assert back.shape == K.shape and (back == K).all()
    # identity table over an in-order pool is a reshape
    pool2 = np.zeros((n_pages, H, P, D), np.float32)
    for i in range(n_pages):
        rows = K[:, i * P:min((i + 1) * P, n)]
        pool2[i, :, :rows.shape[1]] = rows
    assert (oracle.paged_to_contiguous(pool2, np.arange(n_pages), P, n) == K).all()
    q = rng.standard_normal((1, D)).astype(np.float32)
    V = rng.standard_normal((H, n, D)).astype(np.float32)
    poolv = np.zeros_like(pool)
    for i in range(n_pages):
        rows = V[:, i * P:min((i + 1) * P, n)]
        poolv[table[i], :, :rows.shape[1]] = rows
    Vb = oracle.paged_to_contiguous(poolv, table, P, n)
    rows = np.arange(n)
    o1, l1 = oracle.attend(q, K[0], V[0], rows, 0.25)
    o2, l2 = oracle.attend(q, back[0], Vb[0], rows, 0.25)
    assert (o1 == o2).all() and (l1 == l2).all()


def test_fp8_e4m3_decoding_matches_torch_and_the_format_limits():
    import torch
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.fp8_e4m3_to_f32(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    both_nan = np.isnan(ours) & np.isnan(ref)
    assert (both_nan | (ours == ref)).all()
    assert np.isnan(ours).sum() == 2                       # S.1111.111
    assert ours[0x38] == 1.0 and ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9
    assert ours[0x80] == 0.0 and np.signbit(ours[0x80])    # negative zero
