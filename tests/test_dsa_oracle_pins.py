"""Pins of the CPU oracle of the sparse attention's key selection (indexer score
and top-k) against what the pages and the mathematics fix.

None of these compares the oracle with itself: each check is a hand-derived
worked example, a closed form, a number the pages print, brute force on a tiny
input, or an invariant the equations imply.  Sources: "GLM-5 . MoE transformer
block" (open model atlas), section "All 43 steps", the indexer equations
(S_I = 1/(sqrt(32) sqrt(128)) sum_h w ReLU(q.k), S~ = S_I + M, top_2048); nnterp
encyclopedia page glm_moe_dsa, section "Up to 2048 tokens the sparse attention
is plain causal attention".
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import oracle as O
from sigmoid_routed_mixture_b200 import workloads as W

HERE = os.path.dirname(__file__)
GOLDEN = json.load(open(os.path.join(HERE, "golden", "page_constants.json")))
WORKED = json.load(open(os.path.join(HERE, "golden", "dsa_worked_example.json")))


def num(v):
    return -math.inf if v == "-inf" else float(v)


def bf(vals):
    a = np.asarray(vals, dtype=np.float32)
    bits = W.f32_to_bf16_bits(a)
    assert np.array_equal(W.bf16_bits_to_f32(bits), a), "value not exact in bf16"
    return bits


def rand_case(B=2, T=9, S=13, NH=4, D=8, seed=3):
    rng = np.random.default_rng(seed)
    q = W.f32_to_bf16_bits(rng.standard_normal((B, T, NH, D), dtype=np.float32))
    k = W.f32_to_bf16_bits(rng.standard_normal((B, S, D), dtype=np.float32))
    w = rng.standard_normal((B, T, NH)).astype(np.float32)
    return q, k, w


def test_worked_example_scores_and_selection():
    ex = WORKED
    q = bf(ex["q"])[None]
    k = bf(ex["k"])[None]
    w = np.asarray(ex["w"], dtype=np.float32)[None]
    s = O.dsa_scores(q, k, w)[0]
    want = np.array([[num(v) for v in row] for row in ex["scores"]])
    assert np.array_equal(s, want)
    sel, kth, nxt = O.dsa_select(s, 2)
    assert sel.tolist() == ex["top2"]["sel"]
    assert kth.tolist() == [num(v) for v in ex["top2"]["kth"]]
    assert nxt.tolist() == [num(v) for v in ex["top2"]["next"]]
    sel1, _, _ = O.dsa_select(s, 1)
    assert sel1.tolist() == ex["top1"]["sel"]


def test_page_scale_is_one_over_64_with_one_hot_vectors():
    """32 heads of width 128 (the pages' config): with one-hot q and k, q.k is 1
    where the hot dimensions agree and 0 elsewhere, so a key's score is the sum of
    w over the heads that hit it, divided by sqrt(32)*sqrt(128) = 64."""
    cfg = GOLDEN["glm5_indexer"]
    NH, D = cfg["index_n_heads"], cfg["index_head_dim"]
    assert math.sqrt(NH * D) == GOLDEN["glm5_indexer_score_scale_inv"]
    S = 6
    qf = np.zeros((1, 1, NH, D), dtype=np.float32)
    for h in range(NH):
        qf[0, 0, h, h % 4] = 1.0  # head h hits key h % 4
    kf = np.zeros((1, S, D), dtype=np.float32)
    for s in range(S):
        kf[0, s, s] = 1.0  # key s is one-hot in dimension s
    w = (np.arange(NH, dtype=np.float32) + 1.0)[None, None]  # w_h = h + 1
    got = O.dsa_scores(bf(qf), bf(kf), w)[0, 0]
    # key j < 4 is hit by heads h = j + 4i (i = 0..7), each adding w_h = j + 4i + 1:
    # sum_{i=0..7} (j + 4i + 1) = 8j + 4*28 + 8 = 8j + 120; keys 4 and 5 are hit by none
    want = [(8 * j + 120) / 64.0 for j in range(4)] + [0.0, 0.0]
    assert got.tolist() == want


def test_relu_drops_negative_head_dots_whatever_the_weight():
    """A head whose dot product is negative adds nothing, even with a negative w."""
    qf = np.zeros((1, 1, 2, 4), dtype=np.float32)
    qf[0, 0, 0] = [1, 0, 0, 0]
    qf[0, 0, 1] = [-1, 0, 0, 0]  # anti-aligned with key 0
    kf = np.zeros((1, 1, 4), dtype=np.float32)
    kf[0, 0] = [3, 0, 0, 0]
    for w1 in (-5.0, 0.0, 7.0):
        w = np.array([[[2.0, w1]]], dtype=np.float32)
        got = O.dsa_scores(bf(qf), bf(kf), w)[0, 0, 0]
        assert got == 2.0 * 3.0 / math.sqrt(2 * 4)


def test_positive_homogeneity_and_linearity_in_w():
    """ReLU(c a) = c ReLU(a) for c > 0: doubling q (exact in bf16) doubles every
    visible score; the score is linear in w: S(w1 + w2) = S(w1) + S(w2)."""
    q, k, w = rand_case()
    base = O.dsa_scores(q, k, w)
    q2 = W.f32_to_bf16_bits(W.bf16_bits_to_f32(q) * 2.0)
    vis = np.isfinite(base)
    assert np.allclose(O.dsa_scores(q2, k, w)[vis], 2.0 * base[vis], rtol=1e-14, atol=1e-14)
    rng = np.random.default_rng(11)
    mask = rng.random(w.shape) < 0.5
    wa = np.where(mask, w, 0).astype(np.float32)
    wb = np.where(mask, 0, w).astype(np.float32)
    sa, sb = O.dsa_scores(q, k, wa), O.dsa_scores(q, k, wb)
    assert np.allclose(sa[vis] + sb[vis], base[vis], rtol=1e-13, atol=1e-13)


def test_causal_rows_keep_t_plus_one_keys():
    """A prefill (T == S): row t sees keys 0..t, i.e. t + 1 finite scores (page: row t has
    t + 1 nonzero entries); with a cache, query t sits at position S - T + t."""
    q, k, w = rand_case(B=1, T=7, S=7)
    s = O.dsa_scores(q, k, w)[0]
    assert [int(np.isfinite(r).sum()) for r in s] == list(range(1, 8))
    q, k, w = rand_case(B=1, T=3, S=10, seed=4)
    s = O.dsa_scores(q, k, w)[0]
    assert [int(np.isfinite(r).sum()) for r in s] == [8, 9, 10]


def test_short_prompt_selects_every_key():
    """Up to index_topk keys the selection lists every key (page)."""
    q, k, w = rand_case(B=1, T=12, S=12, seed=5)
    sel, _, _ = O.dsa_select(O.dsa_scores(q, k, w), 2048)
    assert sel.shape == (1, 12, 12)
    assert all(r.tolist() == list(range(12)) for r in sel[0])


def brute_force_select(row, n_sel):
    """Key s is taken iff fewer than n_sel keys come before it in the order
    (higher score, or equal score and lower index); listed in ascending index."""
    S = len(row)
    taken = []
    for s in range(S):
        before = sum(1 for j in range(S) if row[j] > row[s] or (row[j] == row[s] and j < s))
        if before < n_sel:
            taken.append(s)
    return taken


@pytest.mark.parametrize("topk", [1, 3, 5, 13, 40])
def test_selection_equals_brute_force(topk):
    q, k, w = rand_case(B=2, T=9, S=13, seed=6)
    s = O.dsa_scores(q, k, w)
    # plant exact ties: equal scores decided by index
    s[0, 8, 3] = s[0, 8, 7]
    s[1, 4, 0] = s[1, 4, 2]
    sel, kth, nxt = O.dsa_select(s, topk)
    for b in range(2):
        for t in range(9):
            want = brute_force_select(s[b, t].tolist(), min(topk, 13))
            assert sel[b, t].tolist() == want
            row = sorted(s[b, t].tolist(), reverse=True)
            assert kth[b, t] == row[min(topk, 13) - 1]
            assert nxt[b, t] == (row[topk] if topk < 13 else -math.inf)


def test_key_permutation_moves_the_selection_with_it():
    """One query at the last position sees every key; relabelling the keys
    relabels the selection (distinct scores)."""
    q, k, w = rand_case(B=1, T=1, S=30, NH=8, D=16, seed=8)
    perm = np.random.default_rng(9).permutation(30)
    s = O.dsa_scores(q, k, w)[0, 0]
    sp = O.dsa_scores(q, k[:, perm], w)[0, 0]
    assert np.array_equal(sp, s[perm])
    assert len(set(s.tolist())) == 30
    sel, _, _ = O.dsa_select(s, 11)
    selp, _, _ = O.dsa_select(sp, 11)
    assert sorted(perm[selp].tolist()) == sel.tolist()


def test_the_2048_key_boundary():
    """At the pages' index_topk = 2048: a query that sees exactly 2048 keys takes
    them all; one that sees 2049 drops exactly its lowest-scored key (the page's
    short-prompt rule and its first exception)."""
    S = 2049
    rng = np.random.default_rng(12)
    scores = np.full((2, S), -np.inf)
    scores[0, :2048] = rng.standard_normal(2048)      # sees keys 0 .. 2047
    scores[1, :] = rng.standard_normal(S)             # sees all 2049
    sel, kth, nxt = O.dsa_select(scores, GOLDEN["glm5_indexer"]["index_topk"])
    assert sel[0].tolist() == list(range(2048)) and nxt[0] == -math.inf
    dropped = int(np.argmin(scores[1]))
    assert sel[1].tolist() == [s for s in range(S) if s != dropped]
    assert nxt[1] == scores[1, dropped]


def test_scores_of_a_cache_query_equal_those_of_a_prefill_row():
    """Query t of a prefill (T = S) and the single query of a cached decode step at
    the same position see the same keys and score them identically."""
    q, k, w = rand_case(B=1, T=10, S=10, seed=13)
    pre = O.dsa_scores(q, k, w)[0]
    for t in (0, 4, 9):
        dec = O.dsa_scores(q[:, t:t + 1], k[:, :t + 1], w[:, t:t + 1])[0, 0]
        assert np.array_equal(dec, pre[t, :t + 1])
