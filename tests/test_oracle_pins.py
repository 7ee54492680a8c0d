"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these compares the oracle with itself: each check is a number the pages
print, a closed form, brute force on a tiny input, an invariant the equations
imply, or a special case that reduces to a library routine (NumPy matmul in
float64).  Sources: "GLM-5 . MoE transformer block" (open model atlas), section
"All 43 steps", Mixture-of-experts equations and the "Parameters" table; nnterp
encyclopedia pages GLM-4.7-Flash and GLM-5, section 03, note "The mixture:
sigmoid scores, a selection bias, renormalized weights".
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

from oracle import oracle as O
from sigmoid_routed_mixture_b200 import workloads as W

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_constants.json")))


def bf(vals):
    """Exact bf16 bit patterns of values that are representable in bf16."""
    a = np.asarray(vals, dtype=np.float32)
    bits = W.f32_to_bf16_bits(a)
    assert np.array_equal(W.bf16_bits_to_f32(bits), a), "value not exact in bf16"
    return bits


def small_case(T=24, H=48, I=80, E=8, K=3, seed=7, scale=2.5):
    rng = np.random.default_rng(seed)
    x = W.f32_to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
    w_r = (rng.standard_normal((E, H)) * 0.3).astype(np.float32)
    b = (rng.standard_normal(E) * 0.1).astype(np.float32)
    w1 = W.f32_to_bf16_bits(rng.standard_normal((E, I, H), dtype=np.float32) * 0.2)
    w3 = W.f32_to_bf16_bits(rng.standard_normal((E, I, H), dtype=np.float32) * 0.2)
    w2 = W.f32_to_bf16_bits(rng.standard_normal((E, H, I), dtype=np.float32) * 0.2)
    ws1 = W.f32_to_bf16_bits(rng.standard_normal((I, H), dtype=np.float32) * 0.2)
    ws3 = W.f32_to_bf16_bits(rng.standard_normal((I, H), dtype=np.float32) * 0.2)
    ws2 = W.f32_to_bf16_bits(rng.standard_normal((H, I), dtype=np.float32) * 0.2)
    return dict(x=x, w_r=w_r, b=b, w1=w1, w3=w3, w2=w2, ws1=ws1, ws3=ws3, ws2=ws2, K=K, scale=scale)


def numpy_swiglu(xf, w1, w3, w2):
    """Dense SwiGLU MLP in float64 through NumPy matmul: down(silu(gate) * up)."""
    g = xf @ W.bf16_bits_to_f32(w1).astype(np.float64).T
    u = xf @ W.bf16_bits_to_f32(w3).astype(np.float64).T
    return ((g / (1.0 + np.exp(-g))) * u) @ W.bf16_bits_to_f32(w2).astype(np.float64).T


# ---------------------------------------------------------------- page numbers

def test_param_count_matches_page():
    g = GOLDEN["glm5"]
    n = O.param_count(g["hidden_size"], g["moe_intermediate_size"], g["n_routed_experts"],
                      g["n_shared_experts"])
    assert n == GOLDEN["glm5_moe_params_per_block"]
    assert g["n_routed_experts"] * GOLDEN["glm5_moe_blocks"] == GOLDEN["glm5_bias_values_whole_model"]


def test_workload_shapes_match_pages():
    g5, g47 = GOLDEN["glm5"], GOLDEN["glm47flash"]
    for name in ("glm5_decode", "glm5_prefill", "glm5_skewed"):
        w = W.WORKLOADS[name]
        assert (w.H, w.I, w.E, w.K, w.scale) == (g5["hidden_size"], g5["moe_intermediate_size"],
                                                 g5["n_routed_experts"], g5["num_experts_per_tok"],
                                                 g5["routed_scaling_factor"])
    w = W.WORKLOADS["glm47flash"]
    assert (w.H, w.I, w.E, w.K) == (g47["hidden_size"], g47["moe_intermediate_size"],
                                    g47["n_routed_experts"], g47["num_experts_per_tok"])


@pytest.mark.parametrize("scale_key", ["gate_sum_glm5", "gate_sum_glm47flash"])
@pytest.mark.parametrize("name", ["tiny", "glm47flash"])
def test_gates_sum_to_page_scale(name, scale_key):
    w = W.WORKLOADS[name]
    if name == "glm47flash":
        w = w.replace(T=512)
    scale = GOLDEN[scale_key]
    x, w_r, b = W.router_inputs(w)
    idx, gate, margin, z = O.route(x, w_r, b, w.K, scale)
    assert np.max(np.abs(gate.sum(axis=1) - scale)) <= 1e-12
    assert np.all(gate > 0)
    # every token selects K distinct experts
    assert all(len(set(r)) == w.K for r in idx.tolist())


# ---------------------------------------------------------------- closed forms

def test_worked_example_by_hand():
    """A 1-token, 4-expert, H=2, I=1 block whose every step is a closed form.

    x = (1, 0), so z_e = W_r[e, 0] = (2, -1, 0.5, 1) and s_e = sigmoid(z_e).
    b = (0, 0.5, 0, 0): keys = s + b rank experts 0, 1, 3, 2, so top-2 = (0, 1)
    although the un-biased ranking would pick (0, 3).
    G_0 = 2.5 s_0/(s_0+s_1), G_1 = 2.5 s_1/(s_0+s_1).
    Expert 0: g = 1, u = 2   -> h = 2 sigmoid(1);       W2 column (1, -0.5)
    Expert 1: g = -2, u = 1  -> h = -2 sigmoid(-2);     W2 column (2, 1)
    Shared:   g = 0.5, u = 4 -> h = 2 sigmoid(0.5);     W2 column (1, 1)
    """
    sig = lambda v: 1.0 / (1.0 + math.exp(-v))  # noqa: E731
    x = bf([[1.0, 0.0]])
    w_r = np.array([[2.0, 7.0], [-1.0, -3.0], [0.5, 1.0], [1.0, 0.25]], dtype=np.float32)
    b = np.array([0.0, 0.5, 0.0, 0.0], dtype=np.float32)
    w1 = bf([[[1.0, 9.0]], [[-2.0, 5.0]], [[3.0, 3.0]], [[4.0, -4.0]]])      # [E, I=1, H=2]
    w3 = bf([[[2.0, -7.0]], [[1.0, 6.0]], [[1.0, 1.0]], [[-1.0, 2.0]]])
    w2 = bf([[[1.0], [-0.5]], [[2.0], [1.0]], [[8.0], [8.0]], [[-8.0], [8.0]]])  # [E, H=2, I=1]
    ws1, ws3, ws2 = bf([[0.5, 11.0]]), bf([[4.0, -13.0]]), bf([[1.0], [1.0]])

    idx, gate, margin, z = O.route(x, w_r, b, 2, 2.5)
    assert idx.tolist() == [[0, 1]]
    s0, s1, s3 = sig(2.0), sig(-1.0), sig(1.0)
    assert gate[0, 0] == pytest.approx(2.5 * s0 / (s0 + s1), rel=1e-15, abs=0)
    assert gate[0, 1] == pytest.approx(2.5 * s1 / (s0 + s1), rel=1e-15, abs=0)
    assert margin[0] == pytest.approx((s1 + 0.5) - s3, rel=1e-14, abs=0)

    y, yr, ys, yk = O.forward(x, w1, w3, w2, ws1, ws3, ws2, idx, gate, want_parts=True)
    e0 = np.array([1.0, -0.5]) * (2.0 * sig(1.0))
    e1 = np.array([2.0, 1.0]) * (-2.0 * sig(-2.0))
    sh = np.array([1.0, 1.0]) * (2.0 * sig(0.5))
    np.testing.assert_allclose(yk[0, 0], gate[0, 0] * e0, rtol=1e-15, atol=0)
    np.testing.assert_allclose(yk[0, 1], gate[0, 1] * e1, rtol=1e-15, atol=0)
    np.testing.assert_allclose(ys[0], sh, rtol=1e-15, atol=0)
    np.testing.assert_allclose(y[0], gate[0, 0] * e0 + gate[0, 1] * e1 + sh, rtol=1e-14, atol=0)


def test_equal_scores_pick_lowest_indices():
    """x = 0 gives z = 0, s = 1/2 for every expert; with b = 0 all keys tie, so the
    selection is experts 0..K-1 in order, every gate is scale/K and the margin is 0."""
    T, H, E, K = 5, 32, 12, 4
    x = np.zeros((T, H), dtype=np.uint16)
    w_r = np.random.default_rng(0).standard_normal((E, H)).astype(np.float32)
    idx, gate, margin, _ = O.route(x, w_r, np.zeros(E, np.float32), K, 2.5)
    assert idx.tolist() == [list(range(K))] * T
    assert np.all(gate == 2.5 / K)
    assert np.all(margin == 0.0)
    # ties among the biased keys only: experts 9 and 3 share the top key -> 3 first
    b = np.zeros(E, np.float32)
    b[[9, 3]] = 0.25
    b[7] = 0.125
    idx, _, margin, _ = O.route(x, w_r, b, 3, 2.5)
    assert idx.tolist() == [[3, 9, 7]] * T
    assert np.all(margin == 0.125)


def test_logits_match_library_matmul():
    c = small_case(T=40, H=96, E=16)
    z = O.logits(c["x"], c["w_r"])
    ref = W.bf16_bits_to_f32(c["x"]).astype(np.float64) @ c["w_r"].astype(np.float64).T
    np.testing.assert_allclose(z, ref, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- brute force

def test_selection_equals_best_subset_brute_force():
    """Top-K of s + b is the K-subset with the largest key sum; among equal sums
    the lexicographically smallest index tuple (lower index wins ties)."""
    rng = np.random.default_rng(3)
    E, K = 8, 3
    for trial in range(200):
        # quantised logits and biases create frequent exact ties
        z = (rng.integers(-3, 4, size=(1, E)) * 0.5).astype(np.float64)
        b = (rng.integers(-2, 3, size=E) * 0.25).astype(np.float32)
        idx, gate, margin = O.select(z, b, K, 2.5)
        key = 1.0 / (1.0 + np.exp(-z[0])) + b.astype(np.float64)
        best = None
        for sub in itertools.combinations(range(E), K):
            tot = sum(key[list(sub)])
            if best is None or tot > best[0] + 1e-12:
                best = (tot, sub)
        assert tuple(sorted(idx[0].tolist())) == best[1]
        # slot order: non-increasing key, equal keys in ascending index
        ks = key[idx[0]]
        for a in range(K - 1):
            assert ks[a] > ks[a + 1] or (ks[a] == ks[a + 1] and idx[0, a] < idx[0, a + 1])
        rest = [e for e in range(E) if e not in best[1]]
        assert margin[0] == pytest.approx(min(key[list(best[1])]) - max(key[rest]), abs=1e-15)


def test_gates_for_given_selection_closed_forms():
    """Gates of a GIVEN selection (the GPU's own choice in every output check):
    G_slot = scale * s_idx[slot] / sum over the selection of s, s = sigmoid(z),
    the un-biased sigmoids ("All 43 steps", G_i; nnterp section 03 note: the
    weights are the un-biased scores renormalised, times the routed scale).

    The 1-token example of test_worked_example_by_hand: z = (2, -1, 0.5, 1).  A
    forced selection (0, 3) -- not the biased choice (0, 1) -- must give
    2.5 s0/(s0+s3), 2.5 s3/(s0+s3) in slot order; the reversed order (3, 0)
    swaps them.  A dropped scale, a sum over all four experts, a sum over the
    biased keys or a gate read at the slot number instead of the expert id each
    fails one of these."""
    sig = lambda v: 1.0 / (1.0 + math.exp(-v))  # noqa: E731
    z = np.array([[2.0, -1.0, 0.5, 1.0]])
    s0, s3 = sig(2.0), sig(1.0)
    g = O.gates_for(z, np.array([[0, 3]], dtype=np.int32), 2.5)
    assert g[0, 0] == pytest.approx(2.5 * s0 / (s0 + s3), rel=1e-15, abs=0)
    assert g[0, 1] == pytest.approx(2.5 * s3 / (s0 + s3), rel=1e-15, abs=0)
    g = O.gates_for(z, np.array([[3, 0]], dtype=np.int32), 1.8)
    assert g[0, 0] == pytest.approx(1.8 * s3 / (s0 + s3), rel=1e-15, abs=0)
    assert g[0, 1] == pytest.approx(1.8 * s0 / (s0 + s3), rel=1e-15, abs=0)
    # one selected expert takes the whole scale, whatever its score
    g = O.gates_for(z, np.array([[1]], dtype=np.int32), 2.5)
    assert g[0, 0] == 2.5
    # equal logits (s = 1/2 everywhere): every gate is scale / K for any selection
    zt = np.zeros((3, 10))
    sel = np.array([[9, 0, 4], [2, 3, 1], [7, 8, 5]], dtype=np.int32)
    assert np.all(O.gates_for(zt, sel, 2.5) == 2.5 / 3)


def test_gates_for_sum_ratio_and_out_of_range():
    """For any selection the gates sum to the scale (to 1e-12) and the ratio of
    two slots' gates is the ratio of their sigmoids, s_a / s_b, exactly the
    ratio of 1/(1+exp(-z)) values (a closed form independent of the sum)."""
    rng = np.random.default_rng(5)
    T, E, K = 40, 16, 5
    z = rng.standard_normal((T, E)) * 3.0
    idx = np.array([rng.permutation(E)[:K] for _ in range(T)], dtype=np.int32)
    g = O.gates_for(z, idx, 2.5)
    assert np.max(np.abs(g.sum(axis=1) - 2.5)) <= 1e-12
    s = 1.0 / (1.0 + np.exp(-z))
    for t in range(T):
        for a in range(1, K):
            assert g[t, a] / g[t, 0] == pytest.approx(s[t, idx[t, a]] / s[t, idx[t, 0]], rel=1e-13)
    # scale enters linearly
    np.testing.assert_allclose(O.gates_for(z, idx, 1.8), g * (1.8 / 2.5), rtol=1e-15, atol=0)
    # the given selection is used as is: select's own choice under a bias that
    # forces experts {1, 4, 6} gives the same gates as the forced selection
    b = np.zeros(E, np.float32)
    b[[1, 4, 6]] = 10.0
    i_b, g_b, _ = O.select(z, b, 3, 2.5)
    np.testing.assert_allclose(O.gates_for(z, i_b, 2.5), g_b, rtol=1e-15, atol=0)
    for bad in (E, -1):
        wrong = idx.copy()
        wrong[3, 2] = bad
        with pytest.raises(ValueError):
            O.gates_for(z, wrong, 2.5)


def test_permute_brute_force_and_invariants():
    rng = np.random.default_rng(11)
    for T, E, K, has_shared in [(37, 8, 3, True), (1, 4, 4, True), (50, 16, 2, False), (0, 8, 2, True)]:
        idx = np.array([rng.permutation(E)[:K] for _ in range(T)], dtype=np.int32).reshape(T, K)
        counts, offsets, srt = O.permute(idx, E, has_shared)
        for g in range(E):
            rows = [t * K + k for t in range(T) for k in range(K) if idx[t, k] == g]
            assert counts[g] == len(rows)
            assert srt[offsets[g]:offsets[g + 1]].tolist() == rows
        assert counts[E] == (T if has_shared else 0)
        if has_shared:
            assert srt[offsets[E]:offsets[E + 1]].tolist() == [T * K + t for t in range(T)]
        assert offsets[0] == 0 and np.all(np.diff(offsets) == counts)
        assert counts[:E].sum() == T * K
        # every assignment appears exactly once
        assert sorted(srt.tolist()) == list(range(T * K + (T if has_shared else 0)))


def test_permute_rejects_out_of_range_ids():
    with pytest.raises(ValueError):
        O.permute(np.array([[0, 9]], dtype=np.int32), 8)


# ---------------------------------------------------------------- invariants

def test_bias_moves_only_the_choice():
    c = small_case(T=64, E=8, K=3)
    z = O.logits(c["x"], c["w_r"])
    E, K = 8, 3
    # force the selection {1, 4, 6} with two different bias magnitudes:
    # the choice is the same and the gates must not move at all
    forced = [1, 4, 6]
    b10 = np.zeros(E, np.float32)
    b10[forced] = 10.0
    b20 = c["b"].copy()
    b20[forced] = 20.0
    i10, g10, _ = O.select(z, b10, K, 2.5)
    i20, g20, _ = O.select(z, b20, K, 2.5)
    assert all(sorted(r) == forced for r in i10.tolist())
    for t in range(z.shape[0]):
        m10 = dict(zip(i10[t].tolist(), g10[t].tolist()))
        m20 = dict(zip(i20[t].tolist(), g20[t].tolist()))
        assert set(m10) == set(m20)
        for e in m10:
            assert m10[e] == pytest.approx(m20[e], rel=1e-15, abs=0)
    # the bias does change the choice for some tokens
    i0, _, _ = O.select(z, np.zeros(E, np.float32), K, 2.5)
    ib, _, _ = O.select(z, c["b"] * 20, K, 2.5)
    assert any(set(a) != set(bb) for a, bb in zip(i0.tolist(), ib.tolist()))


def test_k_equals_e_is_dense_weighted_sum():
    c = small_case(T=16, H=32, I=24, E=6, K=6)
    idx, gate, margin, z = O.route(c["x"], c["w_r"], c["b"], 6, 2.5)
    assert np.all(np.isinf(margin))
    assert all(sorted(r) == list(range(6)) for r in idx.tolist())
    # bias-independent gates: per-expert values identical under another bias
    idx2, gate2, _ = O.select(z, -c["b"], 6, 2.5)
    for t in range(16):
        a = dict(zip(idx[t].tolist(), gate[t].tolist()))
        bb = dict(zip(idx2[t].tolist(), gate2[t].tolist()))
        for e in range(6):
            assert a[e] == pytest.approx(bb[e], rel=1e-15, abs=0)
    # dense sum over ALL experts with G_e = 2.5 s_e / sum_all s  (NumPy float64)
    y = O.forward(c["x"], c["w1"], c["w3"], c["w2"], c["ws1"], c["ws3"], c["ws2"], idx, gate)
    xf = W.bf16_bits_to_f32(c["x"]).astype(np.float64)
    zf = xf @ c["w_r"].astype(np.float64).T
    s = 1.0 / (1.0 + np.exp(-zf))
    G = 2.5 * s / s.sum(axis=1, keepdims=True)
    ref = numpy_swiglu(xf, c["ws1"], c["ws3"], c["ws2"])
    for e in range(6):
        ref = ref + G[:, e:e + 1] * numpy_swiglu(xf, c["w1"][e], c["w3"][e], c["w2"][e])
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-12)


def test_zeroed_routed_weights_leave_only_shared():
    c = small_case()
    idx, gate, _, _ = O.route(c["x"], c["w_r"], c["b"], c["K"], 2.5)
    y, yr, ys, _ = O.forward(c["x"], c["w1"], c["w3"], c["w2"], c["ws1"], c["ws3"], c["ws2"], idx,
                             np.zeros_like(gate), want_parts=True)
    assert np.array_equal(yr, np.zeros_like(yr))
    assert np.array_equal(y, ys)
    xf = W.bf16_bits_to_f32(c["x"]).astype(np.float64)
    np.testing.assert_allclose(ys, numpy_swiglu(xf, c["ws1"], c["ws3"], c["ws2"]), rtol=1e-10,
                               atol=1e-12)


def test_single_expert_unit_gate_is_dense_mlp():
    """E = K = 1, scale 1: the gate is s/s = 1 and the block is one SwiGLU MLP
    (checked with H != I so that a transposed weight cannot pass)."""
    c = small_case(T=20, H=48, I=80, E=1, K=1)
    idx, gate, _, _ = O.route(c["x"], c["w_r"], c["b"], 1, 1.0)
    assert np.all(idx == 0) and np.all(gate == 1.0)
    y = O.forward(c["x"], c["w1"], c["w3"], c["w2"], None, None, None, idx, gate, has_shared=False)
    xf = W.bf16_bits_to_f32(c["x"]).astype(np.float64)
    np.testing.assert_allclose(y, numpy_swiglu(xf, c["w1"][0], c["w3"][0], c["w2"][0]), rtol=1e-10,
                               atol=1e-12)


def test_token_permutation_invariance():
    c = small_case(T=30)
    perm = np.random.default_rng(5).permutation(30)
    idx, gate, margin, _ = O.route(c["x"], c["w_r"], c["b"], c["K"], 2.5)
    idx_p, gate_p, margin_p, _ = O.route(c["x"][perm], c["w_r"], c["b"], c["K"], 2.5)
    assert np.array_equal(idx[perm], idx_p)
    assert np.array_equal(gate[perm], gate_p)
    assert np.array_equal(margin[perm], margin_p)
    y = O.forward(c["x"], c["w1"], c["w3"], c["w2"], c["ws1"], c["ws3"], c["ws2"], idx, gate)
    y_p = O.forward(c["x"][perm], c["w1"], c["w3"], c["w2"], c["ws1"], c["ws3"], c["ws2"], idx_p, gate_p)
    assert np.array_equal(y[perm], y_p)
    # a token subset computes the same rows as the full run
    sub = np.array([29, 3, 3, 17])
    y_s = O.forward(c["x"], c["w1"], c["w3"], c["w2"], c["ws1"], c["ws3"], c["ws2"], idx, gate, tokens=sub)
    assert np.array_equal(y_s, y[sub])


def test_routed_plus_shared_is_output_and_ablation():
    c = small_case(T=32)
    idx, gate, _, _ = O.route(c["x"], c["w_r"], c["b"], c["K"], 2.5)
    y, yr, ys, yk = O.forward(c["x"], c["w1"], c["w3"], c["w2"], c["ws1"], c["ws3"], c["ws2"], idx,
                              gate, want_parts=True)
    np.testing.assert_array_equal(y, yr + ys)
    np.testing.assert_allclose(yr, yk.sum(axis=1), rtol=1e-13, atol=1e-14)
    # ablate expert 3: zero the gate of every slot that chose it, keep the others
    e = 3
    assert np.any(idx == e)
    g_ab = np.where(idx == e, 0.0, gate)
    assert np.all(g_ab.sum(axis=1)[np.any(idx == e, axis=1)] < 2.5)
    y_ab, _, _, yk_ab = O.forward(c["x"], c["w1"], c["w3"], c["w2"], c["ws1"], c["ws3"], c["ws2"], idx,
                                  g_ab, want_parts=True)
    drop = np.where((idx == e)[:, :, None], yk, 0.0).sum(axis=1)
    np.testing.assert_allclose(y - y_ab, drop, rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(np.where((idx == e)[:, :, None], 0.0, yk), yk_ab)


def test_empty_token_batch():
    c = small_case(T=0)
    idx, gate, margin, z = O.route(c["x"], c["w_r"], c["b"], c["K"], 2.5)
    assert idx.shape == (0, c["K"])
    counts, offsets, srt = O.permute(idx, 8)
    assert counts.sum() == 0 and srt.shape == (0,)
    y = O.forward(c["x"], c["w1"], c["w3"], c["w2"], c["ws1"], c["ws3"], c["ws2"], idx, gate)
    assert y.shape == (0, c["x"].shape[1])


# ---------------------------------------------------------------- pre-FFN RMSNorm

def test_rmsnorm_closed_forms():
    """A row of one repeated value c has RMS |c|: out = sign(c) * gamma / sqrt(1 + eps / c^2).
    A row (3, 4) has mean square 12.5."""
    H = 8
    gamma = bf([0.5, 1.0, 2.0, -1.0, 0.25, 4.0, 1.5, -0.75])
    g = W.bf16_bits_to_f32(gamma).astype(np.float64)
    x = bf([[3.0] * H, [-0.5] * H])
    out = O.rmsnorm(x, gamma, 1e-5)
    np.testing.assert_allclose(out[0], g / math.sqrt(1 + 1e-5 / 9.0), rtol=1e-15, atol=0)
    np.testing.assert_allclose(out[1], -g / math.sqrt(1 + 1e-5 / 0.25), rtol=1e-15, atol=0)
    out = O.rmsnorm(bf([[3.0, 4.0]]), bf([1.0, 1.0]), 0.0)
    np.testing.assert_allclose(out[0], [3 / math.sqrt(12.5), 4 / math.sqrt(12.5)], rtol=1e-15)


def test_rmsnorm_scale_invariance_and_unit_rms():
    rng = np.random.default_rng(9)
    x = W.f32_to_bf16_bits(rng.standard_normal((6, 64), dtype=np.float32))
    ones = bf([1.0] * 64)
    out = O.rmsnorm(x, ones, 0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(out ** 2, axis=1)), 1.0, rtol=1e-14)
    x4 = W.f32_to_bf16_bits(W.bf16_bits_to_f32(x) * np.float32(4.0))  # exact: power of two
    np.testing.assert_allclose(O.rmsnorm(x4, ones, 0.0), out, rtol=1e-14, atol=0)
