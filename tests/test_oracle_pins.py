"""Pins of the fp64 oracle against things other than itself.

Each test ties one oracle function to a closed form, a brute-force
enumeration, a special case that reduces to a textbook routine, or an
invariant fixed by "Mixtral of Experts" §2.1, so that a plausible slip in
the oracle (a dropped term, a wrong sign or index, swapped W1/W3, a
transposed operand, a softmax over all experts, the wrong tie rule) fails
one of them.
"""

import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
from scipy.special import expit, softmax

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_layer(rng, T, d, f, E, scale=1.0):
    x = rng.standard_normal((T, d)) * scale
    Wg = rng.standard_normal((E, d)) / math.sqrt(d)
    W1 = rng.standard_normal((E, f, d)) / math.sqrt(d)
    W3 = rng.standard_normal((E, f, d)) / math.sqrt(d)
    W2 = rng.standard_normal((E, d, f)) / math.sqrt(f)
    return x, Wg, W1, W3, W2


def dense_swiglu_loops(xrow, W1, W3, W2):
    """Textbook SwiGLU FFN, plain Python loops, SiLU via scipy's logistic:
    out_i = sum_j W2[i, j] * silu(sum_c W1[j, c] x_c) * (sum_c W3[j, c] x_c)."""
    f, d = W1.shape
    g = []
    for j in range(f):
        a = math.fsum(W1[j, c] * xrow[c] for c in range(d))
        b = math.fsum(W3[j, c] * xrow[c] for c in range(d))
        g.append(a * float(expit(a)) * b)
    return np.array([math.fsum(W2[i, j] * g[j] for j in range(f)) for i in range(d)])


# --------------------------------------------------------------------------
# Worked example with a closed form (tests/golden/worked_example.json)

def test_worked_example_closed_form():
    ex = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    sigma = lambda z: 1.0 / (1.0 + math.exp(-z))  # noqa: E731
    env = {"sigma": sigma}
    x = np.array([ex["x"]])
    y, idx, w = oracle.moe_forward(x, np.array(ex["Wg"]), np.array(ex["W1"]), np.array(ex["W3"]),
                                   np.array(ex["W2"]), ex["k"])
    assert idx[0].tolist() == ex["idx"]
    w_ref = [eval(s, env) for s in ex["w_closed_form"]]
    y_ref = [eval(s, env) for s in ex["y_closed_form"]]
    np.testing.assert_allclose(w[0], w_ref, rtol=1e-15, atol=0)
    np.testing.assert_allclose(y[0], y_ref, rtol=1e-14, atol=0)


# --------------------------------------------------------------------------
# Router logits

def test_router_logits_exact_sum_within_bound():
    """bf16 inputs: every product is exact, so the exact logit is a rational
    number; the oracle's fp64 sum must be within the summation-error bound of
    it (and that bound is tiny)."""
    rng = np.random.default_rng(1)
    x = synth.bf16_bits_to_f64(synth.bf16_round_bits(rng.standard_normal((3, 96)).astype(np.float32)))
    Wg = synth.bf16_bits_to_f64(synth.bf16_round_bits((rng.standard_normal((5, 96)) / 10).astype(np.float32)))
    lg = oracle.router_logits(x, Wg)
    bound = oracle.logit_sum_bound(x, Wg)
    for t in range(3):
        for e in range(5):
            exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(x[t], Wg[e]))
            assert abs(Fraction(float(lg[t, e])) - exact) <= Fraction(float(bound[t, e]))
    assert float(bound.max()) < 1e-12


def test_logit_sum_bound_is_gamma_d_minus_1_times_the_absolute_sum():
    """The near-tie bound against Higham's gamma_{d-1} * sum_i |x_i Wg[e, i]|
    (Accuracy and Stability of Numerical Algorithms, §4.2), worked by hand in
    exact rationals for d = 3: n = d - 1 = 2 and gamma_2 = 2u / (1 - 2u),
    u = 2^-53.  Products (x, Wg rows below):
      token 0, expert 0: |1.5*0.5| + |-2*3| + |0.25*-4|   = 0.75 + 6 + 1     = 31/4
      token 0, expert 1: |1.5*-1| + |-2*0.125| + |0.25*2| = 1.5 + 0.25 + 0.5 = 9/4
      token 1, expert 0: |0.5*0.5| + |0*3| + |-8*-4|      = 0.25 + 0 + 32    = 129/4
      token 1, expert 1: |0.5*-1| + |0*0.125| + |-8*2|    = 0.5 + 0 + 16     = 33/2
    A wrong n (d instead of d - 1), a missing absolute value, a transposed
    operand or a slip of the unit roundoff all miss by far more than the
    few ulps of the fp64 evaluation allowed here."""
    x = np.array([[1.5, -2.0, 0.25], [0.5, 0.0, -8.0]])
    Wg = np.array([[0.5, 3.0, -4.0], [-1.0, 0.125, 2.0]])
    u = Fraction(1, 2 ** 53)
    gamma2 = 2 * u / (1 - 2 * u)
    sums = [[Fraction(31, 4), Fraction(9, 4)], [Fraction(129, 4), Fraction(33, 2)]]
    got = oracle.logit_sum_bound(x, Wg)
    assert got.shape == (2, 2)
    for t in range(2):
        for e in range(2):
            exact = gamma2 * sums[t][e]
            assert abs(Fraction(float(got[t, e])) - exact) <= exact * Fraction(1, 2 ** 50), (t, e)


def test_router_logits_orientation():
    """Wg is stored (n_experts, dim): logit e uses row e.  A transposed or
    mis-indexed router fails on a one-hot x."""
    Wg = np.arange(12, dtype=np.float64).reshape(3, 4)
    for i in range(4):
        x = np.zeros((1, 4))
        x[0, i] = 1.0
        np.testing.assert_array_equal(oracle.router_logits(x, Wg)[0], Wg[:, i])


# --------------------------------------------------------------------------
# TopK and the kept softmax

def test_topk_pair_brute_force():
    """For K = 2 the kept set is the pair with the largest logit sum; slot 0
    holds the larger logit.  Enumerate all C(E, 2) pairs."""
    rng = np.random.default_rng(2)
    for _ in range(300):
        E = int(rng.integers(2, 10))
        lg = rng.standard_normal((1, E))
        idx = oracle.topk_lower_index(lg, 2)[0]
        best = max(itertools.combinations(range(E), 2), key=lambda p: lg[0, p[0]] + lg[0, p[1]])
        assert set(idx.tolist()) == set(best)
        assert lg[0, idx[0]] >= lg[0, idx[1]]


def test_topk_general_k_is_sorted_prefix():
    rng = np.random.default_rng(3)
    lg = rng.standard_normal((50, 8))
    for k in range(1, 9):
        idx = oracle.topk_lower_index(lg, k)
        ref = np.argsort(-lg, axis=1, kind="stable")[:, :k]
        np.testing.assert_array_equal(idx, ref)


def test_tie_rules():
    # x = 0: all logits are 0, so experts 0 and 1 with weights 1/2.
    x = np.zeros((2, 8))
    Wg = np.random.default_rng(4).standard_normal((8, 8))
    idx, w, _ = oracle.route(x, Wg, 2)
    assert idx.tolist() == [[0, 1], [0, 1]]
    np.testing.assert_array_equal(w, 0.5)
    # Two identical dominant router rows: the lower index takes slot 0.
    Wg = np.zeros((8, 4))
    Wg[5] = Wg[3] = [1.0, 2.0, 3.0, 4.0]
    idx, w, _ = oracle.route(np.ones((1, 4)), Wg, 2)
    assert idx[0].tolist() == [3, 5]
    np.testing.assert_array_equal(w, 0.5)
    # A three-way tie for the top: the two lowest indices win.
    Wg = np.zeros((6, 2))
    Wg[[1, 2, 4]] = [1.0, 1.0]
    idx, _, _ = oracle.route(np.ones((1, 2)), Wg, 2)
    assert idx[0].tolist() == [1, 2]


def test_router_scale_and_relabel_invariance():
    rng = np.random.default_rng(5)
    x, Wg, *_ = rand_layer(rng, 40, 16, 4, 8)
    idx, w, _ = oracle.route(x, Wg, 2)
    idx2, _, _ = oracle.route(x, 4.0 * Wg, 2)  # positive scaling: power of 2, exact
    np.testing.assert_array_equal(idx, idx2)
    perm = rng.permutation(8)  # expert e of the new router is old expert perm[e]
    idx3, w3, _ = oracle.route(x, Wg[perm], 2)
    np.testing.assert_array_equal(perm[idx3], idx)
    np.testing.assert_allclose(w3, w, rtol=1e-15)


def test_kept_softmax_closed_forms():
    rng = np.random.default_rng(6)
    lg = rng.standard_normal((200, 8)) * 3
    idx = oracle.topk_lower_index(lg, 2)
    w = oracle.kept_softmax(lg, idx)
    l0 = lg[np.arange(200), idx[:, 0]]
    l1 = lg[np.arange(200), idx[:, 1]]
    np.testing.assert_allclose(w[:, 0], expit(l0 - l1), rtol=1e-15)   # w0 = sigma(l0 - l1)
    np.testing.assert_allclose(w[:, 1], expit(l1 - l0), rtol=1e-14)
    assert (w > 0).all()
    assert np.abs(w.sum(1) - 1).max() <= 4e-16
    assert (w[:, 0] >= w[:, 1]).all()
    # K = E: the kept softmax is the ordinary softmax over all experts.
    idx8 = oracle.topk_lower_index(lg, 8)
    w8 = oracle.kept_softmax(lg, idx8)
    np.testing.assert_allclose(w8, np.take_along_axis(softmax(lg, axis=1), idx8.astype(np.int64), 1),
                               rtol=1e-13)
    # K = 1: the single kept weight is exactly 1.
    idx1 = oracle.topk_lower_index(lg, 1)
    np.testing.assert_array_equal(oracle.kept_softmax(lg, idx1), 1.0)


def test_softmax_not_over_all_experts():
    """Pitfalls, renormalised top-2 weights: a softmax over all eight logits
    followed by picking two would not sum to 1."""
    lg = np.array([[2.0, 1.0, 0.5, 0.0, 0.0, 0.0, 0.0, 0.0]])
    w = oracle.kept_softmax(lg, oracle.topk_lower_index(lg, 2))
    assert abs(w.sum() - 1) < 1e-15
    assert abs(w[0, 0] - 1 / (1 + math.exp(-1))) < 1e-15


# --------------------------------------------------------------------------
# SwiGLU experts and the combine

def test_single_expert_is_dense_swiglu():
    """E = 1, K = 1: the layer is a dense SwiGLU FFN, computed here with
    plain loops and scipy's logistic function."""
    rng = np.random.default_rng(7)
    x, Wg, W1, W3, W2 = rand_layer(rng, 5, 6, 10, 1)
    y, idx, w = oracle.moe_forward(x, Wg, W1, W3, W2, 1)
    assert (idx == 0).all() and (w == 1.0).all()
    for t in range(5):
        np.testing.assert_allclose(y[t], dense_swiglu_loops(x[t], W1[0], W3[0], W2[0]), rtol=1e-12, atol=1e-14)


def test_swiglu_gate_and_up_not_swapped():
    """SiLU acts on W1 x, not on W3 x: a case where the two differ in sign."""
    x = np.array([[1.0]])
    W1 = np.array([[3.0]])
    W3 = np.array([[-2.0]])
    W2 = np.array([[1.0]])
    got = oracle.swiglu_expert(x, W1, W3, W2)[0, 0]
    assert abs(got - 3.0 * expit(3.0) * -2.0) < 1e-14


def test_identical_experts_give_single_expert_output():
    """If all experts are equal the gate weights (summing to 1) drop out:
    y = Expert(x) whatever the routing (§2.1, displays 1-3)."""
    rng = np.random.default_rng(8)
    x, Wg, W1, W3, W2 = rand_layer(rng, 20, 12, 24, 8)
    W1[:] = W1[0]
    W3[:] = W3[0]
    W2[:] = W2[0]
    y, idx, _ = oracle.moe_forward(x, Wg, W1, W3, W2, 2)
    assert len(set(map(tuple, idx.tolist()))) > 3  # routing really varies
    np.testing.assert_allclose(y, oracle.swiglu_expert(x, W1[0], W3[0], W2[0]), rtol=1e-13, atol=1e-14)


def test_layer_brute_force_over_pairs():
    """y = sum over all pairs {i < j} of [pair kept] (sigma(l_i - l_j) E_i(x)
    + sigma(l_j - l_i) E_j(x)), each expert evaluated with plain loops."""
    rng = np.random.default_rng(9)
    E, d, f = 5, 4, 6
    x, Wg, W1, W3, W2 = rand_layer(rng, 6, d, f, E)
    y, _, _ = oracle.moe_forward(x, Wg, W1, W3, W2, 2)
    for t in range(6):
        lg = [math.fsum(x[t, c] * Wg[e, c] for c in range(d)) for e in range(E)]
        best = max(itertools.combinations(range(E), 2), key=lambda p: lg[p[0]] + lg[p[1]])
        ref = np.zeros(d)
        for (i, j) in itertools.combinations(range(E), 2):
            if (i, j) != best:
                continue
            ref += float(expit(lg[i] - lg[j])) * dense_swiglu_loops(x[t], W1[i], W3[i], W2[i])
            ref += float(expit(lg[j] - lg[i])) * dense_swiglu_loops(x[t], W1[j], W3[j], W2[j])
        np.testing.assert_allclose(y[t], ref, rtol=1e-12, atol=1e-14)


def test_linearity_in_w2_and_token_independence():
    rng = np.random.default_rng(10)
    x, Wg, W1, W3, W2 = rand_layer(rng, 12, 8, 16, 8)
    y, _, _ = oracle.moe_forward(x, Wg, W1, W3, W2, 2)
    y2, _, _ = oracle.moe_forward(x, Wg, W1, W3, 2.0 * W2, 2)
    np.testing.assert_allclose(y2, 2.0 * y, rtol=1e-15)
    # Tokens are independent: a subset gives the same rows.
    # (BLAS may block a 3-row product differently from a 12-row one, so the
    # rows agree to rounding, not bit for bit.)
    ys, _, _ = oracle.moe_forward(x, Wg, W1, W3, W2, 2, tokens=[3, 7, 11])
    np.testing.assert_allclose(ys, y[[3, 7, 11]], rtol=1e-13, atol=1e-15)


def test_k_equals_e_is_dense_softmax_mixture():
    """K = E: every expert contributes with the full softmax weight."""
    rng = np.random.default_rng(11)
    E = 4
    x, Wg, W1, W3, W2 = rand_layer(rng, 3, 5, 7, E)
    y, _, _ = oracle.moe_forward(x, Wg, W1, W3, W2, E)
    p = softmax(x @ Wg.T, axis=1)
    ref = sum(p[:, e:e + 1] * oracle.swiglu_expert(x, W1[e], W3[e], W2[e]) for e in range(E))
    np.testing.assert_allclose(y, ref, rtol=1e-12)


# --------------------------------------------------------------------------
# Permutation

@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (37, 8, 2), (200, 8, 1), (64, 3, 3), (500, 64, 2)])
def test_permute_matches_stable_sort(T, E, k):
    rng = np.random.default_rng(T * 131 + E)
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    off, perm, inv = oracle.permute(idx, E)
    flat = idx.ravel()
    np.testing.assert_array_equal(perm, np.argsort(flat, kind="stable"))
    np.testing.assert_array_equal(off, np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))]))
    np.testing.assert_array_equal(inv[perm], np.arange(T * k))
    for e in range(E):
        blk = perm[off[e]:off[e + 1]]
        assert (flat[blk] == e).all() and (np.diff(blk) > 0).all()


def test_permute_empty_experts_and_single_expert():
    idx = np.array([[2, 5], [5, 2], [2, 5]], dtype=np.int32)
    off, perm, inv = oracle.permute(idx, 8)
    assert off.tolist() == [0, 0, 0, 3, 3, 3, 6, 6, 6]
    assert perm.tolist() == [0, 3, 4, 1, 2, 5]
    off, perm, inv = oracle.permute(np.zeros((4, 1), dtype=np.int32), 1)
    assert off.tolist() == [0, 4] and perm.tolist() == [0, 1, 2, 3]


# --------------------------------------------------------------------------
# Workload recipe checks (tab. 1 dims, tab. 5 uniform-routing baselines)

def test_mixtral_parameter_counts_from_table_1():
    """Tab. 1 dims give about 47B stored and 13B active parameters (§3)."""
    s = synth.CONFIGS["prefill"]
    layers, vocab, heads, kv, hd = 32, 32000, 32, 8, 128
    attn = s.d * heads * hd * 2 + s.d * kv * hd * 2
    expert = 3 * s.d * s.f
    norms = 2 * s.d
    per_layer_total = attn + s.E * expert + s.E * s.d + norms
    per_layer_active = attn + s.k * expert + s.E * s.d + norms
    total = layers * per_layer_total + 2 * vocab * s.d + s.d
    active = layers * per_layer_active + 2 * vocab * s.d + s.d
    assert abs(total / 1e9 - 46.7) < 0.05 and abs(active / 1e9 - 12.9) < 0.05


def test_routing_stats_hand_counted():
    idx = np.array([[0, 1], [1, 2], [3, 4], [3, 0], [5, 6], [6, 5]])
    st = oracle.routing_stats(idx, 8)
    # loads 0:2 1:2 2:1 3:2 4:1 5:2 6:2 7:0; first-choice repeats: (3,3) only;
    # overlapping pairs: {1,2}&{0,1}, {3,0}&{3,4}, {6,5}&{5,6}; 5 pairs
    assert st.tolist() == [2, 2, 1, 2, 1, 2, 2, 0, 1, 3, 5]
    # sequences of 3 tokens: pairs (0,1),(1,2),(3,4),(4,5); the (2,3) pair is dropped
    st3 = oracle.routing_stats(idx, 8, seq_len=3)
    assert st3.tolist()[8:] == [0, 2, 4]


@pytest.mark.parametrize("E,k", [(8, 2), (8, 1), (16, 3), (4, 2)])
def test_routing_stats_uniform_closed_forms(E, k):
    """Uniformly random ordered k-subsets: first choices agree with rate 1/E
    and kept sets meet with rate 1 - C(E-k, k)/C(E, k)."""
    rng = np.random.default_rng(E * 10 + k)
    T = 20000
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)])
    st = oracle.routing_stats(idx, E)
    n = st[E + 2]
    p1 = 1.0 / E
    p2 = 1.0 - math.comb(E - k, k) / math.comb(E, k)
    assert n == T - 1 and st[:E].sum() == T * k
    assert abs(st[E] / n - p1) < 4 * math.sqrt(p1 * (1 - p1) / n)
    assert abs(st[E + 1] / n - p2) < 4 * math.sqrt(p2 * (1 - p2) / n)


def test_uniform_routing_baselines_on_synthetic_router():
    """With Wg ~ N(0, 1/d) the synthetic router is close to uniform: the first
    choice repeats on consecutive tokens about 1/8 of the time and the kept
    pairs overlap about 1 - C(6,2)/C(8,2) = 13/28 of the time (the uniform
    baselines quoted with tab. 5)."""
    s = synth.MoEShape("stat", 4096, 256, 8, 8, 2, "bf16")
    t = synth.host_inputs(s, seed=3, with_experts=False)
    idx, _, _ = oracle.route(synth.bf16_bits_to_f64(t["x"]), synth.bf16_bits_to_f64(t["Wg"]), 2)
    st = oracle.routing_stats(idx, 8)
    n = st[10]
    first, overlap = st[8] / n, st[9] / n
    assert abs(first - 1 / 8) < 4 * math.sqrt(1 / 8 * 7 / 8 / n)
    assert abs(overlap - 13 / 28) < 4 * math.sqrt(13 / 28 * 15 / 28 / n)
    load = st[:8] / idx.size
    assert np.abs(load - 1 / 8).max() < 0.03


@pytest.mark.slow
def test_skewed_recipe_hottest_share():
    """The skewed workload (seed 0, T = 16384) gives expert 0 35% of the
    assignments, as calibrated by tests/golden/calibrate_skew.py."""
    s = synth.CONFIGS["skewed"]
    t = synth.host_inputs(s, seed=0, with_experts=False)
    idx, _, _ = oracle.route(synth.bf16_bits_to_f64(t["x"]), synth.bf16_bits_to_f64(t["Wg"]), 2)
    share = np.bincount(idx.ravel(), minlength=8) / idx.size
    assert abs(share[0] - 0.35) < 0.005
    assert (np.diff(share) < 0).all()  # Zipf-shaped: monotone decreasing load
