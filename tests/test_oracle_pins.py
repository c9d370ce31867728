"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each check is chosen so that a plausible slip in the oracle (a dropped term,
a wrong sign or index, a transposed operand, a wrong tie rule) fails it:
brute force over all subsets on tiny inputs, hand-derived worked examples in
tests/golden/, closed forms evaluated with pure-Python math, invariants and
special cases that reduce to a textbook MLP.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
from grouped_gemm_gating_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bits(a):
    return W.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


# ---------------------------------------------------------------- bf16 ----

def test_bf16_decode_known_patterns():
    assert oracle.bf16_to_f64(np.array([0x3F80], np.uint16))[0] == 1.0
    assert oracle.bf16_to_f64(np.array([0xC000], np.uint16))[0] == -2.0
    assert oracle.bf16_to_f64(np.array([0x3F81], np.uint16))[0] == 1.0078125
    assert oracle.bf16_to_f64(np.array([0x0000], np.uint16))[0] == 0.0


# ---------------------------------------------------------------- route ---

def _beats(li, i, lj, j):
    """Selection key: larger logit first, then lower index."""
    return li > lj or (li == lj and i < j)


def _brute_topk(vals, cand, k):
    """Unique k-subset of cand whose every member beats every non-member."""
    winners = []
    for sub in itertools.combinations(cand, k):
        rest = [c for c in cand if c not in sub]
        if all(_beats(vals[a], a, vals[b], b) for a in sub for b in rest):
            winners.append(set(sub))
    assert len(winners) == 1
    return winners[0]


def _check_selection_order(vals, ids):
    for a, b in zip(ids[:-1], ids[1:]):
        assert _beats(vals[a], a, vals[b], b)


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("E,k", [(4, 1), (5, 2), (6, 3), (8, 4), (7, 7)])
def test_route_matches_bruteforce_subsets(seed, E, k):
    rng = np.random.default_rng(seed)
    T = 5
    lg = rng.standard_normal((T, E)).astype(np.float32)
    if seed % 2:
        lg = W.tie_logits(T, E, seed, levels=2)
    ids, _ = oracle.route(lg, k)
    for t in range(T):
        vals = [float(v) for v in lg[t]]
        assert set(ids[t].tolist()) == _brute_topk(vals, list(range(E)), k)
        _check_selection_order(vals, ids[t].tolist())


def _brute_group_scores(vals, n_group, score):
    gs = len(vals) // n_group
    out = []
    for g in range(n_group):
        grp = sorted(vals[g * gs:(g + 1) * gs], reverse=True)
        if score == oracle.GROUP_MAX:
            out.append(grp[0])
        else:
            out.append(float(np.float32(grp[0]) + np.float32(grp[1])))
    return out


@pytest.mark.parametrize("score", [oracle.GROUP_MAX, oracle.GROUP_TOP2SUM])
@pytest.mark.parametrize("seed", range(8))
def test_route_grouped_matches_bruteforce(seed, score):
    E, n_group, topk_group, k = 8, 4, 2, 3
    rng = np.random.default_rng(100 + seed)
    lg = rng.standard_normal((4, E)).astype(np.float32)
    if seed % 3 == 0:
        lg = W.tie_logits(4, E, seed, levels=3)
    ids, _ = oracle.route(lg, k, n_group, topk_group, score)
    gsz = E // n_group
    for t in range(lg.shape[0]):
        vals = [float(v) for v in lg[t]]
        gsc = _brute_group_scores(vals, n_group, score)
        groups = _brute_topk(gsc, list(range(n_group)), topk_group)
        cand = [e for e in range(E) if e // gsz in groups]
        assert set(ids[t].tolist()) == _brute_topk(vals, cand, k)
        _check_selection_order(vals, ids[t].tolist())


def test_route_grouped_golden():
    with open(os.path.join(GOLDEN, "route_groups_tiny.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        lg = np.array([c["logits"]], dtype=np.float32)
        ids, w = oracle.route(lg, c["k"], c["n_group"], c["topk_group"], c["group_score"])
        assert ids[0].tolist() == c["ids"], c["why"]
        assert abs(w.sum() - 1.0) < 1e-12


def test_route_all_equal_logits():
    lg = np.zeros((3, 16), np.float32)
    ids, w = oracle.route(lg, 4)
    assert (ids == np.arange(4)).all()
    assert np.allclose(w, 0.25, rtol=0, atol=1e-15)


def test_route_renormalised_weights_closed_form():
    rng = np.random.default_rng(7)
    lg = rng.standard_normal((6, 10)).astype(np.float32)
    for scaling in (1.0, 2.5):
        ids, w = oracle.route(lg, 3, routed_scaling=scaling)
        for t in range(6):
            chosen = [float(lg[t, e]) for e in ids[t]]
            for j, lj in enumerate(chosen):
                # w_j = 1 / sum_i exp(l_i - l_j): no max shift, pure Python
                ref = scaling / sum(math.exp(li - lj) for li in chosen)
                assert abs(w[t, j] - ref) <= 1e-14 * max(1.0, ref)
            assert abs(w[t].sum() - scaling) < 1e-12


def test_route_full_softmax_weights_closed_form():
    rng = np.random.default_rng(8)
    lg = rng.standard_normal((4, 6)).astype(np.float32)
    ids, w = oracle.route(lg, 2, renormalize=False, routed_scaling=1.5)
    for t in range(4):
        z = sum(math.exp(float(v)) for v in lg[t])
        for j in range(2):
            ref = 1.5 * math.exp(float(lg[t, ids[t, j]])) / z
            assert abs(w[t, j] - ref) < 1e-14
    ids, w = oracle.route(lg, 6, renormalize=False)
    assert np.allclose(w.sum(1), 1.0, atol=1e-12)


def test_route_trivial_grouping_equals_ungrouped():
    rng = np.random.default_rng(9)
    lg = rng.standard_normal((20, 12)).astype(np.float32)
    a = oracle.route(lg, 4)
    b = oracle.route(lg, 4, n_group=1, topk_group=1)
    c = oracle.route(lg, 4, n_group=4, topk_group=4)
    for o in (b, c):
        assert (a[0] == o[0]).all() and np.array_equal(a[1], o[1])


# ---------------------------------------------------------------- align ---

def test_align_golden():
    with open(os.path.join(GOLDEN, "align_tiny.json")) as f:
        g = json.load(f)
    ids = np.array(g["topk_ids"], np.int32)
    st, ex, n, inv = oracle.align(ids, g["E"], g["block_m"])
    assert st.tolist() == g["sorted_token_ids"]
    assert ex.tolist() == g["expert_ids"]
    assert n == g["num_tokens_post_padded"]
    assert inv.tolist() == g["inv_pos"]
    S = ids.size
    assert [int(s) // g["k"] for s in st if s < S] == g["token_of_sorted_valid"]


def _check_align_invariants(ids, E, bm, st, ex, n, inv):
    T, k = ids.shape
    S = T * k
    flat = ids.reshape(-1)
    counts = np.bincount(flat, minlength=E) if S else np.zeros(E, np.int64)
    assert n == sum((int(c) + bm - 1) // bm * bm for c in counts)
    assert st.shape[0] == oracle.max_padded(T, k, E, bm)
    valid = st[st < S]
    assert sorted(valid.tolist()) == list(range(S))          # each slot once
    assert (st[st >= S] == S).all()                           # sentinel = S
    assert (st[n:] == S).all() and (ex[n // bm:] == -1).all()
    live = ex[: n // bm]
    assert (np.diff(live) >= 0).all()                         # non-decreasing
    assert sorted(set(live.tolist())) == [e for e in range(E) if counts[e] > 0]
    for p in range(n):
        if st[p] < S:
            assert flat[st[p]] == ex[p // bm]                    # block expert
            assert inv[st[p]] == p                               # inverse map
            t, j = divmod(int(st[p]), k)                         # slot // top_k
            assert ids[t, j] == ex[p // bm]
    # stable: the valid entries in order equal a stable argsort of the ids
    assert (valid == np.argsort(flat, kind="stable")).all()


@pytest.mark.parametrize("bm", [1, 4, 16, 128])
@pytest.mark.parametrize("case", ["uniform", "skew", "ties_many_empty"])
def test_align_invariants(bm, case):
    T, E, k = 37, 24, 4
    if case == "uniform":
        ids = W.random_topk_ids(T, E, k, seed=bm)
    elif case == "skew":
        ids = W.random_topk_ids(T, E, k, seed=bm + 1, skew=30.0)
    else:
        ids = W.random_topk_ids(T, 8, k, seed=bm + 2)     # experts 8..23 empty
    st, ex, n, inv = oracle.align(ids, E, bm)
    _check_align_invariants(ids, E, bm, st, ex, n, inv)


def test_align_empty():
    ids = np.zeros((0, 2), np.int32)
    st, ex, n, inv = oracle.align(ids, 8, 16)
    assert n == 0 and inv.size == 0
    assert (st == 0).all() and (ex == -1).all()


# -------------------------------------------------------------- forward ---

def _py_silu(z):
    return z / (1.0 + math.exp(-z))


def _py_mlp(xrow, w13, w2, act):
    """Textbook expert MLP in pure Python over decoded bf16 values."""
    W1 = oracle.bf16_to_f64(w13).tolist()
    W2 = oracle.bf16_to_f64(w2).tolist()
    d, F = len(W2), len(W2[0])
    if act == oracle.ACT_SWIGLU:
        g = [sum(W1[f][i] * xrow[i] for i in range(d)) for f in range(F)]
        u = [sum(W1[F + f][i] * xrow[i] for i in range(d)) for f in range(F)]
        h = [_py_silu(g[f]) * u[f] for f in range(F)]
    else:
        a = [sum(W1[f][i] * xrow[i] for i in range(d)) for f in range(F)]
        h = [max(v, 0.0) ** 2 for v in a]
    return [sum(W2[c][f] * h[f] for f in range(F)) for c in range(d)]


def _tiny(seed, T, d, F, E, act=oracle.ACT_SWIGLU, std=0.3):
    rng = np.random.default_rng(seed)
    n1 = 2 * F if act == oracle.ACT_SWIGLU else F
    x = _bits(rng.standard_normal((T, d)))
    w13 = _bits(std * rng.standard_normal((E, n1, d)))
    w2 = _bits(std * rng.standard_normal((E, d, F)))
    return x, w13, w2


@pytest.mark.parametrize("act", [oracle.ACT_SWIGLU, oracle.ACT_RELU2])
def test_forward_single_expert_is_textbook_mlp(act):
    x, w13, w2 = _tiny(1, T=3, d=6, F=5, E=1, act=act)
    ids = np.zeros((3, 1), np.int32)
    w = np.ones((3, 1))
    out = oracle.forward(x, w13, w2, ids, w, act)
    xs = oracle.bf16_to_f64(x).tolist()
    for t in range(3):
        ref = _py_mlp(xs[t], w13[0], w2[0], act)
        assert np.allclose(out[t], ref, rtol=1e-12, atol=1e-12)


def test_forward_k_equals_E_is_dense_softmax_mixture():
    T, d, F, E = 4, 5, 3, 4
    x, w13, w2 = _tiny(2, T, d, F, E)
    lg = np.random.default_rng(3).standard_normal((T, E)).astype(np.float32)
    ids, w = oracle.route(lg, E, renormalize=False)
    out = oracle.forward(x, w13, w2, ids, w, oracle.ACT_SWIGLU)
    xs = oracle.bf16_to_f64(x).tolist()
    for t in range(T):
        z = sum(math.exp(float(v)) for v in lg[t])
        ref = [0.0] * d
        for e in range(E):                       # every expert, no routing
            p = math.exp(float(lg[t, e])) / z
            y = _py_mlp(xs[t], w13[e], w2[e], oracle.ACT_SWIGLU)
            ref = [r + p * yi for r, yi in zip(ref, y)]
        assert np.allclose(out[t], ref, rtol=1e-11, atol=1e-12)


def test_forward_relu2_negative_preactivation_is_zero():
    rng = np.random.default_rng(4)
    x = _bits(np.abs(rng.standard_normal((5, 8))) + 0.1)
    w13 = _bits(-np.abs(rng.standard_normal((3, 4, 8))) - 0.1)
    w2 = _bits(rng.standard_normal((3, 8, 4)))
    ids = W.random_topk_ids(5, 3, 2, seed=4)
    out = oracle.forward(x, w13, w2, ids, np.ones((5, 2)), oracle.ACT_RELU2)
    assert (out == 0.0).all()


def test_forward_token_permutation_equivariance():
    T, d, F, E, k = 9, 16, 8, 6, 2
    x, w13, w2 = _tiny(5, T, d, F, E)
    lg = np.random.default_rng(5).standard_normal((T, E)).astype(np.float32)
    ids, w = oracle.route(lg, k)
    out = oracle.forward(x, w13, w2, ids, w, oracle.ACT_SWIGLU)
    perm = np.random.default_rng(6).permutation(T)
    out_p = oracle.forward(x[perm], w13, w2, ids[perm], w[perm], oracle.ACT_SWIGLU)
    assert np.allclose(out_p, out[perm], rtol=1e-12, atol=1e-14)


def test_forward_expert_relabel_invariance():
    T, d, F, E, k = 7, 12, 8, 5, 2
    x, w13, w2 = _tiny(7, T, d, F, E)
    lg = np.random.default_rng(8).standard_normal((T, E)).astype(np.float32)
    ids, w = oracle.route(lg, k)
    out = oracle.forward(x, w13, w2, ids, w, oracle.ACT_SWIGLU)
    perm = np.random.default_rng(9).permutation(E)      # new id of old expert e
    inv = np.argsort(perm)
    lg2 = lg[:, inv]                                      # column perm[e] holds old e
    ids2, w2r = oracle.route(lg2, k)
    assert (ids2 == perm[ids]).all()
    out2 = oracle.forward(x, w13[inv], w2[inv], ids2, w2r, oracle.ACT_SWIGLU)
    assert np.allclose(out2, out, rtol=1e-12, atol=1e-14)


def test_forward_scaling_w2_doubles_exactly():
    T, d, F, E, k = 6, 8, 4, 4, 2
    x, w13, w2 = _tiny(10, T, d, F, E)
    ids = W.random_topk_ids(T, E, k, seed=10)
    w = np.random.default_rng(10).random((T, k))
    out = oracle.forward(x, w13, w2, ids, w, oracle.ACT_SWIGLU)
    w2x2 = _bits(2.0 * oracle.bf16_to_f64(w2))
    out2 = oracle.forward(x, w13, w2x2, ids, w, oracle.ACT_SWIGLU)
    assert np.array_equal(out2, 2.0 * out)


def test_forward_weights_land_on_their_own_rows():
    """Only slot (t, j) carries weight: out[t] = that expert's output only."""
    T, d, F, E, k = 3, 6, 4, 4, 2
    x, w13, w2 = _tiny(11, T, d, F, E)
    ids = np.array([[0, 1], [2, 3], [1, 3]], np.int32)
    w = np.array([[0.0, 1.0], [1.0, 0.0], [0.0, 0.5]])
    out = oracle.forward(x, w13, w2, ids, w, oracle.ACT_SWIGLU)
    xs = oracle.bf16_to_f64(x).tolist()
    assert np.allclose(out[0], _py_mlp(xs[0], w13[1], w2[1], 0), rtol=1e-12)
    assert np.allclose(out[1], _py_mlp(xs[1], w13[2], w2[2], 0), rtol=1e-12)
    assert np.allclose(out[2], [0.5 * v for v in _py_mlp(xs[2], w13[3], w2[3], 0)], rtol=1e-12)


def test_forward_shared_expert_adds_dense_mlp():
    T, d, F, E, k = 4, 6, 3, 3, 1
    x, w13, w2 = _tiny(12, T, d, F, E)
    xs_, w13s, w2s = _tiny(13, 1, d, F, 1)
    ids = W.random_topk_ids(T, E, k, seed=12)
    w = np.ones((T, k))
    base = oracle.forward(x, w13, w2, ids, w, 0)
    both = oracle.forward(x, w13, w2, ids, w, 0, w13s, w2s)
    xs = oracle.bf16_to_f64(x).tolist()
    for t in range(T):
        assert np.allclose(both[t] - base[t], _py_mlp(xs[t], w13s[0], w2s[0], 0),
                           rtol=1e-10, atol=1e-12)


def test_workload_tiny_route_and_forward_are_sane():
    inp = W.make_inputs(W.CONFIGS["tiny"])
    c = inp.cfg
    ids, w = oracle.route(inp.logits, c.k)
    out = oracle.forward(inp.x, inp.w13, inp.w2, ids, w, c.act)
    rms = float(np.sqrt((out ** 2).mean()))
    assert 1e-3 < rms < 10.0


# ------------------------------------------------------------ router -----

def test_router_one_hot_tokens_read_out_weight_columns():
    """A token that is the i-th unit vector scores expert e with W_g[e, i]."""
    rng = np.random.default_rng(31)
    E, d = 5, 64
    w = _bits(rng.normal(0.0, 0.5, (E, d)))
    x = np.zeros((d, d), np.float32)
    np.fill_diagonal(x, 1.0)
    got = oracle.router_logits(_bits(x), w)
    assert np.array_equal(got, oracle.bf16_to_f64(w).T)


def test_router_matches_python_loops():
    rng = np.random.default_rng(32)
    T, E, d = 3, 4, 8
    x, w = _bits(rng.normal(0, 1, (T, d))), _bits(rng.normal(0, 1, (E, d)))
    xf, wf = oracle.bf16_to_f64(x), oracle.bf16_to_f64(w)
    got = oracle.router_logits(x, w)
    for t in range(T):
        for e in range(E):
            ref = math.fsum(float(xf[t, i]) * float(wf[e, i]) for i in range(d))
            assert got[t, e] == pytest.approx(ref, rel=1e-14, abs=1e-14)


def test_router_permuting_experts_permutes_columns_and_scaling_is_exact():
    rng = np.random.default_rng(33)
    T, E, d = 6, 7, 64
    x, w = _bits(rng.normal(0, 1, (T, d))), _bits(rng.normal(0, 0.1, (E, d)))
    base = oracle.router_logits(x, w)
    perm = rng.permutation(E)
    assert np.array_equal(oracle.router_logits(x, w[perm]), base[:, perm])
    # doubling x doubles every logit exactly (a power of two, no rounding)
    x2 = _bits(oracle.bf16_to_f64(x) * 2.0)
    assert np.array_equal(oracle.router_logits(x2, w), 2.0 * base)


# ------------------------------------------------- randomised properties --

from hypothesis import given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402


@settings(max_examples=60, deadline=None)
@given(st.integers(1, 6), st.integers(1, 7), st.data())
def test_route_selection_is_the_unique_bruteforce_subset(T, E, data):
    """Any logits (ties included, drawn from a few levels): the chosen set is
    the one k-subset whose members all beat every other expert, listed in
    selection order."""
    k = data.draw(st.integers(1, E))
    levels = data.draw(st.lists(st.sampled_from([-1.5, -0.0, 0.0, 0.25, 2.0]), min_size=T * E, max_size=T * E))
    lg = np.array(levels, np.float32).reshape(T, E)
    ids, w = oracle.route(lg, k)
    for t in range(T):
        assert set(ids[t].tolist()) == _brute_topk(lg[t].astype(np.float64), list(range(E)), k)
        _check_selection_order(lg[t].astype(np.float64), ids[t])
        assert abs(w[t].sum() - 1.0) <= 1e-12


@settings(max_examples=60, deadline=None)
@given(st.integers(0, 40), st.integers(1, 9), st.sampled_from([16, 32, 64, 128]), st.data())
def test_align_invariants_on_random_ids(T, E, bm, data):
    k = data.draw(st.integers(1, E))
    flat = data.draw(st.lists(st.integers(0, E - 1), min_size=T * k, max_size=T * k))
    ids = np.array(flat, np.int32).reshape(T, k)
    st_, ex, n, inv = oracle.align(ids, E, bm)
    _check_align_invariants(ids, E, bm, st_, ex, n, inv)
    # the sort is stable: within an expert's run the slots ascend
    order = [int(s) for s in st_[:n] if s < T * k]
    assert order == sorted(range(T * k), key=lambda s: (int(ids.reshape(-1)[s]), s))
