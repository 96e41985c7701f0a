"""Pins for the oracle's router and routing metadata (CPU only).

Each check compares the oracle with something other than itself: brute-force
enumeration, a library routine (scipy softmax, numpy's stable argsort and
bincount), a closed-form identity, or a hand-worked value.
"""
import itertools
import math

import numpy as np
import pytest
import scipy.special

from oracle import moe_ref as ref
from routing_grouped_expert_softmax_b200 import inputs as gen


def brute_force_topk_set(zrow, k):
    """Among all k-subsets with the largest logit sum, the lexicographically smallest."""
    E = len(zrow)
    best, best_key = None, None
    for sub in itertools.combinations(range(E), k):
        s = sum(zrow[e] for e in sub)
        key = (-s, sub)
        if best_key is None or key < best_key:
            best, best_key = sub, key
    return set(best)


@pytest.mark.parametrize("E,k", [(4, 1), (5, 2), (6, 3), (8, 2), (7, 7)])
def test_topk_matches_brute_force_integer_logits(E, k):
    # small integer logits: sums are exact and ties are frequent
    rng = np.random.default_rng(E * 10 + k)
    z = rng.integers(-2, 3, size=(40, E)).astype(np.float64)
    idx = ref.topk_experts(z, k)
    for t in range(z.shape[0]):
        assert set(idx[t].tolist()) == brute_force_topk_set(z[t].tolist(), k)


@pytest.mark.parametrize("E,k", [(8, 2), (6, 4)])
def test_topk_matches_brute_force_normal_logits(E, k):
    z = gen.normal_logits(50, E, seed=3).astype(np.float64)
    idx = ref.topk_experts(z, k)
    for t in range(z.shape[0]):
        assert set(idx[t].tolist()) == brute_force_topk_set(z[t].tolist(), k)


def test_topk_order_descending_ties_lower_index_first():
    z = gen.tied_logits(200, 16, levels=3, seed=1).astype(np.float64)
    idx = ref.topk_experts(z, 5)
    for t in range(200):
        vals = z[t, idx[t]]
        for j in range(4):
            assert vals[j] > vals[j + 1] or (vals[j] == vals[j + 1] and idx[t, j] < idx[t, j + 1])
        assert len(set(idx[t].tolist())) == 5


def test_topk_signed_zero_is_a_tie():
    z = np.array([[0.0, -0.0, -1.0], [-0.0, 0.0, -1.0]])
    assert ref.topk_experts(z, 1).tolist() == [[0], [0]]


def test_all_equal_logits_give_first_k_and_uniform_gates():
    z = np.full((3, 8), 0.7)
    idx, g = ref.route_from_logits(z, 3)
    assert idx.tolist() == [[0, 1, 2]] * 3
    np.testing.assert_allclose(g, 1.0 / 3.0, rtol=0, atol=1e-15)


def test_hand_worked_router_example():
    # logits [1, 3, 2, 3], k = 2: experts 1 and 3 tie at 3, lower index first.
    z = np.array([[1.0, 3.0, 2.0, 3.0]])
    idx, g = ref.route_from_logits(z, 2)
    assert idx.tolist() == [[1, 3]]
    np.testing.assert_allclose(g, [[0.5, 0.5]], atol=1e-15)
    # logits [0, ln 3], k = 2: gates 1/4 and 3/4 listed by descending logit.
    z = np.array([[0.0, math.log(3.0)]])
    idx, g = ref.route_from_logits(z, 2)
    assert idx.tolist() == [[1, 0]]
    np.testing.assert_allclose(g, [[0.75, 0.25]], rtol=1e-14)


def test_softmax_matches_scipy():
    z = gen.normal_logits(30, 9, seed=4).astype(np.float64) * 5
    np.testing.assert_allclose(ref.softmax(z), scipy.special.softmax(z, axis=1), rtol=1e-13)


def test_renormalised_gates_equal_softmax_over_selected_logits():
    # closed form: p_S / sum p_S == softmax(z_S), independent of unselected logits
    z = gen.normal_logits(64, 12, seed=5).astype(np.float64)
    idx, g = ref.route_from_logits(z, 4)
    zs = np.take_along_axis(z, idx.astype(np.int64), axis=1)
    np.testing.assert_allclose(g, scipy.special.softmax(zs, axis=1), rtol=1e-13)
    np.testing.assert_allclose(g.sum(axis=1), 1.0, atol=1e-14)
    assert np.all(np.diff(g, axis=1) <= 1e-15)        # descending like the logits


def test_router_shift_invariance():
    z = gen.normal_logits(32, 8, seed=6).astype(np.float64)
    i1, g1 = ref.route_from_logits(z, 2)
    i2, g2 = ref.route_from_logits(z + 7.25, 2)
    assert np.array_equal(i1, i2)
    np.testing.assert_allclose(g1, g2, rtol=1e-12)


def test_k_equals_E_gives_full_softmax_and_k1_gives_unit_gate():
    z = gen.normal_logits(16, 6, seed=7).astype(np.float64)
    idx, g = ref.route_from_logits(z, 6)
    full = scipy.special.softmax(z, axis=1)
    np.testing.assert_allclose(g, np.take_along_axis(full, idx.astype(np.int64), axis=1), rtol=1e-13)
    idx1, g1 = ref.route_from_logits(z, 1)
    assert np.array_equal(idx1[:, 0], np.argmax(z, axis=1))
    np.testing.assert_allclose(g1, 1.0)


def test_router_logits_bias_and_matmul():
    x = np.array([[1.0, 2.0], [0.5, -1.0]])
    w = np.array([[1.0, 0.0, 2.0], [0.0, 1.0, -1.0]])
    b = np.array([0.0, -1.0, 0.5])
    np.testing.assert_array_equal(ref.router_logits(x, w, b),
                                  [[1.0, 1.0, 0.5], [0.5, -2.0, 2.5]])


# --------------------------- routing metadata ---------------------------

@pytest.mark.parametrize("T,E,k,seed", [(1, 1, 1, 0), (37, 8, 2, 1), (200, 16, 4, 2), (64, 128, 4, 3)])
def test_metadata_against_library_routines(T, E, k, seed):
    idx = gen.skewed_routing_idx(T, E, k, seed=seed) if E >= k else None
    counts, offsets, sop, pos = ref.routing_metadata(idx, E)
    flat = idx.ravel()
    assert np.array_equal(counts, np.bincount(flat, minlength=E))
    assert counts.sum() == T * k
    assert offsets[0] == 0 and np.array_equal(offsets[1:], np.cumsum(counts))
    assert np.array_equal(pos, np.argsort(flat, kind="stable"))      # stable counting sort
    assert np.array_equal(np.sort(sop), np.arange(T * k))             # bijection
    assert np.array_equal(pos[sop], np.arange(T * k))                 # inverse
    for e in range(E):
        seg = pos[offsets[e]:offsets[e + 1]]
        assert np.all(flat[seg] == e)
        assert np.all(np.diff(seg) > 0)                                 # stability


def test_metadata_hand_worked():
    # pairs (t,j) -> experts: t0:(2,0) t1:(0,2) t2:(1,2)
    idx = np.array([[2, 0], [0, 2], [1, 2]])
    counts, offsets, sop, pos = ref.routing_metadata(idx, 4)
    assert counts.tolist() == [2, 1, 3, 0]
    assert offsets.tolist() == [0, 2, 3, 6, 6]
    # expert 0 gets pairs 1, 2; expert 1 gets pair 4; expert 2 gets pairs 0, 3, 5
    assert pos.tolist() == [1, 2, 4, 0, 3, 5]
    assert sop.tolist() == [3, 0, 1, 4, 2, 5]


def test_permute_copies_rows_bitwise():
    x = gen.bf16_round(np.random.default_rng(0).standard_normal((10, 6), dtype=np.float32))
    idx = gen.skewed_routing_idx(10, 5, 3, seed=1)
    _, _, sop, pos = ref.routing_metadata(idx, 5)
    xp = ref.permute(x, pos, 3)
    for i in range(30):
        assert np.array_equal(xp[sop[i]], x[i // 3])


def test_uniform_random_routing_generator_is_valid():
    idx, g = gen.uniform_random_routing(500, 16, 4, seed=0)
    for t in range(500):
        assert len(set(idx[t].tolist())) == 4
    assert idx.min() >= 0 and idx.max() < 16
    np.testing.assert_allclose(g, 0.25)
