"""Pins of the balanced spherical k-means oracle against things other than itself (CPU only).

The clustering step of the FlashHead write-up (section 2.1, with the balance
rule of section 1.2.1) is pinned by a hand-worked fixture, by brute force
(over every balanced assignment of a tiny problem, the oracle's greedy one is
the only stable one: no token prefers a cluster that holds a token it beats
there), by the reduction to the plain argmax assignment when that is already
balanced, by a sequential closed form when every token prefers the same
clusters in the same order, and by recovery of planted clusters. A plausible
slip (similarities sorted ascending, the capacity check off by one, ties
broken the other way, squared distances replaced by distances in the seeding,
centres left unnormalised) fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import kmeans

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _fixture():
    with open(os.path.join(GOLDEN, "kmeans_circle.json")) as f:
        return json.load(f)


def _unit(deg):
    r = math.radians(deg)
    return [math.cos(r), math.sin(r)]


# ---------------------------------------------------------------------------
# hand-worked fixture
# ---------------------------------------------------------------------------
def test_golden_kmeanspp_seeds():
    g = _fixture()["kmeanspp"]
    En = kmeans.normalize_rows(np.array(g["points"], dtype=np.float64))
    seeds = kmeans.kmeanspp_seeds(En, len(g["seeds"]), np.array(g["u"]))
    assert seeds.tolist() == g["seeds"]


def test_golden_kmeanspp_edges():
    g = _fixture()["kmeanspp_edges"]
    En = kmeans.normalize_rows(np.array(g["points"], dtype=np.float64))
    seeds = kmeans.kmeanspp_seeds(En, len(g["seeds"]), np.array(g["u"]))
    assert seeds.tolist() == g["seeds"]


def test_seed_weights_match_the_worked_seeding():
    g = _fixture()["kmeanspp"]
    En = np.array(g["points"], dtype=np.float64)
    assert kmeans.seed_weights(En, [0]).tolist() == [0.0, 2.0, 4.0, 2.0]
    assert kmeans.seed_weights(En, [0, 2]).tolist() == [0.0, 2.0, 0.0, 2.0]
    # the seeding's own draws follow the inverse CDF of these weights
    rng = np.random.default_rng(4)
    X = kmeans.normalize_rows(rng.standard_normal((40, 5)))
    u = rng.uniform(size=8)
    seeds = kmeans.kmeanspp_seeds(X, 8, u)
    for j in range(1, 8):
        cdf = np.cumsum(kmeans.seed_weights(X, seeds[:j]))
        t = seeds[j]
        assert cdf[t] > u[j] * cdf[-1] >= (cdf[t - 1] if t > 0 else 0.0)


def test_golden_balanced_steps():
    g = _fixture()["balanced"]
    E = np.array([_unit(a) for a in g["angles_deg"]])
    C, C2T, assign, iters, history = kmeans.build_clusters(E, 2, init_ids=np.array(g["init_ids"]))
    S1 = E @ E[g["init_ids"]].T
    assert np.argmax(S1, axis=1).tolist() == g["plain_argmax_step1"]
    assert history[0].tolist() == g["assign_step1"]
    assert assign.tolist() == g["assign_final"]
    assert iters == g["iterations"]
    assert C2T.tolist() == g["C2T"]
    want = np.array([_unit(a) for a in g["centre_angles_deg"]])
    assert np.max(np.abs(C - want)) < 1e-12


def test_single_cluster_centre_is_the_mean_direction():
    # Points symmetric about the x axis: the normalised mean is exactly (1, 0).
    E = np.array([_unit(a) for a in (-40.0, 40.0, -10.0, 10.0)]) * np.array([[3.0], [0.5], [2.0], [7.0]])
    C, C2T, assign, iters, _ = kmeans.build_clusters(E, 1, init_ids=np.array([2]))
    assert assign.tolist() == [0, 0, 0, 0]
    assert C2T.tolist() == [[0, 1, 2, 3]]
    assert np.max(np.abs(C[0] - np.array([1.0, 0.0]))) < 1e-15
    assert iters == 2


def test_normalize_rows_keeps_zero_rows():
    X = np.array([[3.0, 4.0], [0.0, 0.0], [0.0, -2.0]])
    En = kmeans.normalize_rows(X)
    assert En.tolist() == [[0.6, 0.8], [0.0, 0.0], [0.0, -1.0]]


# ---------------------------------------------------------------------------
# the balanced assignment
# ---------------------------------------------------------------------------
def _balanced_assignments(v, c):
    """Every map token -> cluster with exactly v/c tokens per cluster."""
    b = v // c
    for perm in itertools.permutations(range(v)):
        a = [0] * v
        ok = True
        for k in range(c):
            grp = perm[k * b:(k + 1) * b]
            if list(grp) != sorted(grp):
                ok = False
                break
            for t in grp:
                a[t] = k
        if ok and (c < 2 or all(perm[k * b] < perm[(k + 1) * b] for k in range(c - 1))):
            yield np.array(a)


def _stable(S, a):
    """No token t prefers a cluster k whose weakest member scores below t there."""
    v, c = S.shape
    for t in range(v):
        for k in range(c):
            if k != a[t] and S[t, k] > S[t, a[t]]:
                if np.min(S[a == k, k]) < S[t, k]:
                    return False
    return True


@pytest.mark.parametrize("v,c,seed", [(6, 3, 0), (6, 3, 1), (6, 2, 2), (8, 2, 3), (8, 4, 4), (9, 3, 5)])
def test_greedy_is_the_unique_stable_balanced_assignment(v, c, seed):
    rng = np.random.default_rng(seed)
    S = rng.standard_normal((v, c))
    # all balanced assignments up to relabelling of the clusters are enumerated with labels
    # fixed by their smallest member; the cluster labels matter here, so expand them
    cands = []
    for a in _balanced_assignments(v, c):
        for lab in itertools.permutations(range(c)):
            cands.append(np.array(lab)[a])
    n_expected = math.factorial(v) // math.factorial(v // c) ** c
    assert len(cands) == n_expected
    stable = [a for a in cands if _stable(S, a)]
    assert len(stable) == 1
    got = kmeans.balanced_assign(S, v // c)
    assert got.tolist() == stable[0].tolist()


@pytest.mark.parametrize("seed", range(4))
def test_balanced_argmax_is_kept(seed):
    rng = np.random.default_rng(10 + seed)
    c, b = 5, 7
    v = c * b
    target = rng.permutation(np.repeat(np.arange(c), b))
    S = rng.uniform(-1, 1, size=(v, c))
    S[np.arange(v), target] += 3.0
    assert np.argmax(S, axis=1).tolist() == target.tolist()
    assert kmeans.balanced_assign(S, b).tolist() == target.tolist()


def test_common_preference_fills_clusters_in_order():
    # Every token ranks the clusters 0 > 1 > 2 > 3 with separated bands, so the
    # greedy walk fills cluster 0 with the b best tokens at cluster 0, then
    # cluster 1 with the b best of the rest at cluster 1, and so on.
    rng = np.random.default_rng(7)
    c, b = 4, 6
    v = c * b
    S = -np.arange(c)[None, :] * 1.0 + rng.uniform(0, 0.5, size=(v, c))
    want = np.full(v, -1)
    free = list(range(v))
    for k in range(c):
        best = sorted(free, key=lambda t: -S[t, k])[:b]
        want[best] = k
        free = [t for t in free if t not in best]
    got = kmeans.balanced_assign(S, b)
    assert got.tolist() == want.tolist()
    assert np.bincount(got, minlength=c).tolist() == [b] * c


def test_ties_go_to_the_lower_token_then_the_lower_cluster():
    S = np.zeros((4, 2))            # every pair ties
    assert kmeans.balanced_assign(S, 2).tolist() == [0, 0, 1, 1]
    S = np.array([[1.0, 1.0], [1.0, 1.0], [0.0, 0.0], [0.0, 0.0]])
    assert kmeans.balanced_assign(S, 2).tolist() == [0, 0, 1, 1]


# ---------------------------------------------------------------------------
# whole builder
# ---------------------------------------------------------------------------
def _planted(c, b, d, noise, seed):
    rng = np.random.default_rng(seed)
    mu = rng.standard_normal((c, d))
    mu /= np.linalg.norm(mu, axis=1, keepdims=True)
    perm = rng.permutation(c * b)
    E = np.empty((c * b, d))
    truth = np.empty(c * b, dtype=np.int64)
    for k in range(c):
        for j in range(b):
            t = perm[k * b + j]
            E[t] = (mu[k] + noise * rng.standard_normal(d) / math.sqrt(d)) * rng.uniform(0.5, 2.0)
            truth[t] = k
    return E, truth, mu


def test_recovers_planted_clusters_from_one_seed_each():
    c, b, d = 8, 16, 32
    E, truth, mu = _planted(c, b, d, 0.1, 3)
    init = np.array([np.flatnonzero(truth == k)[0] for k in range(c)])
    C, C2T, assign, iters, _ = kmeans.build_clusters(E, c, init_ids=init)
    assert assign.tolist() == truth.tolist()
    assert oracle.check_c2t(C2T, c * b)
    assert iters == 2
    cos = np.sum(C * mu, axis=1)
    assert np.min(cos) > 0.99


@pytest.mark.parametrize("seed", range(3))
def test_kmeanspp_run_is_balanced_and_a_fixed_point(seed):
    c, b, d = 6, 8, 16
    E, truth, _ = _planted(c, b, d, 0.3, 20 + seed)
    u = np.random.default_rng(seed).uniform(size=c)
    C, C2T, assign, iters, history = kmeans.build_clusters(E, c, u_init=u)
    assert oracle.check_c2t(C2T, c * b)
    assert np.bincount(assign, minlength=c).tolist() == [b] * c
    assert iters < 1000
    assert np.array_equal(history[-1], assign)
    assert np.allclose(np.linalg.norm(C, axis=1), 1.0, atol=1e-14)
    # seeds were distinct tokens
    seeds = kmeans.kmeanspp_seeds(kmeans.normalize_rows(E), c, u)
    assert len(set(seeds.tolist())) == c


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_stops_at_the_first_repeated_assignment(seed):
    # Unstructured embeddings take several steps; the run ends on the first step
    # that repeats the previous assignment, and the centres it returns are the
    # normalised means of that assignment.
    rng = np.random.default_rng(seed)
    E = rng.standard_normal((48, 8))
    u = rng.uniform(size=6)
    C, C2T, assign, iters, history = kmeans.build_clusters(E, 6, u_init=u)
    assert iters == len(history) >= 3
    assert np.array_equal(history[-1], history[-2])
    assert all(not np.array_equal(history[i], history[i + 1]) for i in range(len(history) - 2))
    En = E / np.linalg.norm(E, axis=1, keepdims=True)
    for k in range(6):
        s = En[assign == k].sum(axis=0)
        assert np.max(np.abs(C[k] - s / np.linalg.norm(s))) < 1e-14


def test_builder_rejects_unbalanced_sizes():
    with pytest.raises(ValueError):
        kmeans.build_clusters(np.ones((10, 4)), 3, init_ids=np.array([0, 1, 2]))


# ---------------------------------------------------------------------------
# the parallel round structure the assignment kernels use
# ---------------------------------------------------------------------------
def _deferred_acceptance(S, b):
    """Rounds of proposals: every unassigned token proposes to its best cluster
    (similarity desc, cluster asc) among those whose b-th held pair it beats at
    the start of the round (or that still have room); every cluster keeps the
    best b of its held tokens and its proposers (similarity desc, token asc)."""
    v, c = S.shape
    held = [[] for _ in range(c)]          # (s, t), best first
    assign = np.full(v, -1)
    rounds = 0
    while np.any(assign < 0):
        rounds += 1
        props = [[] for _ in range(c)]
        for t in np.flatnonzero(assign < 0):
            best = None
            for k in range(c):
                h = held[k]
                if len(h) == b:
                    ws, wt = h[-1]
                    if not (S[t, k] > ws or (S[t, k] == ws and t < wt)):
                        continue
                if best is None or S[t, k] > S[t, best]:
                    best = k
            props[best].append((S[t, best], t))
        for k in range(c):
            if not props[k]:
                continue
            cand = sorted(held[k] + props[k], key=lambda e: (-e[0], e[1]))
            for s_, t in cand[b:]:
                assign[t] = -1
            held[k] = cand[:b]
            for s_, t in held[k]:
                assign[t] = k
    return assign, rounds


@pytest.mark.parametrize("v,c,levels,seed", [(12, 3, 0, 0), (40, 5, 0, 1), (40, 5, 3, 2), (64, 8, 2, 3),
                                             (96, 6, 0, 4), (60, 4, 1, 5)])
def test_round_structure_of_the_kernels_gives_the_greedy_assignment(v, c, levels, seed):
    # levels > 0 quantises the similarities to a few values, so ties decide most pairs
    rng = np.random.default_rng(seed)
    S = rng.standard_normal((v, c))
    if levels:
        S = np.round(S * levels) / levels
    got, rounds = _deferred_acceptance(S, v // c)
    assert got.tolist() == kmeans.balanced_assign(S, v // c).tolist()
    assert rounds >= 1
