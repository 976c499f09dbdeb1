"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test ties one part of the oracle to a fact the FlashHead pages or the
mathematics fix: hand-worked fixtures, brute force in exact rational
arithmetic, closed forms of the Gumbel-max and Plackett-Luce laws, the p = c
reduction to the dense head, and the C2T invariant. A plausible slip in the
oracle (a transposed operand, a wrong gather index, a flipped sign in the
Gumbel transform, temperature multiplied instead of divided, swapped nibbles,
a wrong tie-break) fails at least one of them.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
from scipy import stats

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(x):
    return synth.to_bf16_bits(np.asarray(x, dtype=np.float32))


class _H:  # minimal head record for hand-built heads
    def __init__(self, E, C, C2T, C_q=None, C_scales=None):
        self.E, self.C, self.C2T, self.C_q, self.C_scales = E, C, C2T, C_q, C_scales
        self.v, self.d = E.shape
        self.c, self.b = C2T.shape


# ---------------------------------------------------------------------------
# golden fixtures (hand-worked)
# ---------------------------------------------------------------------------
def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_golden_two_stage_greedy_and_dense():
    g = _load("two_stage_tiny.json")
    head = _H(_bf16(g["E"]), _bf16(g["C"]), np.array(g["C2T"], dtype=np.int32))
    for case in g["cases"]:
        h = _bf16(case["h"])
        s = oracle.centroid_scores(oracle.widen_bf16(head.C), h[None])[0]
        assert s.tolist() == case["scores"]
        z, am = oracle.dense_head(head.E, h[None])
        assert z[0].tolist() == case["dense_logits"] and int(am[0]) == case["dense_argmax"]
        for gr in case["greedy"]:
            ids = oracle.select_greedy(s[None], gr["p"])[0]
            assert sorted(ids.tolist()) == gr["clusters"]
            toks, zc = oracle.candidate_logits(head.E, head.C2T, h, ids)
            assert toks.tolist() == gr["cand_tokens"] and zc.tolist() == gr["cand_logits"]
            tok, _, _ = oracle.decode(head, h[None], gr["p"])
            assert int(tok[0]) == gr["token"]


def test_golden_sampling():
    g = _load("two_stage_tiny.json")
    head = _H(_bf16(g["E"]), _bf16(g["C"]), np.array(g["C2T"], dtype=np.int32))
    case = g["cases"][0]
    h = _bf16(case["h"])
    sm = case["sampling_T1_p2"]
    U = np.array(sm["u_clusters"], dtype=np.float32)[None]
    s = oracle.centroid_scores(oracle.widen_bf16(head.C), h[None])
    keys = oracle.gumbel_keys(s, U, sm["T"])[0]
    np.testing.assert_allclose(keys, sm["keys"], atol=sm["keys_tolerance"])
    ids = oracle.select_sampled(s, U, 2, sm["T"])[0]
    assert sorted(ids.tolist()) == sm["clusters"]
    toks, z = oracle.candidate_logits(head.E, head.C2T, h, ids)
    assert toks.tolist() == sm["cand_tokens"] and z.tolist() == sm["cand_logits"]
    for dr in sm["token_draws"]:
        tok, _, _ = oracle.decode(head, h[None], 2, mode="gumbel", T=sm["T"], U=U,
                                  u_tok=np.array([dr["u_tok"]]))
        assert int(tok[0]) == dr["token"]
    fx = case["token_sampling_fixed_candidates"]
    for dr in fx["draws"]:
        t = oracle.sample_token(np.array(fx["cand_tokens"]), np.array(fx["cand_logits"], float),
                                fx["T"], dr["u_tok"])
        assert t == dr["token"]


def test_golden_int4_nibbles():
    g = _load("int4_nibbles.json")
    d = g["d"]
    q = np.zeros((1, d // 2), dtype=np.uint8)
    q[0, :4] = g["bytes_first"]
    q[0, 16] = g["group1_first_byte"]
    sc = np.array([g["scale_bits"]], dtype=np.uint16)
    deq = oracle.dequantize_int4(q, sc)[0]
    assert deq[:8].tolist() == g["expected_first_values"]
    assert deq[32:34].tolist() == g["expected_group1_first_values"]
    assert np.all(deq[8:32] == 0) and np.all(deq[34:] == 0)


# ---------------------------------------------------------------------------
# INT4 quantiser round trip (quantiser lives in the generator, independent code)
# ---------------------------------------------------------------------------
def test_int4_roundtrip_within_half_step():
    rng = np.random.default_rng(7)
    C = _bf16(rng.standard_normal((64, 256)) * 0.05)
    C[3, 32:64] = 0  # an all-zero group
    q, sc = synth.quantize_int4_g32(C)
    deq = oracle.dequantize_int4(q, sc)
    x = oracle.widen_bf16(C)
    scale = np.repeat(oracle.widen_bf16(sc), 32, axis=1)
    # the rounding step is x/scale -> nearest code; |error| <= scale/2 (+ bf16 scale rounding slack)
    err = np.abs(deq - x)
    assert np.all(err <= 0.5 * scale * (1 + 2 ** -7) + 1e-300)
    assert np.all(deq[3, 32:64] == 0)
    codes = np.rint(deq / np.where(scale > 0, scale, 1))
    assert codes.min() >= -7 and codes.max() <= 7


# ---------------------------------------------------------------------------
# adaptive probe count (reading: smallest p whose top-p softmax mass reaches tau)
# ---------------------------------------------------------------------------
def test_adaptive_probes_closed_forms():
    # equal scores: the top p hold p/c of the mass
    assert oracle.adaptive_probe_count(np.zeros((1, 100)), 0.305, 1, 100)[0] == 31
    assert oracle.adaptive_probe_count(np.zeros((1, 100)), 0.295, 1, 100)[0] == 30
    # "at least tau": a mass of exactly tau (0.5 = 2/4, exact in binary) stops at that p
    assert oracle.adaptive_probe_count(np.zeros((1, 4)), 0.5, 1, 4)[0] == 2
    # ten clusters at ln 9, ninety at 0: weights 9 and 1, mass of the top p = p/20 up to p = 10,
    # then (90 + p - 10) / 180
    S = np.r_[np.full(10, math.log(9.0)), np.zeros(90)][None, :]
    rng = np.random.default_rng(3)
    S = S[:, rng.permutation(100)]
    assert oracle.adaptive_probe_count(S, 0.41, 1, 100)[0] == 9
    assert oracle.adaptive_probe_count(S, 0.61, 1, 100)[0] == 30
    # one dominant cluster: p_min
    D = np.zeros((1, 1000))
    D[0, 17] = 50.0
    assert oracle.adaptive_probe_count(D, 0.99, 4, 512)[0] == 4
    # everything: clamped to p_max
    assert oracle.adaptive_probe_count(np.zeros((1, 100)), 1.0, 1, 64)[0] == 64


def test_adaptive_probes_temperature_and_monotonicity():
    rng = np.random.default_rng(4)
    S = rng.standard_normal((6, 300))
    a = oracle.adaptive_probe_count(S, 0.5, 1, 300, T=0.7)
    assert np.array_equal(a, oracle.adaptive_probe_count(2.0 * S, 0.5, 1, 300, T=1.4))   # depends on s/T only
    assert np.array_equal(a, oracle.adaptive_probe_count(S + 3.0, 0.5, 1, 300, T=0.7))   # shift invariant
    prev = np.zeros(6, dtype=np.int32)
    for tau in (0.1, 0.3, 0.5, 0.7, 0.9, 0.99):
        cur = oracle.adaptive_probe_count(S, tau, 1, 300)
        assert np.all(cur >= prev)
        prev = cur
    # a very high temperature flattens the law: p -> ceil(tau c) within one
    hot = oracle.adaptive_probe_count(S, 0.5, 1, 300, T=1e6)
    assert np.all(np.abs(hot - 150) <= 1)
    # colder is more peaked: never more probes
    assert np.all(oracle.adaptive_probe_count(S, 0.5, 1, 300, T=0.3) <= a)


# ---------------------------------------------------------------------------
# speculative drafting: FlashHead draft, dense-head verification
# ---------------------------------------------------------------------------
def _softmax(x):
    from scipy.special import softmax
    return softmax(np.asarray(x, dtype=np.float64))


def test_speculative_verify_output_follows_the_dense_softmax():
    # draft x ~ q (softmax over the candidates only), then verify: the output
    # law must be softmax(z/T) over the whole vocabulary (chi-square, fixed seed)
    rng = np.random.default_rng(12)
    v, T = 10, 0.8
    z = rng.standard_normal(v) * 1.5
    cand = np.array([1, 4, 7, 8])
    p = _softmax(z / T)
    q = _softmax(z[cand] / T)
    n = 60000
    xs = cand[np.searchsorted(np.cumsum(q), rng.random(n), side="right").clip(0, len(cand) - 1)]
    ua, ur = rng.random(n), rng.random(n)
    out = np.array([oracle.speculative_verify(z, cand, T, int(xs[i]), ua[i], ur[i]) for i in range(n)])
    obs = np.bincount(out, minlength=v)
    chi2, pval = stats.chisquare(obs, p * n)
    assert pval > 1e-3, (obs, p * n)


def test_speculative_verify_accepts_and_resamples_as_defined():
    rng = np.random.default_rng(13)
    v, T = 12, 1.3
    z = rng.standard_normal(v)
    # every token a candidate: q = p, every draft is kept
    for x in range(v):
        assert oracle.speculative_verify(z, np.arange(v), T, x, 0.999999, 0.5) == x
    cand = np.array([0, 2, 3, 9, 11])
    p = _softmax(z / T)
    q = np.zeros(v)
    q[cand] = _softmax(z[cand] / T)
    for x in cand:
        assert oracle.speculative_verify(z, cand, T, int(x), 0.0, 0.5) == x     # u = 0 always keeps
    # a rejected draft is replaced from max(0, p - q): its law on a fine u grid
    x = int(cand[np.argmax(q[cand] - p[cand])])   # the draft most over-weighted by q: ratio < 1
    assert p[x] / q[x] < 1
    M = 20000
    outs = np.array([oracle.speculative_verify(z, cand, T, x, 0.9999999, (i + 0.5) / M) for i in range(M)])
    r = np.maximum(p - q, 0.0)
    r /= r.sum()
    assert np.all(np.abs(np.bincount(outs, minlength=v) / M - r) <= 2.0 / M)
    assert np.all(r[np.bincount(outs, minlength=v) > 0] > 0)


# ---------------------------------------------------------------------------
# INT8 (W8A16) centroids
# ---------------------------------------------------------------------------
def test_golden_int8_codes():
    g = _load("int8_codes.json")
    d = g["d"]
    q = np.zeros((1, d), dtype=np.uint8)
    q[0, :8] = g["bytes_first"]
    q[0, 32:34] = g["group1_first_bytes"]
    sc = np.array([g["scale_bits"]], dtype=np.uint16)
    deq = oracle.dequantize_int8(q, sc)[0]
    assert deq[:8].tolist() == g["expected_first_values"]
    assert deq[32:34].tolist() == g["expected_group1_first_values"]
    assert np.all(deq[8:32] == 0) and np.all(deq[34:] == 0)
    # the same bytes given as int8 codes dequantise identically
    assert np.array_equal(oracle.dequantize_int8(q.view(np.int8), sc)[0], deq)


def test_int8_roundtrip_within_half_step():
    rng = np.random.default_rng(8)
    C = _bf16(rng.standard_normal((64, 256)) * 0.05)
    C[5, 64:96] = 0  # an all-zero group
    q, sc = synth.quantize_int8_g32(C)
    assert q.dtype == np.int8 and q.shape == (64, 256) and sc.shape == (64, 8)
    deq = oracle.dequantize_int8(q, sc)
    x = oracle.widen_bf16(C)
    scale = np.repeat(oracle.widen_bf16(sc), 32, axis=1)
    err = np.abs(deq - x)
    assert np.all(err <= 0.5 * scale * (1 + 2 ** -7) + 1e-300)
    assert np.all(deq[5, 64:96] == 0)
    assert q.min() >= -127 and q.max() <= 127
    # INT8 is the finer grid: its error is far below the INT4 one on the same rows
    q4, sc4 = synth.quantize_int4_g32(C)
    assert np.abs(deq - x).mean() < 0.1 * np.abs(oracle.dequantize_int4(q4, sc4) - x).mean()


def test_int8_values_are_exact_in_fp32_and_split_into_two_bf16():
    # code * scale carries at most 7 + 8 significant bits: exact in fp32, and
    # exactly hi + lo with hi = bf16(x) and lo = x - hi itself a bf16 value
    rng = np.random.default_rng(9)
    C = _bf16(rng.standard_normal((32, 128)))
    q, sc = synth.quantize_int8_g32(C)
    deq = oracle.dequantize_int8(q, sc)
    f32 = deq.astype(np.float32)
    assert np.array_equal(f32.astype(np.float64), deq)
    hi = oracle.widen_bf16(_bf16(f32))
    lo = deq - hi
    assert np.array_equal(oracle.widen_bf16(_bf16(lo.astype(np.float32))), lo)


def test_int8_head_selects_on_its_dequantised_centres():
    # the oracle's INT8 path is the fp64 two-stage head over the dequantised centres
    cfg, head, hid, _ = synth.make_config(0)
    q, sc = synth.quantize_int8_g32(head.C)
    h8 = _H(head.E, head.C, head.C2T)
    h8.C_q8, h8.C_scales8 = q, sc
    Cw = oracle.dequantize_int8(q, sc)
    S = oracle.centroid_scores(Cw, hid.H[:4])
    assert np.array_equal(oracle.centroid_scores(oracle.centroid_matrix(h8), hid.H[:4]), S)
    toks, ids, _ = oracle.decode(h8, hid.H[:4], cfg.p)
    assert np.array_equal(ids, oracle.select_greedy(S, cfg.p))


# ---------------------------------------------------------------------------
# C2T invariant
# ---------------------------------------------------------------------------
def test_c2t_permutation_invariant():
    cfg, head, hid, _ = synth.make_config(0)
    assert head.C2T.shape == (cfg.c, cfg.b)
    assert oracle.check_c2t(head.C2T, cfg.v)
    bad = head.C2T.copy()
    bad[5, 3] = bad[7, 1]                      # duplicate token
    assert not oracle.check_c2t(bad, cfg.v)
    bad = head.C2T.copy()
    bad[0, 0] = cfg.v                          # out of range
    assert not oracle.check_c2t(bad, cfg.v)
    bad = head.C2T.copy()
    bad[0, 0] = -1
    assert not oracle.check_c2t(bad, cfg.v)
    assert not oracle.check_c2t(head.C2T[:, :-1], cfg.v)   # wrong shape


# ---------------------------------------------------------------------------
# brute force in exact rational arithmetic on tiny heads
# ---------------------------------------------------------------------------
def _exact_dot(a_vals, b_vals):
    return sum(Fraction(float(x)) * Fraction(float(y)) for x, y in zip(a_vals, b_vals))


def _brute_topp(keys, p):
    """The unique p-set whose every member beats every non-member under (key desc, id asc)."""
    c = len(keys)
    found = []
    for S in itertools.combinations(range(c), p):
        Sset = set(S)
        ok = all((keys[k] > keys[o]) or (keys[k] == keys[o] and k < o)
                 for k in S for o in range(c) if o not in Sset)
        if ok:
            found.append(S)
    assert len(found) == 1
    return set(found[0])


@pytest.mark.parametrize("seed", range(12))
def test_bruteforce_exact_tiny(seed):
    rng = np.random.default_rng(100 + seed)
    c, b, d = 6, int(rng.integers(1, 4)), 5
    v = c * b
    # small-integer quarter values: exact in bf16 and full of ties
    E = _bf16(rng.integers(-3, 4, size=(v, d)) / 4)
    C = _bf16(rng.integers(-2, 3, size=(c, d)) / 2)
    C2T = rng.permutation(v).astype(np.int32).reshape(c, b)
    head = _H(E, C, C2T)
    Ew, Cw = oracle.widen_bf16(E), oracle.widen_bf16(C)
    for trial in range(4):
        h = _bf16(rng.integers(-2, 3, size=d))
        hw = oracle.widen_bf16(h)
        s_exact = [_exact_dot(Cw[k], hw) for k in range(c)]
        s = oracle.centroid_scores(Cw, h[None])[0]
        assert [Fraction(x) for x in s] == s_exact
        z_exact = [_exact_dot(Ew[t], hw) for t in range(v)]
        for p in range(1, c + 1):
            S = _brute_topp(s_exact, p)
            tokens = [int(C2T[k][j]) for k in S for j in range(b)]
            best = min(tokens, key=lambda t: (-z_exact[t], t))
            tok, ids, mx = oracle.decode(head, h[None], p)
            assert set(ids[0].tolist()) == S
            assert int(tok[0]) == best
            assert Fraction(mx[0]) == z_exact[best]
        zd, am = oracle.dense_head(E, h[None])
        assert int(am[0]) == min(range(v), key=lambda t: (-z_exact[t], t))


# ---------------------------------------------------------------------------
# p = c reduces FlashHead to the dense head
# ---------------------------------------------------------------------------
def test_p_equals_c_is_dense_head():
    cfg, head, hid, _ = synth.make_config(0)
    H = hid.H[:8]
    z, am = oracle.dense_head(head.E, H)
    tok, ids, mx = oracle.decode(head, H, cfg.c)
    assert np.array_equal(tok, am)
    for r in range(H.shape[0]):
        toks, zc = oracle.candidate_logits(head.E, head.C2T, H[r], ids[r])
        assert np.array_equal(np.sort(toks), np.arange(cfg.v))
        np.testing.assert_allclose(zc, z[r, toks], rtol=1e-13, atol=1e-13)
        assert mx[r] == pytest.approx(z[r].max(), abs=1e-13)


def test_max_candidate_logit_monotone_in_p():
    cfg, head, hid, _ = synth.make_config(0)
    H = hid.H[:6]
    prev = np.full(H.shape[0], -np.inf)
    for p in (1, 2, 4, 8, 16, 64, 256):
        _, _, mx = oracle.decode(head, H, p)
        assert np.all(mx >= prev - 1e-12)
        prev = mx


def test_planted_rows_select_their_cluster():
    cfg, head, hid, _ = synth.make_config(0)
    tok, ids, _ = oracle.decode(head, hid.H, cfg.p)
    for r in range(hid.H.shape[0]):
        j = int(hid.planted[r])
        assert j >= 0
        assert j in ids[r]
        assert tok[r] in head.C2T[j]


# ---------------------------------------------------------------------------
# sampling laws
# ---------------------------------------------------------------------------
def _chi2_ok(counts, probs, alpha=1e-3):
    counts = np.asarray(counts, float)
    exp = np.asarray(probs, float) * counts.sum()
    # merge bins until every expected count is >= 5
    order = np.argsort(exp)
    oc, oe, acc_c, acc_e = [], [], 0.0, 0.0
    for i in order:
        acc_c += counts[i]
        acc_e += exp[i]
        if acc_e >= 5:
            oc.append(acc_c)
            oe.append(acc_e)
            acc_c = acc_e = 0.0
    if acc_e > 0:
        if oe:
            oc[-1] += acc_c
            oe[-1] += acc_e
        else:
            oc.append(acc_c)
            oe.append(acc_e)
    if len(oc) < 2:
        return True
    pval = stats.chisquare(oc, oe).pvalue
    return pval > alpha


def test_gumbel_max_p1_is_softmax():
    rng = np.random.default_rng(11)
    s = np.array([0.3, -0.2, 0.9, 0.1, -1.0, 0.5])
    T = 0.7
    n = 60000
    U = rng.random((n, s.size), dtype=np.float32)
    K = oracle.gumbel_keys(np.broadcast_to(s, U.shape), U, T)
    pick = np.argmax(K, axis=1)   # p = 1 of the same keys used by select_sampled
    ids = oracle.select_sampled(np.broadcast_to(s, U.shape)[:2000], U[:2000], 1, T)[:, 0]
    assert np.array_equal(ids, pick[:2000])
    counts = np.bincount(pick, minlength=s.size)
    w = np.exp(s / T)
    assert _chi2_ok(counts, w / w.sum())
    # the wrong temperature placement is rejected by the same test
    w_bad = np.exp(s * T)
    assert not _chi2_ok(counts, w_bad / w_bad.sum())


def _plackett_luce_set_probs(w, p):
    """P(S) for every unordered p-set under sequential sampling without replacement."""
    c = len(w)
    out = {}
    for perm in itertools.permutations(range(c), p):
        prob, rem = 1.0, w.sum()
        for k in perm:
            prob *= w[k] / rem
            rem -= w[k]
        key = frozenset(perm)
        out[key] = out.get(key, 0.0) + prob
    return out


def test_two_stage_sampling_law_plackett_luce():
    rng = np.random.default_rng(5)
    c, b, d, p, T = 5, 2, 4, 2, 0.8
    v = c * b
    E = _bf16(rng.standard_normal((v, d)))
    C = _bf16(rng.standard_normal((c, d)))
    C2T = rng.permutation(v).astype(np.int32).reshape(c, b)
    head = _H(E, C, C2T)
    h = _bf16(rng.standard_normal(d))
    s = oracle.centroid_scores(oracle.widen_bf16(C), h[None])[0]
    z = oracle.widen_bf16(E) @ oracle.widen_bf16(h)
    # exact joint law of the token
    law = np.zeros(v)
    for S, pS in _plackett_luce_set_probs(np.exp(s / T), p).items():
        toks = [int(C2T[k][j]) for k in S for j in range(b)]
        wz = np.exp(z[toks] / T)
        law[toks] += pS * wz / wz.sum()
    assert law.sum() == pytest.approx(1.0, abs=1e-12)
    n = 20000
    H = np.broadcast_to(h, (n, d))
    U = rng.random((n, c), dtype=np.float32)
    ut = rng.random(n, dtype=np.float32)
    tok, _, _ = oracle.decode(head, H, p, mode="gumbel", T=T, U=U, u_tok=ut)
    assert _chi2_ok(np.bincount(tok, minlength=v), law)


def test_p_equals_c_sampling_is_full_softmax():
    rng = np.random.default_rng(9)
    c, b, d, T = 4, 3, 6, 1.3
    v = c * b
    E = _bf16(rng.standard_normal((v, d)))
    C = _bf16(rng.standard_normal((c, d)))
    C2T = rng.permutation(v).astype(np.int32).reshape(c, b)
    head = _H(E, C, C2T)
    h = _bf16(rng.standard_normal(d))
    z = oracle.widen_bf16(E) @ oracle.widen_bf16(h)
    law = np.exp(z / T) / np.exp(z / T).sum()
    n = 20000
    U = rng.random((n, c), dtype=np.float32)
    ut = rng.random(n, dtype=np.float32)
    tok, _, _ = oracle.decode(head, np.broadcast_to(h, (n, d)), c, mode="gumbel", T=T, U=U, u_tok=ut)
    assert _chi2_ok(np.bincount(tok, minlength=v), law)


def test_inverse_cdf_measure_is_exact():
    """With the candidates fixed, the set of u_tok mapping to t has measure w_t / W."""
    rng = np.random.default_rng(3)
    toks = rng.permutation(40).astype(np.int32)
    z = rng.standard_normal(40) * 2
    T = 0.6
    m = 100000
    grid = (np.arange(m) + 0.5) / m
    hits = np.zeros(40)
    pos = {int(t): i for i, t in enumerate(toks)}
    for u in grid:
        hits[pos[oracle.sample_token(toks, z, T, u)]] += 1
    w = np.exp(z / T - (z / T).max())
    np.testing.assert_allclose(hits / m, w / w.sum(), atol=2.0 / m)


def test_zero_temperature_limit_is_greedy():
    cfg, head, hid, _ = synth.make_config(0)
    H = hid.H[:8]
    rng = np.random.default_rng(2)
    U = rng.random((8, cfg.c), dtype=np.float32)
    ut = rng.random(8, dtype=np.float32)
    tg, ig, _ = oracle.decode(head, H, cfg.p)
    ts, is_, _ = oracle.decode(head, H, cfg.p, mode="gumbel", T=1e-9, U=U, u_tok=ut)
    assert np.array_equal(tg, ts)
    for r in range(8):
        assert set(ig[r].tolist()) == set(is_[r].tolist())


def test_uniform_clamp_keeps_keys_finite():
    s = np.zeros((1, 3))
    U = np.array([[0.0, 1.0, 0.5]], dtype=np.float32)
    k = oracle.gumbel_keys(s, U, 1.0)
    assert np.all(np.isfinite(k))
    assert k[0, 0] == pytest.approx(-math.log(-math.log(2.0 ** -126)))
    toks = np.array([2, 0, 1])
    assert oracle.sample_token(toks, np.zeros(3), 1.0, 1.0) == 1   # clamped below 1 -> last
    assert oracle.sample_token(toks, np.zeros(3), 1.0, 0.0) == 2


def test_generator_health_metric():
    cfg, head, hid, _ = synth.make_config(0)
    assert synth.intra_cluster_cosine(head) > 0.6   # the pages' clustering health check
