"""Sampling statistics of the GPU head on a tiny planted head (needs a B200).

The scope's histogram check for the sampling configuration: on the tiny
v = 4096 instance (c = 256 clusters of b = 16, p = 16 probes, T = 0.7), draws
from the batched decode (tensor-core keys, Gumbel top-p, de-duplicated
candidate logits, inverse-CDF token) are compared with the oracle:

(i)   draw by draw on identical uniforms (band rule near CDF steps);
(ii)  with the cluster uniforms fixed, 10^5 draws of the token against the
      exact softmax(z/T) over the fixed candidate set (chi-square, bins merged
      to expected counts >= 5, accepted at p-value > 1e-3);
(iii) with fresh uniforms per draw, 10^5 draws over the whole vocabulary
      against 2 x 10^5 draws of the oracle's two-stage process (two-sample
      chi-square, same rule). The full two-stage law (Plackett-Luce over
      16-of-256 cluster sets) is not enumerable, hence the Monte-Carlo side.
"""
import numpy as np
import pytest

import oracle
import synth
from tests import parity

torch = pytest.importorskip("torch")
scipy_stats = pytest.importorskip("scipy.stats")
pytestmark = pytest.mark.gpu

T = 0.7
BATCH = 1024
CALLS = 98  # 100352 draws


@pytest.fixture(scope="module")
def setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lm_output_head_b200 import build
    build.build()
    import lm_output_head_b200 as fh
    cfg, head, hid, _ = synth.make_config(0)
    dev = "cuda"
    dh = fh.FlashHead(fh.bf16_from_bits(head.E, dev), torch.from_numpy(head.C2T).to(dev),
                      C=fh.bf16_from_bits(head.C, dev), max_batch=BATCH, max_probes=cfg.p)
    # an unplanted hidden state, bf16 of N(0, 64/d) (|h| ~ 8): both stages' laws are far from
    # uniform (scores spread ~0.7 / T) without collapsing onto a handful of tokens
    rng = np.random.default_rng(2024)
    h = rng.normal(0.0, 8.0 / np.sqrt(cfg.d), cfg.d).astype(np.float32)
    h_bits = (np.frombuffer(h.tobytes(), dtype=np.uint32) + 0x8000 >> 16).astype(np.uint16)
    yield fh, cfg, head, dh, h_bits
    dh.close()


def _draw(fh, dh, cfg, h_bits, U, ut):
    B = U.shape[0]
    Hd = fh.bf16_from_bits(np.repeat(h_bits[None], B, axis=0), "cuda")
    tok = dh.decode(Hd, cfg.p, mode="gumbel", T=T, u_clusters=torch.from_numpy(U).cuda(),
                    u_token=torch.from_numpy(ut).cuda())
    return tok.cpu().numpy()


def _chi2_merged(obs, exp):
    """Pearson chi-square with bins merged (in order of expected count) until each expects >= 5."""
    order = np.argsort(exp)
    o, e = obs[order].astype(np.float64), exp[order].astype(np.float64)
    mo, me, acc_o, acc_e = [], [], 0.0, 0.0
    for oi, ei in zip(o, e):
        acc_o += oi
        acc_e += ei
        if acc_e >= 5.0:
            mo.append(acc_o)
            me.append(acc_e)
            acc_o = acc_e = 0.0
    if acc_e > 0 and me:
        mo[-1] += acc_o
        me[-1] += acc_e
    mo, me = np.array(mo), np.array(me)
    stat = float(((mo - me) ** 2 / me).sum())
    return stat, len(mo) - 1


def test_draw_by_draw_matches_oracle(setup):
    fh, cfg, head, dh, h_bits = setup
    rng = np.random.default_rng(11)
    U = rng.random((BATCH, cfg.c), dtype=np.float32)
    ut = rng.random(BATCH, dtype=np.float32)
    tok = _draw(fh, dh, cfg, h_bits, U, ut)
    assert dh.device_status() == 0
    Cw = oracle.centroid_matrix(head)
    rep = parity.Report()
    for r in range(0, BATCH, 16):
        S = oracle.centroid_scores(Cw, h_bits[None])
        K = oracle.gumbel_keys(S, U[r:r + 1], T)
        ids = np.sort(np.argsort(-K[0], kind="stable")[:cfg.p])
        rep.add(parity.check_sampled_token(head, h_bits, ids, int(tok[r]), T, float(ut[r])))
    assert rep.tight_mismatch == 0, rep


def test_fixed_clusters_token_law_is_softmax_over_candidates(setup):
    fh, cfg, head, dh, h_bits = setup
    rng = np.random.default_rng(12)
    u_fixed = rng.random(cfg.c, dtype=np.float32)
    Cw = oracle.centroid_matrix(head)
    S = oracle.centroid_scores(Cw, h_bits[None])
    ids = np.sort(np.argsort(-oracle.gumbel_keys(S, u_fixed[None], T)[0], kind="stable")[:cfg.p])
    toks, z = oracle.candidate_logits(head.E, head.C2T, h_bits, ids)
    y = z / T
    prob = np.exp(y - y.max())
    prob /= prob.sum()
    U = np.repeat(u_fixed[None], BATCH, axis=0)
    counts = {}
    for _ in range(CALLS):
        ut = rng.random(BATCH, dtype=np.float32)
        for t in _draw(fh, dh, cfg, h_bits, U, ut):
            counts[int(t)] = counts.get(int(t), 0) + 1
    assert dh.device_status() == 0
    assert set(counts) <= set(toks.tolist()), "a draw left the fixed candidate set"
    n = BATCH * CALLS
    obs = np.array([counts.get(int(t), 0) for t in toks])
    stat, df = _chi2_merged(obs, prob * n)
    pval = float(scipy_stats.chi2.sf(stat, df))
    assert pval > 1e-3, (stat, df, pval)


def _oracle_two_stage(head, cfg, h_bits, n, rng):
    """n draws of the oracle's two-stage process (vectorised over draws)."""
    Cw = oracle.centroid_matrix(head)
    s = oracle.centroid_scores(Cw, h_bits[None])[0]
    z_all = oracle.widen_bf16(head.E) @ oracle.widen_bf16(h_bits)  # candidate logits of every token
    out = np.empty(n, dtype=np.int64)
    chunk = 10000
    for a in range(0, n, chunk):
        m = min(chunk, n - a)
        u = np.clip(rng.random((m, cfg.c)), 2.0 ** -126, 1.0 - 2.0 ** -24)
        keys = s[None] / T - np.log(-np.log(u))
        sel = np.sort(np.argpartition(-keys, cfg.p - 1, axis=1)[:, :cfg.p], axis=1)
        toks = head.C2T[sel].reshape(m, -1)              # canonical order: cluster asc, slot asc
        y = z_all[toks] / T
        w = np.exp(y - y.max(axis=1, keepdims=True))
        cdf = np.cumsum(w, axis=1)
        ut = np.clip(rng.random(m), 0.0, 1.0 - 2.0 ** -24) * cdf[:, -1]
        idx = np.minimum((cdf > ut[:, None]).argmax(axis=1), toks.shape[1] - 1)
        out[a:a + m] = toks[np.arange(m), idx]
    return out


def test_two_stage_histogram_matches_oracle_monte_carlo(setup):
    fh, cfg, head, dh, h_bits = setup
    rng = np.random.default_rng(13)
    gpu = np.zeros(cfg.v, dtype=np.int64)
    for _ in range(CALLS):
        U = rng.random((BATCH, cfg.c), dtype=np.float32)
        ut = rng.random(BATCH, dtype=np.float32)
        np.add.at(gpu, _draw(fh, dh, cfg, h_bits, U, ut), 1)
    assert dh.device_status() == 0
    ref = np.bincount(_oracle_two_stage(head, cfg, h_bits, 2 * BATCH * CALLS, np.random.default_rng(14)),
                      minlength=cfg.v)
    n1, n2 = gpu.sum(), ref.sum()
    # two-sample chi-square on bins merged (by pooled count) to pooled expected >= 10
    order = np.argsort(gpu + ref)
    o1, o2, groups, acc1, acc2 = [], [], 0, 0, 0
    for i in order:
        acc1 += gpu[i]
        acc2 += ref[i]
        if acc1 + acc2 >= 10:
            o1.append(acc1)
            o2.append(acc2)
            acc1 = acc2 = 0
    if (acc1 or acc2) and o1:
        o1[-1] += acc1
        o2[-1] += acc2
    o1, o2 = np.array(o1, np.float64), np.array(o2, np.float64)
    k1, k2 = np.sqrt(n2 / n1), np.sqrt(n1 / n2)
    stat = float(((k1 * o1 - k2 * o2) ** 2 / (o1 + o2)).sum())
    df = len(o1) - 1
    pval = float(scipy_stats.chi2.sf(stat, df))
    assert pval > 1e-3, (stat, df, pval)
