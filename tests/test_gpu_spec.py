"""Speculative verification of FlashHead drafts (CUDA, through the C ABI) vs the oracle (needs a B200).

Write-up section 4.2: a FlashHead draft is accepted or replaced with the dense
head's probabilities. Checked two ways on the tiny planted head: row by row
against ``oracle.speculative_verify`` on the oracle's own logits and candidate
sets (band rule: a decision may differ only where the oracle's acceptance
ratio or residual CDF lies within a small band of the uniform), and as a law:
with drafts drawn from q, 16384 verified tokens against the dense softmax(z/T)
(chi-square, bins merged to expected >= 5, accepted at p > 1e-3).
"""
import numpy as np
import pytest
from scipy import stats

import oracle
from tests.test_gpu_parity import fh, get_cfg, hid_dev  # noqa: F401
from tests.test_gpu_sampling_stats import _chi2_merged

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _softmax(x):
    y = np.asarray(x, dtype=np.float64)
    w = np.exp(y - y.max())
    return w / w.sum()


def _oracle_candidates(head, H, p):
    S = oracle.centroid_scores(oracle.centroid_matrix(head), H)
    ids = oracle.select_greedy(S, p)
    return np.stack([oracle.candidate_tokens(head.C2T, ids[r]) for r in range(H.shape[0])])


def test_spec_verify_row_by_row(fh):
    cfg, head, hid, _, dh = get_cfg(0, fh, n_states=65, max_batch=65, max_probes=256)
    B, T = 32, 0.8
    H = hid.H[:B]
    cand = _oracle_candidates(head, H, cfg.p)
    z_or, _ = oracle.dense_head(head.E, H)
    rng = np.random.default_rng(41)
    draft = cand[np.arange(B), rng.integers(0, cand.shape[1], size=B)].astype(np.int32)
    ua = rng.random(B, dtype=np.float32)
    ur = rng.random(B, dtype=np.float32)
    _, z_dev = dh.dense_head(hid_dev(H), want_logits=True)
    out = fh.speculative_verify(dh, z_dev, torch.from_numpy(cand.astype(np.int32)).cuda(),
                                torch.from_numpy(draft).cuda(), T, torch.from_numpy(ua).cuda(),
                                torch.from_numpy(ur).cuda()).cpu().numpy()
    assert dh.device_status() == 0
    outside = 0
    for r in range(B):
        want = oracle.speculative_verify(z_or[r], cand[r], T, int(draft[r]), float(ua[r]), float(ur[r]))
        if out[r] == want:
            continue
        p = _softmax(z_or[r] / T)
        q = np.zeros_like(p)
        q[cand[r]] = _softmax(z_or[r][cand[r]] / T)
        ratio = p[draft[r]] / q[draft[r]]
        if abs(float(ua[r]) - ratio) <= 1e-3 * max(1.0, ratio):
            continue                      # the acceptance decision sits on the band
        res = np.maximum(p - q, 0.0)
        cdf = np.cumsum(res)
        t = int(out[r])
        lo = cdf[t - 1] if t > 0 else 0.0
        target = float(ur[r]) * cdf[-1]
        if lo - 1e-3 * cdf[-1] <= target <= cdf[t] + 1e-3 * cdf[-1] and res[t] > 0:
            continue                      # a resampled token within the band of its CDF step
        outside += 1
    assert outside == 0


def test_spec_verify_output_law_is_the_dense_softmax(fh):
    cfg, head, hid, _, dh = get_cfg(0, fh, n_states=65, max_batch=65, max_probes=256)
    T, N = 2.0, 16384
    h = hid.H[5:6]
    cand = _oracle_candidates(head, h, cfg.p)[0]
    z_or, _ = oracle.dense_head(head.E, h)
    p = _softmax(z_or[0] / T)
    q = _softmax(z_or[0][cand] / T)
    rng = np.random.default_rng(42)
    draft = cand[np.searchsorted(np.cumsum(q), rng.random(N), side="right").clip(0, len(cand) - 1)]
    _, z_dev = dh.dense_head(hid_dev(h), want_logits=True)
    Z = z_dev.expand(N, -1).contiguous()
    C = torch.from_numpy(np.repeat(cand[None].astype(np.int32), N, axis=0)).cuda()
    out = fh.speculative_verify(dh, Z, C, torch.from_numpy(draft.astype(np.int32)).cuda(), T,
                                torch.from_numpy(rng.random(N, dtype=np.float32)).cuda(),
                                torch.from_numpy(rng.random(N, dtype=np.float32)).cuda()).cpu().numpy()
    assert dh.device_status() == 0
    assert np.all((out >= 0) & (out < head.v))
    obs = np.bincount(out, minlength=head.v)
    stat, dof = _chi2_merged(obs, p * N)
    assert stats.chi2.sf(stat, dof) > 1e-3, (stat, dof)
    # some drafts were replaced: the law is not just q's
    assert np.any(~np.isin(out, cand))


def test_spec_verify_rejects_a_draft_outside_its_candidates(fh):
    cfg, head, hid, _, dh = get_cfg(0, fh, n_states=65, max_batch=65, max_probes=256)
    h = hid.H[:1]
    cand = _oracle_candidates(head, h, cfg.p)
    bad = np.setdiff1d(np.arange(head.v), cand[0])[:1].astype(np.int32)
    _, z_dev = dh.dense_head(hid_dev(h), want_logits=True)
    half = torch.full((1,), 0.5, dtype=torch.float32, device="cuda")
    out = fh.speculative_verify(dh, z_dev, torch.from_numpy(cand.astype(np.int32)).cuda(),
                                torch.from_numpy(bad).cuda(), 1.0, half, half).cpu().numpy()
    assert out[0] == -1
    assert dh.device_status() == 6   # FH_ERR_OUT_OF_RANGE
    assert dh.device_status() == 0
