"""Adaptive probe count (CUDA, through the C ABI) vs the oracle (needs a B200).

``fh_adaptive_probes`` against ``oracle.adaptive_probe_count``: on equal scores
(closed form ceil(tau c)), and on the tiny and the Llama-3.2-1B-shaped heads'
centroid scores, with a band rule -- the GPU count may differ from the
oracle's only where the oracle's top-p mass at the GPU's count (or one below
it) lies within 1e-4 of tau.
"""
import math

import numpy as np
import pytest

import oracle
from tests.test_gpu_parity import fh, get_cfg, hid_dev  # noqa: F401

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _top_mass(S_row, T, p):
    y = np.sort(np.asarray(S_row, dtype=np.float64) / T)[::-1]
    w = np.exp(y - y[0])
    return float(np.cumsum(w)[p - 1] / w.sum()) if p >= 1 else 0.0


def test_adaptive_probes_on_equal_scores(fh):
    cfg, head, hid, _, dh = get_cfg(0, fh, n_states=65, max_batch=65, max_probes=256)
    S = torch.zeros((3, head.c), dtype=torch.float32, device="cuda")
    for tau, p_min, p_max, want in ((0.3, 1, 256, math.ceil(0.3 * head.c)), (0.3, 100, 256, 100),
                                    (0.9, 1, 64, 64)):
        got = dh.adaptive_probes(S, tau, p_min, p_max).cpu().numpy()
        assert np.all(got == want), (tau, got, want)
        assert np.all(oracle.adaptive_probe_count(np.zeros((3, head.c)), tau, p_min, p_max) == want)


@pytest.mark.parametrize("cfg_id,B,T", [(0, 16, 1.0), (0, 16, 0.3), (1, 4, 1.0)])
def test_adaptive_probes_match_the_oracle(fh, cfg_id, B, T):
    cfg, head, hid, _, dh = get_cfg(cfg_id, fh) if cfg_id else get_cfg(0, fh, n_states=65, max_batch=65,
                                                                           max_probes=256)
    H = hid.H[:B]
    S_gpu = dh.centroid_scores(hid_dev(H))
    S_or = oracle.centroid_scores(oracle.centroid_matrix(head), H)
    for tau in (0.2, 0.5, 0.9):
        got = dh.adaptive_probes(S_gpu, tau, 1, cfg.p, T=T).cpu().numpy()
        want = oracle.adaptive_probe_count(S_or, tau, 1, cfg.p, T=T)
        assert dh.device_status() == 0
        for r in range(B):
            if got[r] == want[r]:
                continue
            g = int(got[r])
            near = abs(_top_mass(S_or[r], T, g) - tau) <= 1e-4 or abs(_top_mass(S_or[r], T, g - 1) - tau) <= 1e-4
            assert near, (tau, r, got[r], want[r])


def test_adaptive_probes_rejects_bad_arguments(fh):
    cfg, head, hid, _, dh = get_cfg(0, fh, n_states=65, max_batch=65, max_probes=256)
    S = torch.zeros((1, head.c), dtype=torch.float32, device="cuda")
    for tau, p_min, p_max in ((0.0, 1, 8), (1.5, 1, 8), (0.5, 0, 8), (0.5, 9, 8), (0.5, 1, head.c + 1)):
        with pytest.raises(fh.FlashHeadError):
            dh.adaptive_probes(S, tau, p_min, p_max)
