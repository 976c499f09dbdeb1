"""Comparison rules between the CUDA path and the fp64 oracle.

Tolerance (stated for the retrieval head): a score or logit may differ from
its fp64 value by at most ``TOL * |row| * |h|`` (fp32 accumulation), where
``row`` is the centroid (dequantised for INT4) or token row. Integer outputs
(cluster ids, token ids) must match exactly, except where the oracle's own
gap at the decision boundary is under that tolerance: there any choice
inside the band is accepted, and the rest of the output is checked for
validity. A second, tight bound -- the fp32 accumulation bound
``2 d 2^-24 sum|row_i h_i|`` -- is reported alongside as the real quality
signal of the kernels.
"""
from __future__ import annotations

import dataclasses

import numpy as np

import oracle

TOL = 2e-3
EPS32 = 2.0 ** -24


def widen(bits):
    return oracle.widen_bf16(bits)


def tight_bound(rows_w: np.ndarray, h_w: np.ndarray) -> np.ndarray:
    """fp32 accumulation bound 2 d 2^-24 sum_i |row_i h_i| per row."""
    d = rows_w.shape[1]
    return 2.0 * d * EPS32 * (np.abs(rows_w) @ np.abs(h_w))


def loose_bound(rows_w: np.ndarray, h_w: np.ndarray) -> np.ndarray:
    return TOL * np.linalg.norm(rows_w, axis=1) * np.linalg.norm(h_w)


@dataclasses.dataclass
class Report:
    n: int = 0
    exempt: int = 0          # decisions inside the loose band
    tight_mismatch: int = 0  # decisions outside the tight band that differ

    def add(self, other: "Report"):
        self.n += other.n
        self.exempt += other.exempt
        self.tight_mismatch += other.tight_mismatch


def check_values(gpu: np.ndarray, ref: np.ndarray, rows_w: np.ndarray, h_w: np.ndarray, what: str):
    """|gpu - ref| <= TOL |row| |h| elementwise; returns the fraction inside the tight bound."""
    tol = loose_bound(rows_w, h_w)
    err = np.abs(np.asarray(gpu, np.float64) - ref)
    bad = np.nonzero(err > tol)[0]
    assert bad.size == 0, f"{what}: {bad.size} values outside tolerance, e.g. index {bad[:5]} " \
                          f"err {err[bad[:5]]} tol {tol[bad[:5]]}"
    tb = tight_bound(rows_w, h_w)
    return float(np.mean(err <= tb + 1e-30))


def check_cluster_set(gpu_ids: np.ndarray, keys: np.ndarray, p: int, tau: np.ndarray,
                      tau_tight: np.ndarray) -> Report:
    """Band rule for a top-p set.

    ``keys`` are the oracle's fp64 keys, ``tau`` per-cluster loose tolerances.
    With s_p the oracle's p-th largest key: every k with key > s_p + tau must
    be chosen, no k with key < s_p - tau may be; ids inside the band may differ.
    """
    ids = np.asarray(gpu_ids, np.int64)
    c = keys.shape[0]
    assert ids.shape == (p,), f"expected {p} ids, got {ids.shape}"
    assert ids.min() >= 0 and ids.max() < c, "cluster id out of range"
    assert np.unique(ids).size == p, "repeated cluster id"
    order = np.lexsort((np.arange(c), -keys))
    sp = keys[order[p - 1]]
    chosen = np.zeros(c, bool)
    chosen[ids] = True
    t = tau.max()
    must = keys > sp + t
    never = keys < sp - t
    assert np.all(chosen[must]), f"missed {np.nonzero(must & ~chosen)[0][:5]} clearly above the threshold"
    assert not np.any(chosen[never]), f"chose {np.nonzero(never & chosen)[0][:5]} clearly below"
    ref = np.zeros(c, bool)
    ref[order[:p]] = True
    diff = chosen != ref
    tt = tau_tight.max()
    outside_tight = diff & ((keys > sp + tt) | (keys < sp - tt))
    return Report(n=1, exempt=int(diff.any()), tight_mismatch=int(outside_tight.sum()))


def candidates_fp64(head, h_bits, cluster_ids):
    toks, z = oracle.candidate_logits(head.E, head.C2T, h_bits, cluster_ids)
    return toks, z


def check_greedy_token(head, h_bits, gpu_cluster_ids, gpu_token: int) -> Report:
    """Re-run the oracle's gather + argmax on the GPU's cluster set and compare the token."""
    toks, z = candidates_fp64(head, h_bits, gpu_cluster_ids)
    hw = widen(h_bits)
    rows = widen(head.E[toks])
    tau = loose_bound(rows, hw)
    tau_t = tight_bound(rows, hw)
    ref_tok, zmax = oracle.greedy_token(toks, z)
    assert gpu_token in set(toks.tolist()), f"token {gpu_token} is not a candidate"
    if gpu_token == ref_tok:
        return Report(n=1)
    i = int(np.nonzero(toks == gpu_token)[0][0])
    j = int(np.nonzero(toks == ref_tok)[0][0])
    gap = zmax - z[i]
    assert gap <= tau[i] + tau[j], f"token {gpu_token} (z={z[i]}) vs argmax {ref_tok} (z={zmax}): gap {gap}"
    return Report(n=1, exempt=1, tight_mismatch=int(gap > tau_t[i] + tau_t[j]))


def check_sampled_token(head, h_bits, gpu_cluster_ids, gpu_token: int, T: float, u_tok: float) -> Report:
    """Inverse-CDF draw on the GPU's cluster set; near a CDF step any neighbour within the band is accepted."""
    toks, z = candidates_fp64(head, h_bits, gpu_cluster_ids)
    hw = widen(h_bits)
    rows = widen(head.E[toks])
    tau = loose_bound(rows, hw)
    ref = oracle.sample_token(toks, z, T, u_tok)
    assert gpu_token in set(toks.tolist()), f"token {gpu_token} is not a candidate"
    if gpu_token == ref:
        return Report(n=1)
    y = z / T
    w = np.exp(y - y.max())
    cdf = np.cumsum(w) / w.sum()
    i = int(np.nonzero(toks == gpu_token)[0][0])
    j = int(np.nonzero(toks == ref)[0][0])
    # relative perturbation of every weight by up to tau/T moves each CDF value by at most 2*max(tau)/T
    band = 4.0 * tau.max() / T
    lo, hi = min(i, j), max(i, j)
    u = min(max(u_tok, 0.0), 1 - 2.0 ** -24)
    steps = cdf[lo:hi]
    assert np.all(np.abs(steps - u) <= band), \
        f"sampled {gpu_token} vs oracle {ref}: u={u} not within {band} of a CDF step between them"
    return Report(n=1, exempt=1)
