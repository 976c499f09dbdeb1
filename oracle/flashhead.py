"""fp64 CPU oracle of the FlashHead retrieval head (test infrastructure only).

THIS IS TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import it. The product path (the CUDA
library and its Python binding) never calls it and shares no code with it.

What it computes, step by step, in the order of the FlashHead write-up
("FlashHead技术解析", www.framerc.cn/news/2430929) and the FlashHead abstract
(arXiv 2603.14591):

* dense head ``z = E h`` (section 1.1) -- the comparison path;
* stage 1, centroid scores ``s = C h`` over all c balanced clusters
  (section 1.2.2; section 1.2.4 allows C to be a low-bit quantisation, here
  symmetric INT4 with one bf16 scale per 32 elements);
* probe selection: the p highest-scoring clusters (multi-probe retrieval,
  section 1.2.2), or, in sampling mode, p clusters drawn without replacement
  by multinomial sampling at temperature T (section 1.2.3), realised as the
  Gumbel-top-p of ``s/T + g`` with ``g = -ln(-ln u)`` from supplied uniforms;
* gather: the b = v/c tokens of each chosen cluster come from the dense
  cluster-to-token map C2T (section 1.2.1), slot ``k*b + j`` <-> ``C2T[k][j]``;
* stage 2, candidate logits ``z_t = E_t h`` for those p*b tokens in full
  precision (section 1.2.4);
* output: argmax of the candidate logits, or a token drawn from
  ``softmax(z/T)`` over the candidates by inverse CDF with a supplied uniform.

All floating point is fp64 over exact widenings of the bf16 / INT4 inputs.
The readings taken where the pages are silent:

* ties in any ranking go to the lower id (cluster id for selection, token id
  for the argmax);
* uniforms are clamped, ``u`` to ``[2^-126, 1 - 2^-24]`` for Gumbel noise and
  ``u_tok`` to ``[0, 1 - 2^-24]`` for the token draw;
* temperature applies to both stages (softmax(z/T) for the token);
* candidates are in the canonical order (cluster id ascending, slot j
  ascending), which fixes the inverse-CDF walk independently of how a
  selection orders its output;
* INT4 codes are two's-complement nibbles, element 2i in the low nibble of
  byte i; a value is ``code * scale`` with the group's bf16 scale.

Every function here is pinned by ``tests/test_oracle_pins.py`` against
something other than itself (brute force in exact rational arithmetic,
closed forms of the Gumbel-max / Plackett-Luce laws, the p = c reduction to
the dense head, hand-worked golden fixtures).
"""
from __future__ import annotations

import numpy as np

U_CLUSTER_MIN = 2.0 ** -126
U_MAX = 1.0 - 2.0 ** -24
INT4_GROUP = 32


# ---------------------------------------------------------------------------
# exact input widening
# ---------------------------------------------------------------------------
def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact float64 values."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def dequantize_int4(C_q: np.ndarray, C_scales: np.ndarray) -> np.ndarray:
    """INT4 group-32 centroids -> exact float64 ``[c, d]``.

    Section 1.2.4 of the write-up quantises the centroids only ("quantize(C)
    @ h", e.g. INT4); the format is symmetric INT4 with one bf16 scale per 32
    elements. Byte i holds element 2i in its low nibble and 2i+1 in its high
    nibble, each a two's-complement code in -8..7. Value = code * scale, which
    is exact in fp64.
    """
    q = np.asarray(C_q, dtype=np.uint8)
    c, half = q.shape
    d = 2 * half
    lo = (q & 0x0F).astype(np.int16)
    hi = (q >> 4).astype(np.int16)
    codes = np.empty((c, d), dtype=np.int16)
    codes[:, 0::2] = lo
    codes[:, 1::2] = hi
    codes = np.where(codes >= 8, codes - 16, codes)            # two's complement nibble
    scale = widen_bf16(C_scales)                                 # [c, d/32]
    if scale.shape != (c, d // INT4_GROUP):
        raise ValueError("scales must be [c, d/32]")
    return codes.astype(np.float64) * np.repeat(scale, INT4_GROUP, axis=1)


def dequantize_int8(C_q: np.ndarray, C_scales: np.ndarray) -> np.ndarray:
    """INT8 group-32 centroids -> exact float64 ``[c, d]``.

    The W8A16 row of the write-up's parameter table (section 5.2) with the
    stage-1 quantisation of section 1.2.4: one two's-complement byte per
    element and one bf16 scale per 32 elements; value = code * scale, exact in
    fp64 (and in fp32: at most 7 + 8 significant bits).
    """
    q = np.asarray(C_q).view(np.int8) if np.asarray(C_q).dtype == np.uint8 else np.asarray(C_q, dtype=np.int8)
    c, d = q.shape
    scale = widen_bf16(C_scales)
    if scale.shape != (c, d // INT4_GROUP) or d % INT4_GROUP:
        raise ValueError("scales must be [c, d/32]")
    return q.astype(np.float64) * np.repeat(scale, INT4_GROUP, axis=1)


def centroid_matrix(head) -> np.ndarray:
    """The stage-1 centroid matrix in fp64: INT8 or INT4 dequantised if present, else bf16 C."""
    if getattr(head, "C_q8", None) is not None:
        return dequantize_int8(head.C_q8, head.C_scales8)
    if getattr(head, "C_q", None) is not None:
        return dequantize_int4(head.C_q, head.C_scales)
    return widen_bf16(head.C)


# ---------------------------------------------------------------------------
# C2T invariant (balanced clustering, section 1.2.1)
# ---------------------------------------------------------------------------
def check_c2t(C2T: np.ndarray, v: int) -> bool:
    """True iff C2T is ``[c, b]`` with ``c*b == v`` and its entries are a permutation of 0..v-1.

    Balanced clustering puts exactly b = v/c tokens in every cluster and every
    token in exactly one cluster.
    """
    m = np.asarray(C2T)
    if m.ndim != 2 or m.shape[0] * m.shape[1] != v:
        return False
    flat = m.reshape(-1).astype(np.int64)
    if flat.min(initial=0) < 0 or flat.max(initial=-1) >= v:
        return False
    seen = np.zeros(v, dtype=np.int64)
    np.add.at(seen, flat, 1)
    return bool(np.all(seen == 1))


# ---------------------------------------------------------------------------
# stage 1: centroid scores
# ---------------------------------------------------------------------------
def centroid_scores(Cw: np.ndarray, H: np.ndarray) -> np.ndarray:
    """``s[r, k] = sum_i C[k, i] * h_r[i]`` in fp64 (section 1.2.2, c x d mat-vec per row)."""
    Hw = widen_bf16(H) if H.dtype == np.uint16 else np.asarray(H, dtype=np.float64)
    return Hw @ Cw.T


# ---------------------------------------------------------------------------
# probe selection
# ---------------------------------------------------------------------------
def _top_p_by_key(keys: np.ndarray, p: int) -> np.ndarray:
    """Ids of the p largest keys, ordered by (key desc, id asc)."""
    ids = np.arange(keys.shape[0])
    order = np.lexsort((ids, -keys))
    return order[:p].astype(np.int32)


def select_greedy(S: np.ndarray, p: int) -> np.ndarray:
    """Deterministic multi-probe selection: the p highest scores per row (section 1.2.2)."""
    S = np.atleast_2d(S)
    return np.stack([_top_p_by_key(S[r], p) for r in range(S.shape[0])])


def gumbel_keys(S: np.ndarray, U: np.ndarray, T: float) -> np.ndarray:
    """Perturbed keys ``s/T + g`` with ``g = -ln(-ln u)`` (sampling reading of section 1.2.3).

    Taking the p largest of these keys draws p clusters without replacement
    with Plackett-Luce probabilities proportional to ``exp(s/T)``.
    """
    if not T > 0:
        raise ValueError("temperature must be > 0")
    u = np.clip(np.asarray(U, dtype=np.float64), U_CLUSTER_MIN, U_MAX)
    g = -np.log(-np.log(u))
    return np.asarray(S, dtype=np.float64) / T + g


def select_sampled(S: np.ndarray, U: np.ndarray, p: int, T: float) -> np.ndarray:
    """Multinomial probe selection at temperature T from supplied uniforms (section 1.2.3)."""
    K = np.atleast_2d(gumbel_keys(S, U, T))
    return np.stack([_top_p_by_key(K[r], p) for r in range(K.shape[0])])


def adaptive_probe_count(S: np.ndarray, tau: float, p_min: int, p_max: int, T: float = 1.0) -> np.ndarray:
    """Probes per row adapted to the spread of its centroid scores (section 1.2.2, "dynamic adjustment").

    The write-up lets the number of probes follow the distribution of the
    hidden state's centroid scores, with fewer probes where it is peaked
    (section 4.2: frequent tokens need fewer). Read here as: the smallest
    ``p`` in ``[p_min, p_max]`` whose top-``p`` clusters hold at least a
    fraction ``tau`` of ``softmax(s / T)`` over all c clusters. The mass of
    the top p depends only on the p largest values, not on how ties among
    them are ordered.
    """
    if not 0.0 < tau <= 1.0 or not 1 <= p_min <= p_max:
        raise ValueError("need 0 < tau <= 1 and 1 <= p_min <= p_max")
    if not T > 0:
        raise ValueError("temperature must be > 0")
    S = np.atleast_2d(np.asarray(S, dtype=np.float64))
    p_max = min(p_max, S.shape[1])
    out = np.empty(S.shape[0], dtype=np.int32)
    for r in range(S.shape[0]):
        y = np.sort(S[r] / T)[::-1]
        w = np.exp(y - y[0])
        mass = np.cumsum(w) / w.sum()
        p = int(np.searchsorted(mass, tau, side="left")) + 1   # first p with mass >= tau
        out[r] = min(max(p, p_min), p_max)
    return out


# ---------------------------------------------------------------------------
# gather + stage 2 candidate logits
# ---------------------------------------------------------------------------
def candidate_tokens(C2T: np.ndarray, cluster_ids: np.ndarray) -> np.ndarray:
    """Token ids of the chosen clusters in canonical order (cluster asc, slot asc).

    Slot arithmetic of section 1.2.1: slot ``k*b + j`` of the flattened map is
    token ``C2T[k][j]``.
    """
    ks = np.sort(np.asarray(cluster_ids, dtype=np.int64))
    b = C2T.shape[1]
    flat = np.asarray(C2T).reshape(-1)
    slots = (ks[:, None] * b + np.arange(b)[None, :]).reshape(-1)
    return flat[slots].astype(np.int32)


def candidate_logits(E: np.ndarray, C2T: np.ndarray, h: np.ndarray, cluster_ids: np.ndarray):
    """``(tokens, z)`` for one hidden state: ``z_t = E_t . h`` over the gathered candidates.

    Stage 2 of section 1.2.4 ("E[top_clusters] @ h", kept at full precision).
    """
    toks = candidate_tokens(C2T, cluster_ids)
    hw = widen_bf16(h) if np.asarray(h).dtype == np.uint16 else np.asarray(h, dtype=np.float64)
    z = widen_bf16(E[toks]) @ hw
    return toks, z


# ---------------------------------------------------------------------------
# output token
# ---------------------------------------------------------------------------
def greedy_token(tokens: np.ndarray, z: np.ndarray):
    """Argmax of the candidate logits; equal logits go to the lowest token id."""
    order = np.lexsort((tokens, -z))
    i = order[0]
    return int(tokens[i]), float(z[i])


def sample_token(tokens: np.ndarray, z: np.ndarray, T: float, u_tok: float) -> int:
    """Draw from ``softmax(z/T)`` over the candidates by inverse CDF (section 1.2.3).

    Weights ``w = exp(z/T - max(z/T))`` are walked in the given (canonical)
    order; the token is the first whose running sum exceeds ``u_tok * sum(w)``.
    """
    if not T > 0:
        raise ValueError("temperature must be > 0")
    y = np.asarray(z, dtype=np.float64) / T
    w = np.exp(y - y.max())
    cdf = np.cumsum(w)
    u = min(max(float(u_tok), 0.0), U_MAX)
    i = int(np.searchsorted(cdf, u * cdf[-1], side="right"))
    return int(tokens[min(i, len(tokens) - 1)])


def speculative_verify(z_full: np.ndarray, cand_tokens: np.ndarray, T: float, draft: int,
                       u_accept: float, u_resample: float) -> int:
    """Check a FlashHead draft token against the dense head (section 4.2, speculative decoding).

    The write-up drafts with FlashHead sampling and accepts or rejects with
    the original head's probabilities. Read as standard speculative
    sampling with the draft law taken given the chosen clusters: ``q`` =
    ``softmax(z/T)`` over the candidate tokens (zero elsewhere), ``p`` =
    ``softmax(z/T)`` over the whole vocabulary. The draft is kept when
    ``u_accept < p(x) / q(x)``; otherwise the token is drawn by inverse CDF
    (token id order, first running sum above ``u_resample`` times the total)
    from ``max(0, p - q)``. For every cluster set the result follows ``p``
    exactly, so the two-stage head's approximation disappears at the cost of
    one dense pass.
    """
    if not T > 0:
        raise ValueError("temperature must be > 0")
    z = np.asarray(z_full, dtype=np.float64) / T
    p = np.exp(z - z.max())
    p /= p.sum()
    toks = np.asarray(cand_tokens, dtype=np.int64)
    zc = z[toks]
    qc = np.exp(zc - zc.max())
    qc /= qc.sum()
    q = np.zeros_like(p)
    q[toks] = qc
    x = int(draft)
    if q[x] <= 0.0:
        raise ValueError("the draft must be one of the candidates")
    if u_accept < p[x] / q[x]:
        return x
    r = np.maximum(p - q, 0.0)
    cdf = np.cumsum(r)
    u = min(max(float(u_resample), 0.0), U_MAX)
    i = int(np.searchsorted(cdf, u * cdf[-1], side="right"))
    return min(i, len(r) - 1)


# ---------------------------------------------------------------------------
# whole path
# ---------------------------------------------------------------------------
def decode(head, H: np.ndarray, p: int, *, mode: str = "greedy", T: float = 1.0,
           U: np.ndarray | None = None, u_tok: np.ndarray | None = None):
    """FlashHead for a batch of hidden states (section 2.2.2: h -> centroid scores ->
    top-p clusters -> token scores -> token).

    Returns ``(tokens [B], cluster_ids [B, p] in selection order, max_logit [B])``.
    """
    H = np.atleast_2d(H)
    Cw = centroid_matrix(head)
    S = centroid_scores(Cw, H)
    if mode == "greedy":
        ids = select_greedy(S, p)
    elif mode == "gumbel":
        ids = select_sampled(S, np.atleast_2d(U), p, T)
    else:
        raise ValueError(mode)
    out = np.empty(H.shape[0], dtype=np.int32)
    mx = np.empty(H.shape[0], dtype=np.float64)
    for r in range(H.shape[0]):
        toks, z = candidate_logits(head.E, head.C2T, H[r], ids[r])
        t_g, m = greedy_token(toks, z)
        mx[r] = m
        out[r] = t_g if mode == "greedy" else sample_token(toks, z, T, float(u_tok[r]))
    return out, ids, mx


def dense_head(E: np.ndarray, H: np.ndarray, *, rows_per_chunk: int = 8192):
    """Dense comparison head ``z = E h`` over the whole vocabulary (section 1.1).

    Returns ``(z [B, v], argmax [B])`` with the lowest-id tie-break. Rows of E
    are widened a slice at a time only to bound memory; each logit is the same
    single dot product either way.
    """
    H = np.atleast_2d(H)
    Hw = widen_bf16(H)
    v = E.shape[0]
    z = np.empty((H.shape[0], v), dtype=np.float64)
    for r0 in range(0, v, rows_per_chunk):
        r1 = min(v, r0 + rows_per_chunk)
        z[:, r0:r1] = Hw @ widen_bf16(E[r0:r1]).T
    return z, np.argmax(z, axis=1).astype(np.int32)   # argmax returns the first (lowest) index on ties
