"""fp64 CPU oracle of FlashHead's offline balanced clustering (test infrastructure only).

THIS IS TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import it. The product path never
calls it and shares no code with it.

What it computes, in the order of the FlashHead write-up ("FlashHead技术解析",
www.framerc.cn/news/2430929), section 2.1 (offline clustering) with the
balance rule of section 1.2.1:

1. every token embedding is L2-normalised (spherical k-means);
2. the c starting centres are chosen by k-means++ seeding;
3. each iteration scores every token against every centre (cosine
   similarity of unit vectors, a v x c product), assigns tokens to clusters
   under the balance rule that every cluster holds exactly b = v/c tokens,
   and moves each centre to the normalised mean of its tokens;
4. the result is the centre matrix C and the dense cluster-to-token map C2T.

Readings taken where the pages are silent:

* "greedy reassignment" under the balance rule is read as the plain global
  greedy: all (token, cluster) pairs are visited by similarity descending
  (ties: lower token id, then lower cluster id) and a pair is taken when its
  token is still unassigned and its cluster still has room;
* k-means++ is the textbook seeding (Arthur and Vassilvitskii, 2007):
  the first centre is token ``floor(u_0 * v)``, every further centre is drawn
  with probability proportional to the squared Euclidean distance to the
  nearest centre chosen so far, by inverse CDF over token order with the
  supplied uniform (the first token whose running weight exceeds ``u * W``);
  if every weight is zero the lowest unchosen token is taken;
* a zero embedding stays zero after normalisation; a cluster whose mean is
  the zero vector keeps its previous centre;
* iteration stops after a step that leaves the assignment unchanged (the
  centres are then a fixed point) or after ``max_iter`` steps (the write-up's
  loop runs 1000);
* within a cluster, C2T lists its tokens in ascending token id.

Every function is pinned by ``tests/test_kmeans_pins.py`` against brute
force (the greedy assignment is the unique stable balanced assignment),
the unconstrained reduction (balanced argmax assignments are kept as is),
hand-worked fixtures and recovery of planted clusters.
"""
from __future__ import annotations

import numpy as np


def normalize_rows(X: np.ndarray) -> np.ndarray:
    """Rows scaled to unit L2 norm in fp64; zero rows stay zero (section 2.1, data preparation)."""
    X = np.asarray(X, dtype=np.float64)
    n = np.sqrt(np.sum(X * X, axis=1, keepdims=True))
    return np.divide(X, n, out=np.zeros_like(X), where=n > 0)


def kmeanspp_seeds(En: np.ndarray, c: int, u: np.ndarray) -> np.ndarray:
    """Token ids of the c starting centres by k-means++ seeding from the uniforms ``u[0..c)``.

    Section 2.1, initialisation ("k-means++"). Weights are the squared
    Euclidean distances ``D(x)^2`` to the nearest centre chosen so far.
    """
    En = np.asarray(En, dtype=np.float64)
    v = En.shape[0]
    u = np.asarray(u, dtype=np.float64)
    if not 1 <= c <= v or u.shape[0] < c:
        raise ValueError("need 1 <= c <= v and c uniforms")
    chosen = np.empty(c, dtype=np.int64)
    chosen[0] = min(int(np.floor(u[0] * v)), v - 1)
    diff = En - En[chosen[0]]
    d2 = np.sum(diff * diff, axis=1)
    taken = np.zeros(v, dtype=bool)
    taken[chosen[0]] = True
    for j in range(1, c):
        cdf = np.cumsum(d2)
        total = cdf[-1]
        if total > 0:
            i = int(np.searchsorted(cdf, u[j] * total, side="right"))
            i = min(i, v - 1)
        else:
            i = int(np.flatnonzero(~taken)[0])
        chosen[j] = i
        taken[i] = True
        diff = En - En[i]
        d2 = np.minimum(d2, np.sum(diff * diff, axis=1))
    return chosen


def seed_weights(En: np.ndarray, chosen) -> np.ndarray:
    """k-means++ weights ``D(x)^2``: squared Euclidean distance of every row to the
    nearest of the rows ``chosen`` (section 2.1, initialisation)."""
    En = np.asarray(En, dtype=np.float64)
    d2 = np.full(En.shape[0], np.inf)
    for i in chosen:
        diff = En - En[int(i)]
        d2 = np.minimum(d2, np.sum(diff * diff, axis=1))
    return d2


def balanced_assign(S: np.ndarray, b: int) -> np.ndarray:
    """Cluster of every token under the balance rule, from similarities ``S [v, c]`` (section 1.2.1).

    Global greedy over (token, cluster) pairs by similarity descending, ties
    to the lower token id then the lower cluster id; a pair is taken when its
    token is unassigned and its cluster holds fewer than b tokens.
    """
    S = np.asarray(S, dtype=np.float64)
    v, c = S.shape
    if v != c * b:
        raise ValueError("balanced clustering needs v == c * b")
    tok = np.repeat(np.arange(v), c)
    clu = np.tile(np.arange(c), v)
    order = np.lexsort((clu, tok, -S.reshape(-1)))
    assign = np.full(v, -1, dtype=np.int64)
    room = np.full(c, b, dtype=np.int64)
    left = v
    for f in order:
        t, k = tok[f], clu[f]
        if assign[t] < 0 and room[k] > 0:
            assign[t] = k
            room[k] -= 1
            left -= 1
            if left == 0:
                break
    return assign


def update_centres(En: np.ndarray, assign: np.ndarray, C_prev: np.ndarray) -> np.ndarray:
    """Each centre moved to the normalised mean of its tokens (section 2.1, centre update)."""
    c = C_prev.shape[0]
    C = np.array(C_prev, dtype=np.float64, copy=True)
    for k in range(c):
        m = En[assign == k].mean(axis=0)
        n = np.sqrt(np.sum(m * m))
        if n > 0:
            C[k] = m / n
    return C


def c2t_from_assignment(assign: np.ndarray, c: int) -> np.ndarray:
    """Dense ``[c, b]`` cluster-to-token map, each row's tokens in ascending id (section 1.2.1)."""
    assign = np.asarray(assign)
    rows = [np.flatnonzero(assign == k) for k in range(c)]
    b = len(rows[0])
    if any(len(r) != b for r in rows):
        raise ValueError("assignment is not balanced")
    return np.stack(rows).astype(np.int32)


def build_clusters(E: np.ndarray, c: int, *, u_init: np.ndarray | None = None,
                   init_ids: np.ndarray | None = None, max_iter: int = 1000):
    """Balanced spherical k-means over token embeddings ``E [v, d]`` (section 2.1).

    Starting centres are the tokens ``init_ids`` if given, else k-means++
    seeds drawn from ``u_init``. Returns ``(C [c, d] fp64 unit rows,
    C2T [c, b] int32, assign [v], iterations run, history)`` where
    ``history`` lists the assignment after every iteration.
    """
    En = normalize_rows(E)
    v = En.shape[0]
    if c < 1 or v % c:
        raise ValueError("balanced clustering needs c | v")
    b = v // c
    if init_ids is None:
        init_ids = kmeanspp_seeds(En, c, u_init)
    C = En[np.asarray(init_ids, dtype=np.int64)].copy()
    assign = None
    history = []
    it = 0
    for it in range(1, max_iter + 1):
        S = En @ C.T                      # cosine similarities of unit vectors
        new = balanced_assign(S, b)
        history.append(new)
        if assign is not None and np.array_equal(new, assign):
            break
        assign = new
        C = update_centres(En, assign, C)
    return C, c2t_from_assignment(assign, c), assign, it, history
