"""Clustering builder (CUDA, through the C ABI) vs the fp64 k-means oracle (needs a B200).

Every step of the offline clustering (FlashHead write-up, section 2.1, with the
balance rule of section 1.2.1) is compared with the oracle on the same seeded
inputs: row normalisation (within one bf16 unit in the last place), the
tensor-core similarity product (fp32 accumulation bound), the balanced
assignment (exactly the oracle's greedy, on the same fp32 similarities, with
random, heavily tied and one-sided preferences), the centre update (one bf16
unit, and the zero-mean rule), the k-means++ seeding (every draw inside the
oracle's inverse-CDF interval for the draws before it), and whole runs
(planted clusters recovered exactly; a k-means++ run that ends on a repeated
assignment).
"""
import ctypes
import math

import numpy as np
import pytest

import oracle
import synth
from oracle import kmeans

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

V, D, C = 2048, 256, 128   # b = 16 tokens per cluster
B = V // C


@pytest.fixture(scope="module")
def fh():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lm_output_head_b200 import build
    build.build()
    import lm_output_head_b200 as m
    return m


@pytest.fixture(scope="module")
def cb(fh):
    from lm_output_head_b200.cluster import ClusterBuilder
    b = ClusterBuilder(V, D, C)
    yield b
    b.close()


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _embeddings(seed):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((V, D)) * rng.uniform(0.2, 3.0, size=(V, 1))
    X[5] = 0.0
    return synth.to_bf16_bits(X.astype(np.float32))


def _planted(seed, noise=0.1):
    rng = np.random.default_rng(seed)
    mu = rng.standard_normal((C, D))
    mu /= np.linalg.norm(mu, axis=1, keepdims=True)
    perm = rng.permutation(V)
    X = np.empty((V, D))
    truth = np.empty(V, dtype=np.int64)
    for k in range(C):
        for j in range(B):
            t = perm[k * B + j]
            X[t] = (mu[k] + noise * rng.standard_normal(D) / math.sqrt(D)) * rng.uniform(0.5, 2.0)
            truth[t] = k
    return synth.to_bf16_bits(X.astype(np.float32)), truth


def _unit_rows(seed, n):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((n, D))
    X /= np.linalg.norm(X, axis=1, keepdims=True)
    return synth.to_bf16_bits(X.astype(np.float32))


def test_normalize_rows(fh, cb):
    bits = _embeddings(0)
    got = _bits(cb.normalize(fh.bf16_from_bits(bits, "cuda")))
    want = synth.to_bf16_bits(kmeans.normalize_rows(oracle.widen_bf16(bits)).astype(np.float32))
    diff = np.abs(got.astype(np.int32) - want.astype(np.int32))
    assert diff.max() <= 1
    assert np.mean(diff == 0) > 0.99
    assert np.all(got[5] == 0)


def test_similarities_match_fp64(fh, cb):
    En = cb.normalize(fh.bf16_from_bits(_embeddings(1), "cuda"))
    Cb = _unit_rows(2, C)
    S = cb.similarities(En, fh.bf16_from_bits(Cb, "cuda")).cpu().numpy()
    Ew, Cw = oracle.widen_bf16(_bits(En)), oracle.widen_bf16(Cb)
    want = Cw @ Ew.T
    scale = np.linalg.norm(Cw, axis=1)[:, None] * np.linalg.norm(Ew, axis=1)[None, :]
    assert np.all(np.abs(S - want) <= 2e-3 * scale + 1e-30)
    tight = 2 * D * 2.0 ** -24 * (np.abs(Cw) @ np.abs(Ew).T)
    assert np.mean(np.abs(S - want) <= tight) >= 0.999


def _check_assign(cb, S_host):
    a, m, rounds = cb.assign(torch.from_numpy(S_host).cuda())
    want = kmeans.balanced_assign(S_host.T.astype(np.float64), B)
    assert a.cpu().numpy().tolist() == want.tolist()
    assert np.array_equal(m.cpu().numpy(), kmeans.c2t_from_assignment(want, C))
    assert rounds >= 1
    assert cb.device_status() == 0
    return rounds


def test_assign_equals_greedy_on_similarities(fh, cb):
    En = cb.normalize(fh.bf16_from_bits(_embeddings(3), "cuda"))
    S = cb.similarities(En, fh.bf16_from_bits(_unit_rows(4, C), "cuda")).cpu().numpy()
    _check_assign(cb, S)


def test_assign_equals_greedy_with_heavy_ties(cb):
    rng = np.random.default_rng(5)
    S = (np.round(rng.standard_normal((C, V)) * 2) / 2).astype(np.float32)
    _check_assign(cb, S)


def test_assign_equals_greedy_when_every_token_prefers_the_same_cluster(cb):
    rng = np.random.default_rng(6)
    S = (-np.arange(C, dtype=np.float64)[:, None] + rng.uniform(0, 0.5, size=(C, V))).astype(np.float32)
    rounds = _check_assign(cb, S)
    assert rounds > 1


def test_update_is_the_normalised_mean(fh, cb):
    bits = _embeddings(7)
    # tokens 100..107 and 200..207 are exact negatives: cluster 0 sums to zero and keeps its centre
    bits[200:208] = bits[100:108] ^ np.uint16(0x8000)
    En = cb.normalize(fh.bf16_from_bits(bits, "cuda"))
    rng = np.random.default_rng(8)
    rest = np.setdiff1d(np.arange(V), np.r_[100:108, 200:208])
    rest = rng.permutation(rest)
    row0 = np.ravel(np.column_stack([np.arange(100, 108), np.arange(200, 208)]))
    m = np.concatenate([row0, rest]).reshape(C, B).astype(np.int32)
    Cprev = _unit_rows(9, C)
    Cd = fh.bf16_from_bits(Cprev, "cuda")
    cb.update(En, torch.from_numpy(m).cuda(), Cd)
    got = _bits(Cd)
    assign = np.empty(V, dtype=np.int64)
    for k in range(C):
        assign[m[k]] = k
    want = kmeans.update_centres(oracle.widen_bf16(_bits(En)), assign, oracle.widen_bf16(Cprev))
    assert np.array_equal(got[0], Cprev[0])
    assert np.max(np.abs(oracle.widen_bf16(got[1:]) - want[1:])) <= 4e-3
    assert cb.device_status() == 0


def test_seed_draws_follow_the_inverse_cdf(fh, cb):
    En = cb.normalize(fh.bf16_from_bits(_embeddings(10), "cuda"))
    u = np.random.default_rng(11).uniform(size=C).astype(np.float32)
    ids = cb.seed(En, torch.from_numpy(u).cuda()).cpu().numpy()
    assert cb.device_status() == 0
    assert ids[0] == min(int(math.floor(float(u[0]) * V)), V - 1)
    assert len(set(ids.tolist())) == C
    X = oracle.widen_bf16(_bits(En))
    w = kmeans.seed_weights(X, ids[:1])
    for j in range(1, C):
        cdf = np.cumsum(w)
        total = cdf[-1]
        target = float(u[j]) * total
        tol = 1e-5 * total + 1e-12
        t = int(ids[j])
        assert w[t] > 0
        assert cdf[t] >= target - tol
        assert (cdf[t - 1] if t > 0 else 0.0) <= target + tol
        w = np.minimum(w, kmeans.seed_weights(X, [t]))


def test_build_recovers_planted_clusters(fh, cb):
    bits, truth = _planted(12)
    init = np.array([np.flatnonzero(truth == k)[0] for k in range(C)], dtype=np.int32)
    Cout, m, it = cb.build(fh.bf16_from_bits(bits, "cuda"), init_ids=torch.from_numpy(init).cuda(), max_iter=50)
    want = np.stack([np.flatnonzero(truth == k) for k in range(C)]).astype(np.int32)
    assert np.array_equal(m.cpu().numpy(), want)
    assert it == 2
    C_or, m_or, _, it_or, _ = kmeans.build_clusters(oracle.widen_bf16(bits), C, init_ids=init)
    assert np.array_equal(m_or, want) and it_or == 2
    assert np.max(np.abs(oracle.widen_bf16(_bits(Cout)) - C_or)) <= 4e-3


def test_build_from_kmeanspp_ends_on_a_repeated_assignment(fh, cb):
    bits = _embeddings(13)
    u = np.random.default_rng(14).uniform(size=C).astype(np.float32)
    E = fh.bf16_from_bits(bits, "cuda")
    Cout, m, it = cb.build(E, u_init=torch.from_numpy(u).cuda(), max_iter=300)
    m = m.cpu().numpy()
    assert oracle.check_c2t(m, V)
    assert np.all(np.diff(m, axis=1) > 0)
    assert 1 <= it < 300
    En = cb.normalize(E)
    _, m2, _ = cb.assign(cb.similarities(En, Cout))
    assert np.array_equal(m2.cpu().numpy(), m)


def test_create_rejects_bad_shapes(fh):
    from lm_output_head_b200 import _lib
    lib = _lib.load()
    h = ctypes.c_void_p()
    assert lib.fh_cluster_create(100, 256, 3, None, ctypes.byref(h)) == _lib.FH_ERR_INVALID_ARG
    assert lib.fh_cluster_create(4096, 250, 64, None, ctypes.byref(h)) == _lib.FH_ERR_INVALID_ARG
    assert lib.fh_cluster_create(4096, 256, 64, None, ctypes.byref(h)) == _lib.FH_ERR_UNSUPPORTED  # b = 64


def test_assign_at_the_llama_shape_has_no_blocking_pair(fh):
    """v 128256, c 8016, d 2048 from k-means++ seeds: the assignment is balanced and,
    on the same fp32 similarities, no token prefers a cluster whose weakest member
    it beats -- the property that makes it the global greedy (unique under the
    order similarity desc, token asc, cluster asc)."""
    from lm_output_head_b200.cluster import ClusterBuilder
    cfg, head, _, _ = synth.make_config(1, n_states=1)
    v, d, c, b = head.v, head.d, head.c, head.b
    cbl = ClusterBuilder(v, d, c)
    try:
        En = cbl.normalize(fh.bf16_from_bits(head.E, "cuda"))
        u = np.random.default_rng(21).uniform(size=c).astype(np.float32)
        ids = cbl.seed(En, torch.from_numpy(u).cuda())
        assert cbl.device_status() == 0
        idh = ids.cpu().numpy()
        assert idh[0] == min(int(math.floor(float(u[0]) * v)), v - 1) and len(set(idh.tolist())) == c
        S = cbl.similarities(En, cbl.gather(En, ids))
        a, m, rounds = cbl.assign(S)
        assert cbl.device_status() == 0
        mh = m.cpu().numpy()
        assert oracle.check_c2t(mh, v) and np.all(np.diff(mh, axis=1) > 0)
        a = a.long()
        t_all = torch.arange(v, device="cuda")
        sa = S[a, t_all]                                    # every token's similarity to its cluster
        ms = S.gather(1, m.long())                          # [c, b] members' similarities
        # weakest member of every cluster: lowest similarity, then highest token id
        ws = ms.min(dim=1).values
        wt = torch.where(ms == ws[:, None], m.long(), torch.full_like(m.long(), -1)).max(dim=1).values
        blocking = 0
        for k0 in range(0, c, 512):
            k1 = min(c, k0 + 512)
            Sc = S[k0:k1]
            kk = torch.arange(k0, k1, device="cuda")[:, None]
            pref = (Sc > sa[None, :]) | ((Sc == sa[None, :]) & (kk < a[None, :]))
            beats = (Sc > ws[k0:k1, None]) | ((Sc == ws[k0:k1, None]) & (t_all[None, :] < wt[k0:k1, None]))
            blocking += int((pref & beats & (kk != a[None, :])).sum().item())
        assert blocking == 0
        assert rounds >= 1
    finally:
        cbl.close()


def test_built_clusters_serve_as_a_head(fh):
    """Cluster a planted vocabulary on the GPU, build a FlashHead from the result (E, C_out,
    C2T_out) and decode: the tokens match the oracle's two-stage head on the same arrays."""
    from lm_output_head_b200.cluster import ClusterBuilder
    from tests import parity
    bits, truth = _planted(15, noise=0.3)
    rng = np.random.default_rng(16)
    u = rng.uniform(size=C).astype(np.float32)
    cbl = ClusterBuilder(V, D, C)
    try:
        E = fh.bf16_from_bits(bits, "cuda")
        Cout, m, it = cbl.build(E, u_init=torch.from_numpy(u).cuda(), max_iter=100)
        assert cbl.device_status() == 0
    finally:
        cbl.close()
    head = synth.Head(v=V, d=D, c=C, b=B, E=bits, C=_bits(Cout), C2T=m.cpu().numpy())
    assert oracle.check_c2t(head.C2T, V)
    dh = fh.FlashHead(E, m, C=Cout, max_batch=4, max_probes=8)
    try:
        Hx = synth.to_bf16_bits((rng.standard_normal((8, D)) * 0.5).astype(np.float32))
        rep = parity.Report()
        for r in range(8):
            tok = int(dh.decode(torch.from_numpy(Hx[r:r + 1].view(np.int16)).view(torch.bfloat16).cuda(), 8).item())
            ids = torch.empty((1, 8), dtype=torch.int32, device="cuda")
            dh.decode(torch.from_numpy(Hx[r:r + 1].view(np.int16)).view(torch.bfloat16).cuda(), 8,
                      out_cluster_ids=ids)
            Cw = oracle.centroid_matrix(head)
            S = oracle.centroid_scores(Cw, Hx[r:r + 1])[0]
            hw = oracle.widen_bf16(Hx[r])
            rep.add(parity.check_cluster_set(ids.cpu().numpy()[0], S, 8, parity.loose_bound(Cw, hw),
                                             parity.tight_bound(Cw, hw)))
            rep.add(parity.check_greedy_token(head, Hx[r], ids.cpu().numpy()[0], tok))
        assert rep.tight_mismatch == 0, rep
        assert dh.device_status() == 0
    finally:
        dh.close()
