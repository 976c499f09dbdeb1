"""Clustering builder at the sizes that reach its full-size paths (needs a B200).

The small-shape tests (v 2048, c 128, d 256) stay inside one 256-centre chunk
of the similarity product and one 128-row tile block. Here, against the same
fp64 k-means oracle (FlashHead write-up, section 2.1, with the balance rule of
section 1.2.1):

* v 16384, d 2048, c 1024, b 16: the similarity step runs four 256-centre
  chunks, each two 128-row tcgen05 blocks, over a 2048-wide contraction;
  the assignment's proposal / accept rounds see 1024 clusters;
* v 8192, d 512, c 256, b 32: b at its limit (one warp holds a cluster's
  list of b held tokens, every lane busy), one full 256-centre chunk.

Checks: similarities within the fp32 accumulation bound (sampled tokens, all
centres), the assignment equal to the oracle's global greedy on the GPU's own
fp32 similarities, the centre update within one bf16 unit of the oracle's
normalised mean, and a whole build on planted clusters recovering them.
"""
import math

import numpy as np
import pytest

import oracle
import synth
from oracle import kmeans

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

SHAPES = [(16384, 2048, 1024), (8192, 512, 256)]


@pytest.fixture(scope="module")
def fh():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lm_output_head_b200 import build
    build.build()
    import lm_output_head_b200 as m
    return m


@pytest.fixture(scope="module", params=SHAPES, ids=lambda s: f"v{s[0]}-d{s[1]}-c{s[2]}")
def shape(request, fh):
    from lm_output_head_b200.cluster import ClusterBuilder
    v, d, c = request.param
    cb = ClusterBuilder(v, d, c)
    yield v, d, c, cb
    cb.close()


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _rows(seed, n, d, spread=True):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((n, d))
    if spread:
        X *= rng.uniform(0.2, 3.0, size=(n, 1))
    else:
        X /= np.linalg.norm(X, axis=1, keepdims=True)
    return synth.to_bf16_bits(X.astype(np.float32))


def test_similarities_over_several_centre_chunks(fh, shape):
    v, d, c, cb = shape
    En = cb.normalize(fh.bf16_from_bits(_rows(31, v, d), "cuda"))
    Cb = _rows(32, c, d, spread=False)
    S = cb.similarities(En, fh.bf16_from_bits(Cb, "cuda")).cpu().numpy()
    assert cb.device_status() == 0
    cols = np.sort(np.random.default_rng(33).choice(v, 1024, replace=False))
    Ew = oracle.widen_bf16(_bits(En)[cols])
    Cw = oracle.widen_bf16(Cb)
    want = Cw @ Ew.T
    got = S[:, cols]
    scale = np.linalg.norm(Cw, axis=1)[:, None] * np.linalg.norm(Ew, axis=1)[None, :]
    assert np.all(np.abs(got - want) <= 2e-3 * scale + 1e-30)
    tight = 2 * d * 2.0 ** -24 * (np.abs(Cw) @ np.abs(Ew).T)
    assert np.mean(np.abs(got - want) <= tight) >= 0.999


def test_assignment_is_the_global_greedy(fh, shape):
    v, d, c, cb = shape
    b = v // c
    En = cb.normalize(fh.bf16_from_bits(_rows(34, v, d), "cuda"))
    S = cb.similarities(En, fh.bf16_from_bits(_rows(35, c, d, spread=False), "cuda"))
    a, m, rounds = cb.assign(S)
    assert cb.device_status() == 0
    S_host = S.cpu().numpy()
    want = kmeans.balanced_assign(S_host.T.astype(np.float64), b)
    assert np.array_equal(a.cpu().numpy(), want)
    assert np.array_equal(m.cpu().numpy(), kmeans.c2t_from_assignment(want, c))
    assert rounds >= 1


def test_update_is_the_normalised_mean(fh, shape):
    v, d, c, cb = shape
    b = v // c
    bits = _rows(36, v, d)
    En = cb.normalize(fh.bf16_from_bits(bits, "cuda"))
    perm = np.random.default_rng(37).permutation(v).astype(np.int32)
    m = perm.reshape(c, b)
    C0 = fh.bf16_from_bits(_rows(38, c, d, spread=False), "cuda")
    Cn = cb.update(En, torch.from_numpy(m).cuda(), C0.clone())
    assert cb.device_status() == 0
    assign = np.empty(v, dtype=np.int64)
    for k in range(c):
        assign[m[k]] = k
    want = kmeans.update_centres(oracle.widen_bf16(_bits(En)), assign, oracle.widen_bf16(_bits(C0)))
    got = _bits(Cn)
    assert np.max(np.abs(oracle.widen_bf16(got) - want)) <= 4e-3
    # fp32 sums of bf16 rows: the rounded result is the oracle's rounded mean but near rounding ties
    want_bits = synth.to_bf16_bits(want.astype(np.float32))
    assert np.mean(got == want_bits) > 0.99


def test_build_recovers_planted_clusters(fh, shape):
    v, d, c, cb = shape
    b = v // c
    rng = np.random.default_rng(39)
    mu = rng.standard_normal((c, d))
    mu /= np.linalg.norm(mu, axis=1, keepdims=True)
    perm = rng.permutation(v)
    truth = np.empty(v, dtype=np.int64)
    truth[perm] = np.repeat(np.arange(c), b)
    X = mu[truth] + 0.1 * rng.standard_normal((v, d)) / math.sqrt(d)
    X *= rng.uniform(0.5, 2.0, size=(v, 1))
    bits = synth.to_bf16_bits(X.astype(np.float32))
    # one seed token from every planted cluster, in a shuffled order
    init = perm.reshape(c, b)[rng.permutation(c), 0].astype(np.int32)
    C, m, it = cb.build(fh.bf16_from_bits(bits, "cuda"), init_ids=torch.from_numpy(init).cuda(), max_iter=20)
    assert cb.device_status() == 0
    mh = m.cpu().numpy()
    assert oracle.check_c2t(mh, v)
    # every built cluster holds exactly one planted cluster's tokens
    for k in range(c):
        assert len(set(truth[mh[k]].tolist())) == 1
    assert 1 <= it <= 20
