"""CUDA path vs fp64 oracle, through the C ABI (needs a B200).

Sizes: the tiny planted head at full size (several tiles, ragged tails) and
the full-size Llama-3.2-1B-, Qwen3-4B- and Gemma-3-shaped heads on sampled
rows, in the same launch configuration the benchmark times. Every entry point
is covered: centroid scores, cluster selection, candidate logits, decode
(greedy and Gumbel sampling, bf16 and INT4 centroids) and the dense head.
"""
import math

import numpy as np
import pytest

import oracle
import synth
from tests import parity

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

_HEADS = {}


@pytest.fixture(scope="session")
def fh():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lm_output_head_b200 import build
    build.build()
    import lm_output_head_b200 as m
    return m


def _to_dev(head, max_batch, max_probes, fh_mod, int4=None):
    dev = "cuda"
    E = fh_mod.bf16_from_bits(head.E, dev)
    C2T = torch.from_numpy(head.C2T).to(dev)
    use_int4 = head.C_q is not None if int4 is None else int4
    if use_int4:
        Cq = torch.from_numpy(head.C_q).to(dev)
        Cs = fh_mod.bf16_from_bits(head.C_scales, dev)
        return fh_mod.FlashHead(E, C2T, C_q=Cq, C_scales=Cs, max_batch=max_batch, max_probes=max_probes)
    C = fh_mod.bf16_from_bits(head.C, dev)
    return fh_mod.FlashHead(E, C2T, C=C, max_batch=max_batch, max_probes=max_probes)


def get_cfg(cfg_id, fh_mod, n_states=None, max_batch=None, max_probes=None):
    if cfg_id == 0:  # one tiny head serves every tiny-case test (B up to 65, p up to c)
        n_states, max_batch, max_probes = 65, 65, 256
    elif cfg_id == 1:
        max_batch = 8
    key = (cfg_id, n_states, max_batch, max_probes)
    if key not in _HEADS:
        cfg, head, hid, uni = synth.make_config(cfg_id, n_states=n_states)
        mb = max_batch or max(cfg.batches)
        mp = max_probes or cfg.p
        _HEADS[key] = (cfg, head, hid, uni, _to_dev(head, mb, mp, fh_mod))
    return _HEADS[key]


def hid_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _score_tols(head, H):
    Cw = oracle.centroid_matrix(head)
    tau = []
    tight = []
    for r in range(H.shape[0]):
        hw = oracle.widen_bf16(H[r])
        tau.append(parity.loose_bound(Cw, hw))
        tight.append(parity.tight_bound(Cw, hw))
    return Cw, np.array(tau), np.array(tight)


# ---------------------------------------------------------------------------
# host-side argument and create-time errors
# ---------------------------------------------------------------------------
def test_create_rejects_bad_c2t(fh):
    cfg, head, hid, _ = synth.make_config(0)
    for mutate in ("dup", "oor"):
        bad = head.C2T.copy()
        if mutate == "dup":
            bad[3, 1] = bad[9, 2]
        else:
            bad[0, 0] = cfg.v + 5
        h2 = synth.Head(v=head.v, d=head.d, c=head.c, b=head.b, E=head.E, C=head.C, C2T=bad)
        with pytest.raises(fh.FlashHeadError) as ei:
            _to_dev(h2, 1, cfg.p, fh)
        assert ei.value.status == 2  # FH_ERR_INVALID_C2T


def test_create_rejects_bad_shapes(fh):
    cfg, head, hid, _ = synth.make_config(0)
    E = fh.bf16_from_bits(head.E)
    C = fh.bf16_from_bits(head.C)
    C2T = torch.from_numpy(head.C2T).cuda()
    with pytest.raises(fh.FlashHeadError) as ei:     # max_probes > c
        fh.FlashHead(E, C2T, C=C, max_batch=1, max_probes=cfg.c + 1)
    assert ei.value.status == 1
    with pytest.raises(fh.FlashHeadError) as ei:     # v != c*b
        fh.FlashHead(E[:-16], C2T, C=C, max_batch=1, max_probes=4)
    assert ei.value.status == 1
    with pytest.raises(fh.FlashHeadError) as ei:     # INT4 needs d % 32 == 0
        Cq = torch.zeros((cfg.c, 4), dtype=torch.uint8, device="cuda")
        Cs = torch.zeros((cfg.c, 1), dtype=torch.bfloat16, device="cuda")
        fh.FlashHead(E[:, :8].contiguous(), C2T, C_q=Cq, C_scales=Cs, max_batch=1, max_probes=4)
    assert ei.value.status == 1


def test_call_argument_errors(fh):
    cfg, head, hid, _, dh = get_cfg(0, fh, n_states=65, max_batch=65)
    H = hid_dev(hid.H[:2])
    for kw in ({"p": 0}, {"p": cfg.c + 1}, {"p": 4, "mode": "gumbel", "T": 0.0},
               {"p": 4, "mode": "gumbel", "T": -1.0}):
        mode = kw.get("mode", "greedy")
        with pytest.raises(fh.FlashHeadError) as ei:
            dh.decode(H, kw["p"], mode=mode, T=kw.get("T", 1.0),
                      u_clusters=torch.zeros((2, cfg.c), device="cuda"),
                      u_token=torch.zeros(2, device="cuda"))
        assert ei.value.status == 1
    with pytest.raises(fh.FlashHeadError) as ei:  # sampling without uniforms
        dh.decode(H, 4, mode="gumbel", T=1.0)
    assert ei.value.status == 1
    with pytest.raises(fh.FlashHeadError) as ei:  # B above max_batch
        dh.decode(hid_dev(np.zeros((66, cfg.d), np.uint16)), 4)
    assert ei.value.status == 1
    with pytest.raises(fh.FlashHeadError) as ei:  # misaligned hidden pointer
        flat = hid_dev(np.zeros(cfg.d + 8, np.uint16))
        dh.decode(flat[1:cfg.d + 1].view(1, cfg.d), 4)
    assert ei.value.status == 1
    assert dh.device_status() == 0


def test_workspace_limit_gives_oom(fh, monkeypatch):
    cfg, head, hid, _ = synth.make_config(0)
    monkeypatch.setenv("FH_TEST_WORKSPACE_LIMIT", "4096")
    with pytest.raises(fh.FlashHeadError) as ei:
        _to_dev(head, 1, cfg.p, fh)
    assert ei.value.status == 4  # FH_ERR_OOM


# ---------------------------------------------------------------------------
# stage 1: centroid scores
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("cfg_id,B", [(0, 1), (0, 7), (0, 8), (0, 32), (0, 64), (0, 65), (1, 1), (2, 1), (2, 4),
                                      (2, 15), (2, 16), (3, 32), (4, 256)])
def test_centroid_scores(fh, cfg_id, B):
    """From B = 8 (bf16) or B = 16 (INT4) the tcgen05 tile GEMM scores the centroids
    (INT4 dequantised as exact hi + lo bf16 pairs); smaller batches stream centroid
    rows on CUDA cores. Both sides of each threshold are covered."""
    cfg, head, hid, _, dh = get_cfg(cfg_id, fh)
    H = hid.H[:B]
    s = dh.centroid_scores(hid_dev(H)).cpu().numpy()
    assert dh.device_status() == 0
    Cw = oracle.centroid_matrix(head)
    S = oracle.centroid_scores(Cw, H)
    rows = range(B) if B <= 32 else range(0, B, 16)
    tight = []
    for r in rows:
        tight.append(parity.check_values(s[r], S[r], Cw, oracle.widen_bf16(H[r]), f"scores row {r}"))
    assert np.mean(tight) >= 0.999


# ---------------------------------------------------------------------------
# selection
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("cfg_id,mode", [(0, "greedy"), (1, "greedy"), (3, "gumbel"), (0, "gumbel")])
def test_select_clusters(fh, cfg_id, mode):
    cfg, head, hid, uni, dh = get_cfg(cfg_id, fh)
    B = min(8, hid.H.shape[0])
    H = hid.H[:B]
    Cw = oracle.centroid_matrix(head)
    S = oracle.centroid_scores(Cw, H)
    # the GPU selects from the oracle's own scores (rounded to fp32), isolating selection
    s32 = torch.from_numpy(S.astype(np.float32)).cuda()
    T = cfg.temperature if mode == "gumbel" else 1.0
    if uni is None:
        rng = np.random.default_rng(77)
        U = rng.random((B, cfg.c), dtype=np.float32)
    else:
        U = uni[0][:B]
    u_dev = torch.from_numpy(U).cuda() if mode == "gumbel" else None
    ids = dh.select_clusters(s32, cfg.p, mode=mode, T=T, u_clusters=u_dev).cpu().numpy()
    assert dh.device_status() == 0
    rep = parity.Report()
    for r in range(B):
        assert np.all(np.diff(ids[r]) > 0), "ids must be ascending"
        S_r = S[r].astype(np.float32).astype(np.float64)
        if mode == "gumbel":
            keys = oracle.gumbel_keys(S_r[None], U[r][None], T)[0]
            g = keys - S_r / T
            tau = np.full(cfg.c, 1e-5) * (1 + np.abs(g)) + np.abs(S_r) * 1e-6 / T
        else:
            keys = S_r
            tau = np.full(cfg.c, 1e-6) * (1 + np.abs(S_r))
        rep.add(parity.check_cluster_set(ids[r], keys, cfg.p, tau, tau))
    assert rep.tight_mismatch == 0


# ---------------------------------------------------------------------------
# candidate logits for given clusters
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("cfg_id,B", [(0, 4), (1, 2), (3, 3)])
def test_candidate_logits(fh, cfg_id, B):
    cfg, head, hid, _, dh = get_cfg(cfg_id, fh)
    H = hid.H[:B]
    rng = np.random.default_rng(cfg_id)
    ids = np.stack([rng.permutation(cfg.c)[:cfg.p] for _ in range(B)]).astype(np.int32)
    toks, logits = dh.candidate_logits(hid_dev(H), torch.from_numpy(ids).cuda())
    toks, logits = toks.cpu().numpy(), logits.cpu().numpy()
    assert dh.device_status() == 0
    tight = []
    for r in range(B):
        t_ref, z_ref = oracle.candidate_logits(head.E, head.C2T, H[r], ids[r])
        assert np.array_equal(toks[r], t_ref), "candidate tokens must match exactly (canonical order)"
        tight.append(parity.check_values(logits[r], z_ref, oracle.widen_bf16(head.E[t_ref]),
                                         oracle.widen_bf16(H[r]), f"logits row {r}"))
    assert np.mean(tight) >= 0.999


def test_candidate_logits_rejects_bad_ids(fh):
    cfg, head, hid, _, dh = get_cfg(0, fh)
    B = 3
    ids = np.stack([np.arange(cfg.p) * 3 for _ in range(B)]).astype(np.int32)
    ids[1, 5] = cfg.c + 2          # out of range
    ids[2, 7] = ids[2, 8]          # repeated
    toks = torch.full((B, cfg.p * cfg.b), -7, dtype=torch.int32, device="cuda")
    logits = torch.full((B, cfg.p * cfg.b), -7.0, device="cuda")
    # call through the C ABI with preset outputs to see that skipped rows stay untouched
    from lm_output_head_b200.head import _ptr, _stream
    st = dh._lib.fh_candidate_logits(dh._h, _ptr(hid_dev(hid.H[:B])), B, cfg.p,
                                     _ptr(torch.from_numpy(ids).cuda()), _ptr(toks), _ptr(logits), _stream())
    assert st == 0
    assert dh.device_status() == 6   # FH_ERR_OUT_OF_RANGE
    assert dh.device_status() == 0   # cleared
    t = toks.cpu().numpy()
    assert np.all(t[1] == -7) and np.all(t[2] == -7)
    t_ref, _ = oracle.candidate_logits(head.E, head.C2T, hid.H[0], ids[0])
    assert np.array_equal(t[0], t_ref)


# ---------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------
def _decode_check_greedy(cfg, head, hid, dh, rows, B, p):
    rep = parity.Report()
    Cw = oracle.centroid_matrix(head)
    for r0 in range(0, len(rows), B):
        idx = rows[r0:r0 + B]
        if len(idx) < B:
            break
        H = hid.H[idx]
        out_ids = torch.empty((B, p), dtype=torch.int32, device="cuda")
        out_max = torch.empty(B, dtype=torch.float32, device="cuda")
        tok = dh.decode(hid_dev(H), p, out_cluster_ids=out_ids, out_max_logit=out_max).cpu().numpy()
        ids = out_ids.cpu().numpy()
        mx = out_max.cpu().numpy()
        assert dh.device_status() == 0
        S = oracle.centroid_scores(Cw, H)
        for r in range(B):
            hw = oracle.widen_bf16(H[r])
            rep.add(parity.check_cluster_set(ids[r], S[r], p, parity.loose_bound(Cw, hw),
                                             parity.tight_bound(Cw, hw)))
            rep.add(parity.check_greedy_token(head, H[r], ids[r], int(tok[r])))
            toks, z = oracle.candidate_logits(head.E, head.C2T, H[r], ids[r])
            i = int(np.nonzero(toks == tok[r])[0][0])
            assert abs(mx[r] - z[i]) <= parity.loose_bound(oracle.widen_bf16(head.E[toks[i:i + 1]]), hw)[0]
    return rep


@pytest.mark.parametrize("cfg_id,B,nrows", [(0, 1, 32), (1, 1, 24), (2, 1, 16), (2, 4, 16), (2, 16, 32),
                                            (4, 256, 256)])
def test_decode_greedy(fh, cfg_id, B, nrows):
    cfg, head, hid, _, dh = get_cfg(cfg_id, fh)
    if B == 1:
        assert dh.fused_b1
    rows = list(range(nrows))
    rep = _decode_check_greedy(cfg, head, hid, dh, rows, B, cfg.p)
    assert rep.tight_mismatch <= max(1, rep.n // 1000), rep


def test_decode_planted_rows_hit_their_cluster(fh):
    cfg, head, hid, _, dh = get_cfg(1, fh)
    rows = [r for r in range(64) if hid.planted[r] >= 0][:16]
    for r in rows:
        ids = torch.empty((1, cfg.p), dtype=torch.int32, device="cuda")
        tok = int(dh.decode(hid_dev(hid.H[r:r + 1]), cfg.p, out_cluster_ids=ids).item())
        assert hid.planted[r] in ids.cpu().numpy()[0]
        assert tok in head.C2T[hid.planted[r]]


@pytest.mark.parametrize("p", [1, 2, 255, 256])
def test_decode_probe_extremes_tiny(fh, p):
    cfg, head, hid, _, dh = get_cfg(0, fh, n_states=65, max_batch=65, max_probes=256)
    rep = _decode_check_greedy(cfg, head, hid, dh, list(range(8)), 1, p)
    assert rep.tight_mismatch == 0
    if p == cfg.c:   # p = c is the dense head
        H = hid.H[:8]
        _, am = oracle.dense_head(head.E, H)
        for r in range(8):
            t = int(dh.decode(hid_dev(H[r:r + 1]), p).item())
            assert t == am[r] or parity.check_greedy_token(head, H[r], np.arange(cfg.c), t).exempt


@pytest.mark.parametrize("B", [2, 63, 64, 65])
def test_decode_batched_tiny(fh, B):
    cfg, head, hid, _, dh = get_cfg(0, fh, n_states=65, max_batch=65, max_probes=256)
    rep = _decode_check_greedy(cfg, head, hid, dh, list(range(B)), B, cfg.p)
    assert rep.tight_mismatch == 0


def test_decode_ragged_hidden_size(fh):
    """d = 288 (not a multiple of the 256-element lane stride) with INT4 centroids, c not a multiple of the warps."""
    head = synth.make_head(2 * 999, 288, 999, seed_base=4242, int4=True)
    hid = synth.make_hidden(head, 6, seed_base=4242)
    for int4 in (False, True):
        dh = _to_dev(head, 3, 64, fh, int4=int4)
        h2 = synth.Head(v=head.v, d=head.d, c=head.c, b=head.b, E=head.E, C=head.C, C2T=head.C2T,
                        C_q=head.C_q if int4 else None, C_scales=head.C_scales if int4 else None)
        rep = _decode_check_greedy(None, h2, hid, dh, list(range(6)), 1, 64)
        rep.add(_decode_check_greedy(None, h2, hid, dh, list(range(6)), 3, 64))
        assert rep.tight_mismatch == 0
        dh.close()


@pytest.mark.parametrize("cfg_id,B", [(0, 1), (0, 4), (1, 1), (1, 3)])
def test_decode_all_scores_tied(fh, cfg_id, B):
    """h = 0: every centroid score and every logit is exactly 0, so the order
    (key desc, id asc) picks clusters 0..p-1 and the lowest candidate token id
    wins. On the Llama-3.2-1B-shaped head all 8016 keys share one histogram
    bin, more than the boundary rank takes, so the tie fallback runs."""
    cfg, head, hid, _, dh = get_cfg(cfg_id, fh)
    p = cfg.p
    out_ids = torch.empty((B, p), dtype=torch.int32, device="cuda")
    tok = dh.decode(hid_dev(np.zeros((B, cfg.d), np.uint16)), p, out_cluster_ids=out_ids).cpu().numpy()
    assert dh.device_status() == 0
    ids = out_ids.cpu().numpy()
    want_tok, _, _ = oracle.decode(head, np.zeros((1, cfg.d), np.uint16), p)
    for r in range(B):
        assert np.array_equal(ids[r], np.arange(p))
        assert tok[r] == int(np.min(head.C2T[:p])) == int(np.asarray(want_tok).ravel()[0])


def test_decode_duplicated_centroids(fh):
    """Centroid rows drawn from three patterns: every key is one of three
    values, so whole groups tie at the boundary; the chosen set is exact
    (lowest ids first within the boundary group) on both paths."""
    cfg, head, hid, _ = synth.make_config(0)
    rng = np.random.default_rng(77)
    pat = rng.integers(0, 3, size=cfg.c)
    C = head.C[np.array([5, 17, 101])[pat]].copy()  # three distinct centroid rows
    h2 = synth.Head(v=head.v, d=head.d, c=head.c, b=head.b, E=head.E, C=C, C2T=head.C2T)
    dh = _to_dev(h2, 4, cfg.p, fh, int4=False)
    H = hid.H[:4]
    Cw = oracle.centroid_matrix(h2)
    S = oracle.centroid_scores(Cw, H)
    for B in (1, 4):
        out_ids = torch.empty((B, cfg.p), dtype=torch.int32, device="cuda")
        tok = dh.decode(hid_dev(H[:B]), cfg.p, out_cluster_ids=out_ids).cpu().numpy()
        assert dh.device_status() == 0
        ids = out_ids.cpu().numpy()
        for r in range(B):
            vals = np.unique(S[r])
            assert len(vals) == 3 and np.min(np.diff(vals)) > 1e-3  # well separated: fp32 keeps the order
            assert np.array_equal(ids[r], np.sort(oracle.select_greedy(S[r:r + 1], cfg.p)[0]))
            rep = parity.check_greedy_token(h2, H[r], ids[r], int(tok[r]))
            assert rep.tight_mismatch == 0
    dh.close()


def _decode_check_gumbel(cfg, head, hid, uni, dh, rows, B, p, T):
    rep = parity.Report()
    Cw = oracle.centroid_matrix(head)
    U, ut = uni
    for r0 in range(0, len(rows), B):
        idx = rows[r0:r0 + B]
        H = hid.H[idx]
        out_ids = torch.empty((B, p), dtype=torch.int32, device="cuda")
        tok = dh.decode(hid_dev(H), p, mode="gumbel", T=T, u_clusters=torch.from_numpy(U[idx]).cuda(),
                        u_token=torch.from_numpy(ut[idx]).cuda(), out_cluster_ids=out_ids).cpu().numpy()
        ids = out_ids.cpu().numpy()
        assert dh.device_status() == 0
        S = oracle.centroid_scores(Cw, H)
        K = oracle.gumbel_keys(S, U[idx], T)
        for r in range(B):
            hw = oracle.widen_bf16(H[r])
            g = K[r] - S[r] / T
            tau = parity.loose_bound(Cw, hw) / T + 1e-5 * (1 + np.abs(g))
            tau_t = parity.tight_bound(Cw, hw) / T + 1e-6 * (1 + np.abs(g))
            rep.add(parity.check_cluster_set(ids[r], K[r], p, tau, tau_t))
            rep.add(parity.check_sampled_token(head, H[r], ids[r], int(tok[r]), T, float(ut[idx[r]])))
    return rep


def test_decode_b1_predicted_thresholds_never_change_results(fh):
    """The fused B = 1 decode predicts where the p-th key lies from the
    previous call and selects through a histogram of that region, falling
    back to a general selector when the prediction misses; results must not
    depend on the prediction."""
    cfg, head, hid, _, dh0 = get_cfg(1, fh)
    dh = fh.FlashHead(dh0.E, dh0.C2T, C=dh0.C, max_batch=1, max_probes=cfg.p)
    try:
        rep = _decode_check_greedy(cfg, head, hid, dh, [0], 1, cfg.p)
        assert dh.last_selection() == (0, True)     # first call: nothing predicted, all keys
        rep.add(_decode_check_greedy(cfg, head, hid, dh, list(range(1, 13)), 1, cfg.p))
        in_range, full = dh.last_selection()
        assert not full and in_range >= cfg.p, (in_range, full)
        assert rep.tight_mismatch <= 1, rep
        # sampling at temperatures far apart: the carried prediction is far off
        # (the region misses the boundary), then recovers
        rng = np.random.default_rng(77)
        U = rng.random((16, cfg.c), dtype=np.float32)
        ut = rng.random(16, dtype=np.float32)
        for i, T in enumerate((0.7, 0.7, 0.02, 50.0, 0.7)):
            r = _decode_check_gumbel(cfg, head, hid, (U, ut), dh, [3 * i, 3 * i + 1, 3 * i + 2], 1, cfg.p, T)
            assert r.tight_mismatch <= 1, (T, r)
        assert dh.device_status() == 0
    finally:
        dh.close()


def test_decode_batch_deduplicates_shared_clusters(fh):
    """Batched decodes group the chosen (row, cluster) pairs by cluster and read each
    distinct cluster's token rows once: a batch of one repeated hidden state gathers
    exactly p clusters, and every row gets the single-row answer."""
    cfg, head, hid, _, dh = get_cfg(0, fh, n_states=65, max_batch=65, max_probes=256)
    H = np.repeat(hid.H[3:4], 64, axis=0)
    tok = dh.decode(hid_dev(H), cfg.p).cpu().numpy()
    assert dh.device_status() == 0
    assert dh.query(1) == cfg.p              # FH_QUERY_LAST_UNION
    ref, _, _ = oracle.decode(head, H[:1], cfg.p)
    assert np.all(tok == tok[0])
    assert parity.check_greedy_token(head, H[0], oracle.select_greedy(
        oracle.centroid_scores(oracle.centroid_matrix(head), H[:1]), cfg.p)[0], int(tok[0])).tight_mismatch == 0
    # distinct rows: the union lies between p and min(c, B p)
    dh.decode(hid_dev(hid.H[:64]), cfg.p)
    u = dh.query(1)
    assert cfg.p <= u <= min(cfg.c, 64 * cfg.p)


def test_decode_gumbel_b1_tiny(fh):
    cfg, head, hid, _, dh = get_cfg(0, fh, n_states=65, max_batch=65, max_probes=256)
    rng = np.random.default_rng(31)
    uni = (rng.random((65, cfg.c), dtype=np.float32), rng.random(65, dtype=np.float32))
    rep = _decode_check_gumbel(cfg, head, hid, uni, dh, list(range(16)), 1, cfg.p, 0.7)
    assert rep.tight_mismatch == 0


def test_decode_gumbel_qwen_b32(fh):
    cfg, head, hid, uni, dh = get_cfg(3, fh)
    rep = _decode_check_gumbel(cfg, head, hid, uni, dh, list(range(64)), 32, cfg.p, cfg.temperature)
    assert rep.tight_mismatch <= max(1, rep.n // 1000), rep


# ---------------------------------------------------------------------------
# dense head
# ---------------------------------------------------------------------------
def _dense_check(cfg, head, hid, dh, B):
    H = hid.H[:B]
    am, z = dh.dense_head(hid_dev(H), want_logits=True)
    am, z = am.cpu().numpy(), z.cpu().numpy()
    assert dh.device_status() == 0
    zr, amr = oracle.dense_head(head.E, H)
    for r in range(B):
        hw = oracle.widen_bf16(H[r])
        sample = np.arange(cfg.v) if cfg.v <= 8192 else np.random.default_rng(r).choice(cfg.v, 4096, False)
        sample = np.union1d(sample, [amr[r], am[r]])
        Ew = oracle.widen_bf16(head.E[sample])
        parity.check_values(z[r, sample], zr[r, sample], Ew, hw, f"dense row {r}")
        if am[r] != amr[r]:
            gap = zr[r, amr[r]] - zr[r, am[r]]
            tau = parity.loose_bound(oracle.widen_bf16(head.E[[am[r], amr[r]]]), hw).sum()
            assert gap <= tau
    # argmax only (no logits written)
    am2 = dh.dense_head(hid_dev(H)).cpu().numpy()
    assert np.array_equal(am2, am)


@pytest.mark.parametrize("cfg_id,B", [(0, 1), (0, 33), (0, 65), (1, 1), (1, 4), (3, 2), (4, 64)])
def test_dense_head(fh, cfg_id, B):
    """B >= 64 runs the tcgen05 tile GEMM with the fused column argmax."""
    cfg, head, hid, _, dh = get_cfg(cfg_id, fh) if cfg_id else get_cfg(0, fh, n_states=65, max_batch=65,
                                                                       max_probes=256)
    _dense_check(cfg, head, hid, dh, B)


@pytest.mark.parametrize("cfg_id,B", [(0, 128), (0, 129), (0, 256), (4, 129), (4, 256)])
def test_dense_head_two_row_blocks(fh, cfg_id, B):
    """B > 128: the tcgen05 GEMM holds two 128-row blocks of hidden states per
    launch, and the fused argmax epilogue keeps a running maximum for each; B = 129
    leaves a one-row second block, B = 128 exactly one full block."""
    if cfg_id == 0:
        key = ("dense256", 0)
        if key not in _HEADS:
            cfg, head, hid, uni = synth.make_config(0, n_states=256)
            _HEADS[key] = (cfg, head, hid, uni, _to_dev(head, 256, 256, fh))
        cfg, head, hid, _, dh = _HEADS[key]
    else:
        cfg, head, hid, _, dh = get_cfg(cfg_id, fh)
    assert hid.H.shape[0] >= B
    _dense_check(cfg, head, hid, dh, B)


# ---------------------------------------------------------------------------
# bounded waits: a device-wide wait that runs out reports FH_ERR_TIMEOUT
# ---------------------------------------------------------------------------
def test_grid_wait_timeout_is_reported_and_recoverable(fh):
    cfg, head, hid, _, dh = get_cfg(0, fh, n_states=65, max_batch=65, max_probes=256)
    assert dh.fused_b1
    dh.set_spin_budget(0)
    dh.decode(hid_dev(hid.H[:1]), cfg.p)
    assert dh.device_status() == 7     # FH_ERR_TIMEOUT
    dh.set_spin_budget(2_000_000_000)
    rep = _decode_check_greedy(cfg, head, hid, dh, [0, 1, 2], 1, cfg.p)
    assert rep.tight_mismatch == 0
    assert dh.device_status() == 0
