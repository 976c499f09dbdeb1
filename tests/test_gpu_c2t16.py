"""The compact uint16 cluster-to-token map (FlashHead write-up, section 2.2.1;
v <= 65536) through the C ABI (needs a B200).

A head built on the uint16 map must give exactly the outputs of the same head
on the int32 map -- cluster sets, tokens, logits and token ids -- on every
path that reads the map (the fused B = 1 decode, the batched decode with its
de-duplicated tensor-core gather and the centroid GEMM, Gumbel sampling,
explicit candidate logits), and those outputs hold against the fp64 oracle.
fh_create checks the uint16 map like the int32 one and refuses it past
v = 65536.
"""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from tests import parity
from tests.test_gpu_parity import _decode_check_greedy, _decode_check_gumbel, hid_dev

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def heads():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lm_output_head_b200 import build
    build.build()
    import lm_output_head_b200 as fh
    cfg, head, hid, _ = synth.make_config(0, n_states=64)
    uni = synth.make_uniforms(64, cfg.c, seed_base=9100)
    E = fh.bf16_from_bits(head.E, "cuda")
    C = fh.bf16_from_bits(head.C, "cuda")
    t32 = torch.from_numpy(head.C2T).cuda()
    t16 = torch.from_numpy(head.C2T.astype(np.uint16).view(np.int16)).cuda()
    h32 = fh.FlashHead(E, t32, C=C, max_batch=64, max_probes=64)
    h16 = fh.FlashHead(E, t16, C=C, max_batch=64, max_probes=64)
    yield fh, cfg, head, hid, uni, h32, h16
    h32.close()
    h16.close()


def _run(dh, H, p, **kw):
    B = H.shape[0]
    ids = torch.empty((B, p), dtype=torch.int32, device="cuda")
    mx = torch.empty(B, dtype=torch.float32, device="cuda")
    tok = dh.decode(hid_dev(H), p, out_cluster_ids=ids, out_max_logit=mx, **kw)
    assert dh.device_status() == 0
    return tok.cpu().numpy(), ids.cpu().numpy(), mx.cpu().numpy()


@pytest.mark.parametrize("B", [1, 4, 64])
def test_greedy_matches_the_int32_map(heads, B):
    fh, cfg, head, hid, uni, h32, h16 = heads
    for r0 in range(0, 8 if B == 1 else B, B):
        H = hid.H[r0:r0 + B]
        a = _run(h32, H, cfg.p)
        b = _run(h16, H, cfg.p)
        for x, y in zip(a, b):
            assert np.array_equal(x, y)
    rep = _decode_check_greedy(cfg, head, hid, h16, list(range(B)), B, cfg.p)
    assert rep.tight_mismatch == 0, rep


@pytest.mark.parametrize("B", [1, 8])
def test_gumbel_matches_the_int32_map(heads, B):
    fh, cfg, head, hid, uni, h32, h16 = heads
    U, ut = uni
    idx = list(range(B))
    kw = dict(mode="gumbel", T=0.7, u_clusters=torch.from_numpy(U[idx]).cuda(),
              u_token=torch.from_numpy(ut[idx]).cuda())
    a = _run(h32, hid.H[idx], cfg.p, **kw)
    b = _run(h16, hid.H[idx], cfg.p, **kw)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    rep = _decode_check_gumbel(cfg, head, hid, uni, h16, idx, B, cfg.p, 0.7)
    assert rep.tight_mismatch == 0, rep


def test_candidate_token_ids_come_from_the_uint16_map(heads):
    fh, cfg, head, hid, uni, h32, h16 = heads
    B, p = 3, 5
    rng = np.random.default_rng(5)
    ids = np.stack([rng.choice(cfg.c, p, replace=False) for _ in range(B)]).astype(np.int32)
    H = hid.H[:B]
    toks, logits = h16.candidate_logits(hid_dev(H), torch.from_numpy(ids).cuda())
    toks, logits = toks.cpu().numpy(), logits.cpu().numpy()
    assert h16.device_status() == 0
    for r in range(B):
        want_t, want_z = oracle.candidate_logits(head.E, head.C2T, H[r], ids[r])
        assert np.array_equal(toks[r], want_t)
        hw = oracle.widen_bf16(H[r])
        parity.check_values(logits[r], want_z, oracle.widen_bf16(head.E[want_t]), hw, f"row {r}")


def test_create_checks_the_uint16_map(heads):
    fh, cfg, head, hid, uni, h32, h16 = heads
    E = fh.bf16_from_bits(head.E, "cuda")
    C = fh.bf16_from_bits(head.C, "cuda")
    bad = head.C2T.astype(np.uint16).copy()
    bad[3, 5] = bad[7, 1]                       # one token twice, another never
    with pytest.raises(fh.FlashHeadError) as ei:
        fh.FlashHead(E, torch.from_numpy(bad.view(np.int16)).cuda(), C=C)
    assert ei.value.status == 2                 # FH_ERR_INVALID_C2T
    # token ids past 65535 do not fit: refused before any device work
    from lm_output_head_b200 import _lib
    lib = _lib.load()
    big = torch.zeros(16, dtype=torch.int16, device="cuda")
    desc = _lib.HeadDesc(v=65552, d=256, c=4097, b=16, E=E.data_ptr(), C=C.data_ptr(), C_q=None, C_scales=None,
                         C2T=big.data_ptr(), fmt=0, max_batch=1, max_probes=16, c2t_format=_lib.FH_C2T_UINT16)
    h = ctypes.c_void_p()
    assert lib.fh_create(ctypes.byref(desc), None, ctypes.byref(h)) == _lib.FH_ERR_INVALID_ARG
    assert not h.value
