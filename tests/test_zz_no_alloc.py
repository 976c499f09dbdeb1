"""The allocation-free dense head (fh_dense_head_noalloc) against fh_dense_head
and against the fp64 oracle's dense head (FlashHead write-up, section 1.1),
through the C ABI. Its own file, collected last; it passes alone too."""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from tests import parity

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lm_output_head_b200 import build
    build.build()
    import lm_output_head_b200 as m
    cfg, head, hid, _ = synth.make_config(0, n_states=70)
    E = m.bf16_from_bits(head.E, "cuda")
    C = m.bf16_from_bits(head.C, "cuda")
    dh = m.FlashHead(E, torch.from_numpy(head.C2T).cuda(), C=C, max_batch=64, max_probes=cfg.p)
    H = torch.from_numpy(np.ascontiguousarray(hid.H).view(np.int16)).view(torch.bfloat16).cuda()
    yield m, m.load(), cfg, E, H, dh
    dh.close()


def _call(lib, E, H, B, logits, am):
    st = torch.cuda.current_stream().cuda_stream
    return lib.fh_dense_head_noalloc(E.data_ptr(), E.shape[0], E.shape[1], H.data_ptr(), B,
                                     logits.data_ptr() if logits is not None else None, am.data_ptr(), st)


@pytest.mark.parametrize("B", [1, 5, 8, 9, 64])
def test_matches_dense_head_on_two_calls_in_a_row(env, B):
    m, lib, cfg, E, H, dh = env
    ref_am, ref_z = dh.dense_head(H[:B], want_logits=True)
    for _ in range(2):  # the second call sees the scratch the first one left behind
        am = torch.full((B,), -1, dtype=torch.int32, device="cuda")
        z = torch.full((B, cfg.v), float("nan"), dtype=torch.float32, device="cuda")
        assert _call(lib, E, H, B, z, am) == 0
        torch.cuda.synchronize()
        assert torch.equal(am, ref_am)
        torch.testing.assert_close(z, ref_z, rtol=1e-6, atol=1e-6)


@pytest.mark.parametrize("B", [3, 9])
def test_matches_the_oracle(env, B):
    # every logit within the fp32 accumulation bound of the oracle's; the argmax equal
    # to the oracle's unless the two candidates' logits lie within that bound
    m, lib, cfg, E, H, dh = env
    _, head, hid, _ = synth.make_config(0, n_states=70)
    am = torch.full((B,), -1, dtype=torch.int32, device="cuda")
    z = torch.full((B, cfg.v), float("nan"), dtype=torch.float32, device="cuda")
    assert _call(lib, E, H, B, z, am) == 0
    torch.cuda.synchronize()
    am, z = am.cpu().numpy(), z.cpu().numpy()
    zr, amr = oracle.dense_head(head.E, hid.H[:B])
    Ew = oracle.widen_bf16(head.E)
    for r in range(B):
        hw = oracle.widen_bf16(hid.H[r])
        parity.check_values(z[r], zr[r], Ew, hw, f"noalloc dense row {r}")
        if am[r] != amr[r]:
            gap = zr[r, amr[r]] - zr[r, am[r]]
            assert gap <= parity.loose_bound(oracle.widen_bf16(head.E[[am[r], amr[r]]]), hw).sum()


def test_argmax_only_and_python_wrapper(env):
    m, lib, cfg, E, H, dh = env
    ref = dh.dense_head(H[:3])
    am = torch.full((3,), -1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        m.dense_head_noalloc(E, H[:3], am)
        torch.cuda.synchronize()
        assert torch.equal(am, ref)


def test_allocates_no_device_memory(env):
    m, lib, cfg, E, H, dh = env
    am = torch.full((8,), -1, dtype=torch.int32, device="cuda")
    z = torch.empty((8, cfg.v), dtype=torch.float32, device="cuda")
    assert _call(lib, E, H, 8, z, am) == 0  # first call on the device: set-up
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(4):
        assert _call(lib, E, H, 8, z, am) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_rejects_more_rows_than_the_fixed_scratch(env):
    m, lib, cfg, E, H, dh = env
    from lm_output_head_b200 import _lib
    B = _lib.FH_NOALLOC_MAX_ROWS + 1
    Hb = H[:1].repeat(B, 1).contiguous()
    am = torch.full((B,), -1, dtype=torch.int32, device="cuda")
    assert _call(lib, E, Hb, B, None, am) == _lib.FH_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert bool((am == -1).all())  # nothing launched
    with pytest.raises(m.FlashHeadError) as ei:
        m.dense_head_noalloc(E, Hb, am)
    assert ei.value.status == _lib.FH_ERR_INVALID_ARG


def test_argument_errors(env):
    m, lib, cfg, E, H, dh = env
    from lm_output_head_b200 import _lib
    am = torch.empty((2,), dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert lib.fh_dense_head_noalloc(None, cfg.v, cfg.d, H.data_ptr(), 2, None, am.data_ptr(), st) == 1
    assert lib.fh_dense_head_noalloc(E.data_ptr(), cfg.v, cfg.d, H.data_ptr(), 0, None, am.data_ptr(), st) == 1
    assert lib.fh_dense_head_noalloc(E.data_ptr(), cfg.v, 12, H.data_ptr(), 2, None, am.data_ptr(), st) == 1
    assert lib.fh_dense_head_noalloc(E.data_ptr(), cfg.v, cfg.d, H.data_ptr() + 2, 2, None, am.data_ptr(),
                                     st) == 1
    assert lib.fh_dense_head_noalloc(E.data_ptr(), cfg.v, 2568, H.data_ptr(), 2, None, am.data_ptr(),
                                     st) == _lib.FH_ERR_UNSUPPORTED
