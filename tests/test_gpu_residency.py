"""Hot-cluster residency: fh_prefetch_clusters through the C ABI (needs a B200).

Write-up section 2.2.1 keeps frequently used clusters close to the compute;
here a caller requests their token rows into L2 ahead of a decode. The call
only warms a cache, so: decodes after it give exactly the tokens, cluster
sets and maxima they give without it (and those hold against the fp64
oracle); an id out of range is skipped and recorded as FH_ERR_OUT_OF_RANGE
in the device status; n = 0 launches nothing; bad arguments are refused on
the host.
"""
import ctypes

import numpy as np
import pytest

from tests.test_gpu_parity import _decode_check_greedy, fh, get_cfg, hid_dev  # noqa: F401

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _run(dh, H, p):
    B = H.shape[0]
    ids = torch.empty((B, p), dtype=torch.int32, device="cuda")
    mx = torch.empty(B, dtype=torch.float32, device="cuda")
    tok = dh.decode(hid_dev(H), p, out_cluster_ids=ids, out_max_logit=mx)
    assert dh.device_status() == 0
    return tok.cpu().numpy(), ids.cpu().numpy(), mx.cpu().numpy()


@pytest.mark.parametrize("B", [1, 8])
def test_decode_is_unchanged_by_a_prefetch(fh, B):
    cfg, head, hid, _, dh = get_cfg(0, fh)
    H = hid.H[:B]
    before = _run(dh, H, cfg.p)
    hot = torch.from_numpy(np.unique(before[1]).astype(np.int32)).cuda()
    dh.prefetch_clusters(hot)
    assert dh.device_status() == 0
    after = _run(dh, H, cfg.p)
    for x, y in zip(before, after):
        assert np.array_equal(x, y)
    rep = _decode_check_greedy(cfg, head, hid, dh, list(range(B)), B, cfg.p)
    assert rep.tight_mismatch == 0, rep


def test_out_of_range_ids_are_recorded(fh):
    cfg, head, hid, _, dh = get_cfg(0, fh)
    ids = torch.tensor([0, cfg.c - 1, cfg.c, -1], dtype=torch.int32, device="cuda")
    dh.prefetch_clusters(ids)
    assert dh.device_status() == 6          # FH_ERR_OUT_OF_RANGE
    assert dh.device_status() == 0          # reading the status cleared it
    _run(dh, hid.H[:1], cfg.p)


def test_host_checks(fh):
    cfg, head, hid, _, dh = get_cfg(0, fh)
    from lm_output_head_b200 import _lib
    lib = _lib.load()
    assert lib.fh_prefetch_clusters(dh._h, None, 0, None) == _lib.FH_OK
    assert lib.fh_prefetch_clusters(dh._h, None, 3, None) == _lib.FH_ERR_INVALID_ARG
    ids = torch.zeros(4, dtype=torch.int32, device="cuda")
    assert lib.fh_prefetch_clusters(dh._h, ctypes.c_void_p(ids.data_ptr()), -1, None) == _lib.FH_ERR_INVALID_ARG
    assert lib.fh_prefetch_clusters(None, ctypes.c_void_p(ids.data_ptr()), 4, None) == _lib.FH_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert dh.device_status() == 0
