"""INT8 group-32 (W8A16) centroids: CUDA path vs the fp64 oracle, through the C ABI (needs a B200).

Every kernel that reads centroid rows has an INT8 form: the fused
single-token decode (register-streamed and bulk-copied rows), the batched
score kernel (B < 16) and the tcgen05 GEMM (B >= 16, codes * scale written as
exact hi + lo bf16 pairs). Cases: the tiny planted head (several tiles,
ragged tails), d = 288 (a ragged lane stride), and the Llama-3.2-1B-shaped
head at one token per call.
"""
import numpy as np
import pytest

import oracle
import synth
from tests import parity
from tests.test_gpu_parity import _decode_check_greedy, _decode_check_gumbel, fh, hid_dev  # noqa: F401

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

_CACHE = {}


def _int8_head(key, v, d, c, seed, n_states):
    if key not in _CACHE:
        head = synth.make_head(v, d, c, seed_base=seed, int8=True)
        hid = synth.make_hidden(head, n_states, seed_base=seed, pure_fraction=0.25)
        _CACHE[key] = (head, hid)
    return _CACHE[key]


def _dev_head(fh, head, max_batch, max_probes):
    E = fh.bf16_from_bits(head.E, "cuda")
    C2T = torch.from_numpy(head.C2T).cuda()
    Cq = torch.from_numpy(head.C_q8).cuda()
    Cs = fh.bf16_from_bits(head.C_scales8, "cuda")
    assert Cq.dtype == torch.int8
    return fh.FlashHead(E, C2T, C_q=Cq, C_scales=Cs, max_batch=max_batch, max_probes=max_probes)


def _oracle_head(head):
    # the oracle sees the INT8 codes only (no INT4, and C is not used for scores)
    return synth.Head(v=head.v, d=head.d, c=head.c, b=head.b, E=head.E, C=head.C, C2T=head.C2T,
                      C_q8=head.C_q8, C_scales8=head.C_scales8)


@pytest.mark.parametrize("shape,B", [("tiny", 1), ("tiny", 32), ("tiny", 64), ("tiny", 65), ("ragged", 3),
                                     ("ragged", 64)])
def test_int8_centroid_scores(fh, shape, B):
    if shape == "tiny":
        head, hid = _int8_head("tiny", 4096, 256, 256, 8100, 65)
    else:
        head, hid = _int8_head("ragged", 1998, 288, 999, 8200, 65)
    dh = _dev_head(fh, head, 65, 64)
    H = hid.H[:B]
    s = dh.centroid_scores(hid_dev(H)).cpu().numpy()
    assert dh.device_status() == 0
    Cw = oracle.centroid_matrix(_oracle_head(head))
    assert np.array_equal(Cw, oracle.dequantize_int8(head.C_q8, head.C_scales8))
    S = oracle.centroid_scores(Cw, H)
    tight = [parity.check_values(s[r], S[r], Cw, oracle.widen_bf16(H[r]), f"scores row {r}") for r in range(B)]
    assert np.mean(tight) >= 0.999
    dh.close()


@pytest.mark.parametrize("shape,B", [("tiny", 1), ("tiny", 4), ("tiny", 64), ("ragged", 1), ("ragged", 3)])
def test_int8_decode_greedy(fh, shape, B):
    if shape == "tiny":
        head, hid = _int8_head("tiny", 4096, 256, 256, 8100, 65)
        p = 16
    else:
        head, hid = _int8_head("ragged", 1998, 288, 999, 8200, 65)
        p = 64
    dh = _dev_head(fh, head, 64, p)
    if B == 1:
        assert dh.fused_b1
    rep = _decode_check_greedy(None, _oracle_head(head), hid, dh, list(range(max(B, 8) if B < 64 else 64)), B, p)
    assert rep.tight_mismatch == 0, rep
    dh.close()


def test_int8_decode_llama_shape_single_token(fh):
    head, hid = _int8_head("llama", 128256, 2048, 8016, 8300, 16)
    dh = _dev_head(fh, head, 1, 512)
    assert dh.fused_b1
    rep = _decode_check_greedy(None, _oracle_head(head), hid, dh, list(range(16)), 1, 512)
    assert rep.tight_mismatch <= 1, rep
    dh.close()


@pytest.mark.parametrize("B", [1, 8, 64])
def test_int8_decode_gumbel(fh, B):
    head, hid = _int8_head("tiny", 4096, 256, 256, 8100, 65)
    dh = _dev_head(fh, head, 64, 16)
    uni = synth.make_uniforms(65, head.c, seed_base=8100)
    rows = list(range(8)) if B == 1 else list(range(B))
    rep = _decode_check_gumbel(None, _oracle_head(head), hid, uni, dh, rows, B, 16, 0.7)
    assert rep.tight_mismatch == 0, rep
    dh.close()
