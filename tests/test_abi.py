"""The C-ABI library loads and exports every entry point the headers under include/ declare (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    inc = os.path.join(ROOT, "include")
    src = "".join(open(os.path.join(inc, f)).read() for f in sorted(os.listdir(inc)) if f.endswith(".h"))
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = set(re.findall(r"\b(fh_[a-z_0-9]+)\s*\(", src))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    from lm_output_head_b200 import build
    build.build()
    return ctypes.CDLL(build.LIB)


def test_header_declares_the_entry_points():
    names = _declared()
    for n in ("fh_create", "fh_centroid_scores", "fh_select_clusters", "fh_candidate_logits",
              "fh_decode", "fh_dense_head"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_lists_every_declared_symbol():
    from lm_output_head_b200 import _lib
    assert sorted(_lib.EXPORTED) == _declared()


def test_status_strings(lib):
    lib.fh_status_string.restype = ctypes.c_char_p
    for code in range(8):
        assert lib.fh_status_string(code)
    assert lib.fh_status_string(99) == b"unknown status"


def test_create_without_device_fails_cleanly(lib):
    """On a machine without a GPU, fh_create returns an error status instead of crashing."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    from lm_output_head_b200 import _lib
    l = _lib.load()
    desc = _lib.HeadDesc(v=32, d=8, c=2, b=16, E=16, C=16, C_q=None, C_scales=None, C2T=16, fmt=0,
                         max_batch=1, max_probes=1)
    h = ctypes.c_void_p()
    st = l.fh_create(ctypes.byref(desc), None, ctypes.byref(h))
    assert st in (3, 5)  # unsupported / CUDA error
    assert not h.value
    assert l.fh_create(None, None, ctypes.byref(h)) == 1
