"""The Python binding fails loudly without its library and checks arguments before any device call (no GPU)."""
import pytest

torch = pytest.importorskip("torch")


def test_missing_library_raises_import_error(monkeypatch, tmp_path):
    from lm_output_head_b200 import _lib
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(ImportError, match="no CPU fallback"):
        _lib.load()


def test_head_rejects_host_tensors():
    from lm_output_head_b200 import FlashHead
    E = torch.zeros((32, 8), dtype=torch.bfloat16)
    C2T = torch.arange(32, dtype=torch.int32).reshape(2, 16)
    C = torch.zeros((2, 8), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        FlashHead(E, C2T, C=C)


def test_cluster_builder_needs_balanced_sizes():
    from lm_output_head_b200.cluster import ClusterBuilder
    with pytest.raises(ValueError, match="c \\| v"):
        ClusterBuilder(100, 256, 3)
