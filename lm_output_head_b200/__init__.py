"""B200-native FlashHead retrieval head (sm_100a CUDA behind a C ABI).

``FlashHead`` binds device tensors to the library in ``libflashhead.so``
(built by ``python -m lm_output_head_b200.build``); ``HostDecoder`` runs the
end-to-end path from pinned host memory. There is no CPU fallback: if the
library is missing, constructing a head raises ImportError.
"""
from ._lib import FlashHeadError, load  # noqa: F401
from .head import FlashHead, HostDecoder, bf16_from_bits, dense_head_noalloc, speculative_verify  # noqa: F401

__all__ = ["FlashHead", "FlashHeadError", "HostDecoder", "bf16_from_bits", "dense_head_noalloc", "load",
           "speculative_verify"]
