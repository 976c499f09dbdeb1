"""fp64 CPU oracle of the FlashHead retrieval head.

Test infrastructure: only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. It shares no code
with the CUDA library.
"""
from .flashhead import (adaptive_probe_count, candidate_logits, candidate_tokens, centroid_matrix, centroid_scores,
                        check_c2t, decode, dense_head, dequantize_int4, dequantize_int8, greedy_token, gumbel_keys,
                        sample_token, select_greedy, select_sampled, speculative_verify, widen_bf16)

__all__ = ["adaptive_probe_count", "candidate_logits", "candidate_tokens", "centroid_matrix", "centroid_scores",
           "check_c2t", "decode", "dense_head", "dequantize_int4", "dequantize_int8", "greedy_token", "gumbel_keys",
           "sample_token", "select_greedy", "select_sampled", "speculative_verify", "widen_bf16"]
