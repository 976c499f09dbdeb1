"""Python face of the C ABI: torch tensors in, ``data_ptr()`` and the current
CUDA stream out to ``libflashhead.so``. Every step of the head runs in the
library's kernels; this module only checks shapes and marshals arguments.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import numpy as np
import torch

from . import _lib
from ._lib import FlashHeadError

_MODES = {"greedy": _lib.FH_GREEDY, "gumbel": _lib.FH_SAMPLE_GUMBEL}


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream] = None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, where: str):
    if status != _lib.FH_OK:
        raise FlashHeadError(status, where)


def _dev(t: torch.Tensor, name: str, dtypes, ndim: int):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype not in dtypes:
        raise ValueError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {ndim}-d tensor")
    return t


_BF16 = (torch.bfloat16, torch.int16, torch.uint16)


def bf16_from_bits(bits: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bit patterns (numpy) -> a torch.bfloat16 tensor on ``device``."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


class FlashHead:
    """A FlashHead retrieval head bound to device tensors (borrowed, kept alive here).

    ``E`` bf16 [v, d]; ``C2T`` int32 [c, b], or uint16 [c, b] (int16 bits are
    read as uint16) for v <= 65536; centroids either ``C`` bf16 [c, d],
    or ``C_q`` with ``C_scales`` bf16 [c, d/32]: uint8 [c, d/2] packed INT4
    codes, or int8 [c, d] INT8 codes (the dtype picks the format).
    """

    def __init__(self, E: torch.Tensor, C2T: torch.Tensor, *, C: Optional[torch.Tensor] = None,
                 C_q: Optional[torch.Tensor] = None, C_scales: Optional[torch.Tensor] = None,
                 max_batch: int = 1, max_probes: Optional[int] = None):
        self._lib = _lib.load()
        self._h = None
        E = _dev(E, "E", _BF16, 2)
        C2T = _dev(C2T, "C2T", (torch.int32, torch.uint16, torch.int16), 2)
        c2t_format = _lib.FH_C2T_INT32 if C2T.dtype == torch.int32 else _lib.FH_C2T_UINT16
        v, d = E.shape
        c, b = C2T.shape
        if C is not None:
            C = _dev(C, "C", _BF16, 2)
            fmt = _lib.FH_CENTROID_BF16
        elif C_q is not None and C_scales is not None:
            C_q = _dev(C_q, "C_q", (torch.uint8, torch.int8), 2)
            C_scales = _dev(C_scales, "C_scales", _BF16, 2)
            fmt = _lib.FH_CENTROID_INT8_G32 if C_q.dtype == torch.int8 else _lib.FH_CENTROID_INT4_G32
        else:
            raise ValueError("give C (bf16) or C_q and C_scales (INT4 uint8 / INT8 int8 codes)")
        self.E, self.C2T, self.C, self.C_q, self.C_scales = E, C2T, C, C_q, C_scales
        self.v, self.d, self.c, self.b = v, d, c, b
        self.fmt = fmt
        self.max_batch = int(max_batch)
        self.max_probes = int(max_probes if max_probes is not None else c)
        desc = _lib.HeadDesc(v=v, d=d, c=c, b=b, E=E.data_ptr(),
                             C=C.data_ptr() if C is not None else None,
                             C_q=C_q.data_ptr() if C_q is not None else None,
                             C_scales=C_scales.data_ptr() if C_scales is not None else None,
                             C2T=C2T.data_ptr(), fmt=fmt, max_batch=self.max_batch,
                             max_probes=self.max_probes, c2t_format=c2t_format)
        h = ctypes.c_void_p()
        with torch.cuda.device(E.device):
            _check(self._lib.fh_create(ctypes.byref(desc), _stream(), ctypes.byref(h)), "fh_create")
        self._h = h
        self.device = E.device

    # ------------------------------------------------------------------ helpers
    def close(self):
        if self._h is not None:
            self._lib.fh_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _hidden(self, hidden: torch.Tensor) -> torch.Tensor:
        hidden = _dev(hidden, "hidden", _BF16, 2)
        if hidden.shape[1] != self.d:
            raise ValueError("hidden must be [B, d]")
        return hidden

    def query(self, key: int) -> int:
        out = ctypes.c_int64()
        _check(self._lib.fh_query(self._h, int(key), ctypes.byref(out)), "fh_query")
        return out.value

    @property
    def workspace_bytes(self) -> int:
        return self.query(_lib.FH_QUERY_WORKSPACE_BYTES)

    @property
    def fused_b1(self) -> bool:
        return bool(self.query(_lib.FH_QUERY_FUSED_B1))

    def last_selection(self):
        """(keys counted near the predicted boundary, selected from a histogram of all keys?)
        of the last fused B = 1 decode."""
        return self.query(_lib.FH_QUERY_LAST_LIST), bool(self.query(_lib.FH_QUERY_LAST_FULL))

    def set_spin_budget(self, cycles: int):
        _check(self._lib.fh_set_spin_budget(self._h, int(cycles)), "fh_set_spin_budget")

    def device_status(self, stream=None) -> int:
        """Synchronise the stream and return (and clear) the device status word."""
        return int(self._lib.fh_get_device_status(self._h, _stream(stream)))

    # ------------------------------------------------------------------ stages
    def centroid_scores(self, hidden: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None):
        hidden = self._hidden(hidden)
        B = hidden.shape[0]
        if out is None:
            out = torch.empty((B, self.c), dtype=torch.float32, device=self.device)
        _check(self._lib.fh_centroid_scores(self._h, _ptr(hidden), B, _ptr(out), _stream(stream)),
               "fh_centroid_scores")
        return out

    def select_clusters(self, scores: torch.Tensor, p: int, *, mode: str = "greedy", T: float = 1.0,
                        u_clusters: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                        stream=None):
        scores = _dev(scores, "scores", (torch.float32,), 2)
        B = scores.shape[0]
        if out is None:
            out = torch.empty((B, p), dtype=torch.int32, device=self.device)
        _check(self._lib.fh_select_clusters(self._h, _ptr(scores), B, int(p), _MODES[mode], float(T),
                                            _ptr(u_clusters), _ptr(out), _stream(stream)),
               "fh_select_clusters")
        return out

    def candidate_logits(self, hidden: torch.Tensor, cluster_ids: torch.Tensor, stream=None):
        hidden = self._hidden(hidden)
        cluster_ids = _dev(cluster_ids, "cluster_ids", (torch.int32,), 2)
        B, p = cluster_ids.shape
        toks = torch.empty((B, p * self.b), dtype=torch.int32, device=self.device)
        logits = torch.empty((B, p * self.b), dtype=torch.float32, device=self.device)
        _check(self._lib.fh_candidate_logits(self._h, _ptr(hidden), B, p, _ptr(cluster_ids), _ptr(toks),
                                             _ptr(logits), _stream(stream)), "fh_candidate_logits")
        return toks, logits

    def adaptive_probes(self, scores: torch.Tensor, tau: float, p_min: int, p_max: int, *, T: float = 1.0,
                        stream=None) -> torch.Tensor:
        """Probes per row: the smallest p in [p_min, p_max] whose top-p clusters hold a fraction tau
        of softmax(scores / T)."""
        scores = _dev(scores, "scores", (torch.float32,), 2)
        B = scores.shape[0]
        out = torch.empty(B, dtype=torch.int32, device=self.device)
        _check(self._lib.fh_adaptive_probes(self._h, _ptr(scores), B, float(tau), int(p_min), int(p_max), float(T),
                                            _ptr(out), _stream(stream)), "fh_adaptive_probes")
        return out

    def prefetch_clusters(self, cluster_ids: torch.Tensor, stream=None):
        """Start reading the token rows of these clusters into L2 (``fh_prefetch_clusters``)."""
        cluster_ids = _dev(cluster_ids, "cluster_ids", (torch.int32,), 1)
        _check(self._lib.fh_prefetch_clusters(self._h, _ptr(cluster_ids), int(cluster_ids.shape[0]),
                                              _stream(stream)), "fh_prefetch_clusters")

    def decode(self, hidden: torch.Tensor, p: int, *, mode: str = "greedy", T: float = 1.0,
               u_clusters: Optional[torch.Tensor] = None, u_token: Optional[torch.Tensor] = None,
               out_tokens: Optional[torch.Tensor] = None, out_cluster_ids: Optional[torch.Tensor] = None,
               out_max_logit: Optional[torch.Tensor] = None, stream=None):
        hidden = self._hidden(hidden)
        B = hidden.shape[0]
        if out_tokens is None:
            out_tokens = torch.empty(B, dtype=torch.int32, device=self.device)
        _check(self._lib.fh_decode(self._h, _ptr(hidden), B, int(p), _MODES[mode], float(T),
                                   _ptr(u_clusters), _ptr(u_token), _ptr(out_tokens),
                                   _ptr(out_cluster_ids), _ptr(out_max_logit), _stream(stream)),
               "fh_decode")
        return out_tokens

    def dense_head(self, hidden: torch.Tensor, *, want_logits: bool = False,
                   out_argmax: Optional[torch.Tensor] = None, stream=None):
        hidden = self._hidden(hidden)
        B = hidden.shape[0]
        logits = torch.empty((B, self.v), dtype=torch.float32, device=self.device) if want_logits else None
        if out_argmax is None:
            out_argmax = torch.empty(B, dtype=torch.int32, device=self.device)
        _check(self._lib.fh_dense_head(self._h, _ptr(hidden), B, _ptr(logits), _ptr(out_argmax),
                                       _stream(stream)), "fh_dense_head")
        return (out_argmax, logits) if want_logits else out_argmax


def speculative_verify(head: FlashHead, logits: torch.Tensor, cand_tokens: torch.Tensor, draft: torch.Tensor,
                       T: float, u_accept: torch.Tensor, u_resample: torch.Tensor, stream=None) -> torch.Tensor:
    """Check FlashHead drafts against the dense logits (``fh_speculative_verify``)."""
    logits = _dev(logits, "logits", (torch.float32,), 2)
    cand_tokens = _dev(cand_tokens, "cand_tokens", (torch.int32,), 2)
    B, n = cand_tokens.shape
    if logits.shape != (B, head.v):
        raise ValueError("logits must be [B, v]")
    out = torch.empty(B, dtype=torch.int32, device=logits.device)
    _check(head._lib.fh_speculative_verify(head._h, _ptr(logits), _ptr(cand_tokens), int(n), int(B), _ptr(draft),
                                           float(T), _ptr(u_accept), _ptr(u_resample), _ptr(out), _stream(stream)),
           "fh_speculative_verify")
    return out


def dense_head_noalloc(E: torch.Tensor, hidden: torch.Tensor, out_argmax: torch.Tensor, *,
                       logits: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Dense head through ``fh_dense_head_noalloc``: no handle and no device
    allocation (the caller passes every output). At most
    ``FH_NOALLOC_MAX_ROWS`` hidden rows per call; calls that may overlap in
    time share one fixed scratch and must be ordered (e.g. one stream)."""
    lib = _lib.load()
    v, d = E.shape
    B = hidden.shape[0]
    _check(lib.fh_dense_head_noalloc(_ptr(E), int(v), int(d), _ptr(hidden), int(B), _ptr(logits),
                                     _ptr(out_argmax), _stream(stream)), "fh_dense_head_noalloc")
    return out_argmax


class HostDecoder:
    """End-to-end decode from pinned host memory: H2D copy of the hidden states
    (and uniforms), ``fh_decode``, D2H copy of the tokens, all on one stream."""

    def __init__(self, head: FlashHead, B: int, p: int, *, mode: str = "greedy", T: float = 1.0):
        self.head, self.B, self.p, self.mode, self.T = head, B, p, mode, T
        dev = head.device
        self.h_dev = torch.empty((B, head.d), dtype=torch.bfloat16, device=dev)
        self.tok_dev = torch.empty(B, dtype=torch.int32, device=dev)
        self.tok_host = torch.empty(B, dtype=torch.int32, pin_memory=True)
        self.u_dev = torch.empty((B, head.c), dtype=torch.float32, device=dev) if mode == "gumbel" else None
        self.ut_dev = torch.empty(B, dtype=torch.float32, device=dev) if mode == "gumbel" else None

    @property
    def h2d_bytes(self) -> int:
        n = self.h_dev.numel() * 2
        if self.u_dev is not None:
            n += self.u_dev.numel() * 4 + self.ut_dev.numel() * 4
        return n

    @property
    def d2h_bytes(self) -> int:
        return self.tok_host.numel() * 4

    def __call__(self, hidden_host: torch.Tensor, u_host=None, ut_host=None, stream=None) -> torch.Tensor:
        s = stream if stream is not None else torch.cuda.current_stream()
        with torch.cuda.stream(s):
            self.h_dev.copy_(hidden_host, non_blocking=True)
            if self.u_dev is not None:
                self.u_dev.copy_(u_host, non_blocking=True)
                self.ut_dev.copy_(ut_host, non_blocking=True)
            self.head.decode(self.h_dev, self.p, mode=self.mode, T=self.T, u_clusters=self.u_dev,
                             u_token=self.ut_dev, out_tokens=self.tok_dev, stream=s)
            self.tok_host.copy_(self.tok_dev, non_blocking=True)
        s.synchronize()
        return self.tok_host
