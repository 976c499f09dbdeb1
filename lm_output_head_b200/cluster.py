"""Python face of the clustering builder in ``include/fh_cluster.h``.

Offline balanced spherical k-means (FlashHead write-up, section 2.1, with the
balance rule of section 1.2.1) on the library's kernels; this module checks
shapes and marshals ``data_ptr()`` and the current CUDA stream, nothing more.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _lib
from .head import _check, _dev, _ptr, _stream


class ClusterBuilder:
    """Workspace for clustering ``v`` token rows of size ``d`` into ``c`` balanced clusters."""

    def __init__(self, v: int, d: int, c: int):
        self._lib = _lib.load()
        self.v, self.d, self.c = int(v), int(d), int(c)
        if self.c < 1 or self.v % self.c:
            raise ValueError("balanced clustering needs c | v")
        self.b = self.v // self.c
        h = ctypes.c_void_p()
        _check(self._lib.fh_cluster_create(self.v, self.d, self.c, _stream(), ctypes.byref(h)),
               "fh_cluster_create")
        self._h = h

    def close(self):
        if getattr(self, "_h", None):
            self._lib.fh_cluster_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- single steps ---------------------------------------------------------
    def normalize(self, E: torch.Tensor) -> torch.Tensor:
        """bf16 ``E [v, d]`` -> unit rows ``En`` (bf16)."""
        _dev(E, "E", (torch.bfloat16,), 2)
        En = torch.empty_like(E)
        _check(self._lib.fh_cluster_normalize(self._h, _ptr(E), _ptr(En), _stream()), "fh_cluster_normalize")
        return En

    def seed(self, En: torch.Tensor, u: torch.Tensor) -> torch.Tensor:
        """k-means++ seeds from uniforms ``u [c]`` (fp32) -> token ids ``[c]`` (int32)."""
        _dev(En, "En", (torch.bfloat16,), 2)
        _dev(u, "u", (torch.float32,), 1)
        ids = torch.empty(self.c, dtype=torch.int32, device=En.device)
        _check(self._lib.fh_cluster_seed(self._h, _ptr(En), _ptr(u), _ptr(ids), _stream()), "fh_cluster_seed")
        return ids

    def gather(self, En: torch.Tensor, ids: torch.Tensor) -> torch.Tensor:
        """Centres ``C[k] = En[ids[k]]`` (bf16 ``[c, d]``)."""
        _dev(ids, "ids", (torch.int32,), 1)
        C = torch.empty((self.c, self.d), dtype=torch.bfloat16, device=En.device)
        _check(self._lib.fh_cluster_gather(self._h, _ptr(En), _ptr(ids), _ptr(C), _stream()), "fh_cluster_gather")
        return C

    def similarities(self, En: torch.Tensor, C: torch.Tensor) -> torch.Tensor:
        """``S[k][t] = C[k] . En[t]`` (fp32 ``[c, v]``)."""
        _dev(C, "C", (torch.bfloat16,), 2)
        S = torch.empty((self.c, self.v), dtype=torch.float32, device=En.device)
        _check(self._lib.fh_cluster_similarities(self._h, _ptr(En), _ptr(C), _ptr(S), _stream()),
               "fh_cluster_similarities")
        return S

    def assign(self, S: torch.Tensor):
        """Balanced assignment of ``S [c, v]`` -> ``(assign [v], C2T [c, b], rounds)``."""
        _dev(S, "S", (torch.float32,), 2)
        a = torch.empty(self.v, dtype=torch.int32, device=S.device)
        m = torch.empty((self.c, self.b), dtype=torch.int32, device=S.device)
        rounds = ctypes.c_int32(0)
        _check(self._lib.fh_cluster_assign(self._h, _ptr(S), _ptr(a), _ptr(m), ctypes.byref(rounds), _stream()),
               "fh_cluster_assign")
        return a, m, rounds.value

    def update(self, En: torch.Tensor, C2T: torch.Tensor, C: torch.Tensor) -> torch.Tensor:
        """Centres moved to the normalised means of their tokens (in place on ``C``)."""
        _dev(C2T, "C2T", (torch.int32,), 2)
        _check(self._lib.fh_cluster_update(self._h, _ptr(En), _ptr(C2T), _ptr(C), _stream()), "fh_cluster_update")
        return C

    def device_status(self) -> int:
        return self._lib.fh_cluster_get_device_status(self._h, _stream())

    # -- whole loop -----------------------------------------------------------
    def build(self, E: torch.Tensor, *, init_ids: Optional[torch.Tensor] = None,
              u_init: Optional[torch.Tensor] = None, max_iter: int = 1000):
        """Cluster ``E`` -> ``(C [c, d] bf16, C2T [c, b] int32, iterations)``."""
        _dev(E, "E", (torch.bfloat16,), 2)
        if init_ids is None and u_init is None:
            raise ValueError("give init_ids or u_init")
        C = torch.empty((self.c, self.d), dtype=torch.bfloat16, device=E.device)
        m = torch.empty((self.c, self.b), dtype=torch.int32, device=E.device)
        it = ctypes.c_int32(0)
        _check(self._lib.fh_cluster_build(self._h, _ptr(E), _ptr(init_ids), _ptr(u_init), int(max_iter), _ptr(C),
                                          _ptr(m), ctypes.byref(it), _stream()), "fh_cluster_build")
        return C, m, it.value
