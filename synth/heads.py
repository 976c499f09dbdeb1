"""Seeded synthetic planted-cluster heads, hidden states and uniforms.

This module only draws inputs. It holds none of the retrieval head's own
arithmetic (no scores, no selection, no candidate logits, no sampling): the
fp64 oracle and the CUDA library both read the arrays it returns, and nothing
else is shared between them.

Everything is returned as raw bit patterns so that both sides see the same
bytes:

* bf16 tensors as ``uint16`` arrays (the upper half of an IEEE fp32),
* INT4 centroids as ``uint8`` arrays, two signed nibbles per byte, element
  ``2i`` in the low nibble of byte ``i`` and element ``2i+1`` in the high one,
  with one bf16 scale per group of 32 elements,
* INT8 centroids as ``int8`` arrays, one two's-complement code per element,
  with one bf16 scale per group of 32 elements,
* the cluster-to-token map ``C2T`` as ``int32 [c, b]``.

Recipe (the planted-cluster head of the FlashHead write-up's shape table):

* cluster directions ``mu_k ~ N(0, I_d)``, normalised to the unit sphere;
* token rows: the ``b`` rows of cluster ``k`` are ``bf16(mu_k + N(0, 0.25^2/d))``
  and are scattered through the vocabulary by a seeded permutation, so
  ``C2T[k][j] = perm[k*b + j]`` (every cluster holds exactly ``b = v/c`` tokens,
  the balanced-clustering invariant of FlashHead section 1.2.1);
* centroids: ``C_k = bf16(normalise(fp64 mean of the cluster's bf16 rows))``;
  the INT4 variant quantises that C symmetrically (codes -7..7, one bf16
  scale ``max|x|/7`` per group of 32), the INT8 variant likewise with codes
  -127..127 and scale ``max|x|/127``;
* hidden states: planted ``bf16(6*mu_j + N(0, 1/d))`` with ``j`` uniform over
  the clusters, or pure ``bf16(N(0, 1/d))`` for flat rows;
* uniforms for Gumbel cluster selection ``[n, c]`` and for the token draw ``[n]``,
  fp32 in [0, 1).

Seeds: ``numpy.random.default_rng(1000*config + stream)`` with streams
0 centroids, 1 token noise, 2 permutation, 3 hidden states, 4 uniforms.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

STREAM_CENTROIDS = 0
STREAM_TOKEN_NOISE = 1
STREAM_PERMUTATION = 2
STREAM_HIDDEN = 3
STREAM_UNIFORMS = 4

INT4_GROUP = 32


# ---------------------------------------------------------------------------
# bf16 bit handling (input encoding only)
# ---------------------------------------------------------------------------
def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round an array to bf16 (round to nearest, ties to even); return uint16 bits."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32)
    bias = ((u >> 16) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def _bf16_inplace(f32: np.ndarray, work: np.ndarray, out: np.ndarray) -> None:
    """Same rounding as :func:`to_bf16_bits`, into preallocated buffers."""
    u = f32.view(np.uint32)
    np.right_shift(u, 16, out=work)
    np.bitwise_and(work, np.uint32(1), out=work)
    work += np.uint32(0x7FFF)
    work += u
    np.right_shift(work, 16, out=work)
    out[...] = work


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------------------
# Configurations (shapes of the FlashHead write-up's target models)
# ---------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class HeadConfig:
    cfg_id: int
    name: str
    v: int
    d: int
    c: int
    p: int
    int4: bool = False
    mode: str = "greedy"          # "greedy" or "gumbel"
    temperature: float = 1.0
    batches: tuple = (1,)
    n_states: int = 32
    pure_fraction: float = 0.0    # share of hidden states drawn as pure noise
    dominant_clusters: int = 0    # >0: planted rows use only this many cluster ids

    @property
    def b(self) -> int:
        return self.v // self.c


CONFIGS = {
    0: HeadConfig(0, "tiny planted head v4096 d256 c256 p16", 4096, 256, 256, 16,
                  batches=(1,), n_states=32),
    1: HeadConfig(1, "Llama-3.2-1B-shaped head v128256 d2048 c8016 p512 bf16", 128256, 2048, 8016, 512,
                  batches=(1,), n_states=1024, pure_fraction=0.25),
    2: HeadConfig(2, "Llama-3.2-1B-shaped head, INT4 g32 centroids", 128256, 2048, 8016, 512,
                  int4=True, batches=(1, 4, 16), n_states=1024, pure_fraction=0.25),
    3: HeadConfig(3, "Qwen3-4B-shaped head v151936 d2560 c9496 p512 Gumbel T0.7", 151936, 2560, 9496, 512,
                  mode="gumbel", temperature=0.7, batches=(32,), n_states=1024, pure_fraction=0.25),
    4: HeadConfig(4, "Gemma-3-shaped head v262144 d1152 c16384 p1024 INT4 B256", 262144, 1152, 16384, 1024,
                  int4=True, batches=(256,), n_states=512, dominant_clusters=64),
}


@dataclasses.dataclass
class Head:
    """A synthetic head: token rows E, centroids C (bf16 and/or INT4), map C2T."""
    v: int
    d: int
    c: int
    b: int
    E: np.ndarray                   # uint16 [v, d] bf16 bits
    C: np.ndarray                   # uint16 [c, d] bf16 bits
    C2T: np.ndarray                 # int32 [c, b]
    C_q: Optional[np.ndarray] = None        # uint8 [c, d/2] packed signed nibbles
    C_scales: Optional[np.ndarray] = None   # uint16 [c, d/32] bf16 bits
    C_q8: Optional[np.ndarray] = None       # int8 [c, d] codes (INT8 variant)
    C_scales8: Optional[np.ndarray] = None  # uint16 [c, d/32] bf16 bits (INT8 variant)
    mu: Optional[np.ndarray] = None         # float64 [c, d] planted directions
    seed_base: int = 0


@dataclasses.dataclass
class Hidden:
    H: np.ndarray                   # uint16 [n, d] bf16 bits
    planted: np.ndarray             # int32 [n], planted cluster id or -1 for pure rows


def _rng(seed_base: int, stream: int) -> np.random.Generator:
    return np.random.default_rng(seed_base + stream)


def quantize_int4_g32(C_bits: np.ndarray):
    """Symmetric INT4 with one bf16 scale per 32 elements (codes -7..7).

    Returns ``(C_q uint8 [c, d/2], C_scales uint16 [c, d/32])``. A group that is
    all zero gets scale 0 and codes 0.
    """
    c, d = C_bits.shape
    if d % INT4_GROUP:
        raise ValueError("INT4 centroids need d % 32 == 0")
    x = bf16_bits_to_f32(C_bits).astype(np.float64).reshape(c, d // INT4_GROUP, INT4_GROUP)
    amax = np.abs(x).max(axis=2)
    scale_bits = to_bf16_bits((amax / 7.0).astype(np.float32))
    scale = bf16_bits_to_f32(scale_bits).astype(np.float64)
    safe = np.where(scale > 0, scale, 1.0)
    q = np.rint(x / safe[:, :, None])
    q = np.where(scale[:, :, None] > 0, q, 0.0)
    q = np.clip(q, -7, 7).astype(np.int8).reshape(c, d)
    nib = (q.astype(np.int16) & 0xF).astype(np.uint8)
    packed = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return np.ascontiguousarray(packed), np.ascontiguousarray(scale_bits)


def _quantize_sym_g32(C_bits: np.ndarray, qmax: int):
    """Symmetric codes -qmax..qmax with one bf16 scale ``max|x|/qmax`` per 32 elements.

    Returns ``(codes int8 [c, d], scale bits uint16 [c, d/32])``. A group that
    is all zero gets scale 0 and codes 0.
    """
    c, d = C_bits.shape
    if d % INT4_GROUP:
        raise ValueError("group-32 centroids need d % 32 == 0")
    x = bf16_bits_to_f32(C_bits).astype(np.float64).reshape(c, d // INT4_GROUP, INT4_GROUP)
    amax = np.abs(x).max(axis=2)
    scale_bits = to_bf16_bits((amax / float(qmax)).astype(np.float32))
    scale = bf16_bits_to_f32(scale_bits).astype(np.float64)
    safe = np.where(scale > 0, scale, 1.0)
    q = np.rint(x / safe[:, :, None])
    q = np.where(scale[:, :, None] > 0, q, 0.0)
    q = np.clip(q, -qmax, qmax).astype(np.int8).reshape(c, d)
    return q, np.ascontiguousarray(scale_bits)


def quantize_int8_g32(C_bits: np.ndarray):
    """Symmetric INT8 with one bf16 scale per 32 elements (codes -127..127).

    Returns ``(C_q int8 [c, d], C_scales uint16 [c, d/32])``.
    """
    q, scale_bits = _quantize_sym_g32(C_bits, 127)
    return np.ascontiguousarray(q), scale_bits


def make_head(v: int, d: int, c: int, *, seed_base: int = 0, int4: bool = False, int8: bool = False,
              keep_mu: bool = True, chunk_clusters: int = 512) -> Head:
    """Draw a balanced planted-cluster head with ``b = v/c`` tokens per cluster."""
    if v % c:
        raise ValueError("v must be a multiple of c (balanced clusters)")
    b = v // c
    rng_mu = _rng(seed_base, STREAM_CENTROIDS)
    mu = rng_mu.standard_normal((c, d))
    mu /= np.linalg.norm(mu, axis=1, keepdims=True)

    perm = _rng(seed_base, STREAM_PERMUTATION).permutation(v).astype(np.int64)
    C2T = perm.reshape(c, b).astype(np.int32)

    E = np.empty((v, d), dtype=np.uint16)
    C = np.empty((c, d), dtype=np.uint16)
    rng_noise = _rng(seed_base, STREAM_TOKEN_NOISE)
    sigma = np.float32(0.25 / math.sqrt(d))
    mu32 = mu.astype(np.float32)
    kc_max = min(chunk_clusters, c)
    rows = np.empty((kc_max * b, d), dtype=np.float32)      # reused: first-touch is slow
    work = np.empty((kc_max * b, d), dtype=np.uint32)
    bits = np.empty((kc_max * b, d), dtype=np.uint16)
    for k0 in range(0, c, chunk_clusters):
        k1 = min(c, k0 + chunk_clusters)
        n = (k1 - k0) * b
        r = rows[:n]
        rng_noise.standard_normal(out=r, dtype=np.float32)
        r *= sigma
        r.reshape(k1 - k0, b, d)[...] += mu32[k0:k1, None, :]
        _bf16_inplace(r, work[:n], bits[:n])
        E[perm[k0 * b:k1 * b]] = bits[:n]
        # widen back (exact) and average in fp64
        np.left_shift(bits[:n], 16, out=work[:n], dtype=np.uint32)
        mean = work[:n].view(np.float32).reshape(k1 - k0, b, d).mean(axis=1, dtype=np.float64)
        norm = np.linalg.norm(mean, axis=1, keepdims=True)
        norm[norm == 0] = 1.0
        C[k0:k1] = to_bf16_bits((mean / norm).astype(np.float32))

    head = Head(v=v, d=d, c=c, b=b, E=E, C=C, C2T=C2T, mu=mu if keep_mu else None,
                seed_base=seed_base)
    if int4:
        head.C_q, head.C_scales = quantize_int4_g32(C)
    if int8:
        head.C_q8, head.C_scales8 = quantize_int8_g32(C)
    return head


def make_hidden(head: Head, n: int, *, seed_base: Optional[int] = None, pure_fraction: float = 0.0,
                dominant_clusters: int = 0, scale: float = 6.0) -> Hidden:
    """Hidden states: planted ``bf16(scale*mu_j + N(0, 1/d))`` or pure ``bf16(N(0, 1/d))``.

    Pure rows are spread evenly: with ``pure_fraction = 1/q`` every q-th row
    (q-1, 2q-1, ...) is pure, so every batch slice carries the same mix.
    With ``dominant_clusters = m > 0`` the planted ids come from a seeded set
    of m distinct clusters shared by all rows.
    """
    if head.mu is None:
        raise ValueError("head was generated without its planted directions")
    sb = head.seed_base if seed_base is None else seed_base
    rng = _rng(sb, STREAM_HIDDEN)
    d, c = head.d, head.c
    if dominant_clusters:
        pool = rng.choice(c, size=dominant_clusters, replace=False)
        j = pool[rng.integers(0, dominant_clusters, size=n)]
    else:
        j = rng.integers(0, c, size=n)
    noise = rng.standard_normal((n, d)) / math.sqrt(d)
    planted = j.astype(np.int32).copy()
    if pure_fraction > 0:
        q = int(round(1.0 / pure_fraction))
        pure = (np.arange(n) % q) == (q - 1)
        planted[pure] = -1
    h = noise.copy()
    pl = planted >= 0
    h[pl] += scale * head.mu[planted[pl]]
    return Hidden(H=to_bf16_bits(h.astype(np.float32)), planted=planted)


def make_uniforms(n: int, c: int, *, seed_base: int):
    """fp32 uniforms in [0, 1): ``(u_clusters [n, c], u_token [n])``."""
    rng = _rng(seed_base, STREAM_UNIFORMS)
    u_clusters = rng.random((n, c), dtype=np.float32)
    u_token = rng.random(n, dtype=np.float32)
    return u_clusters, u_token


def make_config(cfg_id: int, *, n_states: Optional[int] = None):
    """Head + hidden states (+ uniforms for sampling configs) of a named configuration."""
    cfg = CONFIGS[cfg_id]
    sb = 1000 * cfg_id
    head = make_head(cfg.v, cfg.d, cfg.c, seed_base=sb, int4=cfg.int4)
    n = cfg.n_states if n_states is None else n_states
    hid = make_hidden(head, n, seed_base=sb, pure_fraction=cfg.pure_fraction,
                      dominant_clusters=cfg.dominant_clusters)
    uni = make_uniforms(n, cfg.c, seed_base=sb) if cfg.mode == "gumbel" else None
    return cfg, head, hid, uni


def intra_cluster_cosine(head: Head, n_clusters: int = 256) -> float:
    """Mean cosine between token rows and their centroid (health metric; > 0.6 is healthy)."""
    ks = np.arange(min(n_clusters, head.c))
    Cw = bf16_bits_to_f32(head.C[ks]).astype(np.float64)
    tot = 0.0
    for i, k in enumerate(ks):
        rows = bf16_bits_to_f32(head.E[head.C2T[k]]).astype(np.float64)
        cos = rows @ Cw[i] / (np.linalg.norm(rows, axis=1) * np.linalg.norm(Cw[i]) + 1e-300)
        tot += cos.mean()
    return float(tot / len(ks))
