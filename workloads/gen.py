"""Seeded input generators.

Every random quantity comes from its own Philox sub-stream, keyed by
(seed, stream id), so that changing one tensor's size never shifts another's
values.  Streams, in their fixed order:

    0 q          1 k_cache      2 v_cache     3 k_tree      4 v_tree
    5 draft logits               6 target noise
    7 bases of target rows for nodes the draft never expanded
    8 uniforms   9 prefix lengths

Distributions:
    q, K, V          ~ N(0, 1) drawn in fp32, rounded to bf16 (round to nearest even)
    draft logits     ~ N(0, 3^2) drawn in fp32, stored as fp32 or bf16
    target row j     = base_j + N(0, sigma^2) in fp32, stored like the draft;
                       base_j is the stored draft row that the tree assigned to
                       node j, or a fresh N(0, 3^2) row for a node without one
    uniforms         fp32 in [0, 1), layout [B][2][m+1]
    prefix lengths   fixed L, or uniform integers in [L_min, L] for a ragged batch

The key/value cache is [B][Hkv][Lmax][D]; entries past a sequence's prefix
length are filled with random values too (finite), which a correct kernel ignores.

Nothing here computes any part of the verify step.  The one thing that depends
on a tree, `make_target_logits`, only copies whichever draft row the caller
names for each node.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

from .configs import Config

S_Q, S_KC, S_VC, S_KT, S_VT, S_DRAFT, S_NOISE, S_UNEXP, S_UNIF, S_PLEN = range(10)

_CHUNK = 1 << 24  # draw at most this many normals per call (bounded host memory)


def _rng(seed: int, stream: int, row: int = 0) -> np.random.Generator:
    key = np.array([seed, stream], dtype=np.uint64)
    counter = np.array([0, 0, row, 0], dtype=np.uint64)
    return np.random.Generator(np.random.Philox(key=key, counter=counter))


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 with round-to-nearest-even, returned as uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def f32_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal_f32(rng: np.random.Generator, shape, scale: float = 1.0) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        out[s:e] = rng.standard_normal(e - s, dtype=np.float32)
    if scale != 1.0:
        out *= np.float32(scale)
    return out.reshape(shape)


def _store(x_f32: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return np.ascontiguousarray(x_f32, dtype=np.float32)
    if dtype == "bf16":
        return bf16_bits_from_f32(x_f32)
    raise ValueError(dtype)


def stored_to_f32(x: np.ndarray, dtype: str) -> np.ndarray:
    return x.astype(np.float32) if dtype == "f32" else f32_from_bf16_bits(x)


def draft_rows_count(cfg: Config) -> int:
    return cfg.R


@dataclass
class Workload:
    cfg: Config
    seed: int
    prefix_len: np.ndarray            # [B] int32
    Lmax: int
    draft_logits: np.ndarray          # [B][R][V] float32 or uint16 (bf16 bits)
    uniforms: np.ndarray              # [B][2][m+1] float32
    q: Optional[np.ndarray] = None        # [B][m][Hq][D] uint16
    k_cache: Optional[np.ndarray] = None  # [B][Hkv][Lmax][D] uint16
    v_cache: Optional[np.ndarray] = None
    k_tree: Optional[np.ndarray] = None   # [B][m][Hkv][D] uint16
    v_tree: Optional[np.ndarray] = None

    @property
    def logits_dtype(self) -> str:
        return self.cfg.logits_dtype


def gen_prefix_len(cfg: Config, seed: int) -> np.ndarray:
    if cfg.ragged:
        rng = _rng(seed, S_PLEN)
        return rng.integers(cfg.L_min, cfg.L, size=cfg.B, endpoint=True).astype(np.int32)
    return np.full(cfg.B, cfg.L, dtype=np.int32)


def gen_draft_logits(cfg: Config, seed: int) -> np.ndarray:
    x = _normal_f32(_rng(seed, S_DRAFT), (cfg.B, cfg.R, cfg.V), 3.0)
    return _store(x, cfg.logits_dtype)


def gen_uniforms(cfg: Config, seed: int) -> np.ndarray:
    rng = _rng(seed, S_UNIF)
    return rng.random((cfg.B, 2, cfg.m + 1), dtype=np.float32)


def gen_attention_inputs(cfg: Config, seed: int, Lmax: Optional[int] = None):
    Lmax = cfg.L if Lmax is None else Lmax
    B, m, Hq, Hkv, D = cfg.B, cfg.m, cfg.Hq, cfg.Hkv, cfg.D
    q = bf16_bits_from_f32(_normal_f32(_rng(seed, S_Q), (B, m, Hq, D)))
    kc = bf16_bits_from_f32(_normal_f32(_rng(seed, S_KC), (B, Hkv, Lmax, D)))
    vc = bf16_bits_from_f32(_normal_f32(_rng(seed, S_VC), (B, Hkv, Lmax, D)))
    kt = bf16_bits_from_f32(_normal_f32(_rng(seed, S_KT), (B, m, Hkv, D)))
    vt = bf16_bits_from_f32(_normal_f32(_rng(seed, S_VT), (B, m, Hkv, D)))
    return q, kc, vc, kt, vt


def make_workload(cfg: Config, seed: int, attention: bool = True) -> Workload:
    plen = gen_prefix_len(cfg, seed)
    Lmax = cfg.L
    w = Workload(cfg=cfg, seed=seed, prefix_len=plen, Lmax=Lmax,
                 draft_logits=gen_draft_logits(cfg, seed),
                 uniforms=gen_uniforms(cfg, seed))
    if attention:
        w.q, w.k_cache, w.v_cache, w.k_tree, w.v_tree = gen_attention_inputs(cfg, seed, Lmax)
    return w


def make_target_logits(cfg: Config, seed: int, draft_logits: np.ndarray,
                       draft_row: np.ndarray, sigma: Optional[float] = None) -> np.ndarray:
    """Target logits [B][m+1][V] in the config's storage type.

    Row j of sequence b is base + sigma * N(0, 1), with base the stored draft row
    draft_row[b][j] (decoded to fp32) when that index is >= 0, else a fresh
    N(0, 3^2) row drawn from its own counter block (keyed by b and j).  The sum is
    formed in fp32 and then stored (bf16: round to nearest even).
    """
    sigma = cfg.sigma if sigma is None else sigma
    B, n_rows, V = cfg.B, cfg.m + 1, cfg.V
    draft_row = np.asarray(draft_row)
    assert draft_row.shape == (B, n_rows), draft_row.shape
    base = np.empty((B, n_rows, V), dtype=np.float32)
    for b in range(B):
        for j in range(n_rows):
            r = int(draft_row[b, j])
            if r >= 0:
                base[b, j] = stored_to_f32(draft_logits[b, r], cfg.logits_dtype)
            else:
                base[b, j] = _normal_f32(_rng(seed, S_UNEXP, row=b * n_rows + j), (V,), 3.0)
    if sigma != 0.0:
        noise = _normal_f32(_rng(seed, S_NOISE), (B, n_rows, V))
        base += np.float32(sigma) * noise
    return _store(base, cfg.logits_dtype)
