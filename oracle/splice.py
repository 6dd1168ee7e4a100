"""Float64 CPU oracle for the fetch primitive's local compute ("splice").

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / reference arm may import this module.  It shares no code with the CUDA path.

Source: "Move the Query, Not the Cache" (technical summary, Methodology, primitive comparison).
Of the three primitives, fetch brings the whole KV chunk to the requester, adapts its
positions ("splice") and attends locally; the problem statement names the adaptation cost:
cached position encodings are re-rotated to the new offsets.  The transfer itself is a copy and
is not computed here; what remains on one GPU is a page-table-driven row move plus the
re-rotation.

What it computes (plain definitions, one token at a time):

* Row move -- token t in [0, n) of the chunk is logical position ``src_start + t`` of the
  source page list (page ``src_pages[(src_start + t) // Ps]``, slot ``(src_start + t) % Ps``)
  and lands at logical position ``dst_start + t`` of the destination page list (page size Pd).
* The 512-d latent (ckv) carries no position and is copied unchanged.
* The 64-d rope part (kpe) holds keys already rotated to their old positions.  Moving a token
  by delta = new_position - old_position rotates each of its 32 pairs (a_i, b_i) by the angle
  delta * theta_i:  a' = a cos - b sin,  b' = a sin + b cos.  Rotations compose, so this is
  exactly the key rotated to its new position.
* Readings (the pages name no rotary layout or frequencies): theta_i = base^(-2i/64) with a
  caller-given base (10000 by default), or a caller-given frequency table; pairs are
  interleaved (2i, 2i+1) or the two halves (i, i + 32).  Every token of a chunk moves by the
  same delta (a chunk keeps its internal order when it is placed at a new offset).
"""
from __future__ import annotations

import numpy as np

from .attention import bf16_to_f64

__all__ = ["ROPE_DIM", "rope_inv_freq", "rope_pairs", "rerotate", "splice_rows"]

ROPE_DIM = 64
LATENT_DIM = 512


def rope_inv_freq(base: float = 10000.0, rope_dim: int = ROPE_DIM) -> np.ndarray:
    """theta_i = base^(-2i / rope_dim), i = 0 .. rope_dim/2 - 1 (float64)."""
    i = np.arange(rope_dim // 2, dtype=np.float64)
    return np.power(np.float64(base), -2.0 * i / rope_dim)


def rope_pairs(layout: str, rope_dim: int = ROPE_DIM):
    """Index arrays (first, second) of the rotated pairs: interleaved (2i, 2i+1) or halves
    (i, i + rope_dim/2)."""
    half = rope_dim // 2
    i = np.arange(half)
    if layout == "interleaved":
        return 2 * i, 2 * i + 1
    if layout == "halves":
        return i, i + half
    raise ValueError(layout)


def rerotate(x, delta: int, inv_freq, layout: str = "interleaved") -> np.ndarray:
    """Rotate every pair of the last axis of ``x`` by delta * theta_i (float64)."""
    x = np.asarray(x, dtype=np.float64)
    a_idx, b_idx = rope_pairs(layout, x.shape[-1])
    ang = np.float64(delta) * np.asarray(inv_freq, dtype=np.float64)
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., a_idx], x[..., b_idx]
    out = np.empty_like(x)
    out[..., a_idx] = a * c - b * s
    out[..., b_idx] = a * s + b * c
    return out


def splice_rows(src_ckv, src_kpe, src_pages, src_start: int, dst_pages, dst_page_size: int, dst_start: int,
                n_tokens: int, delta: int, inv_freq, layout: str = "interleaved"):
    """Move ``n_tokens`` latent rows from the source page list to the destination page list and
    re-rotate their rope part by ``delta`` positions.

    ``src_ckv`` [num_pages, Ps, 512] and ``src_kpe`` [num_pages, Ps, 64] are bf16 bit patterns.
    Returns ``(dst_page, dst_slot, ckv, kpe)``: int arrays [n] of destination coordinates and
    float64 [n, 512] / [n, 64] destination rows."""
    src_ckv = np.asarray(src_ckv)
    src_kpe = np.asarray(src_kpe)
    ps = src_ckv.shape[1]
    dst_page = np.empty(n_tokens, dtype=np.int64)
    dst_slot = np.empty(n_tokens, dtype=np.int64)
    ckv = np.empty((n_tokens, src_ckv.shape[2]), dtype=np.float64)
    kpe_old = np.empty((n_tokens, src_kpe.shape[2]), dtype=np.float64)
    for t in range(n_tokens):
        ls, ld = src_start + t, dst_start + t
        sp, ss = int(src_pages[ls // ps]), ls % ps
        dst_page[t], dst_slot[t] = int(dst_pages[ld // dst_page_size]), ld % dst_page_size
        ckv[t] = bf16_to_f64(src_ckv[sp, ss])
        kpe_old[t] = bf16_to_f64(src_kpe[sp, ss])
    return dst_page, dst_slot, ckv, rerotate(kpe_old, delta, inv_freq, layout)
