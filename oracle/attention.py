"""Float64 CPU oracle for paged attention, split-KV partials and the exact LSE merge.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / reference arm may import this module.  The product (the CUDA library and its
Python binding) never calls it, and this module shares no code with the product: it has its
own bf16 / e4m3 decoders, its own page-table walk, and its own softmax and merge.

What it computes (definitions; every step is the plain formula, no tiling or online form):

* Page-table walk -- the paged KV cache of the FlashInfer PR #4736 page ("batch_pod.cu:
  flexible stride handling": ``paged_kv_t`` holds page size, KV heads, head dim, K and V base
  pointers with their own strides, and the page index list).  Request r owns pages
  ``kv_indices[kv_indptr[r]:kv_indptr[r+1]]``; its KV length is
  L_r = (n_r - 1) * P + kv_last_page_len[r] (0 when n_r = 0); token t sits at page
  ``kv_indices[kv_indptr[r] + t // P]``, slot ``t % P``.  K and V are read through their own
  views, so independent strides need no special case here.
* GQA head map -- query head h reads KV head h // (Hq / Hk) (reading: contiguous groups; the
  pages do not name a map).
* Attention per (request, query token, query head) -- s_t = scale * q . k_t,
  m = max_t s_t, l = sum_t exp(s_t - m), O = sum_t exp(s_t - m) v_t / l, LSE = m + ln l
  (natural log of the scaled logits; reading: the pages never fix the base).  By default no
  causal mask: every query token of a request attends to all L_r tokens (the shared-KV broadcast
  and the MLA fold both rest on KV being shared by all queries and heads).  Empty KV: O = 0,
  LSE = -inf.
* Causal / multi-token decode (``causal=True``) -- the request's n_q query tokens are its last
  n_q positions; query token i sees keys t <= L_r - n_q + i, and a token that sees no key gets
  O = 0, LSE = -inf.  The FlashInfer PR #3309 page (reviewer feedback) mentions MLA decode with
  multi-token prediction (MTP) but gives no mask indexing; this is the plainest reading.
* Split partials -- the same definition restricted to a page range [a, b) of the request
  ("route": partial attention per KV chunk, returned as (O, LSE), "Move the Query, Not the
  Cache" summary, Methodology / primitive comparison; in-CTA split of the SM110 XQA page,
  section 3 "kernel design").
* merge_states -- exact combination of partial (O_j, LSE_j): M = max_j LSE_j,
  LSE = M + ln sum_j exp(LSE_j - M), O = sum_j exp(LSE_j - LSE) O_j; all states -inf gives
  O = 0, LSE = -inf.  (The pages say only "merged via online softmax"; this is the exact
  result that merge reaches.)
* MLA decode -- the FlashInfer PR #3309 page (MLA decode, seqlen_q folded into heads): one
  latent cache row per token holds a 512-d compressed KV (ckv) and a 64-d rope part (kpe),
  shared by every head; s_t = scale * (q_nope . ckv_t + q_pe . kpe_t), v_t = ckv_t.  Folding
  seqlen_q into heads only re-labels rows, so it does not appear here.
* fp8 cache -- OCP e4m3fn codes decoded exactly and multiplied by the per-tensor scale (the MLA
  latent cache, and the GQA K/V cache: ``kv_dtype="e4m3"``).
"""
from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence

import numpy as np

__all__ = [
    "bf16_to_f64", "e4m3_to_f64", "request_kv_length", "request_token_slots", "causal_visible",
    "paged_attention", "paged_attention_partials", "merge_states", "mla_decode",
    "mla_decode_partials",
]


# ----------------------------------------------------------------------------- storage formats
def bf16_to_f64(bits) -> np.ndarray:
    """bf16 bit pattern -> float64.  bf16 is the upper half of an IEEE binary32, so shifting
    the 16 bits into the top of a 32-bit word gives the same value exactly."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def e4m3_to_f64(codes) -> np.ndarray:
    """OCP FP8 e4m3fn code -> float64, from the format definition: 1 sign bit, 4 exponent bits
    (bias 7), 3 mantissa bits; exponent 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; there
    are no infinities (so S.1111.110 = +-448 is the largest magnitude)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    sub = (m / 8.0) * 2.0 ** -6
    v = sign * np.where(e == 0, sub, normal)
    return np.where((c & 0x7F) == 0x7F, np.nan, v)


# ----------------------------------------------------------------------------- page-table walk
def request_kv_length(kv_indptr, kv_last_page_len, page_size: int, r: int) -> int:
    n = int(kv_indptr[r + 1]) - int(kv_indptr[r])
    return 0 if n == 0 else (n - 1) * page_size + int(kv_last_page_len[r])


def request_token_slots(kv_indptr, kv_indices, kv_last_page_len, page_size: int, r: int,
                        page_begin: int = 0, page_end: Optional[int] = None):
    """(physical page, slot) of every token of request r whose logical page lies in
    [page_begin, page_end), in logical token order."""
    n = int(kv_indptr[r + 1]) - int(kv_indptr[r])
    L = request_kv_length(kv_indptr, kv_last_page_len, page_size, r)
    page_end = n if page_end is None else page_end
    t = np.arange(page_begin * page_size, min(page_end * page_size, L), dtype=np.int64)
    pages = np.asarray(kv_indices, dtype=np.int64)[int(kv_indptr[r]) + t // page_size]
    return pages, t % page_size


def causal_visible(n_q: int, kv_len: int, t) -> np.ndarray:
    """[n_q, len(t)] bool.  The n_q query tokens of a request are its last n_q positions, query
    token i at position kv_len - n_q + i; it sees key t when t <= kv_len - n_q + i (its own key
    and every earlier one).  Reading of causal prefill / multi-token (MTP) decode: the pages name
    the mask but give no indexing."""
    i = np.arange(n_q, dtype=np.int64)[:, None]
    return np.asarray(t, dtype=np.int64)[None, :] <= kv_len - n_q + i


def _token_range(kv_indptr, kv_last_page_len, page_size: int, r: int, page_begin: int, page_end):
    """Logical token ids of request r whose page lies in [page_begin, page_end)."""
    n = int(kv_indptr[r + 1]) - int(kv_indptr[r])
    L = request_kv_length(kv_indptr, kv_last_page_len, page_size, r)
    page_end = n if page_end is None else page_end
    return np.arange(page_begin * page_size, min(page_end * page_size, L), dtype=np.int64), L


# ----------------------------------------------------------------------------- attention core
def _softmax_attend(s: np.ndarray, v: np.ndarray, visible: Optional[np.ndarray] = None):
    """s: [rows, L] scaled logits, v: [L, Dv] -> O [rows, Dv], LSE [rows] (definition).  With
    ``visible`` ([rows, L] bool) each row attends only to its visible keys; a row that sees no
    key gets O = 0, LSE = -inf (the empty-KV convention)."""
    rows = s.shape[0]
    if s.shape[1] == 0:
        return np.zeros((rows, v.shape[1])), np.full(rows, -np.inf)
    if visible is not None:
        o = np.zeros((rows, v.shape[1]))
        lse = np.full(rows, -np.inf)
        for i in range(rows):
            keys = np.flatnonzero(visible[i])
            if keys.size:
                oi, li = _softmax_attend(s[i:i + 1, keys], v[keys])
                o[i], lse[i] = oi[0], li[0]
        return o, lse
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    o = (e @ v) / l
    return o, (m + np.log(l))[:, 0]


def _decode_kv(x, kv_dtype: str, kv_scale: float) -> np.ndarray:
    if kv_dtype == "bf16":
        return bf16_to_f64(x)
    if kv_dtype == "e4m3":
        return e4m3_to_f64(x) * float(kv_scale)
    raise ValueError(kv_dtype)


def _gqa_request(q, k, v, qo_indptr, kv_indptr, kv_indices, kv_last_page_len, page_size, sm_scale,
                 r, heads, page_begin=0, page_end=None, causal=False, kv_dtype="bf16", kv_scale=1.0):
    hq, hk = q.shape[1], k.shape[2]
    g = hq // hk
    pages, slots = request_token_slots(kv_indptr, kv_indices, kv_last_page_len, page_size, r,
                                       page_begin, page_end)
    q_r = bf16_to_f64(q[int(qo_indptr[r]):int(qo_indptr[r + 1])])      # [n_q, Hq, D]
    n_q, dv = q_r.shape[0], v.shape[3]
    vis = None
    if causal:
        t, L = _token_range(kv_indptr, kv_last_page_len, page_size, r, page_begin, page_end)
        vis = causal_visible(n_q, L, t)
    o = np.zeros((n_q, len(heads), dv))
    lse = np.zeros((n_q, len(heads)))
    for kh in sorted({h // g for h in heads}):
        kk = _decode_kv(k[pages, slots, kh], kv_dtype, kv_scale)         # [L, D]
        vv = _decode_kv(v[pages, slots, kh], kv_dtype, kv_scale)         # [L, Dv]
        for j, h in enumerate(heads):
            if h // g != kh:
                continue
            s = sm_scale * (q_r[:, h, :] @ kk.T)                          # [n_q, L]
            o[:, j], lse[:, j] = _softmax_attend(s, vv, vis)
    return o, lse


def paged_attention(q, k, v, qo_indptr, kv_indptr, kv_indices, kv_last_page_len, page_size: int,
                    sm_scale: float, requests: Optional[Iterable[int]] = None,
                    heads: Optional[Sequence[int]] = None, causal: bool = False, kv_dtype: str = "bf16",
                    kv_scale: float = 1.0):
    """GQA attention over a paged KV cache (bf16, or e4m3 codes times the per-tensor ``kv_scale``).

    q: bf16 bits [total_q, Hq, D]; k, v: bf16 bits or e4m3 codes [num_pages, P, Hk, D] (any strides);
    returns O [total_q, |heads|, Dv] and LSE [total_q, |heads|] in float64 (rows of requests
    not in ``requests`` are NaN).  ``causal``: each query token sees only keys up to its own
    position (``causal_visible``)."""
    heads = list(range(q.shape[1])) if heads is None else list(heads)
    requests = range(len(kv_indptr) - 1) if requests is None else requests
    O = np.full((q.shape[0], len(heads), v.shape[3]), np.nan)
    LSE = np.full((q.shape[0], len(heads)), np.nan)
    for r in requests:
        a, b = int(qo_indptr[r]), int(qo_indptr[r + 1])
        O[a:b], LSE[a:b] = _gqa_request(q, k, v, qo_indptr, kv_indptr, kv_indices, kv_last_page_len,
                                        page_size, sm_scale, r, heads, causal=causal, kv_dtype=kv_dtype,
                                        kv_scale=kv_scale)
    return O, LSE


def paged_attention_partials(q, k, v, qo_indptr, kv_indptr, kv_indices, kv_last_page_len,
                             page_size: int, sm_scale: float, split_page_start,
                             requests: Optional[Iterable[int]] = None, causal: bool = False,
                             kv_dtype: str = "bf16", kv_scale: float = 1.0):
    """Per request r and split j over logical pages [split_page_start[r][j], [j+1]): the
    partial (O_j, LSE_j) of every query token and head.  Returns {r: (O [S, n_q, Hq, Dv],
    LSE [S, n_q, Hq])}."""
    heads = list(range(q.shape[1]))
    requests = range(len(kv_indptr) - 1) if requests is None else requests
    out = {}
    for r in requests:
        b = split_page_start[r]
        parts = [_gqa_request(q, k, v, qo_indptr, kv_indptr, kv_indices, kv_last_page_len, page_size,
                              sm_scale, r, heads, b[j], b[j + 1], causal, kv_dtype, kv_scale)
                 for j in range(len(b) - 1)]
        out[r] = (np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    return out


# ----------------------------------------------------------------------------- merge
def merge_states(o_states, lse_states):
    """Exact merge over the leading axis: o_states [S, ..., Dv], lse_states [S, ...].

    M = max_j LSE_j; LSE = M + ln sum_j exp(LSE_j - M); O = sum_j exp(LSE_j - LSE) O_j.
    Where every LSE_j is -inf (no tokens at all) the result is O = 0, LSE = -inf."""
    o_states = np.asarray(o_states, dtype=np.float64)
    lse_states = np.asarray(lse_states, dtype=np.float64)
    S = lse_states.shape[0]
    M = np.full(lse_states.shape[1:], -np.inf)
    for j in range(S):
        M = np.maximum(M, lse_states[j])
    empty = np.isneginf(M)
    Ms = np.where(empty, 0.0, M)
    total = np.zeros_like(Ms)
    for j in range(S):
        total += np.where(np.isneginf(lse_states[j]), 0.0, np.exp(lse_states[j] - Ms))
    lse = np.where(empty, -np.inf, Ms + np.log(np.where(empty, 1.0, total)))
    lse_s = np.where(empty, 0.0, lse)
    o = np.zeros(o_states.shape[1:])
    for j in range(S):
        w = np.where(np.isneginf(lse_states[j]) | empty, 0.0, np.exp(lse_states[j] - lse_s))
        o += w[..., None] * o_states[j]
    return o, lse


# ----------------------------------------------------------------------------- MLA
def _mla_request(q_nope, q_pe, ckv, kpe, kv_indptr, kv_indices, kv_last_page_len, page_size,
                 sm_scale, kv_dtype, kv_scale, r, heads, page_begin=0, page_end=None, causal=False):
    pages, slots = request_token_slots(kv_indptr, kv_indices, kv_last_page_len, page_size, r,
                                       page_begin, page_end)
    c = _decode_kv(ckv[pages, slots], kv_dtype, kv_scale)                 # [L, 512]  (= V)
    kr = _decode_kv(kpe[pages, slots], kv_dtype, kv_scale)                # [L, 64]
    qn = bf16_to_f64(q_nope[r])[:, heads]                                  # [q_len, H', 512]
    qp = bf16_to_f64(q_pe[r])[:, heads]
    q_len, nh = qn.shape[0], qn.shape[1]
    s = sm_scale * (qn.reshape(q_len * nh, -1) @ c.T + qp.reshape(q_len * nh, -1) @ kr.T)
    vis = None
    if causal:   # rows are (decode position i, head): every head of position i shares its mask
        t, L = _token_range(kv_indptr, kv_last_page_len, page_size, r, page_begin, page_end)
        vis = np.repeat(causal_visible(q_len, L, t), nh, axis=0)
    o, lse = _softmax_attend(s, c) if vis is None else _softmax_attend(s, c, vis)
    return o.reshape(q_len, nh, -1), lse.reshape(q_len, nh)


def mla_decode(q_nope, q_pe, ckv, kpe, kv_indptr, kv_indices, kv_last_page_len, page_size: int,
               sm_scale: float, kv_dtype: str = "bf16", kv_scale: float = 1.0,
               requests: Optional[Iterable[int]] = None, heads: Optional[Sequence[int]] = None,
               causal: bool = False):
    """MLA latent attention.  q_nope [B, q_len, H, 512], q_pe [B, q_len, H, 64] (bf16 bits);
    ckv [num_pages, P, 512], kpe [num_pages, P, 64] (bf16 bits or e4m3 codes).  Returns
    O [B, q_len, |heads|, 512], LSE [B, q_len, |heads|] (unrequested requests NaN)."""
    heads = list(range(q_nope.shape[2])) if heads is None else list(heads)
    requests = range(len(kv_indptr) - 1) if requests is None else requests
    B, q_len = q_nope.shape[0], q_nope.shape[1]
    O = np.full((B, q_len, len(heads), ckv.shape[-1]), np.nan)
    LSE = np.full((B, q_len, len(heads)), np.nan)
    for r in requests:
        O[r], LSE[r] = _mla_request(q_nope, q_pe, ckv, kpe, kv_indptr, kv_indices, kv_last_page_len,
                                    page_size, sm_scale, kv_dtype, kv_scale, r, heads, causal=causal)
    return O, LSE


def mla_decode_partials(q_nope, q_pe, ckv, kpe, kv_indptr, kv_indices, kv_last_page_len,
                        page_size: int, sm_scale: float, split_page_start, kv_dtype: str = "bf16",
                        kv_scale: float = 1.0, requests: Optional[Iterable[int]] = None,
                        causal: bool = False):
    """Per request and split (logical page ranges), the MLA partial (O_j, LSE_j)."""
    heads = list(range(q_nope.shape[2]))
    requests = range(len(kv_indptr) - 1) if requests is None else requests
    out = {}
    for r in requests:
        b = split_page_start[r]
        parts = [_mla_request(q_nope, q_pe, ckv, kpe, kv_indptr, kv_indices, kv_last_page_len,
                              page_size, sm_scale, kv_dtype, kv_scale, r, heads, b[j], b[j + 1], causal)
                 for j in range(len(b) - 1)]
        out[r] = (np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    return out
