"""Seeded synthetic inputs (bit patterns + page tables) for the five paged-attention workloads.

Nothing in this module computes attention.  It only

* draws float32 N(0,1) values from numpy's PCG64 (in fixed-size chunks, each from
  its own ``SeedSequence`` child, so the result does not depend on thread count),
* rounds them once to bf16 bit patterns (round-to-nearest-even) or encodes them as
  OCP fp8 e4m3 ("fn": bias 7, no infinities, max 448) codes with a per-tensor scale,
* lays out paged KV caches and page tables (``kv_indptr`` / ``kv_indices`` /
  ``kv_last_page_len``) with the physical pages drawn as a seeded permutation.

Workloads (sizes follow the paged-decode, shared-KV, MLA and route descriptions of
the FlashInfer PR #4736 page (paged FA2 with independent K/V strides), the PyTorch
MPS FlexAttention page (KV batch broadcast), the FlashInfer PR #3309 page (MLA
decode with seqlen_q folding) and the "Move the Query, Not the Cache" summary
(route = per-chunk partial attention + merge)):

1. ``tiny_gqa_case``        4 requests, 8/2 heads, D=64, P=16, L={37,128,200,256}
2. ``llama70b_decode_case`` 64 requests, 64/8 heads, D=128, P=16, L~U[1024,8192]
3. ``shared_kv_prefill_case`` one 16384-token KV, P=64, 32/8 heads, 32 x 128 queries
4. ``mla_decode_case``      32 requests, H in {16,128}, q_len in {1,4}, 512+64 latent
5. ``route_case``           131072-token latent cache, 8 chunks, 256 queries x 16 heads
6. ``fetch_splice_case``    the same corpus fetched chunk by chunk into a requester's paged cache
"""
from __future__ import annotations

import functools
import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

__all__ = [
    "BF16_NAN", "E4M3_NAN", "f32_to_bf16_bits", "bf16_bits_to_f32", "e4m3_encode",
    "normal_f32", "normal_bf16", "build_page_table", "PagedCase", "MlaCase", "RouteCase", "pod_case",
    "tiny_gqa_case", "llama70b_decode_case", "shared_kv_prefill_case", "mla_decode_case",
    "route_case", "even_split_pages", "SpliceCase", "fetch_splice_case",
]

BF16_NAN = np.uint16(0x7FC0)
E4M3_NAN = np.uint8(0x7F)
_CHUNK = 1 << 22


# ----------------------------------------------------------------------------- formats
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 bit patterns, round-to-nearest-even (finite inputs)."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def e4m3_encode(x: np.ndarray, chunk: int = 1 << 24) -> np.ndarray:
    """Encode values as OCP e4m3fn codes: round to nearest, ties to even mantissa, saturating to
    +-448.  Exponent from frexp, mantissa rounded with rint (half-to-even); everything below 2^-6
    is on the subnormal grid m * 2^-9.  (Storage-format conversion for the synthetic fp8 cache.)"""
    x = np.asarray(x)
    flat = x.reshape(-1)
    out = np.empty(flat.shape, dtype=np.uint8)

    def encode(lo: int) -> None:   # chunks are independent; numpy releases the GIL inside them
        v = flat[lo:lo + chunk].astype(np.float64)
        a = np.minimum(np.abs(v), 448.0)
        sub = a < 2.0 ** -6
        mant, ex = np.frexp(np.where(sub, 1.0, a))        # a = mant * 2^ex, mant in [0.5, 1)
        e = ex - 1                                         # a = (2 mant) * 2^e, 2 mant in [1, 2)
        m = np.rint((2.0 * mant - 1.0) * 8.0)
        carry = m == 8.0
        e = np.where(carry, e + 1, e)
        m = np.where(carry, 0.0, m)
        code_n = ((e + 7) << 3).astype(np.int64) | m.astype(np.int64)
        code_s = np.rint(a * 2.0 ** 9).astype(np.int64)   # 0..8 (8 is the smallest normal, code 0x08)
        code = np.minimum(np.where(sub, code_s, code_n), 0x7E).astype(np.uint8)
        out[lo:lo + chunk] = code | np.where(np.signbit(v), np.uint8(0x80), np.uint8(0))

    starts = range(0, flat.size, chunk)
    if len(starts) <= 1:
        for lo in starts:
            encode(lo)
    else:
        with ThreadPoolExecutor(min(8, len(starts))) as ex:
            list(ex.map(encode, starts))
    return out.reshape(x.shape)


# ----------------------------------------------------------------------------- random draws
def normal_f32(seed: int, stream: int, n: int, threads: int = 8) -> np.ndarray:
    """n float32 N(0,1) draws; chunk i comes from SeedSequence(seed, spawn_key=(stream, i))."""
    out = np.empty(n, dtype=np.float32)
    nchunks = max(1, (n + _CHUNK - 1) // _CHUNK)

    def fill(i: int) -> None:
        lo, hi = i * _CHUNK, min(n, (i + 1) * _CHUNK)
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(stream, i))))
        g.standard_normal(out=out[lo:hi], dtype=np.float32)

    if nchunks == 1 or threads <= 1:
        for i in range(nchunks):
            fill(i)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(fill, range(nchunks)))
    return out


def normal_bf16(seed: int, stream: int, shape) -> np.ndarray:
    """bf16 bit patterns of N(0,1) draws, shape ``shape``."""
    n = int(np.prod(shape))
    return f32_to_bf16_bits(normal_f32(seed, stream, n)).reshape(shape)


# ----------------------------------------------------------------------------- page tables
def build_page_table(rng: np.random.Generator, lengths, page_size: int, extra_pages: int = 0,
                     permute: bool = True):
    """Page table for requests of KV length ``lengths``.

    Request r owns n_r = ceil(L_r / P) pages, listed in ``kv_indices[kv_indptr[r]:kv_indptr[r+1]]``;
    ``kv_last_page_len[r]`` = L_r - (n_r - 1) P in [1, P] (0 when n_r = 0).  The physical page ids
    are a seeded permutation of ``num_pages = sum(n_r) + extra_pages``.
    """
    lengths = np.asarray(lengths, dtype=np.int64)
    n = (lengths + page_size - 1) // page_size
    kv_indptr = np.zeros(len(lengths) + 1, dtype=np.int32)
    kv_indptr[1:] = np.cumsum(n)
    num_pages = int(kv_indptr[-1]) + extra_pages
    ids = rng.permutation(num_pages) if permute else np.arange(num_pages)
    kv_indices = ids[: kv_indptr[-1]].astype(np.int32)
    last = np.where(n > 0, lengths - (n - 1) * page_size, 0).astype(np.int32)
    return kv_indptr, kv_indices, last, num_pages


def even_split_pages(kv_indptr, num_splits: int):
    """Per request, ``num_splits`` page ranges, earlier splits taking the extra page
    (ceil first): returns ``split_page_start`` lists (request-relative, length S+1)."""
    out = []
    for r in range(len(kv_indptr) - 1):
        n = int(kv_indptr[r + 1] - kv_indptr[r])
        b = [0]
        for j in range(num_splits):
            rem = n - b[-1]
            b.append(b[-1] + (rem + (num_splits - j) - 1) // (num_splits - j))
        out.append(b)
    return out


# ----------------------------------------------------------------------------- containers
@dataclass
class PagedCase:
    """GQA paged attention input.  ``k`` / ``v`` are numpy views [num_pages, P, Hk, D] of
    bf16 bit patterns over ``k_store`` / ``v_store`` (V may be a column slice of a wider buffer)."""
    name: str
    q: np.ndarray               # uint16 [total_q, Hq, D]
    k_store: np.ndarray         # uint16 buffer holding K
    v_store: np.ndarray         # uint16 buffer holding V (may be K's shape or wider)
    k: np.ndarray               # view [num_pages, P, Hk, D]
    v: np.ndarray               # view [num_pages, P, Hk, D]
    qo_indptr: np.ndarray       # int32 [B+1]
    kv_indptr: np.ndarray       # int32 [B+1]
    kv_indices: np.ndarray      # int32 [nnz]
    kv_last_page_len: np.ndarray  # int32 [B]
    page_size: int
    num_qo_heads: int
    num_kv_heads: int
    head_dim: int
    sm_scale: float
    num_pages: int
    split_page_start: Optional[list] = None   # per request list of page boundaries
    meta: dict = field(default_factory=dict)
    kv_dtype: str = "bf16"      # "bf16": k/v hold bf16 bits; "e4m3": OCP e4m3fn codes (uint8)
    kv_scale: float = 1.0       # per-tensor dequantisation scale of the e4m3 codes

    @property
    def batch(self) -> int:
        return len(self.kv_indptr) - 1

    def kv_lengths(self) -> np.ndarray:
        n = np.diff(self.kv_indptr).astype(np.int64)
        return np.where(n > 0, (n - 1) * self.page_size + self.kv_last_page_len, 0)


@dataclass
class MlaCase:
    """MLA latent decode input.  ``ckv`` / ``kpe`` are views [num_pages, P, 512] / [.., 64] of the
    combined 576-wide cache ``cache`` (bf16 bits, or e4m3 codes with ``kv_scale``)."""
    name: str
    q_nope: np.ndarray          # uint16 [B, q_len, H, 512]
    q_pe: np.ndarray            # uint16 [B, q_len, H, 64]
    cache: np.ndarray           # uint16 or uint8 [num_pages, P, 576]
    ckv: np.ndarray
    kpe: np.ndarray
    kv_dtype: str               # "bf16" | "e4m3"
    kv_scale: float
    kv_indptr: np.ndarray
    kv_indices: np.ndarray
    kv_last_page_len: np.ndarray
    page_size: int
    num_heads: int
    q_len: int
    sm_scale: float
    num_pages: int
    meta: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return len(self.kv_indptr) - 1

    def kv_lengths(self) -> np.ndarray:
        n = np.diff(self.kv_indptr).astype(np.int64)
        return np.where(n > 0, (n - 1) * self.page_size + self.kv_last_page_len, 0)


@dataclass
class RouteCase:
    """Route-and-merge input: one latent cache split into chunks; per (query, chunk) a sorted
    list of selected token ids.  ``as_mla(chunk)`` views chunk c's selections as an MLA case
    with page_size 1 (page id = global token id)."""
    name: str
    q_nope: np.ndarray          # uint16 [Q, 1, H, 512]
    q_pe: np.ndarray            # uint16 [Q, 1, H, 64]
    cache: np.ndarray           # uint16 [N_tokens, 576]
    sel: np.ndarray             # int32 [Q, C, K] global token ids, sorted within (q, c)
    num_chunks: int
    chunk_tokens: int
    num_heads: int
    sm_scale: float

    def as_mla(self, chunk: int) -> MlaCase:
        Q, _, K = self.sel.shape
        kv_indptr = (np.arange(Q + 1, dtype=np.int64) * K).astype(np.int32)
        kv_indices = np.ascontiguousarray(self.sel[:, chunk, :]).reshape(-1).astype(np.int32)
        last = np.ones(Q, dtype=np.int32)
        c3 = self.cache.reshape(self.cache.shape[0], 1, 576)
        return MlaCase(f"{self.name}/chunk{chunk}", self.q_nope, self.q_pe, c3, c3[..., :512], c3[..., 512:],
                       "bf16", 1.0, kv_indptr, kv_indices, last, 1, self.num_heads, 1, self.sm_scale,
                       self.cache.shape[0])

    def union_mla(self) -> MlaCase:
        """All chunks' selections of each query concatenated (the unsplit reference problem)."""
        Q, C, K = self.sel.shape
        kv_indptr = (np.arange(Q + 1, dtype=np.int64) * C * K).astype(np.int32)
        kv_indices = self.sel.reshape(-1).astype(np.int32)
        last = np.ones(Q, dtype=np.int32)
        c3 = self.cache.reshape(self.cache.shape[0], 1, 576)
        return MlaCase(f"{self.name}/union", self.q_nope, self.q_pe, c3, c3[..., :512], c3[..., 512:],
                       "bf16", 1.0, kv_indptr, kv_indices, last, 1, self.num_heads, 1, self.sm_scale,
                       self.cache.shape[0])


# ----------------------------------------------------------------------------- helpers
def _poison_paged(k_view, v_view, kv_indptr, kv_indices, last, page_size, num_pages, kv_dtype="bf16"):
    used = np.zeros(num_pages, dtype=bool)
    used[kv_indices] = True
    nan = BF16_NAN if kv_dtype == "bf16" else E4M3_NAN
    k_view[~used] = nan
    v_view[~used] = nan
    # a huge V in the tail slots: 1e4 in bf16, the largest e4m3 code (448) otherwise
    sentinel = f32_to_bf16_bits(np.array([1.0e4], dtype=np.float32))[0] if kv_dtype == "bf16" else np.uint8(0x7E)
    for r in range(len(kv_indptr) - 1):
        n = kv_indptr[r + 1] - kv_indptr[r]
        if n == 0:
            continue
        p = kv_indices[kv_indptr[r + 1] - 1]
        k_view[p, last[r]:] = nan
        v_view[p, last[r]:] = sentinel


def _make_paged(name, seed, lengths, q_len, hq, hk, d, page_size, independent_v, extra_pages=0,
                poison=False, qo_lens=None, kv_dtype="bf16"):
    rng = np.random.Generator(np.random.PCG64(seed))
    kv_indptr, kv_indices, last, num_pages = build_page_table(rng, lengths, page_size, extra_pages)
    b = len(lengths)
    qo_lens = np.full(b, q_len, dtype=np.int64) if qo_lens is None else np.asarray(qo_lens, np.int64)
    qo_indptr = np.zeros(b + 1, dtype=np.int32)
    qo_indptr[1:] = np.cumsum(qo_lens)
    q = normal_bf16(seed, 1, (int(qo_indptr[-1]), hq, d))
    v_shape = (num_pages, page_size, hk, 2 * d if independent_v else d)
    kv_scale = 1.0
    if kv_dtype == "bf16":
        k_store = normal_bf16(seed, 2, (num_pages, page_size, hk, d))
        v_store = normal_bf16(seed, 3, v_shape)
    elif kv_dtype == "e4m3":
        # N(0,1) draws encoded as e4m3 codes with one scale for K and V: amax / 448
        kf = normal_f32(seed, 2, num_pages * page_size * hk * d)
        vf = normal_f32(seed, 3, int(np.prod(v_shape)))
        kv_scale = float(np.float32(max(float(np.max(np.abs(kf))), float(np.max(np.abs(vf)))) / 448.0))
        k_store = e4m3_encode(kf / np.float64(kv_scale)).reshape(num_pages, page_size, hk, d)
        v_store = e4m3_encode(vf / np.float64(kv_scale)).reshape(v_shape)
    else:
        raise ValueError(kv_dtype)
    v = v_store[..., :d] if independent_v else v_store
    k = k_store
    if poison:
        _poison_paged(k, v, kv_indptr, kv_indices, last, page_size, num_pages, kv_dtype)
    return PagedCase(name, q, k_store, v_store, k, v, qo_indptr, kv_indptr, kv_indices, last, page_size,
                     hq, hk, d, 1.0 / math.sqrt(d), num_pages, kv_dtype=kv_dtype, kv_scale=kv_scale)


# ----------------------------------------------------------------------------- workloads
def tiny_gqa_case(poison: bool = False, independent_v: bool = False, seed: int = 1) -> PagedCase:
    """4 requests, q_len 1, 8 query / 2 KV heads, D=64, P=16, L={37,128,200,256}; 64 physical
    pages (the 40 used ones a seeded permutation), scale 1/8, 2 KV splits per request."""
    c = _make_paged("tiny_gqa", seed, [37, 128, 200, 256], 1, 8, 2, 64, 16, independent_v,
                    extra_pages=64 - 40, poison=poison)
    c.split_page_start = even_split_pages(c.kv_indptr, 2)
    return c


def llama70b_decode_case(independent_v: bool = False, batch: int = 64, seed: int = 2,
                         len_range=(1024, 8192), poison: bool = False, kv_dtype: str = "bf16",
                         q_len: int = 1) -> PagedCase:
    """Llama-3.1-70B-shaped decode: q_len 1, 64 query / 8 KV heads, D=128, P=16,
    L ~ U[1024, 8192]; V optionally a column slice of a [.., 8, 256] buffer; K/V bf16, or e4m3
    codes with one per-tensor scale (``kv_dtype="e4m3"``)."""
    rng = np.random.Generator(np.random.PCG64(seed + 1000))
    lengths = rng.integers(len_range[0], len_range[1] + 1, size=batch)
    name = "llama70b_decode" + ("_indep_v" if independent_v else "") + ("_e4m3" if kv_dtype == "e4m3" else "")
    return _make_paged(name, seed, lengths, q_len, 64, 8, 128, 16, independent_v, poison=poison, kv_dtype=kv_dtype)


def pod_case(num_decode: int = 48, prefill_q=(1024, 1024), prefill_kv=(2048, 2048), seed: int = 6,
             decode_len_range=(1024, 8192)) -> PagedCase:
    """A POD batch (prefill on decode) with Llama-3.1-70B heads (64 query / 8 KV, D=128, P=16):
    ``num_decode`` decode requests (one query token, KV lengths U[1024, 8192]) followed by prefill
    requests of ``prefill_q`` query tokens over ``prefill_kv`` KV tokens (every query token sees the
    request's whole KV), bf16 N(0,1), randomly permuted pages."""
    rng = np.random.Generator(np.random.PCG64(seed + 3000))
    dec_lens = rng.integers(decode_len_range[0], decode_len_range[1] + 1, size=num_decode)
    lengths = np.concatenate([dec_lens, np.asarray(prefill_kv, np.int64)])
    qo_lens = np.concatenate([np.ones(num_decode, np.int64), np.asarray(prefill_q, np.int64)])
    return _make_paged("pod_llama70b", seed, lengths, 1, 64, 8, 128, 16, False, qo_lens=qo_lens)


def shared_kv_prefill_case(replicated: bool = False, n_batches: int = 32, q_len: int = 128,
                           kv_len: int = 16384, seed: int = 3) -> PagedCase:
    """One kv_len-token KV sequence (P=64, 32 query / 8 KV heads, D=128) shared by n_batches
    query batches of q_len tokens, no mask.  ``replicated`` stores a private copy of the KV
    pages per batch (same values) instead of listing the same pages in every request."""
    hq, hk, d, P = 32, 8, 128, 64
    rng = np.random.Generator(np.random.PCG64(seed))
    n = kv_len // P if kv_len % P == 0 else kv_len // P + 1
    base_pages = rng.permutation(n).astype(np.int32)
    k1 = normal_bf16(seed, 2, (n, P, hk, d))
    v1 = normal_bf16(seed, 3, (n, P, hk, d))
    last_len = kv_len - (n - 1) * P
    qo_indptr = (np.arange(n_batches + 1) * q_len).astype(np.int32)
    q = normal_bf16(seed, 1, (n_batches * q_len, hq, d))
    kv_indptr = (np.arange(n_batches + 1) * n).astype(np.int32)
    last = np.full(n_batches, last_len, dtype=np.int32)
    if not replicated:
        # logical page j of the shared sequence lives at physical page base_pages[j]
        k_store = np.empty_like(k1)
        v_store = np.empty_like(v1)
        k_store[base_pages] = k1
        v_store[base_pages] = v1
        kv_indices = np.tile(base_pages, n_batches)
        num_pages = n
    else:
        perm = rng.permutation(n * n_batches).astype(np.int32)
        k_store = np.empty((n * n_batches, P, hk, d), dtype=np.uint16)
        v_store = np.empty_like(k_store)
        kv_indices = perm
        for b in range(n_batches):
            ids = perm[b * n:(b + 1) * n]
            k_store[ids] = k1
            v_store[ids] = v1
        num_pages = n * n_batches
    return PagedCase("shared_kv_prefill" + ("_replicated" if replicated else ""), q, k_store, v_store,
                     k_store, v_store, qo_indptr, kv_indptr, kv_indices, last, P, hq, hk, d,
                     1.0 / math.sqrt(d), num_pages, meta={"kv_len": kv_len, "q_len": q_len})


@functools.lru_cache(maxsize=4)
def _latent_cache(seed: int, num_pages: int, page_size: int, kv_dtype: str):
    """[num_pages, P, 576] latent cache (read-only, shared between MLA sub-configurations)."""
    raw = normal_f32(seed, 3, num_pages * page_size * 576).reshape(num_pages, page_size, 576)
    if kv_dtype == "bf16":
        cache, kv_scale = f32_to_bf16_bits(raw), 1.0
    elif kv_dtype == "e4m3":
        amax = float(np.max(np.abs(raw)))
        kv_scale = float(np.float32(amax / 448.0))
        cache = e4m3_encode(raw / np.float64(kv_scale))
    else:
        raise ValueError(kv_dtype)
    cache.setflags(write=False)
    return cache, kv_scale


def mla_decode_case(num_heads: int = 16, q_len: int = 1, kv_dtype: str = "bf16", batch: int = 32,
                    seed: int = 4, len_range=(4096, 32768), page_size: int = 64,
                    poison: bool = False) -> MlaCase:
    """DeepSeek-V3-shaped MLA decode: 512-d latent + 64-d rope part (576 per token), P=64,
    L ~ U[4096, 32768], scale 1/sqrt(192); bf16 cache or e4m3 cache with per-tensor scale
    amax/448."""
    rng = np.random.Generator(np.random.PCG64(seed + 2000))
    lengths = rng.integers(len_range[0], len_range[1] + 1, size=batch)
    kv_indptr, kv_indices, last, num_pages = build_page_table(rng, lengths, page_size, 0)
    q_nope = normal_bf16(seed, 1 + 10 * num_heads + q_len, (batch, q_len, num_heads, 512))
    q_pe = normal_bf16(seed, 2 + 10 * num_heads + q_len, (batch, q_len, num_heads, 64))
    cache, kv_scale = _latent_cache(seed, num_pages, page_size, kv_dtype)
    if poison:
        cache = cache.copy()
        used = np.zeros(num_pages, dtype=bool)
        used[kv_indices] = True
        nan = BF16_NAN if kv_dtype == "bf16" else E4M3_NAN
        big = f32_to_bf16_bits(np.array([1.0e4], np.float32))[0] if kv_dtype == "bf16" else np.uint8(0x7E)
        cache[~used] = nan
        for r in range(batch):
            p = kv_indices[kv_indptr[r + 1] - 1]
            cache[p, last[r]:, 512:] = nan
            cache[p, last[r]:, :512] = big
    return MlaCase(f"mla_h{num_heads}_q{q_len}_{kv_dtype}", q_nope, q_pe, cache, cache[..., :512],
                   cache[..., 512:], kv_dtype, kv_scale, kv_indptr, kv_indices, last, page_size,
                   num_heads, q_len, 1.0 / math.sqrt(192.0), num_pages)


def route_case(num_queries: int = 256, num_chunks: int = 8, chunk_tokens: int = 16384,
               per_chunk: int = 2048, num_heads: int = 16, seed: int = 5) -> RouteCase:
    """Route-and-merge: a (num_chunks x chunk_tokens)-token latent cache; each query selects
    ``per_chunk`` distinct tokens per chunk (seeded uniform sampling without replacement,
    sorted ascending)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    n_tok = num_chunks * chunk_tokens
    cache = normal_bf16(seed, 3, (n_tok, 576))
    q_nope = normal_bf16(seed, 1, (num_queries, 1, num_heads, 512))
    q_pe = normal_bf16(seed, 2, (num_queries, 1, num_heads, 64))
    sel = np.empty((num_queries, num_chunks, per_chunk), dtype=np.int32)
    for q in range(num_queries):
        for c in range(num_chunks):
            ids = np.sort(rng.choice(chunk_tokens, size=per_chunk, replace=False))
            sel[q, c] = ids + c * chunk_tokens
    return RouteCase("route_merge", q_nope, q_pe, cache, sel, num_chunks, chunk_tokens, num_heads,
                     1.0 / math.sqrt(192.0))


@dataclass
class SpliceCase:
    """Fetch-primitive input: a latent corpus held in a paged cache (the chunk holder) and a
    requester's paged cache.  Chunk c is corpus positions [c*T, (c+1)*T) (logical positions
    ``src_start[c]`` .. of ``src_pages``); it lands at logical position ``dst_start[c]`` of
    ``dst_pages`` and moves by ``delta[c]`` positions."""
    name: str
    src: np.ndarray             # uint16 [src_num_pages, Ps, 576]
    src_pages: np.ndarray       # int32 corpus page list (logical order)
    dst_pages: np.ndarray       # int32 requester page list (logical order)
    dst_num_pages: int
    dst_page_size: int
    chunk_tokens: int
    src_start: np.ndarray       # int64 [C]
    dst_start: np.ndarray       # int64 [C]
    delta: np.ndarray           # int64 [C]
    rope_theta: float

    @property
    def num_chunks(self) -> int:
        return len(self.src_start)


def fetch_splice_case(num_chunks: int = 8, chunk_tokens: int = 16384, src_page_size: int = 64,
                      dst_page_size: int = 64, context: int = 1000, seed: int = 5,
                      rope_theta: float = 10000.0) -> SpliceCase:
    """The route corpus (same draws as ``route_case``: num_chunks x chunk_tokens rows of 576 bf16
    values) placed on seeded random physical pages of size ``src_page_size``; the requester holds
    ``context`` tokens of its own and fetches the chunks in a seeded random order, each appended
    after the previous one, so chunk c moves by delta = new position - c * chunk_tokens."""
    rng = np.random.Generator(np.random.PCG64(seed + 6000))
    n_tok = num_chunks * chunk_tokens
    corpus = normal_bf16(seed, 3, (n_tok, 576))
    n_src = -(-n_tok // src_page_size)
    pad = n_src * src_page_size - n_tok
    if pad:
        corpus = np.concatenate([corpus, np.zeros((pad, 576), np.uint16)])
    src_pages = rng.permutation(n_src).astype(np.int32)
    src = np.empty((n_src, src_page_size, 576), np.uint16)
    src[src_pages] = corpus.reshape(n_src, src_page_size, 576)
    n_dst_used = -(-(context + n_tok) // dst_page_size)
    dst_num_pages = n_dst_used + 3
    dst_pages = rng.permutation(dst_num_pages)[:n_dst_used].astype(np.int32)
    order = rng.permutation(num_chunks)
    src_start = np.arange(num_chunks, dtype=np.int64) * chunk_tokens
    dst_start = np.empty(num_chunks, np.int64)
    dst_start[order] = context + np.arange(num_chunks, dtype=np.int64) * chunk_tokens
    return SpliceCase(f"fetch_splice_{num_chunks}x{chunk_tokens}", src, src_pages, dst_pages, dst_num_pages,
                      dst_page_size, chunk_tokens, src_start, dst_start, dst_start - src_start, rope_theta)
