"""Upload the generator's numpy bit patterns to torch tensors (CUDA or CPU) with the same views.

Glue only: no attention arithmetic.  K/V keep their strides (a V that is a column slice of a
wider buffer stays a strided view of the uploaded buffer).
"""
from __future__ import annotations

import numpy as np

from .gen import MlaCase, PagedCase, RouteCase, SpliceCase


def bf16_tensor(bits: np.ndarray, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def i32_tensor(a, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(np.asarray(a, dtype=np.int32))).to(device)


def _kv_tensor(codes: np.ndarray, kv_dtype: str, device):
    import torch
    if kv_dtype == "bf16":
        return bf16_tensor(codes, device)
    return torch.from_numpy(np.ascontiguousarray(codes)).to(device).view(torch.float8_e4m3fn)


def paged_to_device(c: PagedCase, device):
    """dict of device tensors for a PagedCase: q, k, v (views), k_store, v_store, page table
    (K/V as bf16, or as float8_e4m3fn codes for an e4m3 case)."""
    kd = getattr(c, "kv_dtype", "bf16")
    k_store = _kv_tensor(c.k_store, kd, device)
    v_store = _kv_tensor(c.v_store, kd, device)
    d = c.head_dim
    v = v_store[..., :d] if c.v_store.shape[-1] != d else v_store
    return dict(q=bf16_tensor(c.q, device), k=k_store, v=v, k_store=k_store, v_store=v_store,
                qo_indptr=i32_tensor(c.qo_indptr, device), kv_indptr=i32_tensor(c.kv_indptr, device),
                kv_indices=i32_tensor(c.kv_indices, device),
                kv_last_page_len=i32_tensor(c.kv_last_page_len, device))


def mla_to_device(c: MlaCase, device):
    import torch
    if c.kv_dtype == "bf16":
        cache = bf16_tensor(c.cache, device)
    else:
        cache = torch.from_numpy(np.ascontiguousarray(c.cache)).to(device).view(torch.float8_e4m3fn)
    return dict(q_nope=bf16_tensor(c.q_nope, device), q_pe=bf16_tensor(c.q_pe, device), cache=cache,
                ckv=cache[..., :512], kpe=cache[..., 512:], kv_indptr=i32_tensor(c.kv_indptr, device),
                kv_indices=i32_tensor(c.kv_indices, device),
                kv_last_page_len=i32_tensor(c.kv_last_page_len, device))


def route_to_device(c: RouteCase, device):
    cache = bf16_tensor(c.cache, device).view(c.cache.shape[0], 1, 576)
    return dict(q_nope=bf16_tensor(c.q_nope, device), q_pe=bf16_tensor(c.q_pe, device), cache=cache,
                ckv=cache[..., :512], kpe=cache[..., 512:],
                sel_cqk=i32_tensor(np.ascontiguousarray(c.sel.transpose(1, 0, 2)), device))


def splice_to_device(c: SpliceCase, device, fill_bits: int = 0x40E0):
    """Source cache views, a destination cache [dst_num_pages, Pd, 576] pre-filled with one bf16
    pattern (7.0 by default, so rows the splice must not touch can be checked), page lists."""
    import torch
    src = bf16_tensor(c.src, device)
    dst = torch.full((c.dst_num_pages, c.dst_page_size, 576), 0, dtype=torch.int16, device=device)
    dst.fill_(int(np.int16(np.uint16(fill_bits))))
    dst = dst.view(torch.bfloat16)
    return dict(src=src, src_ckv=src[..., :512], src_kpe=src[..., 512:], dst=dst, dst_ckv=dst[..., :512],
                dst_kpe=dst[..., 512:], src_pages=i32_tensor(c.src_pages, device),
                dst_pages=i32_tensor(c.dst_pages, device))
