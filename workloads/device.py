"""Upload the generator's numpy bit patterns to torch tensors (CUDA or CPU) with the same views.

Glue only: no attention arithmetic.  K/V keep their strides (a V that is a column slice of a
wider buffer stays a strided view of the uploaded buffer).
"""
from __future__ import annotations

import numpy as np

from .gen import MlaCase, PagedCase, RouteCase


def bf16_tensor(bits: np.ndarray, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def i32_tensor(a, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(np.asarray(a, dtype=np.int32))).to(device)


def paged_to_device(c: PagedCase, device):
    """dict of device tensors for a PagedCase: q, k, v (views), k_store, v_store, page table."""
    k_store = bf16_tensor(c.k_store, device)
    v_store = bf16_tensor(c.v_store, device)
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
