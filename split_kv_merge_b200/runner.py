"""High-level calls: plan on the host, copy the plan to the device, allocate outputs with torch,
launch through the C ABI.  These are the calls a user makes; they add no arithmetic."""
from __future__ import annotations

from typing import Optional

import numpy as np

from . import (Plan, mla_decode_fwd, merge_states, paged_attn_fwd, plan_mla, plan_paged)


def _dev_i32(a, device, non_blocking=False):
    import torch
    if isinstance(a, torch.Tensor):
        return a.to(device=device, dtype=torch.int32, non_blocking=non_blocking)
    t = torch.from_numpy(np.ascontiguousarray(np.asarray(a, dtype=np.int32)))
    if non_blocking:
        t = t.pin_memory()
    return t.to(device, non_blocking=non_blocking)


def paged_attention(q, k_cache, v_cache, qo_indptr_h, kv_indptr_h, kv_indices, kv_last_page_len_h, *,
                    sm_scale: Optional[float] = None, policy="balanced", param: int = 0,
                    split_page_start=None, o_dtype=None, num_pages: Optional[int] = None,
                    kv_indptr=None, kv_last_page_len=None, plan: Optional[Plan] = None,
                    status=None, stream=None):
    """GQA attention over a paged cache.  Host page-table shape arrays (``*_h``) feed the planner;
    ``kv_indices`` (and optionally ``kv_indptr`` / ``kv_last_page_len``) are device tensors.
    Returns (o, lse, extras) with extras = {"plan", "o_part", "lse_part"}."""
    import torch
    dev = q.device
    hq, d = q.shape[1], q.shape[2]
    hk = k_cache.shape[2]
    if plan is None:
        plan = plan_paged(qo_indptr_h, kv_indptr_h, kv_last_page_len_h, k_cache.shape[1], hq, hk, d, policy,
                          param, split_page_start)
    if plan.device is None:
        plan.to(dev)
    kv_indptr = _dev_i32(kv_indptr_h, dev) if kv_indptr is None else kv_indptr
    kv_last_page_len = _dev_i32(kv_last_page_len_h, dev) if kv_last_page_len is None else kv_last_page_len
    o = torch.empty(q.shape[0], hq, d, dtype=o_dtype or torch.float32, device=dev)
    lse = torch.empty(q.shape[0], hq, dtype=torch.float32, device=dev)
    n_part = plan.info.num_partial_rows
    o_part = torch.empty(n_part, hq, d, dtype=torch.float32, device=dev) if n_part else None
    lse_part = torch.empty(n_part, hq, dtype=torch.float32, device=dev) if n_part else None
    paged_attn_fwd(q, k_cache, v_cache, kv_indptr, kv_indices, kv_last_page_len, plan, o, lse, o_part, lse_part,
                   status, sm_scale, num_pages, stream)
    return o, lse, {"plan": plan, "o_part": o_part, "lse_part": lse_part}


def mla_decode(q_nope, q_pe, ckv, kpe, kv_indptr_h, kv_indices, kv_last_page_len_h, *,
               sm_scale: Optional[float] = None, kv_scale: float = 1.0, policy="balanced", param: int = 0,
               split_page_start=None, o_dtype=None, num_pages: Optional[int] = None, kv_indptr=None,
               kv_last_page_len=None, plan: Optional[Plan] = None, status=None, stream=None, o=None, lse=None):
    """MLA latent decode over a paged latent cache (bf16 or e4m3 codes).  Returns (o, lse, extras)."""
    import torch
    dev = q_nope.device
    B, q_len, H = q_nope.shape[:3]
    if plan is None:
        kd = "bf16" if ckv.dtype == torch.bfloat16 else "e4m3"
        plan = plan_mla(q_len, kv_indptr_h, kv_last_page_len_h, ckv.shape[1], H, policy, param, split_page_start, kd)
    if plan.device is None:
        plan.to(dev)
    kv_indptr = _dev_i32(kv_indptr_h, dev) if kv_indptr is None else kv_indptr
    kv_last_page_len = _dev_i32(kv_last_page_len_h, dev) if kv_last_page_len is None else kv_last_page_len
    if o is None:
        o = torch.empty(B, q_len, H, 512, dtype=o_dtype or torch.float32, device=dev)
    if lse is None:
        lse = torch.empty(B, q_len, H, dtype=torch.float32, device=dev)
    n_part = plan.info.num_partial_rows
    o_part = torch.empty(n_part, H, 512, dtype=torch.float32, device=dev) if n_part else None
    lse_part = torch.empty(n_part, H, dtype=torch.float32, device=dev) if n_part else None
    mla_decode_fwd(q_nope, q_pe, ckv, kpe, kv_indptr, kv_indices, kv_last_page_len, plan, o, lse, o_part, lse_part,
                   status, sm_scale, kv_scale, num_pages, stream)
    return o, lse, {"plan": plan, "o_part": o_part, "lse_part": lse_part}


class RouteMerge:
    """Route-and-merge on one GPU: each KV chunk "holder" computes the partial MLA attention of
    every query over that query's selected rows of the chunk (page size 1: a page id is a token
    id), then ``merge_states`` combines the chunk partials per query (the route primitive of
    "Move the Query, Not the Cache")."""

    def __init__(self, sel_h: np.ndarray, num_heads: int, device):
        import torch
        Q, C, K = sel_h.shape
        self.Q, self.C, self.K, self.H = Q, C, K, num_heads
        self.kv_indptr_h = (np.arange(Q + 1, dtype=np.int64) * K).astype(np.int32)
        self.last_h = np.ones(Q, dtype=np.int32)
        self.plan = plan_mla(1, self.kv_indptr_h, self.last_h, 1, num_heads, "none").to(device)
        self.kv_indptr = _dev_i32(self.kv_indptr_h, device)
        self.last = _dev_i32(self.last_h, device)
        self.o_states = torch.empty(C, Q, 1, num_heads, 512, dtype=torch.float32, device=device)
        self.lse_states = torch.empty(C, Q, 1, num_heads, dtype=torch.float32, device=device)

    def __call__(self, q_nope, q_pe, ckv, kpe, sel_cqk, *, sm_scale=None, status=None, stream=None, o=None,
                 lse=None):
        """sel_cqk: device int32 [C, Q, K], chunk-major (per chunk and query, the selected global
        token ids), so that each chunk's index list is one contiguous block."""
        import torch
        dev = q_nope.device
        for c in range(self.C):
            mla_decode_fwd(q_nope, q_pe, ckv, kpe, self.kv_indptr, sel_cqk[c], self.last, self.plan, self.o_states[c],
                           self.lse_states[c], None, None, status, sm_scale, 1.0, ckv.shape[0], stream)
        if o is None:
            o = torch.empty(self.Q, self.H, 512, dtype=torch.float32, device=dev)
        if lse is None:
            lse = torch.empty(self.Q, self.H, dtype=torch.float32, device=dev)
        merge_states(self.o_states.view(self.C, self.Q, self.H, 512), self.lse_states.view(self.C, self.Q, self.H),
                     o, lse, stream=stream)
        return o, lse
