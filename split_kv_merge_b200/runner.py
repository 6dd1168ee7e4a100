"""High-level calls: plan on the host, copy the plan to the device, allocate outputs with torch,
launch through the C ABI.  These are the calls a user makes; they add no arithmetic."""
from __future__ import annotations

import ctypes
from typing import Optional

import numpy as np

from . import (OK, ERR_WORKSPACE, Plan, PlanInfo, _POLICY, _check, _paged_fwd, _paged_params, _plan_paged, _ptr_i32,
               causal_tables, mla_decode_fwd, merge_states, paged_attn_fwd, plan_mla, plan_paged, plan_paged_subset,
               pod_attn_fwd)


def _dev_i32(a, device, non_blocking=False):
    import torch
    if isinstance(a, torch.Tensor):
        return a.to(device=device, dtype=torch.int32, non_blocking=non_blocking)
    t = torch.from_numpy(np.ascontiguousarray(np.asarray(a, dtype=np.int32)))
    if non_blocking:
        t = t.pin_memory()
    return t.to(device, non_blocking=non_blocking)


def causal_split_tables(q_lens, kv_indptr_h, kv_indices_h, kv_last_page_len_h, page_size: int) -> dict:
    """Host tables that turn causal attention into two unmasked passes and a merge
    (``skv_causal_tables``): ``prefix`` -- each request cut to the keys all its query tokens see;
    ``diag`` -- one page-size-1 request per query token over the token rows (page * P + slot) it
    sees beyond that prefix."""
    qo = np.concatenate([[0], np.cumsum(np.asarray(q_lens, dtype=np.int64))])
    return causal_tables(qo, kv_indptr_h, kv_indices_h, kv_last_page_len_h, page_size)


def _rows_view(cache, page_size: int):
    """[num_pages, P, ...] cache -> [num_pages * P, 1, ...] view of its token rows (pages must be
    laid out back to back: stride[0] == P * stride[1])."""
    st = list(cache.stride())
    if st[0] != page_size * st[1]:
        raise ValueError("causal attention needs each cache's pages back to back (stride[0] == P * stride[1])")
    return cache.as_strided((cache.shape[0] * page_size, 1, *cache.shape[2:]), (st[1], st[1], *st[2:]))


def paged_attention(q, k_cache, v_cache, qo_indptr_h, kv_indptr_h, kv_indices, kv_last_page_len_h, *,
                    sm_scale: Optional[float] = None, policy="balanced", param: int = 0,
                    split_page_start=None, o_dtype=None, num_pages: Optional[int] = None,
                    kv_indptr=None, kv_last_page_len=None, plan: Optional[Plan] = None,
                    status=None, stream=None, causal: bool = False, kv_indices_h=None, o_out=None,
                    lse_out=None, kv_scale: float = 1.0):
    """GQA attention over a paged cache.  Host page-table shape arrays (``*_h``) feed the planner;
    ``kv_indices`` (and optionally ``kv_indptr`` / ``kv_last_page_len``) are device tensors.
    K/V are bf16, or e4m3 codes (float8_e4m3fn) with the per-tensor ``kv_scale``.
    Returns (o, lse, extras) with extras = {"plan", "o_part", "lse_part"}.

    ``causal``: a request's query tokens are its last positions and each sees keys up to its own
    (needs the host page list ``kv_indices_h``); computed as a prefix pass, a diagonal pass over
    token rows and an exact merge (``causal_split_tables``)."""
    import torch
    dev = q.device
    hq, d = q.shape[1], q.shape[2]
    hk = k_cache.shape[2]
    if causal:
        if kv_indices_h is None:
            raise ValueError("causal attention needs the host page list kv_indices_h")
        P = k_cache.shape[1]
        qo = np.asarray(qo_indptr_h, dtype=np.int64)
        tab = causal_split_tables(np.diff(qo), kv_indptr_h, kv_indices_h, kv_last_page_len_h, P)
        rows = q.shape[0]
        pi, px, pl = tab["prefix"]
        di, dx, dl = tab["diag"]
        n_rows = (k_cache.shape[0] if num_pages is None else num_pages) * P
        prefix = lambda oo, ll: paged_attention(  # noqa: E731
            q, k_cache, v_cache, qo_indptr_h, pi, _dev_i32(px, dev), pl, sm_scale=sm_scale, policy=policy,
            param=param, o_dtype=o_dtype, num_pages=num_pages, status=status, stream=stream, o_out=oo, lse_out=ll)
        diag = lambda oo, ll: paged_attention(  # noqa: E731
            q, _rows_view(k_cache, P), _rows_view(v_cache, P), np.arange(rows + 1), di, _dev_i32(dx, dev), dl,
            sm_scale=sm_scale, policy="none", o_dtype=o_dtype, num_pages=n_rows, status=status, stream=stream,
            o_out=oo, lse_out=ll)
        if int(di[-1]) == 0 or int(pi[-1]) == 0:  # one pass sees nothing: the other is the answer
            o, lse, _ = (prefix if int(di[-1]) == 0 else diag)(None, None)
            return o, lse, {"plan": None, "tables": tab}
        o_st = torch.empty(2, rows, hq, d, dtype=torch.float32, device=dev)
        lse_st = torch.empty(2, rows, hq, dtype=torch.float32, device=dev)
        prefix(o_st[0], lse_st[0])
        diag(o_st[1], lse_st[1])
        o = torch.empty(rows, hq, d, dtype=o_dtype or torch.float32, device=dev)
        lse = torch.empty(rows, hq, dtype=torch.float32, device=dev)
        merge_states(o_st, lse_st, o, lse, stream=stream)
        return o, lse, {"plan": None, "o_states": o_st, "lse_states": lse_st, "tables": tab}
    if plan is None:
        plan = plan_paged(qo_indptr_h, kv_indptr_h, kv_last_page_len_h, k_cache.shape[1], hq, hk, d, policy,
                          param, split_page_start)
    if plan.device is None:
        plan.to(dev)
    kv_indptr = _dev_i32(kv_indptr_h, dev) if kv_indptr is None else kv_indptr
    kv_last_page_len = _dev_i32(kv_last_page_len_h, dev) if kv_last_page_len is None else kv_last_page_len
    o = torch.empty(q.shape[0], hq, d, dtype=o_dtype or torch.float32, device=dev) if o_out is None else o_out
    lse = torch.empty(q.shape[0], hq, dtype=torch.float32, device=dev) if lse_out is None else lse_out
    n_part = plan.info.num_partial_rows
    o_part = torch.empty(n_part, hq, d, dtype=torch.float32, device=dev) if n_part else None
    lse_part = torch.empty(n_part, hq, dtype=torch.float32, device=dev) if n_part else None
    paged_attn_fwd(q, k_cache, v_cache, kv_indptr, kv_indices, kv_last_page_len, plan, o, lse, o_part, lse_part,
                   status, sm_scale, num_pages, stream, kv_scale=kv_scale)
    return o, lse, {"plan": plan, "o_part": o_part, "lse_part": lse_part}


def pod_decode_sms(decode_kv_bytes: float, prefill_flops: float, num_sms: int = 148) -> int:
    """SMs a POD launch gives to its decode slices: the decode part's share of the two parts'
    standalone times (decode KV bytes at 6.0 TB/s, prefill FLOPs at 0.9 PFLOP/s -- what the two
    kernels reach alone on B200), kept within [16, num_sms - 16]."""
    t_dec, t_pre = float(decode_kv_bytes) / 6.0e12, float(prefill_flops) / 0.9e15
    share = t_dec / (t_dec + t_pre) if t_dec + t_pre > 0 else 0.5
    return int(min(num_sms - 16, max(16, round(num_sms * share))))


class PodAttention:
    """One batch mixing prefill and decode requests (POD: prefill on decode, FlashInfer PR #4736
    page, batch_pod.cu), planned once: requests with at most ``decode_q_max`` query tokens (default:
    what the all-KV-heads decode kernel holds, 8 // group) on the decode plan, whose KV slices are
    balanced over ``decode_sms`` persistent CTAs, and the rest on the 128-row prefill plan
    (``skv_plan_paged_subset`` twice).  ``fused``: both plans run in ONE attention launch
    (``skv_pod_attn_fwd``: the decode CTAs stream the KV cache while the prefill CTAs fill the
    other SMs); otherwise one launch per plan.  Each call runs on the batch's own q, page table and
    outputs; each plan keeps its own partial buffers."""

    def __init__(self, qo_indptr_h, kv_indptr_h, kv_last_page_len_h, page_size: int, num_qo_heads: int,
                 num_kv_heads: int, head_dim: int, device, *, decode_q_max: Optional[int] = None,
                 decode_sms: Optional[int] = None, num_sms: int = 148, policy="balanced", fused: bool = True):
        import torch
        qo = np.asarray(qo_indptr_h, dtype=np.int64)
        q_lens = np.diff(qo)
        g = num_qo_heads // num_kv_heads
        if decode_q_max is None:
            decode_q_max = max(1, 8 // max(1, g))
        dec, pre = np.flatnonzero(q_lens <= decode_q_max), np.flatnonzero(q_lens > decode_q_max)
        kv_ip = np.asarray(kv_indptr_h, dtype=np.int64)
        n_pages = np.diff(kv_ip)
        lengths = np.where(n_pages > 0, (n_pages - 1) * page_size + np.asarray(kv_last_page_len_h, np.int64), 0)
        if decode_sms is None:
            dec_bytes = float(lengths[dec].sum()) * num_kv_heads * head_dim * 4
            pre_flops = float(np.sum(q_lens[pre] * lengths[pre])) * num_qo_heads * 4 * head_dim
            decode_sms = pod_decode_sms(dec_bytes, pre_flops, num_sms) if len(pre) else num_sms
        self.decode_sms = int(decode_sms)
        args = (qo_indptr_h, kv_indptr_h, kv_last_page_len_h, page_size, num_qo_heads, num_kv_heads, head_dim)
        self.decode_plan = plan_paged_subset(*args, dec, policy, self.decode_sms).to(device)
        self.prefill_plan = plan_paged_subset(*args, pre, policy, max(1, num_sms - self.decode_sms) if len(dec)
                                              else num_sms).to(device)
        self.requests = (dec, pre)
        self.fused = bool(fused) and len(dec) > 0 and len(pre) > 0 and self.decode_plan.info.kernel == 3 \
            and self.prefill_plan.info.kernel == 4
        f32 = dict(dtype=torch.float32, device=device)

        def parts(plan):
            n = plan.info.num_partial_rows
            return (torch.empty(n, num_qo_heads, head_dim, **f32), torch.empty(n, num_qo_heads, **f32)) if n \
                else (None, None)
        self.decode_part, self.prefill_part = parts(self.decode_plan), parts(self.prefill_plan)

    @property
    def plans(self):
        return [p for p, r in ((self.decode_plan, self.requests[0]), (self.prefill_plan, self.requests[1])) if len(r)]

    def launches(self) -> int:
        """Kernel launches per call (attention, then each plan's merge pass if it has merge rows)."""
        merges = sum(1 for p in self.plans if p.info.num_merge_rows > 0)
        return (1 if self.fused else len(self.plans)) + merges

    def __call__(self, q, k_cache, v_cache, kv_indptr, kv_indices, kv_last_page_len, o, lse, *, sm_scale=None,
                 num_pages: Optional[int] = None, status=None, stream=None):
        if self.fused:
            pod_attn_fwd(q, k_cache, v_cache, kv_indptr, kv_indices, kv_last_page_len, self.decode_plan,
                         self.prefill_plan, o, lse, *self.decode_part, *self.prefill_part, status, sm_scale, num_pages,
                         stream)
            return o, lse
        for plan, (op, lp) in ((self.decode_plan, self.decode_part), (self.prefill_plan, self.prefill_part)):
            if plan.info.num_work > 0:
                paged_attn_fwd(q, k_cache, v_cache, kv_indptr, kv_indices, kv_last_page_len, plan, o, lse, op, lp,
                               status, sm_scale, num_pages, stream)
        return o, lse


def pod_attention(q, k_cache, v_cache, qo_indptr_h, kv_indptr_h, kv_indices, kv_last_page_len_h, *,
                  decode_q_max: Optional[int] = None, sm_scale: Optional[float] = None, policy="balanced",
                  decode_sms: Optional[int] = None, o_dtype=None, num_pages: Optional[int] = None, status=None,
                  stream=None, fused: bool = True):
    """A batch that mixes prefill and decode requests (``PodAttention``), planned and run once: by
    default in one attention launch, with ``fused=False`` one launch per plan.
    Returns (o, lse, {"plans": [...], "pod": the PodAttention})."""
    import torch
    dev = q.device
    hq, d = q.shape[1], q.shape[2]
    hk = k_cache.shape[2]
    pod = PodAttention(qo_indptr_h, kv_indptr_h, kv_last_page_len_h, k_cache.shape[1], hq, hk, d, dev,
                       decode_q_max=decode_q_max, decode_sms=decode_sms, policy=policy, fused=fused)
    kv_indptr = _dev_i32(kv_indptr_h, dev)
    kv_last = _dev_i32(kv_last_page_len_h, dev)
    o = torch.empty(q.shape[0], hq, d, dtype=o_dtype or torch.float32, device=dev)
    lse = torch.empty(q.shape[0], hq, dtype=torch.float32, device=dev)
    pod(q, k_cache, v_cache, kv_indptr, kv_indices, kv_last, o, lse, sm_scale=sm_scale, num_pages=num_pages,
        status=status, stream=stream)
    return o, lse, {"plans": pod.plans, "pod": pod}


def mla_decode(q_nope, q_pe, ckv, kpe, kv_indptr_h, kv_indices, kv_last_page_len_h, *,
               sm_scale: Optional[float] = None, kv_scale: float = 1.0, policy="balanced", param: int = 0,
               split_page_start=None, o_dtype=None, num_pages: Optional[int] = None, kv_indptr=None,
               kv_last_page_len=None, plan: Optional[Plan] = None, status=None, stream=None, o=None, lse=None,
               causal: bool = False, kv_indices_h=None):
    """MLA latent decode over a paged latent cache (bf16 or e4m3 codes).  Returns (o, lse, extras).

    ``causal`` (multi-token decode): the q_len decode positions are each request's last positions
    and each sees keys up to its own (needs ``kv_indices_h``); a prefix pass keeps the fold of
    q_len into rows, a diagonal pass over token rows adds the few keys only later positions see,
    and ``merge_states`` combines them exactly."""
    import torch
    dev = q_nope.device
    B, q_len, H = q_nope.shape[:3]
    if causal:
        if kv_indices_h is None:
            raise ValueError("causal attention needs the host page list kv_indices_h")
        P = ckv.shape[1]
        tab = causal_split_tables(np.full(B, q_len), kv_indptr_h, kv_indices_h, kv_last_page_len_h, P)
        pi, px, pl = tab["prefix"]
        di, dx, dl = tab["diag"]
        n_rows = (ckv.shape[0] if num_pages is None else num_pages) * P
        if o is None:
            o = torch.empty(B, q_len, H, 512, dtype=o_dtype or torch.float32, device=dev)
        if lse is None:
            lse = torch.empty(B, q_len, H, dtype=torch.float32, device=dev)
        prefix = lambda oo, ll: mla_decode(  # noqa: E731
            q_nope, q_pe, ckv, kpe, pi, _dev_i32(px, dev), pl, sm_scale=sm_scale, kv_scale=kv_scale, policy=policy,
            param=param, num_pages=num_pages, status=status, stream=stream, o=oo, lse=ll)
        diag = lambda oo, ll: mla_decode(  # noqa: E731
            q_nope.reshape(B * q_len, 1, H, 512), q_pe.reshape(B * q_len, 1, H, 64), _rows_view(ckv, P),
            _rows_view(kpe, P), di, _dev_i32(dx, dev), dl, sm_scale=sm_scale, kv_scale=kv_scale, policy="none",
            num_pages=n_rows, status=status, stream=stream, o=oo.view(B * q_len, 1, H, 512),
            lse=ll.view(B * q_len, 1, H))
        if int(di[-1]) == 0 or int(pi[-1]) == 0:  # one pass sees nothing: the other is the answer
            (prefix if int(di[-1]) == 0 else diag)(o, lse)
            return o, lse, {"plan": None, "tables": tab}
        o_st = torch.empty(2, B, q_len, H, 512, dtype=torch.float32, device=dev)
        lse_st = torch.empty(2, B, q_len, H, dtype=torch.float32, device=dev)
        prefix(o_st[0], lse_st[0])
        diag(o_st[1], lse_st[1])
        merge_states(o_st.view(2, B * q_len, H, 512), lse_st.view(2, B * q_len, H), o.view(B * q_len, H, 512),
                     lse.view(B * q_len, H), stream=stream)
        return o, lse, {"plan": None, "o_states": o_st, "lse_states": lse_st, "tables": tab}
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


class CausalMlaDecode:
    """Causal multi-token MLA decode planned once and launched many times (the per-call form of
    ``mla_decode(causal=True)`` without host planning): every decode step of a fixed batch runs
    the prefix pass (each request cut to the keys all its q_len positions see, q_len folded into
    rows), the diagonal pass (one page-size-1 request per query position over the few keys only
    later positions see) and the exact merge of the two states."""

    def __init__(self, q_len: int, num_heads: int, kv_indptr_h, kv_indices_h, kv_last_page_len_h,
                 page_size: int, num_pages: int, device, kv_dtype: str = "bf16", policy="balanced",
                 param: int = 0):
        import torch
        B = len(kv_indptr_h) - 1
        self.B, self.q_len, self.H, self.P, self.num_pages = B, q_len, num_heads, page_size, num_pages
        tab = causal_split_tables(np.full(B, q_len), kv_indptr_h, kv_indices_h, kv_last_page_len_h, page_size)
        pi, px, pl = tab["prefix"]
        di, dx, dl = tab["diag"]
        self.has_prefix, self.has_diag = int(pi[-1]) > 0, int(di[-1]) > 0
        self.prefix = (_dev_i32(pi, device), _dev_i32(px, device), _dev_i32(pl, device))
        self.diag = (_dev_i32(di, device), _dev_i32(dx, device), _dev_i32(dl, device))
        self.prefix_plan = plan_mla(q_len, pi, pl, page_size, num_heads, policy, param, None, kv_dtype).to(device)
        self.diag_plan = plan_mla(1, di, dl, 1, num_heads, "none", 0, None, kv_dtype).to(device)
        f32 = dict(dtype=torch.float32, device=device)
        self.o_st = torch.empty(2, B, q_len, num_heads, 512, **f32)
        self.lse_st = torch.empty(2, B, q_len, num_heads, **f32)
        n_pre, n_diag = self.prefix_plan.info.num_partial_rows, self.diag_plan.info.num_partial_rows
        self.pre_part = (torch.empty(n_pre, num_heads, 512, **f32), torch.empty(n_pre, num_heads, **f32)) \
            if n_pre else (None, None)
        self.diag_part = (torch.empty(n_diag, num_heads, 512, **f32), torch.empty(n_diag, num_heads, **f32)) \
            if n_diag else (None, None)

    def launches(self) -> int:
        """Kernel launches per call (attention passes, their plans' merge passes, the final merge)."""
        n = 0
        for on, plan in ((self.has_prefix, self.prefix_plan), (self.has_diag, self.diag_plan)):
            if on:
                n += 1 + (1 if plan.info.num_merge_rows > 0 else 0)
        return n + (1 if self.has_prefix and self.has_diag else 0)

    def __call__(self, q_nope, q_pe, ckv, kpe, o, lse, *, sm_scale=None, kv_scale: float = 1.0, status=None,
                 stream=None):
        B, q, H = self.B, self.q_len, self.H
        both = self.has_prefix and self.has_diag
        o_pre, l_pre = (self.o_st[0], self.lse_st[0]) if both else (o, lse)
        o_dg, l_dg = (self.o_st[1], self.lse_st[1]) if both else (o, lse)
        if self.has_prefix:
            ip, ix, la = self.prefix
            mla_decode_fwd(q_nope, q_pe, ckv, kpe, ip, ix, la, self.prefix_plan, o_pre, l_pre, *self.pre_part, status,
                           sm_scale, kv_scale, self.num_pages, stream)
        if self.has_diag:
            ip, ix, la = self.diag
            mla_decode_fwd(q_nope.reshape(B * q, 1, H, 512), q_pe.reshape(B * q, 1, H, 64), _rows_view(ckv, self.P),
                           _rows_view(kpe, self.P), ip, ix, la, self.diag_plan, o_dg.view(B * q, 1, H, 512),
                           l_dg.view(B * q, 1, H), *self.diag_part, status, sm_scale, kv_scale,
                           self.num_pages * self.P, stream)
        if both:
            merge_states(self.o_st.view(2, B * q, H, 512), self.lse_st.view(2, B * q, H), o.view(B * q, H, 512),
                         lse.view(B * q, H), stream=stream)
        return o, lse


class PagedDecodePipeline:
    """Serving-loop helper for repeated paged attention over a device-resident KV cache, with the
    step's inputs and outputs in host memory.

    ``submit`` takes one step's query (a pinned host bf16 tensor [rows, Hq, D]) and page table
    (host int arrays), plans it on the host (``skv_plan_paged`` written straight into a pinned
    buffer, followed there by the page table), copies query and [plan | page table] to the device
    on an input stream (two copies), runs the attention and merge passes on a compute stream
    (one ``skv_paged_attn_fwd`` call on launch arguments kept per buffer set) and copies O and LSE
    back into pinned host buffers on an output stream; it returns a ticket and does not wait.
    ``depth`` sets of host and device buffers alternate, so the host planning and the copies of
    the next steps overlap the kernels of the current one; ``result(ticket)`` waits for that
    step's output copy and returns views of its pinned O and LSE (valid until the same buffer set
    is reused, ``depth`` submits later).  Nothing is allocated per step once the buffers have
    grown to the largest step."""

    def __init__(self, k_cache, v_cache, num_qo_heads: int, *, max_rows: int, max_batch: int, max_page_ids: int,
                 sm_scale: Optional[float] = None, num_pages: Optional[int] = None, o_dtype=None, policy="balanced",
                 param: int = 0, depth: int = 2, plan_words: int = 1 << 14):
        import torch
        self.torch = torch
        self.k, self.v = k_cache, v_cache
        dev = k_cache.device
        self.dev = dev
        self.hq, self.hk, self.d, self.P = num_qo_heads, k_cache.shape[2], k_cache.shape[3], k_cache.shape[1]
        self.sm_scale, self.num_pages = sm_scale, num_pages
        self.policy = _POLICY[policy] if isinstance(policy, str) else int(policy)
        self.param = param
        self.o_dtype = o_dtype or torch.float32
        self.max_rows, self.max_batch, self.max_page_ids = max_rows, max_batch, max_page_ids
        self.s_in, self.s_run, self.s_out = (torch.cuda.Stream(dev) for _ in range(3))
        self.p_in, self.p_run, self.p_out = (int(s.cuda_stream) for s in (self.s_in, self.s_run, self.s_out))
        pin = dict(pin_memory=True)
        self.slots = []
        for _ in range(depth):
            slot = dict(
                o_h=torch.empty(max_rows, num_qo_heads, self.d, dtype=self.o_dtype, **pin),
                lse_h=torch.empty(max_rows, num_qo_heads, dtype=torch.float32, **pin),
                q=torch.empty(max_rows, num_qo_heads, self.d, dtype=torch.bfloat16, device=dev),
                o=torch.empty(max_rows, num_qo_heads, self.d, dtype=self.o_dtype, device=dev),
                lse=torch.empty(max_rows, num_qo_heads, dtype=torch.float32, device=dev),
                o_part=torch.empty(0, device=dev), lse_part=torch.empty(0, device=dev),
                ev_in=torch.cuda.Event(), ev_run=torch.cuda.Event(), ev_out=torch.cuda.Event(), rows=0, used=False)
            self._size_inputs(slot, plan_words)
            self.slots.append(slot)
        self.count = 0
        self.h2d_bytes = self.d2h_bytes = 0

    @staticmethod
    def _align(n: int) -> int:
        return (n + 15) & ~15  # 64-byte segments

    def _size_inputs(self, slot, plan_cap: int):
        """(Re)allocate the slot's pinned [plan | kv_indptr | kv_indices | last] buffer and its
        device twin for a plan of up to plan_cap words; launch arguments are rebuilt."""
        torch = self.torch
        n = (self._align(plan_cap) + self._align(self.max_batch + 1) + self._align(max(1, self.max_page_ids))
             + self._align(self.max_batch))
        slot["in_h"] = torch.empty(n, dtype=torch.int32, pin_memory=True)
        slot["in_np"] = slot["in_h"].numpy()
        slot["in_d"] = torch.empty(n, dtype=torch.int32, device=self.dev)
        slot["plan_cap"] = plan_cap
        slot["params"] = None

    def _params(self, slot):
        """Launch arguments of the slot's fixed device buffers (built once, pointers patched per step)."""
        if slot["params"] is None:
            in_d = slot["in_d"]
            slot["params"] = _paged_params(slot["q"], self.k, self.v, in_d[:2], in_d, in_d[:1], slot["o"], slot["lse"],
                                           slot["o_part"] if slot["o_part"].numel() else None,
                                           slot["lse_part"] if slot["lse_part"].numel() else None, None,
                                           self.sm_scale, self.num_pages)
        return slot["params"]

    def submit(self, q_h, qo_indptr_h, kv_indptr_h, kv_indices_h, kv_last_page_len_h) -> int:
        torch = self.torch
        slot = self.slots[self.count % len(self.slots)]
        if slot["used"]:
            slot["ev_out"].synchronize()  # the previous step of this buffer set has been read back
        qo, ki, la = (np.ascontiguousarray(np.asarray(x, dtype=np.int32)) for x in (qo_indptr_h, kv_indptr_h,
                                                                               kv_last_page_len_h))
        kx = np.ascontiguousarray(np.asarray(kv_indices_h, dtype=np.int32))
        rows = q_h.shape[0]
        if rows > self.max_rows or la.size > self.max_batch or kx.size > self.max_page_ids:
            raise ValueError("step larger than the pipeline's max_rows / max_batch / max_page_ids")
        b = len(ki) - 1
        info = PlanInfo()
        while True:  # plan straight into the front of the pinned input buffer
            buf = slot["in_np"]
            code = _plan_paged(b, _ptr_i32(qo), _ptr_i32(ki), _ptr_i32(la), self.P, self.hq, self.hk, self.d,
                               self.policy, self.param, None, None, _ptr_i32(buf), slot["plan_cap"], ctypes.byref(info))
            if code == OK:
                break
            if code != ERR_WORKSPACE:
                _check(code, "skv_plan_paged")
            self._size_inputs(slot, max(info.plan_words, 2 * slot["plan_cap"]))
        nw = max(1, info.plan_words)
        o_ki = self._align(nw)
        o_kx = o_ki + self._align(ki.size)
        o_la = o_kx + self._align(max(1, kx.size))
        end = o_la + la.size
        buf = slot["in_np"]
        buf[o_ki: o_ki + ki.size] = ki
        buf[o_kx: o_kx + kx.size] = kx
        buf[o_la: end] = la
        n_part = info.num_partial_rows
        if n_part > slot["o_part"].shape[0]:  # grows to the largest plan seen, then stays
            slot["o_part"] = torch.empty(n_part, self.hq, self.d, dtype=torch.float32, device=self.dev)
            slot["lse_part"] = torch.empty(n_part, self.hq, dtype=torch.float32, device=self.dev)
            slot["params"] = None
        p = self._params(slot)
        base = slot["in_d"].data_ptr()
        p.kv_indptr, p.kv_indices, p.kv_last_page_len = base + 4 * o_ki, base + 4 * o_kx, base + 4 * o_la
        p.batch, p.total_q = b, rows
        if slot["used"]:
            self.s_in.wait_event(slot["ev_run"])  # the slot's device buffers are free again
        with torch.cuda.stream(self.s_in):
            slot["q"][:rows].copy_(q_h, non_blocking=True)
            slot["in_d"][:end].copy_(slot["in_h"][:end], non_blocking=True)
        slot["ev_in"].record(self.s_in)
        self.s_run.wait_event(slot["ev_in"])
        _check(_paged_fwd(ctypes.byref(p), base, ctypes.byref(info), self.p_run), "skv_paged_attn_fwd")
        slot["ev_run"].record(self.s_run)
        self.s_out.wait_event(slot["ev_run"])
        with torch.cuda.stream(self.s_out):
            slot["o_h"][:rows].copy_(slot["o"][:rows], non_blocking=True)
            slot["lse_h"][:rows].copy_(slot["lse"][:rows], non_blocking=True)
        slot["ev_out"].record(self.s_out)
        slot["used"], slot["rows"] = True, rows
        self.h2d_bytes += q_h.numel() * q_h.element_size() + 4 * end
        self.d2h_bytes += rows * self.hq * (self.d * slot["o_h"].element_size() + 4)
        self.count += 1
        return self.count - 1

    def result(self, ticket: int):
        """Wait for step ``ticket``'s output copy; returns (O, LSE) views of its pinned host buffers."""
        if ticket < self.count - len(self.slots):
            raise ValueError("that step's buffers have been reused")
        slot = self.slots[ticket % len(self.slots)]
        slot["ev_out"].synchronize()
        return slot["o_h"][: slot["rows"]], slot["lse_h"][: slot["rows"]]

