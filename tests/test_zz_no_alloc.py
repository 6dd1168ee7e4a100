"""skv_paged_attn_fwd_static_scratch: the decode entry point for callers that cannot allocate
device memory (for example a serving engine that gives all free device memory to its KV cache at
start-up, or a C caller with no device allocator).  It keeps the split partials in the library's
own fixed device array instead of caller buffers.

Checked through the C ABI against skv_paged_attn_fwd (caller-provided partial buffers) on the
same inputs, twice in a row (the shared array keeps the previous call's contents, which must not
matter), with the tolerances of the other parity tests; and a plan too large for the array must
be rejected before anything runs.  This file is collected last so that a failure here comes after
every other test has run."""
import ctypes

import numpy as np
import pytest
import torch

import split_kv_merge_b200 as skv
from workloads import llama70b_decode_case
from workloads.device import paged_to_device

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL = 1e-2, 1e-3
DEV = "cuda:0"


def _reference(c, d, plan):
    o, lse, ex = skv.paged_attention(d["q"], d["k"], d["v"], c.qo_indptr, c.kv_indptr, d["kv_indices"],
                                     c.kv_last_page_len, sm_scale=c.sm_scale, num_pages=c.num_pages, plan=plan)
    return o, lse


@pytest.mark.parametrize("indep", [False, True])
def test_static_scratch_matches_regular_entry_point_twice(indep):
    c = llama70b_decode_case(independent_v=indep, batch=16)
    d = paged_to_device(c, DEV)
    plan = skv.plan_paged(c.qo_indptr, c.kv_indptr, c.kv_last_page_len, c.page_size, c.num_qo_heads,
                          c.num_kv_heads, c.head_dim, "balanced", 0).to(DEV)
    assert plan.info.num_partial_rows > 0          # the path really goes through split partials
    o_ref, lse_ref = _reference(c, d, plan)
    for call in range(2):
        o = torch.full_like(o_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        skv.paged_attn_fwd_static_scratch(d["q"], d["k"], d["v"], d["kv_indptr"], d["kv_indices"],
                                          d["kv_last_page_len"], plan, o, lse, status, c.sm_scale, c.num_pages)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"call {call}: device status {int(status.item())}"
        err_o = float((o - o_ref).abs().max())
        err_l = float((lse - lse_ref).abs().max())
        assert err_o <= O_TOL and err_l <= LSE_TOL, (call, err_o, err_l)


def test_static_scratch_rejects_oversized_plan():
    c = llama70b_decode_case(batch=4, len_range=(100, 200))
    d = paged_to_device(c, DEV)
    plan = skv.plan_paged(c.qo_indptr, c.kv_indptr, c.kv_last_page_len, c.page_size, c.num_qo_heads,
                          c.num_kv_heads, c.head_dim, "fixed", 2).to(DEV)
    big = skv.PlanInfo.from_buffer_copy(plan.info)
    big.num_partial_rows = 1 << 16                 # 64 heads x 129 floats x 65536 rows >> 32 MiB
    o = torch.empty(c.q.shape[0], c.num_qo_heads, c.head_dim, device=DEV)
    p = skv._paged_params(d["q"], d["k"], d["v"], d["kv_indptr"], d["kv_indices"], d["kv_last_page_len"], o, None,
                          None, None, None, c.sm_scale, c.num_pages)
    code = skv._paged_static(ctypes.byref(p), plan.device.data_ptr(), ctypes.byref(big),
                             torch.cuda.current_stream().cuda_stream)
    assert code == skv.ERR_WORKSPACE
