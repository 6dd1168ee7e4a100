"""skv_paged_attn_fwd_static_scratch: the decode entry point for callers that cannot allocate
device memory (for example a serving engine that gives all free device memory to its KV cache at
start-up, or a C caller with no device allocator).  It keeps the split partials in the library's
own fixed device array instead of caller buffers.

Checked through the C ABI against skv_paged_attn_fwd (caller-provided partial buffers) and
against the float64 oracle on the same inputs, twice in a row, after the shared array was first
filled by a different plan with more partial rows (the array keeps the previous call's contents;
a partial row the kernel failed to write would then show the other plan's values), with the
tolerances of the other parity tests; and a plan too large for the array must be rejected before
anything runs.  This file is collected last so that a failure here comes after every other test
has run."""
import ctypes

import numpy as np
import pytest
import torch

import oracle.attention as OA
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


def _static(c, d, plan, o, lse, status):
    skv.paged_attn_fwd_static_scratch(d["q"], d["k"], d["v"], d["kv_indptr"], d["kv_indices"],
                                      d["kv_last_page_len"], plan, o, lse, status, c.sm_scale, c.num_pages)


@pytest.mark.parametrize("indep", [False, True])
def test_static_scratch_matches_regular_entry_point_and_oracle_twice(indep):
    # another batch and plan first, with more partial rows than the case under test: its values
    # stay in the shared array
    c0 = llama70b_decode_case(independent_v=not indep, batch=32, seed=7, len_range=(1024, 4096))
    d0 = paged_to_device(c0, DEV)
    plan0 = skv.plan_paged(c0.qo_indptr, c0.kv_indptr, c0.kv_last_page_len, c0.page_size, c0.num_qo_heads,
                           c0.num_kv_heads, c0.head_dim, "fixed", 8).to(DEV)   # 256 partial rows
    o0 = torch.empty(c0.q.shape[0], c0.num_qo_heads, c0.head_dim, device=DEV)
    lse0 = torch.empty(c0.q.shape[0], c0.num_qo_heads, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    _static(c0, d0, plan0, o0, lse0, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0

    c = llama70b_decode_case(independent_v=indep, batch=16)
    d = paged_to_device(c, DEV)
    plan = skv.plan_paged(c.qo_indptr, c.kv_indptr, c.kv_last_page_len, c.page_size, c.num_qo_heads,
                          c.num_kv_heads, c.head_dim, "balanced", 0).to(DEV)
    assert 0 < plan.info.num_partial_rows < plan0.info.num_partial_rows   # split partials, stale rows beyond
    o_ref, lse_ref = _reference(c, d, plan)
    O, LSE = OA.paged_attention(c.q, c.k, c.v, c.qo_indptr, c.kv_indptr, c.kv_indices, c.kv_last_page_len,
                                c.page_size, c.sm_scale)
    for call in range(2):
        o = torch.full_like(o_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        status.zero_()
        _static(c, d, plan, o, lse, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"call {call}: device status {int(status.item())}"
        err_o = float((o - o_ref).abs().max())
        err_l = float((lse - lse_ref).abs().max())
        assert err_o <= O_TOL and err_l <= LSE_TOL, (call, err_o, err_l)
        on, ln = o.cpu().numpy(), lse.cpu().numpy()
        err_o = float(np.max(np.abs(on - O)))
        err_l = float(np.max(np.abs(ln - LSE)))
        assert err_o <= O_TOL and err_l <= LSE_TOL, ("oracle", call, err_o, err_l)


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
