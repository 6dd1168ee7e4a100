"""Host logic of the composed calls (no GPU).  Mixed prefill + decode (POD) batches: ``runner.pod_attention`` plans the
decode requests and the prefill requests of one batch separately (``skv_plan_paged_subset``) and
launches both plans on the batch's own buffers.  With the launch replaced by a float64 stand-in
that computes exactly the requests of the plan it is given (and writes only their rows), the two
launches must together give the oracle's attention for the whole batch, each plan on the kernel
that suits its requests."""
import math

import numpy as np
import torch

import oracle.attention as OA
import split_kv_merge_b200 as skv
import split_kv_merge_b200.runner as R
from workloads import build_page_table, normal_bf16


def _bits(t):
    return t.view(torch.int16).numpy().view(np.uint16)


def _tb(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def test_pod_batch_composition(monkeypatch):
    launches = []
    real_subset = R.plan_paged_subset

    def plan_paged_subset(qo, *a, **k):
        plan = real_subset(qo, *a, **k)
        plan.qo = np.asarray(qo, dtype=np.int32)
        return plan

    def paged_attn_fwd(q, k_cache, v_cache, kv_indptr, kv_indices, kv_last_page_len, plan, o, lse, o_part, lse_part,
                       status, sm_scale, num_pages, stream, kv_scale=1.0):
        w = plan.words[: 8 * plan.info.num_work].reshape(-1, 8)
        reqs = sorted(set(w[:, 0].tolist()))
        launches.append((plan.info.kernel, reqs))
        O, LSE = OA.paged_attention(_bits(q), _bits(k_cache), _bits(v_cache), plan.qo, kv_indptr.numpy(),
                                    kv_indices.numpy(), kv_last_page_len.numpy(), k_cache.shape[1], sm_scale,
                                    requests=reqs)
        for r in reqs:
            a, b = int(plan.qo[r]), int(plan.qo[r + 1])
            o[a:b] = torch.from_numpy(O[a:b])
            lse[a:b] = torch.from_numpy(LSE[a:b])

    monkeypatch.setattr(R, "plan_paged_subset", plan_paged_subset)
    monkeypatch.setattr(R, "paged_attn_fwd", paged_attn_fwd)
    rng = np.random.Generator(np.random.PCG64(71))
    lengths, q_lens, P, hq, hk, d = [300, 17, 0, 64, 200, 5], [1, 40, 1, 1, 128, 0], 16, 64, 8, 128
    kv_indptr, kv_indices, last, num_pages = build_page_table(rng, lengths, P, extra_pages=2)
    qo = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    q = normal_bf16(71, 1, (int(qo[-1]), hq, d))
    k = normal_bf16(71, 2, (num_pages, P, hk, d))
    v = normal_bf16(71, 3, (num_pages, P, hk, d))
    scale = 1 / math.sqrt(d)
    o, lse, ex = R.pod_attention(_tb(q), _tb(k), _tb(v), qo, kv_indptr, torch.from_numpy(kv_indices), last,
                                 sm_scale=scale, policy="none", fused=False)
    # decode requests (one query token) on the all-KV-heads decode kernel, the rest on the prefill kernel
    assert launches == [(3, [0, 2, 3]), (4, [1, 4])]
    O, LSE = OA.paged_attention(q, k, v, qo, kv_indptr, kv_indices, last, P, scale)
    np.testing.assert_allclose(o.numpy(), O, rtol=0, atol=1e-6)
    np.testing.assert_array_equal(np.isneginf(lse.numpy()), np.isneginf(LSE))
    fin = np.isfinite(LSE)
    np.testing.assert_allclose(lse.numpy()[fin], LSE[fin], rtol=0, atol=1e-6)


def test_pod_fused_composition(monkeypatch):
    """The one-launch form: ``PodAttention`` hands both plans (decode subset on the all-KV-heads
    kernel with its CTAs = the SMs given to decode, prefill subset on the 128-row kernel) and their
    own partial buffers to ONE ``skv_pod_attn_fwd`` call; a stand-in computing exactly the requests
    of each plan gives the oracle's attention for the whole batch."""
    calls = []
    real_subset = R.plan_paged_subset

    def plan_paged_subset(qo, *a, **k):
        plan = real_subset(qo, *a, **k)
        plan.qo = np.asarray(qo, dtype=np.int32)
        return plan

    def pod_attn_fwd(q, k_cache, v_cache, kv_indptr, kv_indices, kv_last_page_len, dplan, pplan, o, lse, dop, dlp,
                     pop, plp, status, sm_scale, num_pages, stream):
        calls.append((dplan.info.kernel, dplan.info.num_ctas, pplan.info.kernel))
        for plan in (dplan, pplan):
            w = plan.words[: 8 * plan.info.num_work].reshape(-1, 8)
            reqs = sorted(set(w[:, 0].tolist()))
            O, LSE = OA.paged_attention(_bits(q), _bits(k_cache), _bits(v_cache), plan.qo, kv_indptr.numpy(),
                                        kv_indices.numpy(), kv_last_page_len.numpy(), k_cache.shape[1], sm_scale,
                                        requests=reqs)
            for r in reqs:
                a, b = int(plan.qo[r]), int(plan.qo[r + 1])
                o[a:b] = torch.from_numpy(O[a:b])
                lse[a:b] = torch.from_numpy(LSE[a:b])

    monkeypatch.setattr(R, "plan_paged_subset", plan_paged_subset)
    monkeypatch.setattr(R, "pod_attn_fwd", pod_attn_fwd)
    rng = np.random.Generator(np.random.PCG64(72))
    lengths, q_lens, P, hq, hk, d = [300, 170, 0, 640, 200, 5, 64], [1, 40, 1, 1, 128, 0, 1], 16, 64, 8, 128
    kv_indptr, kv_indices, last, num_pages = build_page_table(rng, lengths, P, extra_pages=2)
    qo = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    q = normal_bf16(72, 1, (int(qo[-1]), hq, d))
    k = normal_bf16(72, 2, (num_pages, P, hk, d))
    v = normal_bf16(72, 3, (num_pages, P, hk, d))
    scale = 1 / math.sqrt(d)
    o, lse, ex = R.pod_attention(_tb(q), _tb(k), _tb(v), qo, kv_indptr, torch.from_numpy(kv_indices), last,
                                 sm_scale=scale, decode_sms=40)
    # one launch; the decode slices on at most the 40 CTAs given (the planner leaves CTAs idle
    # rather than hand out slices smaller than a work item's fixed cost)
    assert len(calls) == 1 and calls[0][0] == 3 and 1 <= calls[0][1] <= 40 and calls[0][2] == 4
    assert ex["pod"].fused and ex["pod"].launches() >= 1
    O, LSE = OA.paged_attention(q, k, v, qo, kv_indptr, kv_indices, last, P, scale)
    np.testing.assert_allclose(o.numpy(), O, rtol=0, atol=1e-6)
    fin = np.isfinite(LSE)
    np.testing.assert_array_equal(np.isneginf(lse.numpy()), np.isneginf(LSE))
    np.testing.assert_allclose(lse.numpy()[fin], LSE[fin], rtol=0, atol=1e-6)


def test_pod_decode_sms_share():
    """The SMs given to decode follow the decode part's share of the two standalone times and stay
    within [16, SMs - 16]."""
    assert R.pod_decode_sms(6.0e12 * 100e-6, 0.9e15 * 100e-6) == 74        # equal times: half the SMs
    assert R.pod_decode_sms(6.0e12 * 300e-6, 0.9e15 * 100e-6) == 111
    assert R.pod_decode_sms(1.0, 1.0e15) == 16 and R.pod_decode_sms(1.0e13, 1.0) == 132


def test_subset_planner_rejects_bad_lists():
    qo, ip, la = np.array([0, 1, 2]), np.array([0, 1, 2]), np.array([3, 3])
    for bad in ([0, 0], [2], [-1]):
        try:
            skv.plan_paged_subset(qo, ip, la, 16, 8, 2, 64, bad, "none")
        except skv.SkvError as e:
            assert e.code == skv.ERR_INVALID
        else:
            raise AssertionError(f"accepted {bad}")
    plan = skv.plan_paged_subset(qo, ip, la, 16, 8, 2, 64, [], "none")
    assert plan.info.num_work == 0


def test_route_merge_composition(monkeypatch):
    """``RouteMerge``: one partial launch per KV chunk over each query's selected rows (page size 1,
    a page id is a token row), then the merge over chunks -- with the launches replaced by oracle
    stand-ins the result equals unsplit attention over the union of the selections."""
    from workloads import route_case

    def mla_decode_fwd(q_nope, q_pe, ckv, kpe, kv_indptr, kv_indices, kv_last_page_len, plan, o, lse, o_part,
                       lse_part, status, sm_scale, kv_scale, num_pages, stream):
        O, LSE = OA.mla_decode(_bits(q_nope), _bits(q_pe), _bits(ckv), _bits(kpe), kv_indptr.numpy(),
                               kv_indices.reshape(-1).numpy(), kv_last_page_len.numpy(), ckv.shape[1], sm_scale)
        o.copy_(torch.from_numpy(O))
        lse.copy_(torch.from_numpy(LSE))

    def merge_states(o_states, lse_states, o_out, lse_out=None, state_indptr=None, num_states=0, stream=None):
        O, LSE = OA.merge_states(o_states.double().numpy(), lse_states.double().numpy())
        o_out.copy_(torch.from_numpy(O))
        lse_out.copy_(torch.from_numpy(LSE))

    monkeypatch.setattr(R, "mla_decode_fwd", mla_decode_fwd)
    monkeypatch.setattr(R, "merge_states", merge_states)
    c = route_case(num_queries=5, num_chunks=3, chunk_tokens=64, per_chunk=10)
    cache = _tb(c.cache).view(c.cache.shape[0], 1, 576)
    rm = R.RouteMerge(c.sel, c.num_heads, "cpu")
    sel_cqk = torch.from_numpy(np.ascontiguousarray(c.sel.transpose(1, 0, 2)).astype(np.int32))
    o, lse = rm(_tb(c.q_nope), _tb(c.q_pe), cache[..., :512], cache[..., 512:], sel_cqk, sm_scale=c.sm_scale)
    u = c.union_mla()
    O, LSE = OA.mla_decode(u.q_nope, u.q_pe, u.ckv, u.kpe, u.kv_indptr, u.kv_indices, u.kv_last_page_len, 1,
                           u.sm_scale)
    np.testing.assert_allclose(o.numpy(), O[:, 0], rtol=0, atol=1e-6)
    np.testing.assert_allclose(lse.numpy(), LSE[:, 0], rtol=0, atol=1e-6)
