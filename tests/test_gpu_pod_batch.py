"""GPU parity of mixed prefill + decode (POD) batches.  ``pod_attention`` plans the decode requests
on the all-KV-heads decode kernel and the prefill requests on the 128-row prefill kernel
(``skv_plan_paged_subset``) and runs both in ONE attention launch (``skv_pod_attn_fwd``: the first
CTAs stream the decode slices, the rest take prefill units), on the batch's own q, page table and
outputs.  Checked against the oracle over the whole batch (O max-abs <= 1e-2, LSE <= 1e-3), and
bit for bit against the same two plans run as two separate launches (each CTA runs the same body
either way), for several SM shares given to decode, both output types, batches with only one
kind of request, and the Llama-shaped POD workload (sampled)."""
import math

import numpy as np
import pytest
import torch

import oracle.attention as OA
import split_kv_merge_b200 as skv
from workloads import build_page_table, normal_bf16, pod_case
from workloads.device import bf16_tensor, i32_tensor, paged_to_device

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _batch(seed, lengths, q_lens, P=16, hq=64, hk=8, d=128):
    rng = np.random.Generator(np.random.PCG64(seed))
    kv_indptr, kv_indices, last, num_pages = build_page_table(rng, lengths, P, extra_pages=2)
    qo = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    q = normal_bf16(seed, 1, (int(qo[-1]), hq, d))
    k = normal_bf16(seed, 2, (num_pages, P, hk, d))
    v = normal_bf16(seed, 3, (num_pages, P, hk, d))
    return dict(q=q, k=k, v=v, qo=qo, kv_indptr=kv_indptr, kv_indices=kv_indices, last=last, P=P,
                scale=1 / math.sqrt(d))


def _run(b, **kw):
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse, ex = skv.pod_attention(bf16_tensor(b["q"], DEV), bf16_tensor(b["k"], DEV), bf16_tensor(b["v"], DEV),
                                   b["qo"], b["kv_indptr"], i32_tensor(b["kv_indices"], DEV), b["last"],
                                   sm_scale=b["scale"], status=status, **kw)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, skv.status_str(int(status.item()))
    return o, lse, ex


def _check(b, o, lse, rows=None):
    O, LSE = OA.paged_attention(b["q"], b["k"], b["v"], b["qo"], b["kv_indptr"], b["kv_indices"], b["last"], b["P"],
                                b["scale"])
    o, lse = o.float().cpu().numpy(), lse.cpu().numpy()
    assert np.array_equal(np.isneginf(lse), np.isneginf(LSE))
    fin = np.isfinite(LSE)
    assert float(np.max(np.abs(o - O))) <= 1e-2
    assert float(np.max(np.abs(lse[fin] - LSE[fin]))) <= 1e-3


MIXED = ([3000, 170, 0, 640, 2000, 50, 1, 900], [1, 40, 1, 1, 128, 0, 1, 300])


@pytest.mark.parametrize("o_dtype", [torch.float32, torch.bfloat16])
def test_pod_batch_one_launch(o_dtype):
    b = _batch(81, *MIXED)
    o, lse, ex = _run(b, o_dtype=o_dtype)
    assert [p.info.kernel for p in ex["plans"]] == [3, 4]
    assert ex["pod"].fused
    _check(b, o, lse)


@pytest.mark.parametrize("decode_sms", [16, 74, 132])
def test_pod_one_launch_equals_two_launches(decode_sms):
    b = _batch(82, *MIXED)
    o1, l1, ex1 = _run(b, decode_sms=decode_sms)
    o2, l2, ex2 = _run(b, decode_sms=decode_sms, fused=False)
    assert ex1["pod"].fused and not ex2["pod"].fused
    assert 1 <= ex1["plans"][0].info.num_ctas <= decode_sms
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    _check(b, o1, l1)


@pytest.mark.parametrize("kind", ["decode_only", "prefill_only"])
def test_pod_one_kind_only(kind):
    lengths, q_lens = ([500, 1200, 33], [1, 1, 1]) if kind == "decode_only" else ([500, 1200, 33], [64, 200, 17])
    b = _batch(83, lengths, q_lens)
    o, lse, ex = _run(b)
    assert not ex["pod"].fused and len(ex["plans"]) == 1
    _check(b, o, lse)


def test_pod_llama70b_workload_sampled():
    c = pod_case()
    d = paged_to_device(c, DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse, ex = skv.pod_attention(d["q"], d["k"], d["v"], c.qo_indptr, c.kv_indptr, d["kv_indices"],
                                   c.kv_last_page_len, sm_scale=c.sm_scale, status=status, num_pages=c.num_pages)
    torch.cuda.synchronize()
    assert int(status.item()) == 0 and ex["pod"].fused
    reqs = [0, 17, c.batch - 2, c.batch - 1]        # decode requests and both prefill requests
    O, LSE = OA.paged_attention(c.q, c.k, c.v, c.qo_indptr, c.kv_indptr, c.kv_indices, c.kv_last_page_len,
                                c.page_size, c.sm_scale, requests=reqs)
    rows = np.concatenate([np.arange(c.qo_indptr[r], c.qo_indptr[r + 1]) for r in reqs])
    on, ln = o.cpu().numpy()[rows], lse.cpu().numpy()[rows]
    assert float(np.max(np.abs(on - O[rows]))) <= 1e-2
    assert float(np.max(np.abs(ln - LSE[rows]))) <= 1e-3
