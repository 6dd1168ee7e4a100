"""GPU parity of mixed prefill + decode (POD) batches: ``pod_attention`` runs the decode requests
on the all-KV-heads decode kernel and the prefill requests on the 128-row prefill kernel, both on
the batch's own q, page table and outputs (``skv_plan_paged_subset``), against the oracle over the
whole batch.  Tolerances: O max-abs <= 1e-2, LSE <= 1e-3."""
import math

import numpy as np
import pytest
import torch

import oracle.attention as OA
import split_kv_merge_b200 as skv
from workloads import build_page_table, normal_bf16
from workloads.device import bf16_tensor, i32_tensor

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.mark.parametrize("o_dtype", [torch.float32, torch.bfloat16])
def test_pod_batch(o_dtype):
    rng = np.random.Generator(np.random.PCG64(81))
    lengths, q_lens, P, hq, hk, d = [3000, 170, 0, 640, 2000, 50, 1], [1, 40, 1, 1, 128, 0, 1], 16, 64, 8, 128
    kv_indptr, kv_indices, last, num_pages = build_page_table(rng, lengths, P, extra_pages=2)
    qo = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    q = normal_bf16(81, 1, (int(qo[-1]), hq, d))
    k = normal_bf16(81, 2, (num_pages, P, hk, d))
    v = normal_bf16(81, 3, (num_pages, P, hk, d))
    scale = 1 / math.sqrt(d)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse, ex = skv.pod_attention(bf16_tensor(q, DEV), bf16_tensor(k, DEV), bf16_tensor(v, DEV), qo, kv_indptr,
                                   i32_tensor(kv_indices, DEV), last, sm_scale=scale, o_dtype=o_dtype, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert [p.info.kernel for p in ex["plans"]] == [3, 4]
    O, LSE = OA.paged_attention(q, k, v, qo, kv_indptr, kv_indices, last, P, scale)
    o, lse = o.float().cpu().numpy(), lse.cpu().numpy()
    assert np.array_equal(np.isneginf(lse), np.isneginf(LSE))
    fin = np.isfinite(LSE)
    assert float(np.max(np.abs(o - O))) <= 1e-2
    assert float(np.max(np.abs(lse[fin] - LSE[fin]))) <= 1e-3
