"""GPU parity of ``PagedDecodePipeline`` (the serving-loop helper: host planning into pinned buffers,
input / compute / output streams, two alternating buffer sets): successive steps with different
queries and page tables -- a step's host work and copies overlapping the previous step's kernels
-- give, step by step, the oracle's attention (O max-abs <= 1e-2, LSE <= 1e-3), also when the
pinned plan buffers start too small and grow, and oversized steps are refused."""
import numpy as np
import pytest
import torch

import oracle.attention as OA
import split_kv_merge_b200 as skv
from workloads import llama70b_decode_case
from workloads.device import bf16_tensor

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.mark.parametrize("plan_words", [1 << 14, 16])  # 16: the plan buffers grow on the first steps
def test_pipeline_steps_match_oracle(plan_words):
    cases = [llama70b_decode_case(batch=b, seed=s, len_range=(200, 3000)) for b, s in ((6, 91), (9, 92), (6, 93), (3, 94))]
    # one cache holds every step's pages: steps use disjoint page ranges of a shared buffer
    offs = np.cumsum([0] + [c.num_pages for c in cases])
    k = torch.empty(int(offs[-1]), 16, 8, 128, dtype=torch.bfloat16, device=DEV)
    v = torch.empty_like(k)
    for c, o in zip(cases, offs):
        k[o:o + c.num_pages] = bf16_tensor(c.k, DEV)
        v[o:o + c.num_pages] = bf16_tensor(c.v, DEV)
    pipe = skv.PagedDecodePipeline(k, v, 64, max_rows=9, max_batch=9, max_page_ids=max(len(c.kv_indices) for c in cases),
                                   sm_scale=cases[0].sm_scale, num_pages=int(offs[-1]), plan_words=plan_words)
    qs = [torch.from_numpy(np.ascontiguousarray(c.q).view(np.int16)).view(torch.bfloat16).pin_memory() for c in cases]
    tickets = []
    results = {}
    for i, (c, o) in enumerate(zip(cases, offs)):
        tickets.append(pipe.submit(qs[i], c.qo_indptr, c.kv_indptr, c.kv_indices + o, c.kv_last_page_len))
        if i >= 1:  # read the previous step while this one runs
            oo, ll = pipe.result(tickets[i - 1])
            results[i - 1] = (oo.clone(), ll.clone())
    oo, ll = pipe.result(tickets[-1])
    results[len(cases) - 1] = (oo.clone(), ll.clone())
    for i, c in enumerate(cases):
        O, LSE = OA.paged_attention(c.q, c.k, c.v, c.qo_indptr, c.kv_indptr, c.kv_indices, c.kv_last_page_len,
                                    c.page_size, c.sm_scale)
        o_g, l_g = results[i][0].float().numpy(), results[i][1].numpy()
        assert float(np.max(np.abs(o_g - O))) <= 1e-2, i
        assert float(np.max(np.abs(l_g - LSE))) <= 1e-3, i
    with pytest.raises(ValueError):
        big = llama70b_decode_case(batch=12, seed=95, len_range=(16, 64))
        pipe.submit(torch.zeros(12, 64, 128, dtype=torch.bfloat16).pin_memory(), big.qo_indptr, big.kv_indptr,
                    big.kv_indices, big.kv_last_page_len)
