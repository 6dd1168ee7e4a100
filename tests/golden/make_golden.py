"""Writes tests/golden/tiny_gqa.json from the float64 oracle only.

The pages print no worked numerical example, so this fixture is not from them: it records
what the oracle gives on the tiny paged GQA decode workload (4 requests, 8 query / 2 KV heads,
D=64, P=16, KV lengths {37,128,200,256}, 2 KV splits per request: the "ceil first" split of
the tiny configuration) so that a change in the oracle's arithmetic shows up as a diff.
Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle.attention as OA  # noqa: E402
from workloads import tiny_gqa_case  # noqa: E402


def build():
    c = tiny_gqa_case()
    O, LSE = OA.paged_attention(c.q, c.k, c.v, c.qo_indptr, c.kv_indptr, c.kv_indices,
                                c.kv_last_page_len, c.page_size, c.sm_scale)
    parts = OA.paged_attention_partials(c.q, c.k, c.v, c.qo_indptr, c.kv_indptr, c.kv_indices,
                                        c.kv_last_page_len, c.page_size, c.sm_scale, c.split_page_start)
    return {
        "workload": "tiny paged GQA decode, seed 1",
        "split_page_start": c.split_page_start,
        "lse": [[float.hex(float(x)) for x in row] for row in LSE],
        "o_head0": [[float.hex(float(x)) for x in O[r, 0]] for r in range(4)],
        "o_head7": [[float.hex(float(x)) for x in O[r, 7]] for r in range(4)],
        "lse_partials": [[[float.hex(float(x)) for x in parts[r][1][j, 0]] for j in range(2)] for r in range(4)],
    }


if __name__ == "__main__":
    with open(os.path.join(HERE, "tiny_gqa.json"), "w") as f:
        json.dump(build(), f, indent=1)
