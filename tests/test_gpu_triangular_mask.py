"""GPU parity of causal / multi-token attention (each query token sees keys up to its own
position) against the oracle's causal attention: GQA decode with several query tokens, GQA
causal prefill, and MLA multi-token decode, through ``runner.paged_attention`` /
``runner.mla_decode`` with ``causal=True`` (a prefix pass, a diagonal pass over token rows and
the exact merge).  Tolerances as for the unmasked paths: O max-abs <= 1e-2 (the e4m3 cache too,
inside its 3e-2 allowance), LSE <= 1e-3; rows that see no key must give O = 0, LSE = -inf."""
import math

import numpy as np
import pytest
import torch

import oracle.attention as OA
import split_kv_merge_b200 as skv
from workloads import build_page_table, mla_decode_case, normal_bf16
from workloads.device import bf16_tensor, i32_tensor, mla_to_device

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _cmp(o, lse, O, LSE, tol, where):
    o, lse = o.float().cpu().numpy(), lse.float().cpu().numpy()
    assert np.array_equal(np.isneginf(lse), np.isneginf(LSE)), where
    fin = np.isfinite(LSE)
    err_o = float(np.max(np.abs(o - O)))
    err_l = float(np.max(np.abs(lse[fin] - LSE[fin]))) if fin.any() else 0.0
    assert err_o <= tol, f"{where}: O max-abs {err_o}"
    assert err_l <= 1e-3, f"{where}: LSE max-abs {err_l}"


@pytest.mark.parametrize("shape", ["mtp_decode", "prefill", "one_token_each", "no_common_prefix"])
def test_causal_gqa(shape):
    rng = np.random.Generator(np.random.PCG64(61))
    if shape == "mtp_decode":      # Llama-70B-shaped heads, 1-4 query tokens per request
        hq, hk, d, P = 64, 8, 128, 16
        lengths, q_lens = [1, 700, 0, 3, 257, 512], [2, 4, 1, 4, 3, 1]
    elif shape == "one_token_each":  # no diagonal keys: the prefix pass alone
        hq, hk, d, P = 64, 8, 128, 16
        lengths, q_lens = [1, 700, 0, 257], [1, 1, 1, 1]
    elif shape == "no_common_prefix":  # every request shorter than its query block: the diagonal pass alone
        hq, hk, d, P = 64, 8, 128, 16
        lengths, q_lens = [1, 0, 2, 3], [2, 3, 3, 4]
    else:                          # shared-KV prefill heads, 128-token query blocks
        hq, hk, d, P = 32, 8, 128, 64
        lengths, q_lens = [300, 500, 128], [128, 128, 128]
    kv_indptr, kv_indices, last, num_pages = build_page_table(rng, lengths, P, extra_pages=2)
    qo = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    q = normal_bf16(61, 1, (int(qo[-1]), hq, d))
    k = normal_bf16(61, 2, (num_pages, P, hk, d))
    v = normal_bf16(61, 3, (num_pages, P, hk, d))
    scale = 1 / math.sqrt(d)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse, _ = skv.paged_attention(bf16_tensor(q, DEV), bf16_tensor(k, DEV), bf16_tensor(v, DEV), qo, kv_indptr,
                                    i32_tensor(kv_indices, DEV), last, sm_scale=scale, causal=True,
                                    kv_indices_h=kv_indices, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    O, LSE = OA.paged_attention(q, k, v, qo, kv_indptr, kv_indices, last, P, scale, causal=True)
    _cmp(o, lse, O, LSE, 1e-2, f"causal gqa {shape}")


@pytest.mark.parametrize("kv_dtype", ["bf16", "e4m3"])
@pytest.mark.parametrize("q_len", [2, 4])
def test_causal_mla_multi_token(q_len, kv_dtype):
    c = mla_decode_case(16, q_len, kv_dtype, batch=5, len_range=(1, 600), seed=12)
    c.kv_last_page_len = c.kv_last_page_len.copy()
    d = mla_to_device(c, DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse, _ = skv.mla_decode(d["q_nope"], d["q_pe"], d["ckv"], d["kpe"], c.kv_indptr, d["kv_indices"],
                               c.kv_last_page_len, sm_scale=c.sm_scale, kv_scale=c.kv_scale, causal=True,
                               kv_indices_h=c.kv_indices, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    O, LSE = OA.mla_decode(c.q_nope, c.q_pe, c.ckv, c.kpe, c.kv_indptr, c.kv_indices, c.kv_last_page_len,
                           c.page_size, c.sm_scale, c.kv_dtype, c.kv_scale, causal=True)
    _cmp(o, lse, O, LSE, 1e-2, f"causal mla q{q_len} {kv_dtype}")
