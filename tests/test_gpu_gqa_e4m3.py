"""GPU parity of GQA decode over an fp8 e4m3 K/V cache (one per-tensor scale for K and V) on the
all-KV-heads tensor-core kernel, against the float64 oracle reading the same decoded codes.

The kernel multiplies the raw e4m3 cache tiles on the tensor cores and splits the other operand
of each product (queries, softmax weights) into two exact e4m3 terms, so only the cache is fp8:
outputs are held to the bf16 paths' bar, O max-abs <= 1e-2 and LSE <= 1e-3 (inside the fp8
case's 3e-2).  Cases: every GQA group size the kernel takes (8, 4, 2, 1 query heads per KV head
with 1, 2, 4, 8 query tokens), page sizes 16 / 64 / 256, ragged lengths around tile and page
boundaries, empty requests and a request without query rows, poisoned unused pages (NaN codes)
and tails (NaN K, the largest code in V), equal and independent K/V strides, split and unsplit
plans, rising scores (forced maximum raises), and the Llama-3.1-70B-shaped batch sampled."""
import numpy as np
import pytest
import torch

import oracle.attention as OA
import split_kv_merge_b200 as skv
from workloads import llama70b_decode_case
from workloads.device import paged_to_device
from workloads.gen import _make_paged, e4m3_encode

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL = 1e-2, 1e-3
DEV = "cuda:0"


def _np(t):
    return t.detach().float().cpu().numpy()


def _cmp(o, lse, O, LSE, where):
    assert np.array_equal(np.isneginf(lse), np.isneginf(LSE)), where
    fin = np.isfinite(LSE)
    assert np.all(np.isfinite(o)), where
    err_o = float(np.max(np.abs(o - O))) if O.size else 0.0
    err_l = float(np.max(np.abs(lse[fin] - LSE[fin]))) if fin.any() else 0.0
    assert err_o <= O_TOL, f"{where}: O max-abs {err_o}"
    assert err_l <= LSE_TOL, f"{where}: LSE max-abs {err_l}"
    return err_o, err_l


def _run(c, policy="balanced", param=0, o_dtype=torch.float32):
    d = paged_to_device(c, DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse, ex = skv.paged_attention(d["q"], d["k"], d["v"], c.qo_indptr, c.kv_indptr, d["kv_indices"],
                                     c.kv_last_page_len, sm_scale=c.sm_scale, policy=policy, param=param,
                                     o_dtype=o_dtype, num_pages=c.num_pages, status=status, kv_scale=c.kv_scale)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, skv.status_str(int(status.item()))
    assert ex["plan"].info.kernel == 3
    return o, lse, ex


def _oracle(c, requests=None):
    return OA.paged_attention(c.q, c.k, c.v, c.qo_indptr, c.kv_indptr, c.kv_indices, c.kv_last_page_len,
                              c.page_size, c.sm_scale, requests=requests, kv_dtype="e4m3", kv_scale=c.kv_scale)


@pytest.mark.parametrize("hq,q_len", [(64, 1), (32, 2), (16, 4), (8, 8)])
@pytest.mark.parametrize("policy,param", [("none", 0), ("fixed", 3), ("balanced", 148)])
def test_e4m3_group_sizes_and_splits(hq, q_len, policy, param):
    c = _make_paged(f"e4m3_g{hq // 8}", 41 + hq, [0, 16, 17, 1, 300, 1000, 2049], q_len, hq, 8, 128, 16, True,
                    extra_pages=3, poison=True, qo_lens=[q_len, q_len, 0, q_len, q_len, q_len, q_len], kv_dtype="e4m3")
    o, lse, ex = _run(c, policy, param)
    assert ex["plan"].info.q_tile == q_len
    O, LSE = _oracle(c)
    _cmp(_np(o), _np(lse), O, LSE, f"e4m3 hq{hq} q{q_len} {policy}")


@pytest.mark.parametrize("page_size", [64, 256])
@pytest.mark.parametrize("indep", [False, True])
def test_e4m3_page_sizes_and_strides(page_size, indep):
    c = _make_paged("e4m3_pages", 52, [1, 63, 64, 65, 511, 1500], 1, 64, 8, 128, page_size, indep,
                    extra_pages=2, poison=True, kv_dtype="e4m3")
    o, lse, _ = _run(c, "fixed", 2)
    O, LSE = _oracle(c)
    _cmp(_np(o), _np(lse), O, LSE, f"e4m3 P{page_size} indep={indep}")


def test_e4m3_bf16_output_is_rounded_fp32_output():
    c = _make_paged("e4m3_bf16out", 53, [900, 77, 3000], 1, 64, 8, 128, 16, False, kv_dtype="e4m3")
    o, lse, _ = _run(c, "fixed", 2)
    ob, lb, _ = _run(c, "fixed", 2, torch.bfloat16)
    O, LSE = _oracle(c)
    _cmp(_np(o), _np(lse), O, LSE, "e4m3 fp32 out")
    assert torch.equal(ob.cpu(), o.cpu().to(torch.bfloat16))
    assert float(np.max(np.abs(_np(lb) - LSE))) <= LSE_TOL


def test_e4m3_rising_scores():
    """Keys scaled up along each sequence (re-encoded with the scale of the scaled cache) so the
    running maximum of every row keeps rising: the lazy raise and the O rescale in TMEM."""
    c = _make_paged("e4m3_rising", 54, [3000, 700, 129], 1, 64, 8, 128, 16, False, kv_dtype="e4m3")
    k = OA.e4m3_to_f64(c.k) * c.kv_scale
    v = OA.e4m3_to_f64(c.v) * c.kv_scale
    for r in range(c.batch):
        pages, slots = OA.request_token_slots(c.kv_indptr, c.kv_indices, c.kv_last_page_len, 16, r)
        L = len(pages)
        k[pages, slots] *= (1.0 + 9.0 * np.arange(L) / max(1, L))[:, None, None]
    scale = float(np.float32(max(np.abs(k).max(), np.abs(v).max()) / 448.0))
    c.k_store = e4m3_encode(k / scale)
    c.v_store = e4m3_encode(v / scale)
    c.k, c.v, c.kv_scale = c.k_store, c.v_store, scale
    o, lse, _ = _run(c, "fixed", 2)
    O, LSE = _oracle(c)
    _cmp(_np(o), _np(lse), O, LSE, "e4m3 rising")


@pytest.mark.parametrize("indep", [False, True])
def test_e4m3_llama70b_full_sampled(indep):
    c = llama70b_decode_case(independent_v=indep, kv_dtype="e4m3")
    o, lse, _ = _run(c, "balanced", 0)
    L = c.kv_lengths()
    reqs = sorted({int(np.argmin(L)), int(np.argmax(L)), 7, 40})
    O, LSE = _oracle(c, requests=reqs)
    _cmp(_np(o)[reqs], _np(lse)[reqs], O[reqs], LSE[reqs], f"e4m3 llama70b indep={indep}")


def test_e4m3_other_kernels_rejected():
    """Shapes the all-KV-heads kernel does not take are refused for an e4m3 cache (no silent
    fallback): 4 KV heads here."""
    c = _make_paged("e4m3_4kv", 55, [100, 200], 1, 16, 4, 128, 16, False, kv_dtype="e4m3")
    d = paged_to_device(c, DEV)
    with pytest.raises(skv.SkvError) as err:
        skv.paged_attention(d["q"], d["k"], d["v"], c.qo_indptr, c.kv_indptr, d["kv_indices"], c.kv_last_page_len,
                            sm_scale=c.sm_scale, num_pages=c.num_pages, kv_scale=c.kv_scale)
    assert err.value.code == skv.ERR_UNSUPPORTED
