"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle on the same seeded
inputs.  Tolerances: O max-abs <= 1e-2, LSE abs <= 1e-3; page gather bit-exact; broadcast KV vs
replicated KV bit-exact; repeated runs bit-identical.  The e4m3 MLA cache is held to the same
1e-2 as bf16 (its tensor-core path splits the bf16 operand into two exact e4m3 terms, so only the
cache is fp8, and the oracle reads the same decoded cache), which is tighter than the 3e-2 the
fp8 case is allowed.  bf16 outputs: the fp32 value a kernel rounds is checked at 1e-2 and the
rounding to bf16 bit for bit (a bf16 number of magnitude 4 or more is up to 2^-6 from the real
value it stands for, so no kernel's bf16 output can be held to 1e-2 there).

Sizes: reduced workloads the oracle finishes in seconds (several tiles, ragged tails) checked
element by element, and the full workload sizes checked on seeded samples of requests
(shortest, longest and random ones; every head)."""
import math

import numpy as np
import pytest
import torch

import oracle.attention as OA
import split_kv_merge_b200 as skv
from workloads import (even_split_pages, llama70b_decode_case, mla_decode_case, route_case,
                       shared_kv_prefill_case, tiny_gqa_case)
from workloads.device import mla_to_device, paged_to_device, route_to_device

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL, O_TOL_FP8 = 1e-2, 1e-3, 3e-2
assert O_TOL <= O_TOL_FP8   # the e4m3 cases below are held to O_TOL, inside the fp8 allowance
DEV = "cuda:0"


def _np(t):
    return t.detach().float().cpu().numpy()


def _cmp(o_gpu, lse_gpu, o_ref, lse_ref, o_tol=O_TOL, where=""):
    o_ref = np.asarray(o_ref)
    lse_ref = np.asarray(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), np.isneginf(lse_ref)), where
    fin = np.isfinite(lse_ref)
    assert np.all(np.isfinite(o_gpu)), where
    err_o = float(np.max(np.abs(o_gpu - o_ref))) if o_ref.size else 0.0
    err_l = float(np.max(np.abs(lse_gpu[fin] - lse_ref[fin]))) if fin.any() else 0.0
    assert err_o <= o_tol, f"{where}: O max-abs {err_o}"
    assert err_l <= LSE_TOL, f"{where}: LSE max-abs {err_l}"
    return err_o, err_l


def _run_paged(c, policy="balanced", param=0, o_dtype=torch.float32, sps=None, status=None):
    d = paged_to_device(c, DEV)
    o, lse, ex = skv.paged_attention(d["q"], d["k"], d["v"], c.qo_indptr, c.kv_indptr, d["kv_indices"],
                                     c.kv_last_page_len, sm_scale=c.sm_scale, policy=policy, param=param,
                                     split_page_start=sps, o_dtype=o_dtype, num_pages=c.num_pages, status=status)
    torch.cuda.synchronize()
    return o, lse, ex, d


def _oracle_paged(c, requests=None):
    return OA.paged_attention(c.q, c.k, c.v, c.qo_indptr, c.kv_indptr, c.kv_indices, c.kv_last_page_len,
                              c.page_size, c.sm_scale, requests=requests)


# ----------------------------------------------------------------------------- tiny GQA decode
@pytest.mark.parametrize("o_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("variant", ["plain", "poison", "indep_v"])
def test_tiny_gqa_decode_with_partials(variant, o_dtype):
    c = tiny_gqa_case(poison=variant == "poison", independent_v=variant == "indep_v")
    o, lse, ex, _ = _run_paged(c, "fixed", 2, o_dtype)
    O, LSE = _oracle_paged(c)
    _cmp(_np(o), _np(lse), O, LSE, where="tiny O")
    # per-split partials: row part_base + i * S + j, here request r split j -> row 2r + j
    parts = OA.paged_attention_partials(c.q, c.k, c.v, c.qo_indptr, c.kv_indptr, c.kv_indices,
                                        c.kv_last_page_len, c.page_size, c.sm_scale, c.split_page_start)
    po, pl = _np(ex["o_part"]), _np(ex["lse_part"])
    for r in range(4):
        for j in range(2):
            _cmp(po[2 * r + j], pl[2 * r + j], parts[r][0][j, 0], parts[r][1][j, 0], where=f"part r{r} j{j}")


def test_tiny_matches_stored_fixture():
    import json
    import os
    c = tiny_gqa_case()
    o, lse, _, _ = _run_paged(c, "fixed", 2)
    with open(os.path.join(os.path.dirname(__file__), "golden", "tiny_gqa.json")) as f:
        g = json.load(f)
    lse_ref = np.array([[float.fromhex(x) for x in row] for row in g["lse"]])
    o0 = np.array([[float.fromhex(x) for x in row] for row in g["o_head0"]])
    assert np.max(np.abs(_np(lse) - lse_ref)) <= LSE_TOL
    assert np.max(np.abs(_np(o)[:, 0] - o0)) <= O_TOL


def test_random_explicit_splits_merge_to_unsplit():
    c = tiny_gqa_case()
    rng = np.random.Generator(np.random.PCG64(7))
    sps = []
    for r in range(4):
        n = int(c.kv_indptr[r + 1] - c.kv_indptr[r])
        cuts = np.sort(rng.integers(0, n + 1, size=int(rng.integers(0, 5))))
        sps.append([0, *cuts.tolist(), n])
    o, lse, _, _ = _run_paged(c, "explicit", 0, sps=sps)
    O, LSE = _oracle_paged(c)
    _cmp(_np(o), _np(lse), O, LSE, where="explicit splits")


# ----------------------------------------------------------------------------- gather hook
@pytest.mark.parametrize("indep", [False, True])
def test_page_gather_bit_exact(indep):
    c = llama70b_decode_case(independent_v=indep, batch=6, len_range=(1, 300))
    d = paged_to_device(c, DEV)
    L = c.kv_lengths()
    tok_indptr = np.concatenate([[0], np.cumsum(L)]).astype(np.int32)
    T = int(tok_indptr[-1])
    k_out = torch.empty(T, 8, 128, dtype=torch.bfloat16, device=DEV)
    v_out = torch.empty_like(k_out)
    skv.paged_kv_gather(d["k"], d["v"], d["kv_indptr"], d["kv_indices"], d["kv_last_page_len"],
                        torch.from_numpy(tok_indptr).to(DEV), T, k_out, v_out, num_pages=c.num_pages)
    torch.cuda.synchronize()
    kb = k_out.view(torch.int16).cpu().numpy().view(np.uint16)
    vb = v_out.view(torch.int16).cpu().numpy().view(np.uint16)
    for r in range(c.batch):
        pages, slots = OA.request_token_slots(c.kv_indptr, c.kv_indices, c.kv_last_page_len, 16, r)
        np.testing.assert_array_equal(kb[tok_indptr[r]:tok_indptr[r + 1]], c.k[pages, slots])
        np.testing.assert_array_equal(vb[tok_indptr[r]:tok_indptr[r + 1]], c.v[pages, slots])


# ----------------------------------------------------------------------------- Llama-70B decode
@pytest.mark.parametrize("indep", [False, True])
@pytest.mark.parametrize("policy", ["none", "balanced"])
def test_llama70b_decode_reduced(indep, policy):
    c = llama70b_decode_case(independent_v=indep, batch=8)
    o, lse, ex, _ = _run_paged(c, policy, 148)
    O, LSE = _oracle_paged(c)
    _cmp(_np(o), _np(lse), O, LSE, where=f"llama reduced {policy}")


@pytest.mark.parametrize("indep", [False, True])
def test_llama70b_decode_full_sampled(indep):
    c = llama70b_decode_case(independent_v=indep)
    o, lse, ex, _ = _run_paged(c, "balanced", 0)
    assert ex["plan"].info.max_splits >= 2
    L = c.kv_lengths()
    rng = np.random.Generator(np.random.PCG64(99))
    reqs = sorted({int(np.argmin(L)), int(np.argmax(L)), *rng.choice(c.batch, 4, replace=False).tolist()})
    O, LSE = _oracle_paged(c, requests=reqs)
    _cmp(_np(o)[reqs], _np(lse)[reqs], O[reqs], LSE[reqs], where="llama full sampled")


# ----------------------------------------------------------------------------- shared-KV prefill
def test_shared_kv_prefill_reduced_and_broadcast_bit_exact():
    kw = dict(n_batches=4, q_len=24, kv_len=1000)
    a = shared_kv_prefill_case(replicated=False, **kw)
    b = shared_kv_prefill_case(replicated=True, **kw)
    oa, la, _, _ = _run_paged(a, "none")
    ob, lb, _, _ = _run_paged(b, "none")
    assert torch.equal(oa, ob) and torch.equal(la, lb)
    O, LSE = _oracle_paged(a)
    _cmp(_np(oa), _np(la), O, LSE, where="shared-kv reduced")


def test_shared_kv_prefill_full_broadcast_bit_exact_and_sampled():
    a = shared_kv_prefill_case(replicated=False)
    oa, la, _, _ = _run_paged(a, "none")
    b = shared_kv_prefill_case(replicated=True)
    ob, lb, _, _ = _run_paged(b, "none")
    assert torch.equal(oa, ob) and torch.equal(la, lb)
    del ob, lb
    rng = np.random.Generator(np.random.PCG64(3))
    rows = rng.choice(a.q.shape[0], 6, replace=False)
    for row in rows:
        r = int(np.searchsorted(a.qo_indptr, row, side="right") - 1)
        qrow = slice(int(row), int(row) + 1)
        sub = dict(q=a.q[qrow], qo_indptr=np.array([0, 1], np.int32), kv_indptr=a.kv_indptr[r:r + 2] - a.kv_indptr[r],
                   kv_indices=a.kv_indices[a.kv_indptr[r]:a.kv_indptr[r + 1]], kv_last_page_len=a.kv_last_page_len[r:r + 1])
        O, LSE = OA.paged_attention(sub["q"], a.k, a.v, sub["qo_indptr"], sub["kv_indptr"], sub["kv_indices"],
                                    sub["kv_last_page_len"], a.page_size, a.sm_scale)
        _cmp(_np(oa)[row:row + 1], _np(la)[row:row + 1], O, LSE, where=f"shared-kv row {row}")


# ----------------------------------------------------------------------------- MLA decode
def _run_mla(c, policy="balanced", param=0, o_dtype=torch.float32):
    d = mla_to_device(c, DEV)
    o, lse, ex = skv.mla_decode(d["q_nope"], d["q_pe"], d["ckv"], d["kpe"], c.kv_indptr, d["kv_indices"],
                                c.kv_last_page_len, sm_scale=c.sm_scale, kv_scale=c.kv_scale, policy=policy,
                                param=param, o_dtype=o_dtype, num_pages=c.num_pages)
    torch.cuda.synchronize()
    return o, lse, ex


def _oracle_mla(c, requests=None):
    return OA.mla_decode(c.q_nope, c.q_pe, c.ckv, c.kpe, c.kv_indptr, c.kv_indices, c.kv_last_page_len,
                         c.page_size, c.sm_scale, c.kv_dtype, c.kv_scale, requests=requests)


@pytest.mark.parametrize("kv_dtype", ["bf16", "e4m3"])
@pytest.mark.parametrize("H,q_len", [(16, 1), (16, 4), (128, 1), (128, 4)])
def test_mla_reduced(H, q_len, kv_dtype):
    c = mla_decode_case(H, q_len, kv_dtype, batch=3, len_range=(100, 900), poison=True)
    o, lse, ex = _run_mla(c, "fixed", 3)
    info = ex["plan"].info
    rows = {12: 16, 13: 32, 14: 64}.get(info.kernel, 128)   # rows per tile of the kernel the planner chose
    assert info.q_tile == (skv.mla_fold_ratio(H, q_len, rows) if H <= rows else 1)
    O, LSE = _oracle_mla(c)
    _cmp(_np(o), _np(lse), O, LSE, O_TOL, where=f"mla {H} {q_len} {kv_dtype}")


@pytest.mark.parametrize("kv_dtype", ["bf16", "e4m3"])
@pytest.mark.parametrize("H,q_len", [(16, 1), (16, 4), (128, 1), (128, 4)])
def test_mla_full_sampled(H, q_len, kv_dtype):
    c = mla_decode_case(H, q_len, kv_dtype)
    o, lse, ex = _run_mla(c, "balanced", 0)
    L = c.kv_lengths()
    reqs = sorted({int(np.argmin(L)), int(np.argmax(L)), 5})
    O, LSE = _oracle_mla(c, requests=reqs)
    _cmp(_np(o)[reqs], _np(lse)[reqs], O[reqs], LSE[reqs], O_TOL, where=f"mla full {H} {q_len} {kv_dtype}")


def _empty_request(c, j):
    """Remove request j's pages from the page table (an empty KV: O = 0, LSE = -inf)."""
    a, b = int(c.kv_indptr[j]), int(c.kv_indptr[j + 1])
    c.kv_indices = np.concatenate([c.kv_indices[:a], c.kv_indices[b:]]).astype(np.int32)
    c.kv_indptr = c.kv_indptr.copy()
    c.kv_indptr[j + 1:] -= b - a
    return c


@pytest.mark.parametrize("kv_dtype", ["bf16", "e4m3"])
@pytest.mark.parametrize("page_size", [16, 128])
@pytest.mark.parametrize("policy,param", [("none", 0), ("balanced", 148)])
def test_mla_tensor_core_page_sizes_and_edges(kv_dtype, page_size, policy, param):
    """Both MLA tensor-core kernels at other page sizes (several pages per 64-token tile, several
    tiles per page): ragged lengths around tile and page boundaries, an empty request, poisoned
    unused pages and tails (NaN rope, huge V), split or whole KV."""
    c = mla_decode_case(16, 1, kv_dtype, batch=5, len_range=(1, 700), page_size=page_size, poison=True, seed=9)
    c = _empty_request(c, 2)
    o, lse, ex = _run_mla(c, policy, param)
    assert ex["plan"].info.kernel == 12
    O, LSE = _oracle_mla(c)
    _cmp(_np(o), _np(lse), O, LSE, O_TOL, where=f"mla edges {kv_dtype} P{page_size} {policy}")


@pytest.mark.parametrize("H,q_len", [(64, 3), (128, 2), (32, 4)])
@pytest.mark.parametrize("page_size", [16, 128])
@pytest.mark.parametrize("policy,param", [("none", 0), ("balanced", 148), ("fixed", 2)])
def test_mla_64_row_groups(H, q_len, page_size, policy, param):
    """The 64-row kernel with CTA groups: every (query tile, head group) of a KV slice on its own
    co-resident CTA (groups of 3, 4 and 2 CTAs here), ragged lengths around tile and page
    boundaries, an empty request, poisoned unused pages and tails, split or whole KV."""
    c = mla_decode_case(H, q_len, "bf16", batch=5, len_range=(1, 900), page_size=page_size, poison=True, seed=13)
    c = _empty_request(c, 1)
    o, lse, ex = _run_mla(c, policy, param)
    info = ex["plan"].info
    assert info.kernel == 14 and info.q_tile == (skv.mla_fold_ratio(H, q_len, 64) if H <= 64 else 1)
    O, LSE = _oracle_mla(c)
    _cmp(_np(o), _np(lse), O, LSE, O_TOL, where=f"mla 64-row H{H} q{q_len} P{page_size} {policy}")


@pytest.mark.parametrize("H,q_len", [(16, 1), (16, 2), (128, 1)])
def test_mla_page_size_one_gather(H, q_len):
    """Page size 1 (a page id is a token row) on the bf16 tensor-core kernel, rows fetched with
    tile::gather4: permuted rows, lengths not a multiple of the 64-token tile, an empty request,
    explicit uneven splits."""
    c = mla_decode_case(H, q_len, "bf16", batch=4, len_range=(1, 300), page_size=1, poison=True, seed=11)
    c = _empty_request(c, 1)
    n = np.diff(c.kv_indptr)
    sps = [[0] + ([int(n[r]) // 3] if n[r] > 3 else []) + [int(n[r])] for r in range(c.batch)]
    o, lse, ex = _run_mla(c, "none", 0)
    assert ex["plan"].info.kernel in (12, 13)
    O, LSE = _oracle_mla(c)
    _cmp(_np(o), _np(lse), O, LSE, where=f"mla P1 H{H} q{q_len}")
    d = mla_to_device(c, DEV)
    o2, lse2, ex2 = skv.mla_decode(d["q_nope"], d["q_pe"], d["ckv"], d["kpe"], c.kv_indptr, d["kv_indices"],
                                   c.kv_last_page_len, sm_scale=c.sm_scale, kv_scale=c.kv_scale, policy="explicit",
                                   split_page_start=sps, num_pages=c.num_pages)
    torch.cuda.synchronize()
    _cmp(_np(o2), _np(lse2), O, LSE, where=f"mla P1 H{H} q{q_len} explicit splits")


# ----------------------------------------------------------------------------- route + merge
def _route(c):
    d = route_to_device(c, DEV)
    rm = skv.RouteMerge(c.sel, c.num_heads, DEV)
    o, lse = rm(d["q_nope"], d["q_pe"], d["ckv"], d["kpe"], d["sel_cqk"], sm_scale=c.sm_scale)
    torch.cuda.synchronize()
    return o, lse, rm


def test_route_merge_reduced():
    c = route_case(num_queries=12, num_chunks=8, chunk_tokens=512, per_chunk=100)
    o, lse, rm = _route(c)
    u = c.union_mla()
    O, LSE = OA.mla_decode(u.q_nope, u.q_pe, u.ckv, u.kpe, u.kv_indptr, u.kv_indices, u.kv_last_page_len, 1,
                           u.sm_scale)
    _cmp(_np(o), _np(lse), O[:, 0], LSE[:, 0], where="route reduced")
    # each chunk holder's partial equals the oracle's partial over that chunk's selection
    for ch in (0, 7):
        m = c.as_mla(ch)
        Oc, Lc = OA.mla_decode(m.q_nope, m.q_pe, m.ckv, m.kpe, m.kv_indptr, m.kv_indices, m.kv_last_page_len, 1,
                               m.sm_scale)
        _cmp(_np(rm.o_states[ch]), _np(rm.lse_states[ch]), Oc, Lc, where=f"route chunk {ch}")


def test_route_merge_full_sampled():
    c = route_case()
    o, lse, _ = _route(c)
    u = c.union_mla()
    qs = [0, 77, 255]
    O, LSE = OA.mla_decode(u.q_nope, u.q_pe, u.ckv, u.kpe, u.kv_indptr, u.kv_indices, u.kv_last_page_len, 1,
                           u.sm_scale, requests=qs)
    _cmp(_np(o)[qs], _np(lse)[qs], O[qs, 0], LSE[qs, 0], where="route full sampled")


# ----------------------------------------------------------------------------- merge_states
def test_merge_states_direct_layouts():
    rng = np.random.Generator(np.random.PCG64(17))
    rows, H, D = 37, 16, 512
    counts = rng.integers(0, 6, size=rows)
    indptr = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    n = int(indptr[-1])
    o_st = rng.standard_normal((n, H, D)).astype(np.float32)
    lse_st = (rng.standard_normal((n, H)) * 3).astype(np.float32)
    lse_st[rng.random((n, H)) < 0.2] = -np.inf
    o_out = torch.empty(rows, H, D, device=DEV)
    lse_out = torch.empty(rows, H, device=DEV)
    skv.merge_states(torch.from_numpy(o_st).to(DEV), torch.from_numpy(lse_st).to(DEV), o_out, lse_out,
                     state_indptr=torch.from_numpy(indptr).to(DEV))
    torch.cuda.synchronize()
    for r in range(rows):
        a, b = indptr[r], indptr[r + 1]
        if b == a:
            ro, rl = np.zeros((H, D)), np.full(H, -np.inf)
        else:
            ro, rl = OA.merge_states(o_st[a:b], lse_st[a:b])
        _cmp(_np(o_out[r]), _np(lse_out[r]), ro, rl, o_tol=1e-5, where=f"merge row {r}")
    # state-major uniform layout
    S = 5
    o2 = rng.standard_normal((S, rows, H, D)).astype(np.float32)
    l2 = (rng.standard_normal((S, rows, H)) * 3).astype(np.float32)
    skv.merge_states(torch.from_numpy(o2).to(DEV), torch.from_numpy(l2).to(DEV), o_out, lse_out)
    torch.cuda.synchronize()
    ro, rl = OA.merge_states(o2, l2)
    _cmp(_np(o_out), _np(lse_out), ro, rl, o_tol=1e-5, where="merge uniform")


# ----------------------------------------------------------------------------- edge cases
def test_edge_empty_requests_and_full_last_page():
    from workloads.gen import _make_paged
    c = _make_paged("edge", 9, [0, 16, 17, 1, 32], 1, 8, 2, 128, 16, False, extra_pages=2,
                    qo_lens=[1, 2, 0, 1, 3])
    for policy, param in [("none", 0), ("fixed", 3), ("balanced", 148)]:
        o, lse, _, _ = _run_paged(c, policy, param)
        O, LSE = _oracle_paged(c)
        _cmp(_np(o), _np(lse), O, LSE, where=f"edge {policy}")


def test_page_size_one():
    from workloads.gen import _make_paged
    c = _make_paged("p1", 10, [5, 33, 64], 1, 16, 2, 64, 1, True)
    o, lse, _, _ = _run_paged(c, "fixed", 2)
    O, LSE = _oracle_paged(c)
    _cmp(_np(o), _np(lse), O, LSE, where="page size 1")


def test_out_of_range_page_id_sets_status():
    c = tiny_gqa_case()
    c.kv_indices = c.kv_indices.copy()
    c.kv_indices[5] = c.num_pages + 3
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    _run_paged(c, "none", status=status)
    assert int(status.item()) == skv.DEV_PAGE_OOB


def test_deterministic_bitwise():
    c = llama70b_decode_case(batch=8)
    o1, l1, _, _ = _run_paged(c, "balanced", 148)
    o2, l2, _, _ = _run_paged(c, "balanced", 148)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# ----------------------------------------------------------------------------- kernel coverage
@pytest.mark.parametrize("page_size", [16, 64])
@pytest.mark.parametrize("policy,param", [("none", 0), ("fixed", 3), ("balanced", 148)])
def test_all_heads_decode_edges(page_size, policy, param):
    """The all-KV-heads decode kernel (8 KV heads, 8 query rows each): empty requests, a request
    with no query rows, lengths around page and tile boundaries, poisoned unused pages/tails."""
    from workloads.gen import _make_paged
    c = _make_paged("wide_edge", 21, [0, 16, 17, 1, 32, 300, 1000], 1, 64, 8, 128, page_size, True,
                    extra_pages=3, poison=True, qo_lens=[1, 1, 0, 1, 1, 1, 1])
    o, lse, ex, _ = _run_paged(c, policy, param)
    assert ex["plan"].info.kernel == 3
    O, LSE = _oracle_paged(c)
    _cmp(_np(o), _np(lse), O, LSE, where=f"wide edge P{page_size} {policy}")


def test_all_heads_decode_two_query_tokens():
    """g = 4 with two query tokens per request also fills the 8 columns per KV head."""
    from workloads.gen import _make_paged
    c = _make_paged("wide_q2", 22, [700, 33, 2048], 2, 32, 8, 128, 16, False)
    o, lse, ex, _ = _run_paged(c, "fixed", 2)
    assert ex["plan"].info.kernel == 3 and ex["plan"].info.q_tile == 2
    O, LSE = _oracle_paged(c)
    _cmp(_np(o), _np(lse), O, LSE, where="wide q2")


def test_per_head_tensor_core_decode():
    """Shapes the all-heads kernel does not take (4 KV heads, 4 query rows each) run on the
    per-KV-head tensor-core kernel."""
    from workloads.gen import _make_paged
    c = _make_paged("perhead", 23, [500, 64, 1500, 0], 1, 16, 4, 128, 32, True, poison=True)
    o, lse, ex, _ = _run_paged(c, "fixed", 2)
    assert ex["plan"].info.kernel == 2
    O, LSE = _oracle_paged(c)
    _cmp(_np(o), _np(lse), O, LSE, where="per-head tc")


@pytest.mark.parametrize("policy,param", [("none", 0), ("fixed", 3)])
def test_all_heads_decode_rising_scores(policy, param):
    """Scores that keep growing along the sequence (K scaled up with the token position, and one
    dominant key near the end) make the running maximum rise many times, exercising the rescale
    of l and of O in tensor memory."""
    from workloads.gen import _make_paged, bf16_bits_to_f32, f32_to_bf16_bits
    import oracle.attention as OA_
    c = _make_paged("rising", 24, [40, 333, 1200, 2047], 1, 64, 8, 128, 16, False)
    k = bf16_bits_to_f32(c.k_store).copy()
    for r in range(c.batch):
        pages, slots = OA_.request_token_slots(c.kv_indptr, c.kv_indices, c.kv_last_page_len, 16, r)
        L = len(pages)
        ramp = (1.0 + 6.0 * np.arange(L) / max(1, L)).astype(np.float32)
        k[pages, slots] *= ramp[:, None, None]
        if L > 8:  # a dominant key near the end, aligned with query head 0 of each KV head
            q0 = bf16_bits_to_f32(c.q[c.qo_indptr[r]]).reshape(8, 8, 128)[:, 0, :]
            k[pages[L - 5], slots[L - 5]] = 30.0 * q0 / np.linalg.norm(q0, axis=1, keepdims=True)
    c.k_store = f32_to_bf16_bits(k).reshape(c.k_store.shape)
    c.k = c.k_store
    o, lse, ex, _ = _run_paged(c, policy, param)
    assert ex["plan"].info.kernel == 3
    O, LSE = _oracle_paged(c)
    _cmp(_np(o), _np(lse), O, LSE, where=f"rising {policy}")


PREFILL_SHAPES = {
    # name: (hq, hk, page_size, kv lengths, query lengths, independent V)
    "g4_p64": (32, 8, 64, [0, 1, 63, 64, 65, 1000, 3000], [5, 0, 40, 33, 1, 128, 70], False),
    "g1_p128": (4, 4, 128, [129, 1, 700, 384], [130, 17, 1, 64], True),
    "g1_p256": (2, 2, 256, [1000, 255, 256, 3], [20, 200, 9, 33], False),
    "g8_p16": (64, 8, 16, [17, 300, 2049], [3, 16, 40], True),
    "g16_p32": (32, 2, 32, [500, 31, 1025], [8, 2, 9], False),
}


@pytest.mark.parametrize("shape", sorted(PREFILL_SHAPES))
@pytest.mark.parametrize("policy,param", [("none", 0), ("fixed", 3), ("balanced", 148)])
def test_prefill_tensor_core(shape, policy, param):
    """Shapes with more query rows per KV head than a decode tile holds run on the 128-row
    prefill kernel: group sizes 1 to 16, page sizes 16 to 256 (several pages per 128-key tile and
    several tiles per page), empty requests and requests with no query rows, ragged key tails,
    poisoned unused slots, independent V strides, whole and split KV."""
    from workloads.gen import _make_paged
    hq, hk, P, lens, qlens, indep = PREFILL_SHAPES[shape]
    c = _make_paged("prefill_" + shape, 31, lens, 1, hq, hk, 128, P, indep, extra_pages=2, poison=True,
                    qo_lens=qlens)
    o, lse, ex, _ = _run_paged(c, policy, param)
    assert ex["plan"].info.kernel == 4 and ex["plan"].info.q_tile == 128 // (hq // hk)
    O, LSE = _oracle_paged(c)
    _cmp(_np(o), _np(lse), O, LSE, where=f"prefill {shape} {policy}")


def test_prefill_tensor_core_rising_scores_fp32_and_bf16_out():
    """fp32 and bf16 output, with keys scaled up along the sequence so the running maximum of every row keeps
    rising (the rescale of l and of the row of O in tensor memory)."""
    from workloads.gen import _make_paged, bf16_bits_to_f32, f32_to_bf16_bits
    c = _make_paged("prefill_rising", 32, [3000, 700, 129], 1, 32, 8, 128, 64, False, qo_lens=[50, 9, 128])
    k = bf16_bits_to_f32(c.k_store).copy()
    for r in range(c.batch):
        pages, slots = OA.request_token_slots(c.kv_indptr, c.kv_indices, c.kv_last_page_len, 64, r)
        L = len(pages)
        k[pages, slots] *= (1.0 + 9.0 * np.arange(L) / max(1, L)).astype(np.float32)[:, None, None]
    c.k_store = f32_to_bf16_bits(k).reshape(c.k_store.shape)
    c.k = c.k_store
    O, LSE = _oracle_paged(c)
    o, lse, ex, _ = _run_paged(c, "fixed", 2)
    assert ex["plan"].info.kernel == 4
    _cmp(_np(o), _np(lse), O, LSE, where="prefill rising")
    # bf16 output (rows here are close to single V rows, so |O| reaches 4 and more): the fp32
    # value checked above, rounded once to bf16 (nearest even), bit for bit
    ob, lb, _, _ = _run_paged(c, "fixed", 2, o_dtype=torch.bfloat16)
    assert float(np.abs(O).max()) >= 4.0        # the case really has values bf16 cannot hold to 1e-2
    assert torch.equal(ob.cpu(), o.cpu().to(torch.bfloat16)), "bf16 output is not the rounded fp32 output"
    assert float(np.max(np.abs(_np(lb) - LSE))) <= LSE_TOL


# ----------------------------------------------------------------------------- failure detection
def test_bounded_wait_reports_timeout_and_context_stays_usable():
    """A wait on a barrier nothing arrives on gives up after its limit and reports SKV_DEV_TIMEOUT;
    the context keeps working afterwards (no trap, no hang)."""
    import time
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    t0 = time.perf_counter()
    skv.test_wait_timeout(status, 50_000_000)   # 50 ms
    torch.cuda.synchronize()
    assert int(status.item()) == skv.DEV_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    c = tiny_gqa_case()
    o, lse, _, _ = _run_paged(c, "fixed", 2)
    O, LSE = _oracle_paged(c)
    _cmp(_np(o), _np(lse), O, LSE, where="after timeout")
