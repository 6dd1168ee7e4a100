"""Host logic of causal attention (no GPU): the prefix / diagonal tables of
``causal_split_tables`` and the composition in ``runner.paged_attention`` / ``runner.mla_decode``
(two unmasked passes, token-row views of the caches, an exact merge) are run with the three
launches replaced by float64 stand-ins built on the oracle, on CPU tensors, and must reproduce
the oracle's causal attention.  What this leaves to the GPU tests is the kernels themselves."""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle.attention as OA
import split_kv_merge_b200 as skv
import split_kv_merge_b200.runner as R
from workloads import build_page_table, normal_bf16


def _bits(t):
    """bf16 torch tensor (any strides) -> numpy uint16 view with the same strides."""
    return t.view(torch.int16).numpy().view(np.uint16)


class _Fakes:
    """Stand-ins for the three launches, computing with the oracle on the tensors they are given."""

    def __init__(self, monkeypatch):
        real_plan = R.plan_paged

        def plan_paged(qo_indptr, *a, **k):
            plan = real_plan(qo_indptr, *a, **k)
            plan.qo = np.asarray(qo_indptr, dtype=np.int32)
            return plan

        def paged_attn_fwd(q, k_cache, v_cache, kv_indptr, kv_indices, kv_last_page_len, plan, o, lse, o_part,
                           lse_part, status, sm_scale, num_pages, stream, kv_scale=1.0):
            O, LSE = OA.paged_attention(_bits(q), _bits(k_cache), _bits(v_cache), plan.qo, kv_indptr.numpy(),
                                        kv_indices.numpy(), kv_last_page_len.numpy(), k_cache.shape[1], sm_scale)
            o.copy_(torch.from_numpy(O))
            lse.copy_(torch.from_numpy(LSE))

        def mla_decode_fwd(q_nope, q_pe, ckv, kpe, kv_indptr, kv_indices, kv_last_page_len, plan, o, lse, o_part,
                           lse_part, status, sm_scale, kv_scale, num_pages, stream):
            O, LSE = OA.mla_decode(_bits(q_nope), _bits(q_pe), _bits(ckv), _bits(kpe), kv_indptr.numpy(),
                                   kv_indices.numpy(), kv_last_page_len.numpy(), ckv.shape[1], sm_scale)
            o.copy_(torch.from_numpy(O))
            lse.copy_(torch.from_numpy(LSE))

        def merge_states(o_states, lse_states, o_out, lse_out=None, state_indptr=None, num_states=0, stream=None):
            assert state_indptr is None
            O, LSE = OA.merge_states(o_states.double().numpy(), lse_states.double().numpy())
            o_out.copy_(torch.from_numpy(O))
            lse_out.copy_(torch.from_numpy(LSE))

        monkeypatch.setattr(R, "plan_paged", plan_paged)
        monkeypatch.setattr(R, "paged_attn_fwd", paged_attn_fwd)
        monkeypatch.setattr(R, "mla_decode_fwd", mla_decode_fwd)
        monkeypatch.setattr(R, "merge_states", merge_states)


def _tb(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


@pytest.mark.parametrize("indep_v", [False, True])
def test_causal_gqa_composition(monkeypatch, indep_v):
    _Fakes(monkeypatch)
    rng = np.random.Generator(np.random.PCG64(51))
    lengths, q_lens, P, hq, hk, d = [13, 0, 3, 40, 9, 64], [3, 2, 5, 4, 1, 7], 4, 8, 2, 64
    kv_indptr, kv_indices, last, num_pages = build_page_table(rng, lengths, P, extra_pages=2)
    qo = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    q = normal_bf16(51, 1, (int(qo[-1]), hq, d))
    k = normal_bf16(51, 2, (num_pages, P, hk, d))
    v_store = normal_bf16(51, 3, (num_pages, P, hk, 2 * d if indep_v else d))
    v = v_store[..., :d]
    tv = _tb(v_store)[..., :d] if indep_v else _tb(v_store)
    o, lse, ex = R.paged_attention(_tb(q), _tb(k), tv, qo, kv_indptr, torch.from_numpy(kv_indices), last,
                                   sm_scale=1 / math.sqrt(d), policy="none", causal=True, kv_indices_h=kv_indices)
    O, LSE = OA.paged_attention(q, k, v, qo, kv_indptr, kv_indices, last, P, 1 / math.sqrt(d), causal=True)
    np.testing.assert_allclose(o.numpy(), O, rtol=0, atol=1e-6)
    np.testing.assert_array_equal(np.isneginf(lse.numpy()), np.isneginf(LSE))
    fin = np.isfinite(LSE)
    np.testing.assert_allclose(lse.numpy()[fin], LSE[fin], rtol=0, atol=1e-6)
    assert np.isneginf(LSE).any() and fin.any()
    # the diagonal pass has one pseudo-request per query token with i keys (fewer near the start)
    di = ex["tables"]["diag"][0]
    assert len(di) == int(qo[-1]) + 1


@pytest.mark.parametrize("case", ["one_token_each", "all_prefix_empty"])
def test_causal_single_pass_cases(monkeypatch, case):
    """With one query token per request there are no diagonal keys, and with every request shorter
    than its query block there is no common prefix: one pass gives the answer, no merge."""
    _Fakes(monkeypatch)
    rng = np.random.Generator(np.random.PCG64(54))
    if case == "one_token_each":
        lengths, q_lens = [13, 0, 40, 7], [1, 1, 1, 1]
    else:
        lengths, q_lens = [1, 0, 2, 3], [2, 3, 3, 5]
    P, hq, hk, d = 4, 8, 2, 64
    kv_indptr, kv_indices, last, num_pages = build_page_table(rng, lengths, P, extra_pages=1)
    qo = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    q, k, v = (normal_bf16(54, i, s) for i, s in ((1, (int(qo[-1]), hq, d)), (2, (num_pages, P, hk, d)),
                                                   (3, (num_pages, P, hk, d))))
    o, lse, ex = R.paged_attention(_tb(q), _tb(k), _tb(v), qo, kv_indptr, torch.from_numpy(kv_indices), last,
                                   sm_scale=0.125, policy="none", causal=True, kv_indices_h=kv_indices)
    assert "o_states" not in ex                      # a single pass, no merge
    O, LSE = OA.paged_attention(q, k, v, qo, kv_indptr, kv_indices, last, P, 0.125, causal=True)
    np.testing.assert_allclose(o.numpy(), O, rtol=0, atol=1e-6)
    np.testing.assert_array_equal(np.isneginf(lse.numpy()), np.isneginf(LSE))
    fin = np.isfinite(LSE)
    np.testing.assert_allclose(lse.numpy()[fin], LSE[fin], rtol=0, atol=1e-6)


def test_empty_page_list_is_passed_as_a_placeholder():
    """An empty page list (no request has pages) reaches the library as a non-NULL buffer."""
    empty = torch.zeros(0, dtype=torch.int32)
    assert skv._index_ptr(empty) not in (None, 0)
    full = torch.arange(3, dtype=torch.int32)
    assert skv._index_ptr(full) == full.data_ptr() and skv._index_ptr(None) is None


def test_causal_mla_composition(monkeypatch):
    _Fakes(monkeypatch)
    rng = np.random.Generator(np.random.PCG64(52))
    lengths, q_len, P, H = [11, 2, 70, 0], 3, 16, 16
    kv_indptr, kv_indices, last, num_pages = build_page_table(rng, lengths, P, extra_pages=1)
    B = len(lengths)
    q_nope = normal_bf16(52, 1, (B, q_len, H, 512))
    q_pe = normal_bf16(52, 2, (B, q_len, H, 64))
    cache = normal_bf16(52, 3, (num_pages, P, 576))
    tc = _tb(cache)
    scale = 1 / math.sqrt(192.0)
    o, lse, ex = R.mla_decode(_tb(q_nope), _tb(q_pe), tc[..., :512], tc[..., 512:], kv_indptr,
                              torch.from_numpy(kv_indices), last, sm_scale=scale, policy="none", causal=True,
                              kv_indices_h=kv_indices)
    O, LSE = OA.mla_decode(q_nope, q_pe, cache[..., :512], cache[..., 512:], kv_indptr, kv_indices, last, P, scale,
                           causal=True)
    np.testing.assert_allclose(o.numpy(), O, rtol=0, atol=1e-6)
    np.testing.assert_array_equal(np.isneginf(lse.numpy()), np.isneginf(LSE))
    fin = np.isfinite(LSE)
    np.testing.assert_allclose(lse.numpy()[fin], LSE[fin], rtol=0, atol=1e-6)


def test_causal_tables_cover_each_visible_key_once():
    """Prefix keys + diagonal keys of every query token = exactly the keys the mask shows it."""
    rng = np.random.Generator(np.random.PCG64(53))
    for trial in range(20):
        B = int(rng.integers(1, 6))
        P = int(rng.choice([1, 4, 16]))
        lengths = rng.integers(0, 60, size=B).tolist()
        q_lens = rng.integers(0, 8, size=B)      # requests without query tokens included
        kv_indptr, kv_indices, last, num_pages = build_page_table(rng, lengths, P, extra_pages=0)
        tab = R.causal_split_tables(q_lens, kv_indptr, kv_indices, last, P)
        pi, px, pl = tab["prefix"]
        di, dx, dl = tab["diag"]
        row = 0
        for r in range(B):
            L = lengths[r]
            pages = kv_indices[kv_indptr[r]:kv_indptr[r + 1]]
            n_p = pi[r + 1] - pi[r]
            Lp = 0 if n_p == 0 else (n_p - 1) * P + pl[r]
            assert n_p <= len(pages) and Lp <= L          # the prefix never leaves the request
            assert np.array_equal(px[pi[r]:pi[r + 1]], pages[:n_p]) and 1 <= pl[r] <= P
            prefix_rows = [pages[t // P] * P + t % P for t in range(Lp)]
            for i in range(int(q_lens[r])):
                want = sorted(pages[t // P] * P + t % P for t in range(L) if t <= L - q_lens[r] + i)
                got = sorted(prefix_rows + dx[di[row]:di[row + 1]].tolist())
                assert got == want, (trial, r, i)
                row += 1
        assert row == len(di) - 1 and np.all(dl == 1)


def test_causal_tables_validation_and_sizing():
    qo, ip, ix, la = [np.asarray(a, np.int32) for a in ([0, 2, 5], [0, 2, 3], [4, 1, 7], [3, 2])]
    B = 2
    outs = [np.zeros(B + 1, np.int32), np.zeros(3, np.int32), np.zeros(B, np.int32), np.zeros(6, np.int32),
            np.zeros(64, np.int32), np.zeros(5, np.int32)]
    need = ctypes.c_int64(-1)

    def call(qo=qo, ip=ip, la=la, P=4, cap=64, rows=outs[4]):
        p = skv._ptr_i32
        return skv._causal(B, p(qo), p(ip), p(ix), p(la), P, p(outs[0]), p(outs[1]), p(outs[2]), p(outs[3]),
                           p(rows), p(outs[5]), cap, ctypes.byref(need))

    # request 0: L = 7, 2 query tokens -> prefix 6 keys, token 1 sees 1 more; request 1: L = 2 and
    # 3 query tokens -> prefix 0 keys, tokens 1 and 2 see 1 and 2 keys: 4 diagonal rows
    assert call(cap=0) == skv.ERR_WORKSPACE and need.value == 4
    assert call() == skv.OK and need.value == 4
    assert outs[0].tolist() == [0, 2, 2] and outs[2].tolist() == [2, 1]
    assert outs[3].tolist() == [0, 0, 1, 1, 2, 4]
    assert outs[4][:4].tolist() == [1 * 4 + 2, 7 * 4 + 0, 7 * 4 + 0, 7 * 4 + 1]
    assert call(la=np.asarray([5, 2], np.int32)) == skv.ERR_INVALID      # last page length > page size
    assert call(qo=np.asarray([0, 3, 2], np.int32)) == skv.ERR_INVALID   # decreasing query offsets
    assert call(P=0) == skv.ERR_INVALID


def test_causal_needs_host_page_list():
    with pytest.raises(ValueError):
        R.paged_attention(torch.zeros(1, 8, 64, dtype=torch.bfloat16), torch.zeros(2, 4, 2, 64, dtype=torch.bfloat16),
                          torch.zeros(2, 4, 2, 64, dtype=torch.bfloat16), [0, 1], [0, 1], torch.zeros(1), [2],
                          causal=True)
