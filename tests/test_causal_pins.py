"""Pins for the oracle's causal / multi-token (MTP) mask, checked against things other than
itself:

* a library routine: torch's float64 ``scaled_dot_product_attention`` with a boolean mask built by
  ``torch.tril`` (diagonal L - n_q, the library's own alignment of a lower triangle to the last
  n_q rows), on a dense KV the test gathers from the pages itself, and ``torch.logsumexp`` of the
  masked scores for the LSE -- for GQA and for MLA (K = [ckv | kpe], V = ckv);
* special cases: with one query token per request the mask changes nothing; the last query
  token of a request sees every key;
* the page table: query token i equals unmasked attention over the request truncated to its first
  L - n_q + 1 + i keys (a shorter page list and last-page length);
* the split invariant: merging causal partials over any split of the pages equals unsplit causal
  attention, splits that some tokens cannot see included;
* mutation tests: plausible mistakes planted in the oracle (on the CPU) must each fail a pin.
"""
import ast
import contextlib
import inspect
import math
import textwrap

import numpy as np
import pytest
import torch

import oracle.attention as OA
from workloads import build_page_table, normal_bf16


def _tiny(seed=41, lengths=(13, 0, 3, 40, 9), q_lens=(3, 2, 5, 4, 1), hq=4, hk=2, d=8, P=4):
    rng = np.random.Generator(np.random.PCG64(seed))
    kv_indptr, kv_indices, last, num_pages = build_page_table(rng, list(lengths), P, extra_pages=2)
    qo_indptr = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    return dict(q=normal_bf16(seed, 1, (int(qo_indptr[-1]), hq, d)), k=normal_bf16(seed, 2, (num_pages, P, hk, d)),
                v=normal_bf16(seed, 3, (num_pages, P, hk, d)), qo_indptr=qo_indptr, kv_indptr=kv_indptr,
                kv_indices=kv_indices, kv_last_page_len=last, page_size=P, sm_scale=1.0 / math.sqrt(d),
                lengths=list(lengths), q_lens=list(q_lens))


def _run(c, **kw):
    return OA.paged_attention(c["q"], c["k"], c["v"], c["qo_indptr"], c["kv_indptr"], c["kv_indices"],
                              c["kv_last_page_len"], c["page_size"], c["sm_scale"], **kw)


def _f64(bits):
    return torch.from_numpy((np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)).double()


def _dense(c, r, x):
    """Request r's logical rows of cache x, gathered by reshaping its pages (the test's own walk)."""
    P = c["page_size"]
    pages = c["kv_indices"][c["kv_indptr"][r]:c["kv_indptr"][r + 1]]
    return x[pages].reshape(len(pages) * P, *x.shape[2:])[:c["lengths"][r]]


def _torch_causal(scores, v, n_q, L):
    """Masked softmax attention by torch: mask = tril(ones(n_q, L), L - n_q); rows without a
    visible key are reported as (0, -inf)."""
    mask = torch.tril(torch.ones(n_q, L, dtype=torch.bool), diagonal=L - n_q)
    masked = scores.masked_fill(~mask, -math.inf)
    lse = torch.logsumexp(masked, dim=-1) if L else torch.full((n_q,), -math.inf, dtype=torch.float64)
    o = torch.softmax(masked, dim=-1) @ v if L else torch.zeros(n_q, v.shape[-1], dtype=torch.float64)
    none = ~mask.any(dim=-1) if L else torch.ones(n_q, dtype=torch.bool)
    o[none] = 0.0
    return o, lse


# ----------------------------------------------------------------------------- pins
def pin_gqa_vs_torch_mask():
    c = _tiny()
    O, LSE = _run(c, causal=True)
    hq, hk = c["q"].shape[1], c["k"].shape[2]
    g = hq // hk
    for r, (L, n_q) in enumerate(zip(c["lengths"], c["q_lens"])):
        a = int(c["qo_indptr"][r])
        kd, vd = _f64(_dense(c, r, c["k"])), _f64(_dense(c, r, c["v"]))
        q = _f64(c["q"][a:a + n_q])
        for h in range(hq):
            kk, vv = kd[:, h // g], vd[:, h // g]
            ref_o = torch.nn.functional.scaled_dot_product_attention(
                q[None, None, :, h], kk[None, None], vv[None, None],
                attn_mask=torch.tril(torch.ones(n_q, L, dtype=torch.bool), diagonal=L - n_q),
                scale=c["sm_scale"])[0, 0] if L else None
            o_t, lse_t = _torch_causal(c["sm_scale"] * q[:, h] @ kk.T, vv, n_q, L)
            sees = torch.tril(torch.ones(n_q, L, dtype=torch.bool), diagonal=L - n_q).any(-1) if L else \
                torch.zeros(n_q, dtype=torch.bool)
            np.testing.assert_allclose(O[a:a + n_q, h], o_t.numpy(), rtol=0, atol=1e-12)
            if ref_o is not None:
                np.testing.assert_allclose(O[a:a + n_q, h][sees.numpy()], ref_o[sees].numpy(), rtol=0, atol=1e-12)
            np.testing.assert_array_equal(np.isneginf(LSE[a:a + n_q, h]), ~sees.numpy())
            fin = sees.numpy()
            np.testing.assert_allclose(LSE[a:a + n_q, h][fin], lse_t.numpy()[fin], rtol=0, atol=1e-12)
    # the case holds rows that see nothing (L = 0, and L = 3 < n_q = 5) and rows that see all keys
    assert np.isneginf(LSE).any() and np.isfinite(LSE).any()


def pin_single_token_and_last_token():
    c = _tiny(q_lens=(1, 1, 1, 1, 1))
    O0, L0 = _run(c)
    O1, L1 = _run(c, causal=True)
    np.testing.assert_allclose(O1, O0, rtol=0, atol=1e-14)
    np.testing.assert_array_equal(np.isneginf(L1), np.isneginf(L0))
    fin = np.isfinite(L0)
    np.testing.assert_allclose(L1[fin], L0[fin], rtol=0, atol=1e-14)
    c = _tiny()
    O0, L0 = _run(c)
    O1, L1 = _run(c, causal=True)
    last = c["qo_indptr"][1:] - 1
    np.testing.assert_allclose(O1[last], O0[last], rtol=0, atol=1e-14)
    fin = np.isfinite(L0[last])
    np.testing.assert_allclose(L1[last][fin], L0[last][fin], rtol=0, atol=1e-14)
    np.testing.assert_array_equal(np.isneginf(L1[last]), np.isneginf(L0[last]))


def pin_truncated_page_table():
    """Query token i of request r = unmasked attention of that token alone over the request cut
    to its first L - n_q + 1 + i keys."""
    c = _tiny()
    O, LSE = _run(c, causal=True)
    P = c["page_size"]
    for r, (L, n_q) in enumerate(zip(c["lengths"], c["q_lens"])):
        a = int(c["qo_indptr"][r])
        pages = c["kv_indices"][c["kv_indptr"][r]:c["kv_indptr"][r + 1]]
        for i in range(n_q):
            Li = L - n_q + 1 + i
            if Li <= 0:
                assert np.all(O[a + i] == 0) and np.all(np.isneginf(LSE[a + i]))
                continue
            n = (Li + P - 1) // P
            sub = dict(c, q=c["q"][a + i:a + i + 1], qo_indptr=np.array([0, 1], np.int32),
                       kv_indptr=np.array([0, n], np.int32), kv_indices=pages[:n].astype(np.int32),
                       kv_last_page_len=np.array([Li - (n - 1) * P], np.int32))
            Oi, Li_lse = _run(sub)
            np.testing.assert_allclose(O[a + i], Oi[0], rtol=0, atol=1e-13)
            np.testing.assert_allclose(LSE[a + i], Li_lse[0], rtol=0, atol=1e-13)


def pin_split_merge():
    c = _tiny(seed=43, lengths=(37, 21, 64), q_lens=(6, 3, 9), P=4)
    O, LSE = _run(c, causal=True)
    rng = np.random.Generator(np.random.PCG64(44))
    for trial in range(4):
        sps = []
        for r in range(3):
            n = int(c["kv_indptr"][r + 1] - c["kv_indptr"][r])
            cuts = np.sort(rng.choice(np.arange(1, n), size=min(n - 1, 1 + trial), replace=False))
            sps.append([0, *cuts.tolist(), n])
        parts = OA.paged_attention_partials(c["q"], c["k"], c["v"], c["qo_indptr"], c["kv_indptr"],
                                            c["kv_indices"], c["kv_last_page_len"], c["page_size"],
                                            c["sm_scale"], sps, causal=True)
        for r in range(3):
            a, b = int(c["qo_indptr"][r]), int(c["qo_indptr"][r + 1])
            mo, ml = OA.merge_states(*parts[r])
            np.testing.assert_allclose(mo, O[a:b], rtol=0, atol=1e-12)
            np.testing.assert_allclose(ml, LSE[a:b], rtol=0, atol=1e-12)
        # the last split is invisible to the earliest tokens when it is short
        assert any(np.isneginf(parts[r][1][-1]).any() for r in range(3)) or trial < 3


def pin_mla_vs_torch_mask():
    rng = np.random.Generator(np.random.PCG64(45))
    P, H, q_len, lengths = 4, 3, 3, [11, 2, 6]
    kv_indptr, kv_indices, last, num_pages = build_page_table(rng, lengths, P, extra_pages=1)
    B = len(lengths)
    q_nope = normal_bf16(45, 1, (B, q_len, H, 512))
    q_pe = normal_bf16(45, 2, (B, q_len, H, 64))
    cache = normal_bf16(45, 3, (num_pages, P, 576))
    ckv, kpe = cache[..., :512], cache[..., 512:]
    scale = 1.0 / math.sqrt(192.0)
    O, LSE = OA.mla_decode(q_nope, q_pe, ckv, kpe, kv_indptr, kv_indices, last, P, scale, causal=True)
    for r, L in enumerate(lengths):
        pages = kv_indices[kv_indptr[r]:kv_indptr[r + 1]]
        rows = _f64(cache[pages].reshape(-1, 576)[:L])
        for h in range(H):
            q = torch.cat([_f64(q_nope[r, :, h]), _f64(q_pe[r, :, h])], dim=-1)
            o_t, lse_t = _torch_causal(scale * q @ rows.T, rows[:, :512], q_len, L)
            np.testing.assert_allclose(O[r, :, h], o_t.numpy(), rtol=0, atol=1e-12)
            fin = np.isfinite(lse_t.numpy())
            np.testing.assert_array_equal(np.isfinite(LSE[r, :, h]), fin)
            np.testing.assert_allclose(LSE[r, :, h][fin], lse_t.numpy()[fin], rtol=0, atol=1e-12)
    assert np.isneginf(LSE[1]).any()   # L = 2 < q_len = 3: the first token sees nothing


PINS = [pin_gqa_vs_torch_mask, pin_single_token_and_last_token, pin_truncated_page_table, pin_split_merge,
        pin_mla_vs_torch_mask]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


# ----------------------------------------------------------------------------- mutation tests
def _code_signature(src):
    """The syntax tree of a function's source without its docstring (comments are not in it):
    equal when only a docstring or a comment changed."""
    body = ast.parse(src).body[0].body
    if body and isinstance(body[0], ast.Expr) and isinstance(getattr(body[0], "value", None), ast.Constant) \
            and isinstance(body[0].value.value, str):
        body = body[1:]
    return ast.dump(ast.Module(body=body, type_ignores=[]))


@contextlib.contextmanager
def _mutated(func_name, old, new):
    fn = getattr(OA, func_name)
    src = textwrap.dedent(inspect.getsource(fn))
    assert old in src, (func_name, old)
    ns = OA.__dict__
    exec(compile(src.replace(old, new, 1), OA.__file__, "exec"), ns)
    try:
        assert _code_signature(src.replace(old, new, 1)) != _code_signature(src), \
            f"mutation of {func_name} changes no code"
        yield
    finally:
        ns[func_name] = fn


MUTATIONS = [
    ("causal_visible", "[None, :] <= kv_len - n_q + i", "[None, :] < kv_len - n_q + i"),
    ("causal_visible", "[None, :] <= kv_len - n_q + i", "[None, :] <= kv_len - 1 - i"),
    ("causal_visible", "[None, :] <= kv_len - n_q + i", "[None, :] <= n_q - 1 + i"),
    ("_softmax_attend", "keys = np.flatnonzero(visible[i])", "keys = np.arange(visible.shape[1])"),
    ("_token_range", "np.arange(page_begin * page_size,", "np.arange(0,"),
    ("_mla_request", "np.repeat(causal_visible(q_len, L, t), nh, axis=0)",
     "np.tile(causal_visible(q_len, L, t), (nh, 1))"),
]


@pytest.mark.parametrize("mut", MUTATIONS, ids=lambda m: f"{m[0]}:{m[2][:28]}")
def test_mutation_is_caught(mut):
    caught = []
    with _mutated(*mut):
        for pin in PINS:
            try:
                pin()
            except (AssertionError, ValueError, IndexError):
                caught.append(pin.__name__)
    assert caught, f"no pin catches mutation {mut}"
