"""Pins for the float64 oracle: it is checked against things other than itself.

* brute force on tiny inputs (pure-Python scalar loops, an independent bf16 decode via
  ``struct``, and 60-digit ``decimal`` arithmetic on <= 8 tokens);
* library routines: torch's float64 ``scaled_dot_product_attention`` on a dense KV that the
  test scatters into pages itself, and torch's ``float8_e4m3fn`` / ``bfloat16`` casts;
* closed forms (identical keys -> mean of V and LSE = s + ln L; one dominant key -> its V);
* invariants from the pages: merging the partials of any KV split equals unsplit attention
  (route / in-CTA split), permuting physical pages changes nothing (paged KV), a KV shared by
  many query batches equals an explicitly replicated KV (KV batch broadcast);
* mutation tests: plausible mistakes planted in the oracle (on the CPU) must each fail a pin.
"""
import ast
import contextlib
import decimal
import inspect
import math
import struct
import textwrap

import numpy as np
import pytest
import torch

import oracle.attention as OA
from workloads import (build_page_table, e4m3_encode, f32_to_bf16_bits, mla_decode_case,
                       normal_bf16, shared_kv_prefill_case)


# ----------------------------------------------------------------------------- helpers
def _bf16_scalar(bits: int) -> float:
    return struct.unpack("<f", struct.pack("<I", int(bits) << 16))[0]


def _tiny_case(seed=11, lengths=(13, 0, 7, 40), hq=4, hk=2, d=8, P=4, q_lens=(1, 2, 1, 3)):
    rng = np.random.Generator(np.random.PCG64(seed))
    kv_indptr, kv_indices, last, num_pages = build_page_table(rng, list(lengths), P, extra_pages=3)
    qo_indptr = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    q = normal_bf16(seed, 1, (int(qo_indptr[-1]), hq, d))
    k = normal_bf16(seed, 2, (num_pages, P, hk, d))
    v = normal_bf16(seed, 3, (num_pages, P, hk, d))
    return dict(q=q, k=k, v=v, qo_indptr=qo_indptr, kv_indptr=kv_indptr, kv_indices=kv_indices,
                kv_last_page_len=last, page_size=P, sm_scale=1.0 / math.sqrt(d))


def _brute(c):
    """Pure-Python scalar attention: explicit page walk, full softmax, fsum."""
    q, k, v = c["q"], c["k"], c["v"]
    P, scale = c["page_size"], c["sm_scale"]
    hq, hk, d = q.shape[1], k.shape[2], q.shape[2]
    g = hq // hk
    O = np.zeros((q.shape[0], hq, d))
    LSE = np.zeros((q.shape[0], hq))
    for r in range(len(c["kv_indptr"]) - 1):
        n = int(c["kv_indptr"][r + 1] - c["kv_indptr"][r])
        L = 0 if n == 0 else (n - 1) * P + int(c["kv_last_page_len"][r])
        for i in range(int(c["qo_indptr"][r]), int(c["qo_indptr"][r + 1])):
            for h in range(hq):
                kh = h // g
                qv = [_bf16_scalar(q[i, h, x]) for x in range(d)]
                scores, vals = [], []
                for t in range(L):
                    page = int(c["kv_indices"][int(c["kv_indptr"][r]) + t // P])
                    slot = t % P
                    kv = [_bf16_scalar(k[page, slot, kh, x]) for x in range(d)]
                    scores.append(scale * math.fsum(a * b for a, b in zip(qv, kv)))
                    vals.append([_bf16_scalar(v[page, slot, kh, x]) for x in range(d)])
                if L == 0:
                    O[i, h] = 0.0
                    LSE[i, h] = -math.inf
                    continue
                m = max(scores)
                w = [math.exp(s - m) for s in scores]
                l = math.fsum(w)
                O[i, h] = [math.fsum(w[t] * vals[t][x] for t in range(L)) / l for x in range(d)]
                LSE[i, h] = m + math.log(l)
    return O, LSE


def _run(c, **kw):
    return OA.paged_attention(c["q"], c["k"], c["v"], c["qo_indptr"], c["kv_indptr"], c["kv_indices"],
                              c["kv_last_page_len"], c["page_size"], c["sm_scale"], **kw)


# ----------------------------------------------------------------------------- pins
def pin_brute_force():
    for seed in (11, 12):
        c = _tiny_case(seed)
        O, LSE = _run(c)
        Ob, Lb = _brute(c)
        np.testing.assert_allclose(O, Ob, rtol=0, atol=1e-12)
        np.testing.assert_array_equal(np.isneginf(LSE), np.isneginf(Lb))
        fin = np.isfinite(Lb)
        np.testing.assert_allclose(LSE[fin], Lb[fin], rtol=0, atol=1e-12)


def pin_decimal():
    """60-digit decimal arithmetic on a <= 8-token request."""
    c = _tiny_case(21, lengths=(7,), q_lens=(1,), hq=2, hk=1, d=4, P=3)
    O, LSE = _run(c)
    decimal.getcontext().prec = 60
    D = decimal.Decimal
    q, k, v = c["q"], c["k"], c["v"]
    scale = D(1) / D(2)  # 1/sqrt(4), exact
    assert c["sm_scale"] == 0.5
    for h in range(2):
        s, vs = [], []
        for t in range(7):
            page = int(c["kv_indices"][t // 3])
            slot = t % 3
            s.append(scale * sum(D(_bf16_scalar(q[0, h, x])) * D(_bf16_scalar(k[page, slot, 0, x]))
                                 for x in range(4)))
            vs.append([D(_bf16_scalar(v[page, slot, 0, x])) for x in range(4)])
        m = max(s)
        w = [(x - m).exp() for x in s]
        l = sum(w)
        for x in range(4):
            ref = sum(w[t] * vs[t][x] for t in range(7)) / l
            assert abs(float(ref) - O[0, h, x]) <= 1e-14 * max(1.0, abs(float(ref)))
        assert abs(float(m + l.ln()) - LSE[0, h]) <= 1e-14 * max(1.0, abs(float(m + l.ln())))


def pin_sdpa_library():
    """Against torch's float64 SDPA on a dense KV the test scatters into permuted pages."""
    rng = np.random.Generator(np.random.PCG64(31))
    hq, hk, d, P, L, nq = 8, 2, 16, 5, 47, 3
    dense_k = normal_bf16(31, 2, (L, hk, d))
    dense_v = normal_bf16(31, 3, (L, hk, d))
    q = normal_bf16(31, 1, (nq, hq, d))
    n = (L + P - 1) // P
    num_pages = n + 4
    perm = rng.permutation(num_pages)[:n].astype(np.int32)
    k = normal_bf16(31, 4, (num_pages, P, hk, d))   # junk everywhere else
    v = normal_bf16(31, 5, (num_pages, P, hk, d))
    for j in range(n):
        rows = dense_k[j * P:(j + 1) * P]
        k[perm[j], :len(rows)] = rows
        v[perm[j], :len(rows)] = dense_v[j * P:(j + 1) * P]
    c = dict(q=q, k=k, v=v, qo_indptr=np.array([0, nq], np.int32), kv_indptr=np.array([0, n], np.int32),
             kv_indices=perm, kv_last_page_len=np.array([L - (n - 1) * P], np.int32), page_size=P,
             sm_scale=0.3)
    O, LSE = _run(c)
    tq = torch.from_numpy(q.astype(np.int16)).view(torch.bfloat16).double().permute(1, 0, 2)[None]
    tk = torch.from_numpy(dense_k.astype(np.int16)).view(torch.bfloat16).double().permute(1, 0, 2)[None]
    tv = torch.from_numpy(dense_v.astype(np.int16)).view(torch.bfloat16).double().permute(1, 0, 2)[None]
    tk = tk.repeat_interleave(hq // hk, dim=1)
    tv = tv.repeat_interleave(hq // hk, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=0.3)[0].permute(1, 0, 2)
    np.testing.assert_allclose(O, ref.numpy(), rtol=0, atol=1e-12)
    lse_ref = torch.logsumexp(0.3 * tq @ tk.transpose(-1, -2), dim=-1)[0].T.numpy()
    np.testing.assert_allclose(LSE, lse_ref, rtol=0, atol=1e-12)


def pin_closed_forms():
    # identical keys: O = mean_t v_t, LSE = s + ln L
    hq, hk, d, P, L = 4, 1, 8, 4, 10
    rng = np.random.Generator(np.random.PCG64(41))
    kv_indptr, kv_indices, last, num_pages = build_page_table(rng, [L], P)
    key = normal_bf16(41, 1, (d,))
    k = np.broadcast_to(key, (num_pages, P, hk, d)).copy()
    v = normal_bf16(41, 2, (num_pages, P, hk, d))
    q = normal_bf16(41, 3, (1, hq, d))
    c = dict(q=q, k=k, v=v, qo_indptr=np.array([0, 1], np.int32), kv_indptr=kv_indptr,
             kv_indices=kv_indices, kv_last_page_len=last, page_size=P, sm_scale=0.25)
    O, LSE = _run(c)
    vt = np.stack([OA.bf16_to_f64(v[kv_indices[t // P], t % P, 0]) for t in range(L)])
    kf = np.array([_bf16_scalar(x) for x in key])
    for h in range(hq):
        qf = np.array([_bf16_scalar(x) for x in q[0, h]])
        np.testing.assert_allclose(O[0, h], vt.mean(axis=0), rtol=0, atol=1e-13)
        assert abs(LSE[0, h] - (0.25 * float(qf @ kf) + math.log(L))) < 1e-12
    # one dominant key: O = v_j, LSE ~= s_j
    d, L, j = 64, 29, 17
    kv_indptr, kv_indices, last, num_pages = build_page_table(rng, [L], P)
    q = normal_bf16(42, 1, (1, 1, d))
    qf = OA.bf16_to_f64(q[0, 0])
    small = (np.random.Generator(np.random.PCG64(43)).standard_normal((num_pages, P, 1, d)) * 0.01)
    k = f32_to_bf16_bits(small.astype(np.float32))
    k[kv_indices[j // P], j % P, 0] = f32_to_bf16_bits((50.0 * qf / np.linalg.norm(qf)).astype(np.float32))
    v = normal_bf16(42, 2, (num_pages, P, 1, d))
    c = dict(q=q, k=k, v=v, qo_indptr=np.array([0, 1], np.int32), kv_indptr=kv_indptr,
             kv_indices=kv_indices, kv_last_page_len=last, page_size=P, sm_scale=1.0 / 8.0)
    O, LSE = _run(c)
    vj = OA.bf16_to_f64(v[kv_indices[j // P], j % P, 0])
    sj = (1.0 / 8.0) * float(qf @ OA.bf16_to_f64(k[kv_indices[j // P], j % P, 0]))
    np.testing.assert_allclose(O[0, 0], vj, rtol=0, atol=1e-9)
    assert abs(LSE[0, 0] - sj) < 1e-9


def pin_split_merge():
    """(a) merging the partials of any KV split equals unsplit attention."""
    c = _tiny_case(51, lengths=(13, 0, 7, 40, 64), q_lens=(1, 2, 1, 3, 2))
    O, LSE = _run(c)
    rng = np.random.Generator(np.random.PCG64(52))
    for trial in range(6):
        sps = []
        for r in range(len(c["kv_indptr"]) - 1):
            n = int(c["kv_indptr"][r + 1] - c["kv_indptr"][r])
            S = int(rng.integers(1, 5))
            cuts = np.sort(rng.integers(0, n + 1, size=S - 1))   # empty splits allowed
            sps.append([0, *cuts.tolist(), n])
        parts = OA.paged_attention_partials(c["q"], c["k"], c["v"], c["qo_indptr"], c["kv_indptr"],
                                            c["kv_indices"], c["kv_last_page_len"], c["page_size"],
                                            c["sm_scale"], sps)
        for r, (po, pl) in parts.items():
            a, b = int(c["qo_indptr"][r]), int(c["qo_indptr"][r + 1])
            mo, ml = OA.merge_states(po, pl)
            np.testing.assert_allclose(mo, O[a:b], rtol=0, atol=1e-12)
            np.testing.assert_array_equal(np.isneginf(ml), np.isneginf(LSE[a:b]))
            fin = np.isfinite(ml)
            np.testing.assert_allclose(ml[fin], LSE[a:b][fin], rtol=0, atol=1e-12)
            # merge is order-free
            perm = rng.permutation(po.shape[0])
            mo2, _ = OA.merge_states(po[perm], pl[perm])
            np.testing.assert_allclose(mo2, mo, rtol=0, atol=1e-13)


def pin_merge_special():
    o = np.random.Generator(np.random.PCG64(5)).standard_normal((1, 3, 4))
    lse = np.array([[0.5, -np.inf, 2.0]])
    mo, ml = OA.merge_states(o, lse)              # one state -> itself (empty stays empty)
    np.testing.assert_allclose(mo[[0, 2]], o[0, [0, 2]], rtol=0, atol=1e-15)
    np.testing.assert_array_equal(mo[1], 0.0)
    assert np.isneginf(ml[1]) and abs(ml[0] - 0.5) < 1e-15
    # two equal-mass states: LSE + ln 2, mean of O
    o2 = np.stack([o[0], -o[0]])
    mo, ml = OA.merge_states(o2, np.array([[1.0, 1.0, 1.0], [1.0, 1.0, 1.0]]))
    np.testing.assert_allclose(mo, 0.0, atol=1e-15)
    np.testing.assert_allclose(ml, 1.0 + math.log(2.0), atol=1e-15)


def pin_permutation():
    """(b) permuting physical pages and the page table leaves outputs bit-identical."""
    c = _tiny_case(61)
    O, LSE = _run(c)
    perm = np.random.Generator(np.random.PCG64(62)).permutation(c["k"].shape[0])
    k2 = np.empty_like(c["k"]); k2[perm] = c["k"]
    v2 = np.empty_like(c["v"]); v2[perm] = c["v"]
    c2 = dict(c, k=k2, v=v2, kv_indices=perm[c["kv_indices"]].astype(np.int32))
    O2, LSE2 = _run(c2)
    np.testing.assert_array_equal(O, O2)
    np.testing.assert_array_equal(LSE, LSE2)


def pin_broadcast():
    """(c) one KV listed by every query batch equals an explicitly replicated KV."""
    kw = dict(n_batches=3, q_len=4, kv_len=300)
    a = shared_kv_prefill_case(replicated=False, **kw)
    b = shared_kv_prefill_case(replicated=True, **kw)
    heads = [0, 5, 31]
    Oa, La = OA.paged_attention(a.q, a.k, a.v, a.qo_indptr, a.kv_indptr, a.kv_indices,
                                a.kv_last_page_len, a.page_size, a.sm_scale, heads=heads)
    Ob, Lb = OA.paged_attention(b.q, b.k, b.v, b.qo_indptr, b.kv_indptr, b.kv_indices,
                                b.kv_last_page_len, b.page_size, b.sm_scale, heads=heads)
    np.testing.assert_array_equal(Oa, Ob)
    np.testing.assert_array_equal(La, Lb)
    # batches see the same KV: identical queries would give identical rows; here check the KV
    # length each batch sees is the full shared sequence
    assert all(OA.request_kv_length(a.kv_indptr, a.kv_last_page_len, a.page_size, r) == 300
               for r in range(3))


def pin_mla():
    """MLA: against torch SDPA with K = [ckv | kpe], V = ckv; q_pe = 0 reduces to the GQA
    oracle with one KV head whose K and V are the 512-d latent."""
    c = mla_decode_case(num_heads=4, q_len=2, batch=2, len_range=(5, 150), page_size=8, seed=71)
    O, LSE = OA.mla_decode(c.q_nope, c.q_pe, c.ckv, c.kpe, c.kv_indptr, c.kv_indices,
                           c.kv_last_page_len, c.page_size, c.sm_scale)
    for r in range(c.batch):
        pages, slots = OA.request_token_slots(c.kv_indptr, c.kv_indices, c.kv_last_page_len, c.page_size, r)
        K = torch.from_numpy(c.cache[pages, slots].astype(np.int16)).view(torch.bfloat16).double()
        qn = torch.from_numpy(c.q_nope[r].astype(np.int16)).view(torch.bfloat16).double()
        qp = torch.from_numpy(c.q_pe[r].astype(np.int16)).view(torch.bfloat16).double()
        qq = torch.cat([qn, qp], dim=-1).permute(1, 0, 2)          # [H, q_len, 576]
        ref = torch.nn.functional.scaled_dot_product_attention(qq, K[None].expand(4, -1, -1),
                                                               K[None, :, :512].expand(4, -1, -1),
                                                               scale=c.sm_scale)
        np.testing.assert_allclose(O[r], ref.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)
        lse_ref = torch.logsumexp(c.sm_scale * qq @ K.T, dim=-1).T.numpy()
        np.testing.assert_allclose(LSE[r], lse_ref, rtol=0, atol=1e-12)
    qpe0 = np.zeros_like(c.q_pe)
    O0, L0 = OA.mla_decode(c.q_nope, qpe0, c.ckv, c.kpe, c.kv_indptr, c.kv_indices,
                           c.kv_last_page_len, c.page_size, c.sm_scale)
    B, ql, H = c.q_nope.shape[:3]
    q_g = c.q_nope.reshape(B * ql, H, 512)
    ckv4 = c.ckv[:, :, None, :]
    qo_indptr = (np.arange(B + 1) * ql).astype(np.int32)
    Og, Lg = OA.paged_attention(q_g, ckv4, ckv4, qo_indptr, c.kv_indptr, c.kv_indices,
                                c.kv_last_page_len, c.page_size, c.sm_scale)
    np.testing.assert_allclose(O0.reshape(B * ql, H, 512), Og, rtol=0, atol=1e-13)
    np.testing.assert_allclose(L0.reshape(B * ql, H), Lg, rtol=0, atol=1e-13)


def pin_e4m3():
    codes = np.arange(256, dtype=np.uint8)
    got = OA.e4m3_to_f64(codes)
    # values fixed by the OCP e4m3fn definition
    named = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0,
             0x39: 1.125, 0x40: 2.0, 0x7E: 448.0, 0xBE: -1.75, 0xB8: -1.0, 0xFE: -448.0}
    for cde, val in named.items():
        assert got[cde] == val, (hex(cde), got[cde], val)
    assert np.isnan(got[0x7F]) and np.isnan(got[0xFF])
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])
    # the generator's encoder is the decoder's inverse on representable values
    np.testing.assert_array_equal(e4m3_encode(got[ok]), codes[ok])


def pin_gqa_e4m3():
    """GQA over an e4m3 K/V cache with per-tensor scale 2^-3 equals GQA over the bf16 cache holding
    the same dequantised values (exact in bf16: at most 4 significant bits), computed by torch's
    float64 SDPA on the dense rows the test gathers itself -- and differs from ignoring the scale."""
    c = _tiny_case(71, hq=4, hk=2, d=8, P=4)
    rng = np.random.Generator(np.random.PCG64(72))
    kc = e4m3_encode(rng.standard_normal(c["k"].shape) * 40)
    vc = e4m3_encode(rng.standard_normal(c["v"].shape) * 40)
    scale = 2.0 ** -3
    O, LSE = OA.paged_attention(c["q"], kc, vc, c["qo_indptr"], c["kv_indptr"], c["kv_indices"],
                                c["kv_last_page_len"], c["page_size"], c["sm_scale"], kv_dtype="e4m3", kv_scale=scale)
    kf = torch.from_numpy(kc).view(torch.float8_e4m3fn).double() * scale
    vf = torch.from_numpy(vc).view(torch.float8_e4m3fn).double() * scale
    assert torch.equal(kf.bfloat16().double(), kf) and torch.equal(vf.bfloat16().double(), vf)
    P, hq, hk = c["page_size"], 4, 2
    for r in range(len(c["kv_indptr"]) - 1):
        n = int(c["kv_indptr"][r + 1] - c["kv_indptr"][r])
        L = 0 if n == 0 else (n - 1) * P + int(c["kv_last_page_len"][r])
        a, b = int(c["qo_indptr"][r]), int(c["qo_indptr"][r + 1])
        if L == 0 or a == b:
            continue
        pages = torch.from_numpy(c["kv_indices"][c["kv_indptr"][r]:c["kv_indptr"][r + 1]].astype(np.int64))
        kd = kf[pages].reshape(n * P, hk, -1)[:L]
        vd = vf[pages].reshape(n * P, hk, -1)[:L]
        qd = torch.from_numpy(OA.bf16_to_f64(c["q"][a:b]))
        for h in range(hq):
            ref = torch.nn.functional.scaled_dot_product_attention(
                qd[None, None, :, h], kd[None, None, :, h // 2], vd[None, None, :, h // 2], scale=c["sm_scale"])
            np.testing.assert_allclose(O[a:b, h], ref[0, 0].numpy(), rtol=0, atol=1e-12)
    O1, _ = OA.paged_attention(c["q"], kc, vc, c["qo_indptr"], c["kv_indptr"], c["kv_indices"],
                               c["kv_last_page_len"], c["page_size"], c["sm_scale"], kv_dtype="e4m3", kv_scale=1.0)
    fin = np.isfinite(LSE)
    assert np.max(np.abs(O1[fin] - O[fin])) > 0.1


def pin_bf16():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = OA.bf16_to_f64(bits)
    ref = torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])


def test_e4m3_encoder_is_nearest_even():
    """The generator's fp8 encoder picks the nearest e4m3fn value, ties to the even code."""
    pos = OA.e4m3_to_f64(np.arange(0x7F, dtype=np.uint8))
    rng = np.random.Generator(np.random.PCG64(8))
    x = np.concatenate([rng.standard_normal(20000) * 60, rng.standard_normal(2000) * 1e-3,
                        (pos[1:] + pos[:-1]) / 2, -(pos[1:] + pos[:-1]) / 2, [500.0, -1e9, 0.0]])
    got = OA.e4m3_to_f64(e4m3_encode(x))
    a = np.minimum(np.abs(x), 448.0)
    d = np.abs(pos[None, :] - a[:, None])
    best = d.min(axis=1)
    assert np.all(np.abs(np.abs(got) - a) == best)
    ties = (d == best[:, None]).sum(axis=1) > 1
    codes = e4m3_encode(x) & 0x7F
    assert np.all(codes[ties] % 2 == 0)


PINS = [pin_brute_force, pin_decimal, pin_sdpa_library, pin_closed_forms, pin_split_merge,
        pin_merge_special, pin_permutation, pin_broadcast, pin_mla, pin_e4m3, pin_gqa_e4m3, pin_bf16]


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
    """Re-define oracle.attention.<func_name> with ``old`` replaced by ``new`` in its source."""
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
    ("request_kv_length", "(n - 1) * page_size + int(kv_last_page_len[r])", "n * page_size"),
    ("request_token_slots", "t % page_size", "(t + 1) % page_size"),
    ("_gqa_request", "if h // g != kh", "if h % hk != kh"),
    ("_gqa_request", "s = sm_scale * (q_r[:, h, :] @ kk.T)", "s = (q_r[:, h, :] @ kk.T)"),
    ("_softmax_attend", "(m + np.log(l))[:, 0]", "np.log(l)[:, 0]"),
    ("_softmax_attend", "o = (e @ v) / l", "o = (e @ v)"),
    ("merge_states", "np.exp(lse_states[j] - lse_s)", "np.exp(lse_states[j] - Ms)"),
    ("merge_states", "Ms + np.log(np.where(empty, 1.0, total))", "Ms + np.where(empty, 1.0, total)"),
    ("e4m3_to_f64", "e.astype(np.float64) - 7.0", "e.astype(np.float64) - 8.0"),
    ("e4m3_to_f64", "(m / 8.0) * 2.0 ** -6", "(m / 8.0) * 2.0 ** -7"),
    ("_mla_request", "+ qp.reshape(q_len * nh, -1) @ kr.T", ""),
    ("_mla_request", "o, lse = _softmax_attend(s, c)", "o, lse = _softmax_attend(s, np.concatenate([c[:, 64:], c[:, :64]], 1))"),
    ("bf16_to_f64", "<< np.uint32(16)", "<< np.uint32(15)"),
    ("_gqa_request", "kk = _decode_kv(k[pages, slots, kh], kv_dtype, kv_scale)",
     "kk = _decode_kv(k[pages, slots, kh], kv_dtype, 1.0)"),
]


@pytest.mark.parametrize("mut", MUTATIONS, ids=lambda m: f"{m[0]}:{m[2][:24]}")
def test_mutation_is_caught(mut):
    caught = []
    with _mutated(*mut):
        for pin in PINS:
            try:
                pin()
            except (AssertionError, ValueError, IndexError, FloatingPointError):
                caught.append(pin.__name__)
    assert caught, f"no pin catches mutation {mut}"
