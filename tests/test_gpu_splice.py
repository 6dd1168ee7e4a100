"""GPU parity of skv_mla_splice (the fetch primitive's local compute) against the float64 splice
oracle on the same seeded inputs.

Bar: the 512-d latent is copied bit for bit; every rope value is within the bf16 rounding of
the exact rotation, |got - exact| <= 2^-8 |exact| + 1e-5 (round to nearest in bf16 moves a value
by at most 2^-8 of itself; the slack covers the fp32 rotation); rows the call does not own keep
their old contents.  Reduced sizes element by element; the full 8 x 16384-token corpus with the
latent checked everywhere, the rope part on seeded samples and through properties (pair lengths
kept, a move by -delta restores the source)."""
import numpy as np
import pytest
import torch

import oracle.splice as OS
import split_kv_merge_b200 as skv
from workloads import fetch_splice_case, normal_bf16
from workloads.device import bf16_tensor, i32_tensor, splice_to_device

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
FILL = 7.0


def _f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _check_rows(dst, pg, sl, ckv_ref, kpe_ref, where=""):
    rows = dst[torch.as_tensor(pg, device=dst.device), torch.as_tensor(sl, device=dst.device)]
    got = _f64(rows)
    assert np.array_equal(got[:, :512], ckv_ref), f"{where}: latent not copied exactly"
    err = np.abs(got[:, 512:] - kpe_ref)
    bound = 2.0 ** -8 * np.abs(kpe_ref) + 1e-5
    assert np.all(err <= bound), f"{where}: rope max err {err.max()} (worst ratio {(err / bound).max()})"
    return float(err.max())


def _owned_mask(c, chunks=None):
    """[dst_num_pages, Pd] True where some spliced chunk writes."""
    m = np.zeros((c.dst_num_pages, c.dst_page_size), bool)
    for ch in (range(c.num_chunks) if chunks is None else chunks):
        pos = c.dst_start[ch] + np.arange(c.chunk_tokens)
        m[c.dst_pages[pos // c.dst_page_size], pos % c.dst_page_size] = True
    return m


def _chunk_rows(c, chunks):
    return [(int(c.src_start[ch]), int(c.dst_start[ch]), c.chunk_tokens, int(c.delta[ch])) for ch in chunks]


def _splice(c, d, chunks, layout="interleaved", status=None, inv_freq=None, dst_pages=None):
    """One skv_mla_splice call moving the given chunks of the case."""
    skv.mla_splice(d["src_ckv"], d["src_kpe"], d["src_pages"], d["dst_ckv"], d["dst_kpe"],
                   d["dst_pages"] if dst_pages is None else dst_pages, _chunk_rows(c, chunks),
                   rope_theta=c.rope_theta, rope_layout=layout, inv_freq=inv_freq, status=status)


def _oracle_chunk(c, ch, layout="interleaved", inv_freq=None):
    freq = OS.rope_inv_freq(c.rope_theta) if inv_freq is None else inv_freq
    return OS.splice_rows(c.src[..., :512], c.src[..., 512:], c.src_pages, int(c.src_start[ch]), c.dst_pages,
                          c.dst_page_size, int(c.dst_start[ch]), c.chunk_tokens, int(c.delta[ch]), freq, layout)


# ----------------------------------------------------------------------------- reduced sizes
@pytest.mark.parametrize("layout", ["interleaved", "halves"])
@pytest.mark.parametrize("ps,pd,context", [(16, 64, 37), (64, 16, 0), (1, 8, 5), (8, 8, 1000)])
@pytest.mark.parametrize("calls", ["one", "per_chunk"])
def test_splice_reduced(layout, ps, pd, context, calls):
    c = fetch_splice_case(num_chunks=3, chunk_tokens=213, src_page_size=ps, dst_page_size=pd, context=context,
                          seed=21)
    d = splice_to_device(c, DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    if calls == "one":
        _splice(c, d, range(c.num_chunks), layout, status)
    else:
        for ch in range(c.num_chunks):
            _splice(c, d, [ch], layout, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for ch in range(c.num_chunks):
        pg, sl, ckv, kpe = _oracle_chunk(c, ch, layout)
        _check_rows(d["dst"], pg, sl, ckv, kpe, f"chunk {ch}")
    untouched = _f64(d["dst"])[~_owned_mask(c)]
    assert np.all(untouched == FILL)


def test_splice_zero_delta_is_a_bit_exact_copy():
    c = fetch_splice_case(num_chunks=2, chunk_tokens=300, src_page_size=16, dst_page_size=32, context=7, seed=22)
    d = splice_to_device(c, DEV)
    skv.mla_splice(d["src_ckv"], d["src_kpe"], d["src_pages"], d["dst_ckv"], d["dst_kpe"], d["dst_pages"],
                   [(int(c.src_start[ch]), int(c.dst_start[ch]), c.chunk_tokens, 0) for ch in range(c.num_chunks)])
    torch.cuda.synchronize()
    for ch in range(c.num_chunks):
        pg, sl, ckv, kpe = OS.splice_rows(c.src[..., :512], c.src[..., 512:], c.src_pages, int(c.src_start[ch]),
                                          c.dst_pages, c.dst_page_size, int(c.dst_start[ch]), c.chunk_tokens, 0,
                                          OS.rope_inv_freq(c.rope_theta))
        got = d["dst"][torch.as_tensor(pg, device=DEV), torch.as_tensor(sl, device=DEV)]
        assert np.array_equal(_f64(got), np.concatenate([ckv, kpe], 1))


@pytest.mark.parametrize("layout", ["interleaved", "halves"])
def test_splice_in_place(layout):
    """Re-rotating rows where they stand (source rows = destination rows)."""
    P, n_pages, n, start, delta = 16, 20, 250, 9, -31000
    bits = normal_bf16(23, 1, (n_pages, P, 576))
    pages = np.random.Generator(np.random.PCG64(23)).permutation(n_pages)[:17].astype(np.int32)
    cache = bf16_tensor(bits, DEV)
    pl = i32_tensor(pages, DEV)
    skv.mla_splice(cache[..., :512], cache[..., 512:], pl, cache[..., :512], cache[..., 512:], pl,
                   [(start, start, n, delta)], rope_layout=layout)
    torch.cuda.synchronize()
    pg, sl, ckv, kpe = OS.splice_rows(bits[..., :512], bits[..., 512:], pages, start, pages, P, start, n, delta,
                                      OS.rope_inv_freq(10000.0), layout)
    _check_rows(cache, pg, sl, ckv, kpe, "in place")
    mask = np.zeros((n_pages, P), bool)
    mask[pg, sl] = True
    got = _f64(cache)[~mask]
    ref = (bits[~mask].astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    assert np.array_equal(got, ref)


def test_splice_frequency_table():
    """A caller-given per-pair frequency table (a scaled-RoPE table, for instance) replaces
    base^(-2i/64)."""
    c = fetch_splice_case(num_chunks=2, chunk_tokens=150, src_page_size=32, dst_page_size=16, context=3, seed=24)
    freq32 = (np.random.Generator(np.random.PCG64(24)).random(32) * 0.9 + 1e-4).astype(np.float32)
    d = splice_to_device(c, DEV)
    tf = torch.from_numpy(freq32).to(DEV)
    _splice(c, d, range(c.num_chunks), "halves", inv_freq=tf)
    torch.cuda.synchronize()
    for ch in range(c.num_chunks):
        pg, sl, ckv, kpe = _oracle_chunk(c, ch, "halves", inv_freq=freq32.astype(np.float64))
        _check_rows(d["dst"], pg, sl, ckv, kpe, f"chunk {ch}")


def test_splice_bad_page_id_sets_status_and_skips_only_its_rows():
    c = fetch_splice_case(num_chunks=1, chunk_tokens=100, src_page_size=16, dst_page_size=16, context=0, seed=25)
    d = splice_to_device(c, DEV)
    bad = c.dst_pages.copy()
    bad[2] = c.dst_num_pages + 5          # tokens 32..47 point outside the destination cache
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    _splice(c, d, [0], status=status, dst_pages=i32_tensor(bad, DEV))
    torch.cuda.synchronize()
    assert int(status.item()) == skv.DEV_PAGE_OOB
    pg, sl, ckv, kpe = _oracle_chunk(c, 0)
    keep = (np.arange(100) // 16) != 2
    _check_rows(d["dst"], pg[keep], sl[keep], ckv[keep], kpe[keep], "good rows")
    assert np.all(_f64(d["dst"][int(c.dst_pages[2])]) == FILL)


def test_splice_many_chunks_with_empty_ones():
    """70 chunks in one call (more than one launch's 64), with empty chunks among them and
    lengths from 1 token up; every chunk has its own delta."""
    rng = np.random.Generator(np.random.PCG64(27))
    lens = rng.integers(0, 40, size=70)
    lens[[0, 5, 6, 63, 64, 69]] = 0
    lens[[1, 65]] = 1
    n_tok = int(lens.sum())
    P = 16
    n_pages = -(-n_tok // P) + 2
    bits = normal_bf16(27, 1, (n_pages, P, 576))
    src_pages = rng.permutation(n_pages).astype(np.int32)
    dst_pages = rng.permutation(n_pages + 4).astype(np.int32)
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]])
    dst_order = rng.permutation(70)
    dst_starts = np.empty(70, np.int64)
    dst_starts[dst_order] = np.concatenate([[0], np.cumsum(lens[dst_order])[:-1]]) + 3
    deltas = rng.integers(-50000, 50000, size=70)
    chunks = [(int(a), int(b), int(n), int(dl)) for a, b, n, dl in zip(starts, dst_starts, lens, deltas)]
    src = bf16_tensor(bits, DEV)
    dst = torch.zeros(n_pages + 4, P, 576, dtype=torch.bfloat16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    skv.mla_splice(src[..., :512], src[..., 512:], i32_tensor(src_pages, DEV), dst[..., :512], dst[..., 512:],
                   i32_tensor(dst_pages, DEV), chunks, rope_layout="halves", status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    freq = OS.rope_inv_freq(10000.0)
    for (s0, d0, n, dl) in chunks:
        pg, sl, ckv, kpe = OS.splice_rows(bits[..., :512], bits[..., 512:], src_pages, s0, dst_pages, P, d0, n, dl,
                                          freq, "halves")
        if n:
            _check_rows(dst, pg, sl, ckv, kpe, f"chunk {(s0, d0, n, dl)}")


# ----------------------------------------------------------------------------- full size
def test_splice_full_corpus_sampled():
    """8 x 16384-token corpus (page size 64 on both sides): the latent everywhere, the rope part
    on 512 seeded tokens against the oracle, pair lengths everywhere, and the way back."""
    c = fetch_splice_case()
    d = splice_to_device(c, DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    _splice(c, d, range(c.num_chunks), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    T, Ps, Pd = c.chunk_tokens, c.src.shape[1], c.dst_page_size
    n_tok = c.num_chunks * T
    spos = np.arange(n_tok)
    dpos = np.concatenate([c.dst_start[ch] + np.arange(T) for ch in range(c.num_chunks)])
    s_pg = torch.as_tensor(c.src_pages[spos // Ps], device=DEV).long()
    s_sl = torch.as_tensor(spos % Ps, device=DEV).long()
    d_pg = torch.as_tensor(c.dst_pages[dpos // Pd], device=DEV).long()
    d_sl = torch.as_tensor(dpos % Pd, device=DEV).long()
    src_rows = d["src"][s_pg, s_sl]
    dst_rows = d["dst"][d_pg, d_sl]
    assert torch.equal(dst_rows[:, :512].view(torch.int16), src_rows[:, :512].view(torch.int16))
    a_idx, b_idx = OS.rope_pairs("interleaved")
    r_in = torch.hypot(src_rows[:, 512:][:, a_idx].float(), src_rows[:, 512:][:, b_idx].float())
    r_out = torch.hypot(dst_rows[:, 512:][:, a_idx].float(), dst_rows[:, 512:][:, b_idx].float())
    assert torch.all((r_out - r_in).abs() <= 2.0 ** -7 * r_in + 1e-5)
    assert int((~torch.from_numpy(_owned_mask(c)).to(DEV) & (d["dst"][..., 0] != FILL)).sum()) == 0
    # seeded samples against the oracle
    rng = np.random.Generator(np.random.PCG64(26))
    freq = OS.rope_inv_freq(c.rope_theta)
    for tok in rng.choice(n_tok, size=512, replace=False):
        ch, t = divmod(int(tok), T)
        pg, sl, ckv, kpe = OS.splice_rows(c.src[..., :512], c.src[..., 512:], c.src_pages, int(c.src_start[ch]) + t,
                                          c.dst_pages, Pd, int(c.dst_start[ch]) + t, 1, int(c.delta[ch]), freq)
        _check_rows(d["dst"], pg, sl, ckv, kpe, f"token {tok}")
    # the way back: moving every chunk by -delta into a fresh copy of the corpus layout
    back = torch.zeros_like(d["src"])
    skv.mla_splice(d["dst_ckv"], d["dst_kpe"], d["dst_pages"], back[..., :512], back[..., 512:], d["src_pages"],
                   [(int(c.dst_start[ch]), int(c.src_start[ch]), T, -int(c.delta[ch])) for ch in range(c.num_chunks)])
    torch.cuda.synchronize()
    diff = (back[s_pg, s_sl].float() - src_rows.float()).abs()
    assert float(diff[:, :512].max()) == 0.0
    # two roundings, each moving a pair by at most 2^-8 of its length
    rad = torch.empty_like(diff[:, 512:])
    rad[:, a_idx] = r_in
    rad[:, b_idx] = r_in
    assert torch.all(diff[:, 512:] <= 2.0 ** -7 * rad + 2e-5)
