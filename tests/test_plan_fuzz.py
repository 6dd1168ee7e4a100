"""Randomised host checks of the planners (no GPU): for random page tables (empty requests, requests
without query rows, ragged lengths), page sizes, head shapes, split policies and both MLA cache
types, every plan must

* cover, for every query row of every request, the request's pages exactly once, split by split in
  order (page ranges contiguous from 0 to n_r);
* write each query row either directly (one split) or through partial rows that its merge item
  lists exactly, with no partial row written twice and every partial row inside the buffer;
* hand the work to persistent CTAs through a monotone CTA index that ends at the work count."""
import numpy as np
import pytest

import split_kv_merge_b200 as skv
from workloads import build_page_table


def _items(plan):
    nw, nm = plan.info.num_work, plan.info.num_merge_rows
    return plan.words[: 8 * nw].reshape(-1, 8), plan.words[8 * nw: 8 * nw + 4 * nm].reshape(-1, 4)


def _grouped(plan, qo, num_heads, kv_dtype="bf16"):
    """Work items as the CTAs run them.  A plan of the 64-row MLA kernel (kernel 14), or of the
    e4m3 MLA kernels (12 / 13), lists query tile 0 of each piece only: the CTAs of a slice's group
    take query tile t = 0 .. q_len / q_tile - 1 by shifting the item's rows by t * q_tile and its
    partial rows by t * q_tile * part_stride (every head group of a tile runs the same rows).
    Returns (items, CTAs per slice)."""
    w, _ = _items(plan)
    rows = {12: 16, 13: 32, 14: 64}.get(plan.info.kernel, 0)
    if not (plan.info.kernel == 14 or (rows and kv_dtype == "e4m3")):
        return w, 1
    q_len = int(qo[1] - qo[0]) if len(qo) > 1 else 0
    qt_count = q_len // plan.info.q_tile
    assert q_len == qt_count * plan.info.q_tile and np.all(np.diff(qo) == q_len)
    out = []
    for row in w.tolist():
        r, qs, qc, pb, pe, prow, pstride, j = row
        assert qs == qo[r] and qc == plan.info.q_tile   # query tile 0 of the request
        for t in range(qt_count):
            out.append([r, qs + t * qc, qc, pb, pe, prow + t * qc * pstride if prow >= 0 else prow, pstride, j])
    group = qt_count * (num_heads // rows if num_heads > rows else 1)
    return np.array(out, dtype=np.int64).reshape(-1, 8), group


def _check(plan, qo, n_pages, num_heads=0, kv_dtype="bf16"):
    info = plan.info
    w, group = _grouped(plan, qo, num_heads, kv_dtype)
    _, m = _items(plan)
    B = len(n_pages)
    part_owner = {}
    direct = {}
    spans = {}
    for r, qs, qc, pb, pe, prow, pstride, j in w.tolist():
        assert 0 <= r < B and qc >= 1 and qo[r] <= qs and qs + qc <= qo[r + 1], (r, qs, qc)
        assert 0 <= pb <= pe <= n_pages[r]
        for i in range(qc):
            row = qs + i
            spans.setdefault(row, []).append((j, pb, pe))
            if prow < 0:
                assert row not in direct, f"row {row} written directly twice"
                direct[row] = True
            else:
                p = prow + i * pstride
                assert 0 <= p < info.num_partial_rows and p not in part_owner, (row, p)
                part_owner[p] = row
    merged = {}
    for out_row, sb, sc, _ in m.tolist():
        assert out_row not in merged and out_row not in direct
        assert sorted(p for p, row in part_owner.items() if row == out_row) == list(range(sb, sb + sc))
        merged[out_row] = sc
    assert len(part_owner) == sum(merged.values()) == info.num_partial_rows
    for r in range(B):
        for row in range(qo[r], qo[r + 1]):
            assert (row in direct) != (row in merged), f"row {row}: direct and merged, or neither"
            sp = sorted(spans[row])
            assert [j for j, _, _ in sp] == list(range(len(sp)))
            assert sp[0][1] == 0 and sp[-1][2] == n_pages[r]
            assert all(sp[k][2] == sp[k + 1][1] for k in range(len(sp) - 1))
    if info.num_ctas:
        assert info.num_ctas % group == 0
        cta = plan.words[info.cta_offset: info.cta_offset + info.num_ctas // group + 1]
        assert cta[0] == 0 and cta[-1] == info.num_work and np.all(np.diff(cta) >= 0)
        assert info.cta_offset + info.num_ctas // group + 1 == info.plan_words


def _random_table(rng, P, max_len, q_max):
    B = int(rng.integers(1, 30))
    lengths = rng.integers(0, max_len + 1, size=B)
    lengths[rng.random(B) < 0.15] = 0
    q_lens = rng.integers(0, q_max + 1, size=B)
    kv_indptr, kv_indices, last, _ = build_page_table(rng, lengths.tolist(), P, extra_pages=0)
    return q_lens, kv_indptr, last


def _policy(rng, n_pages):
    kind = rng.choice(["none", "fixed", "balanced", "balanced_small", "explicit"])
    if kind == "fixed":
        return "fixed", int(rng.integers(1, 6)), None
    if kind == "balanced":
        return "balanced", 148, None
    if kind == "balanced_small":
        return "balanced", int(rng.integers(1, 40)), None
    if kind == "explicit":
        sps = []
        for n in n_pages:
            k = int(rng.integers(1, 4))
            cuts = np.sort(rng.integers(0, n + 1, size=k - 1)) if n >= 0 else []
            sps.append([0, *[int(x) for x in cuts], int(n)])
        return "explicit", 0, sps
    return "none", 0, None


@pytest.mark.parametrize("seed", range(12))
def test_paged_plans(seed):
    rng = np.random.Generator(np.random.PCG64(1000 + seed))
    for _ in range(15):
        hq, hk, d = [(64, 8, 128), (32, 8, 128), (8, 2, 64), (16, 4, 128), (8, 8, 64)][int(rng.integers(0, 5))]
        P = int(rng.choice([1, 4, 16, 64]))
        q_max = int(rng.choice([1, 4, 40, 200]))
        q_lens, kv_indptr, last = _random_table(rng, P, 3000, q_max)
        qo = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
        n_pages = np.diff(kv_indptr)
        policy, param, sps = _policy(rng, n_pages)
        plan = skv.plan_paged(qo, kv_indptr, last, P, hq, hk, d, policy, param, sps)
        _check(plan, qo, n_pages)


@pytest.mark.parametrize("seed", range(12))
def test_mla_plans(seed):
    rng = np.random.Generator(np.random.PCG64(2000 + seed))
    for _ in range(15):
        H = int(rng.choice([16, 32, 64, 128]))
        q_len = int(rng.integers(1, 5))
        P = int(rng.choice([1, 4, 16, 64, 128]))
        kv_dtype = str(rng.choice(["bf16", "e4m3"]))
        _, kv_indptr, last = _random_table(rng, P, 5000, 1)
        B = len(kv_indptr) - 1
        qo = (np.arange(B + 1) * q_len).astype(np.int32)
        n_pages = np.diff(kv_indptr)
        policy, param, sps = _policy(rng, n_pages)
        plan = skv.plan_mla(q_len, kv_indptr, last, P, H, policy, param, sps, kv_dtype=kv_dtype)
        _check(plan, qo, n_pages, H, kv_dtype)


@pytest.mark.parametrize("seed", range(8))
def test_paged_subset_plans(seed):
    """A plan for a subset of the requests covers exactly those requests' query rows (pages once per
    split, partials consistent) and nothing of the others; two complementary subsets together
    cover the batch."""
    rng = np.random.Generator(np.random.PCG64(3000 + seed))
    for _ in range(12):
        hq, hk, d = [(64, 8, 128), (32, 8, 128), (8, 2, 64)][int(rng.integers(0, 3))]
        P = int(rng.choice([1, 16, 64]))
        q_lens, kv_indptr, last = _random_table(rng, P, 2000, int(rng.choice([1, 8, 130])))
        B = len(q_lens)
        qo = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
        n_pages = np.diff(kv_indptr)
        chosen = rng.random(B) < 0.5
        policy = str(rng.choice(["none", "fixed", "balanced"]))
        param = {"none": 0, "fixed": int(rng.integers(1, 4)), "balanced": 148}[policy]
        covered = np.zeros(int(qo[-1]), bool)
        for subset in (np.flatnonzero(chosen), np.flatnonzero(~chosen)):
            plan = skv.plan_paged_subset(qo, kv_indptr, last, P, hq, hk, d, subset, policy, param)
            w, _ = _items(plan)
            assert set(w[:, 0].tolist()) <= set(subset.tolist())
            # rows of the other requests must not appear: check against a table where they are empty
            keep = np.zeros(B, bool)
            keep[subset] = True
            rows_sub = np.concatenate([np.arange(qo[r], qo[r + 1]) for r in subset] + [np.zeros(0, int)])
            _check_subset(plan, qo, n_pages, keep)
            assert not covered[rows_sub].any()
            covered[rows_sub] = True
        assert covered.all()


def _check_subset(plan, qo, n_pages, keep):
    """_check restricted to the requests in ``keep``: the others must have no rows at all."""
    w, m = _items(plan)
    for r, qs, qc, *_ in w.tolist():
        assert keep[r] and qo[r] <= qs and qs + qc <= qo[r + 1]
    q2 = [0]
    for r in range(len(n_pages)):
        q2.append(q2[-1] + (qo[r + 1] - qo[r] if keep[r] else 0))
    # rebase the plan's rows onto the kept requests only, then run the full check on that table
    shift = {}
    for r in range(len(n_pages)):
        shift[r] = q2[r] - qo[r]
    w2 = w.copy()
    for row in w2:
        row[1] += shift[int(row[0])]
    m2 = m.copy()
    row_req = np.searchsorted(qo, np.arange(qo[-1]), side="right") - 1
    for row in m2:
        row[0] += shift[int(row_req[row[0]])]
    words = plan.words.copy()
    words[: w2.size] = w2.reshape(-1)
    words[w2.size: w2.size + m2.size] = m2.reshape(-1)
    _check(skv.Plan(words, plan.info), np.asarray(q2), np.where(keep, n_pages, 0))
