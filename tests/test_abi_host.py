"""Host-side checks of the C ABI (no GPU): the library loads and exports every declared symbol,
the planner lays out splits / partial rows / merges as documented, and argument validation
returns its error codes before anything is launched."""
import ctypes
import os
import re
import shutil
import subprocess

import numpy as np
import pytest

import split_kv_merge_b200 as skv
from workloads import even_split_pages, llama70b_decode_case, tiny_gqa_case

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"SKV_API\s+[\w\s\*]+?\b(skv_\w+)\s*\(", src))
    return names


def test_library_exports_every_declared_symbol():
    declared = _declared_symbols()
    assert len(declared) >= 9
    lib = ctypes.CDLL(skv.library_path())
    for name in declared:
        assert hasattr(lib, name), name
    assert set(skv.SYMBOLS) <= declared


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs a C compiler")
def _scratch_dir():
    """Build products of the C tests go to the repository's ignored build folder."""
    d = os.path.join(ROOT, "_build", "c_tests")
    os.makedirs(d, exist_ok=True)
    return d


def test_binding_structs_match_the_c_header():
    """Every ctypes structure of the binding has the size, field offsets and field sizes of the C
    struct it mirrors (compiled from include/splitkv.h with gcc)."""
    pairs = [(skv.PlanInfo, "skv_plan_info"), (skv.PagedParams, "skv_paged_params"),
             (skv.MlaParams, "skv_mla_params"), (skv.SpliceParams, "skv_splice_params"),
             (skv.SpliceChunk, "skv_splice_chunk")]
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "splitkv.h"', "int main(void) {"]
    for cls, cname in pairs:
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for field, _ in cls._fields_:
            lines.append(f'  printf("{cname} {field} %zu %zu\\n", offsetof({cname}, {field}), '
                         f'sizeof((({cname}*)0)->{field}));')
    lines += ["  return 0;", "}"]
    src = os.path.join(_scratch_dir(), "layout.c")
    with open(src, "w") as f:
        f.write("\n".join(lines) + "\n")
    exe = os.path.join(_scratch_dir(), "layout")
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), src, "-o", exe], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    c_layout = {tuple(l.split()[:2]): [int(x) for x in l.split()[2:]] for l in out if l.strip()}
    for cls, cname in pairs:
        assert c_layout[(cname, "size")] == [ctypes.sizeof(cls)], cname
        for field, _ in cls._fields_:
            desc = getattr(cls, field)
            assert c_layout[(cname, field)] == [desc.offset, desc.size], (cname, field)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs a C compiler")
def test_plain_c_consumer():
    """tests/c/host_calls.c, compiled against include/splitkv.h and linked to libsplitkv.so, runs the
    host-only entry points from C (planners, causal planner, validation, status strings)."""
    lib_dir = os.path.dirname(skv.library_path())
    exe = os.path.join(_scratch_dir(), "host_calls")
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "host_calls.c"),
                    "-L", lib_dir, "-lsplitkv", f"-Wl,-rpath,{lib_dir}", "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stderr


def test_version_and_status_strings():
    assert skv.version() >= 1
    assert skv.status_str(0) == "ok"
    for code in (1, 2, 3, 4, 5, 16, 17, 18):
        assert skv.status_str(code) != "unknown status"


@pytest.mark.parametrize("H,q_len,F", [(16, 1, 1), (16, 4, 4), (128, 1, 1), (128, 4, 1), (32, 4, 4),
                                       (64, 4, 2), (48, 6, 2), (16, 16, 8), (1, 3, 3)])
def test_mla_fold_ratio(H, q_len, F):
    # largest divisor F of q_len with H * F <= 128
    assert skv.mla_fold_ratio(H, q_len, 128) == F


def _items(plan):
    nw, nm = plan.info.num_work, plan.info.num_merge_rows
    w = plan.words[: 8 * nw].reshape(-1, 8)
    m = plan.words[8 * nw: 8 * nw + 4 * nm].reshape(-1, 4)
    return w, m


def test_tiny_fixed_two_splits_layout():
    c = tiny_gqa_case()
    plan = skv.plan_paged(c.qo_indptr, c.kv_indptr, c.kv_last_page_len, 16, 8, 2, 64, "fixed", 2)
    w, m = _items(plan)
    info = plan.info
    assert info.num_work == 8 and info.max_splits == 2 and info.total_splits == 8
    assert info.num_partial_rows == 8 and info.num_merge_rows == 4
    # splits (2,1), (4,4), (7,6), (8,8) pages, ceil first
    by_req = {}
    for r, qs, qc, pb, pe, prow, pstride, j in w:
        by_req.setdefault(int(r), {})[int(j)] = (int(pb), int(pe), int(prow), int(pstride))
    assert [by_req[r][0][1] - by_req[r][0][0] for r in range(4)] == [2, 4, 7, 8]
    assert [by_req[r][1][1] - by_req[r][1][0] for r in range(4)] == [1, 4, 6, 8]
    for r in range(4):
        assert by_req[r][0][2] + 1 == by_req[r][1][2]   # partial rows part_base + j
        assert by_req[r][0][3] == 2
    # merge items: out_row r, states [2r, 2r+2)
    assert sorted(map(tuple, m[:, :3].tolist())) == [(r, 2 * r, 2) for r in range(4)]
    # equals the generator's ceil-first split
    assert [[0, by_req[r][0][1], by_req[r][1][1]] for r in range(4)] == even_split_pages(c.kv_indptr, 2)


def test_plan_explicit_and_empty_splits():
    kv_indptr = np.array([0, 3, 3, 8], np.int32)
    last = np.array([5, 0, 16], np.int32)
    qo = np.array([0, 2, 3, 4], np.int32)
    sps = [[0, 0, 2, 3], [0, 0], [0, 5]]
    plan = skv.plan_paged(qo, kv_indptr, last, 16, 4, 2, 128, "explicit", 0, sps)
    w, m = _items(plan)
    assert plan.info.num_partial_rows == 2 * 3   # request 0: 2 query tokens x 3 splits
    assert plan.info.num_merge_rows == 2
    r0 = w[w[:, 0] == 0]
    assert sorted(r0[:, 7].tolist()) == [0, 1, 2]
    # query token i, split j -> row i*S + j
    for row in r0:
        assert row[5] == 0 * 3 + row[7] and row[6] == 3
    # request with no pages still gets a work item (writes O=0, LSE=-inf)
    r1 = w[w[:, 0] == 1]
    assert len(r1) == 1 and r1[0, 3] == 0 and r1[0, 4] == 0 and r1[0, 5] == -1


def test_plan_balanced_covers_every_page_once():
    """Balanced plan for the persistent all-heads decode kernel: every page of every request is in
    exactly one work item, and the CTAs' costs (16-token tiles plus three tiles per work item, the
    planner's charge for a work item's start and end) are equal up to one small piece; no CTA is
    far above the mean (the last one takes what remains, so it may fall a little further below)."""
    c = llama70b_decode_case(batch=64)
    plan = skv.plan_paged(c.qo_indptr, c.kv_indptr, c.kv_last_page_len, 16, 64, 8, 128, "balanced", 148)
    info = plan.info
    w, m = _items(plan)
    n = np.diff(c.kv_indptr)
    for r in range(64):
        rows = w[w[:, 0] == r]
        spans = sorted((int(a), int(b)) for a, b in rows[:, 3:5])
        assert spans[0][0] == 0 and spans[-1][1] == n[r]
        assert all(spans[i][1] == spans[i + 1][0] for i in range(len(spans) - 1))
    assert info.num_ctas == 148 and info.cta_offset == 8 * info.num_work + 4 * info.num_merge_rows
    cta = plan.words[info.cta_offset: info.cta_offset + info.num_ctas + 1]
    assert cta[0] == 0 and cta[-1] == info.num_work and np.all(np.diff(cta) >= 1)
    L = c.kv_lengths()
    tiles = np.array([sum(-(-(min(b * 16, L[r]) - a * 16) // 16) for r, _, _, a, b, *_ in w[cta[i]:cta[i + 1]])
                      for i in range(info.num_ctas)])
    assert tiles.sum() == np.sum(-(-L // 16))
    cost = tiles + 3 * np.diff(cta)
    assert cost.max() <= cost.mean() + 5 and cost.min() >= cost.mean() - 10
    assert info.total_splits < 64 + 2 * 148       # each CTA boundary cuts at most one request


def test_plan_persistent_fixed_assigns_longest_first():
    c = llama70b_decode_case(batch=16)
    plan = skv.plan_paged(c.qo_indptr, c.kv_indptr, c.kv_last_page_len, 16, 64, 8, 128, "fixed", 3)
    info = plan.info
    assert info.num_ctas == min(148, info.num_work)
    cta = plan.words[info.cta_offset: info.cta_offset + info.num_ctas + 1]
    assert cta[-1] == info.num_work


@pytest.mark.parametrize("bad", ["last_zero", "last_big", "hq_not_multiple", "head_dim", "indptr_decreasing",
                                 "explicit_bad_end", "fixed_zero"])
def test_plan_rejects_bad_input(bad):
    kv_indptr = np.array([0, 2, 5], np.int32)
    last = np.array([3, 16], np.int32)
    qo = np.array([0, 1, 2], np.int32)
    args = dict(hq=8, hk=2, d=64, policy="none", param=0, sps=None)
    if bad == "last_zero":
        last = np.array([0, 16], np.int32)
    elif bad == "last_big":
        last = np.array([17, 16], np.int32)
    elif bad == "hq_not_multiple":
        args["hq"] = 6; args["hk"] = 4
    elif bad == "head_dim":
        args["d"] = 96
    elif bad == "indptr_decreasing":
        kv_indptr = np.array([0, 2, 1], np.int32)
    elif bad == "explicit_bad_end":
        args["policy"] = "explicit"; args["sps"] = [[0, 1], [0, 2]]
    elif bad == "fixed_zero":
        args["policy"] = "fixed"
    with pytest.raises(skv.SkvError) as e:
        skv.plan_paged(qo, kv_indptr, last, 16, args["hq"], args["hk"], args["d"], args["policy"], args["param"],
                       args["sps"])
    assert e.value.code in (skv.ERR_INVALID, skv.ERR_UNSUPPORTED)


def test_launch_validation_returns_before_launch():
    """Invalid arguments come back as status codes without touching the GPU (the pointers here
    are never dereferenced)."""
    info = skv.PlanInfo()
    info.num_work, info.q_tile, info.kernel = 1, 1, 1
    p = skv.PagedParams()
    fake = 1 << 20  # 16-byte aligned, never dereferenced
    p.q = p.k_cache = p.v_cache = p.kv_indptr = p.kv_indices = p.kv_last_page_len = p.o = fake
    for i in range(3):
        p.k_stride[i] = p.v_stride[i] = [2048, 128, 64][i]
    p.batch, p.total_q, p.num_pages, p.page_size = 1, 1, 4, 16
    p.num_qo_heads, p.num_kv_heads, p.head_dim, p.sm_scale = 8, 2, 64, 0.125
    fwd = skv._paged_fwd

    def call(**kw):
        q = skv.PagedParams.from_buffer_copy(p)
        for k, v in kw.items():
            setattr(q, k, v)
        return fwd(ctypes.byref(q), fake, ctypes.byref(info), None)

    assert call(head_dim=96) == skv.ERR_UNSUPPORTED
    assert call(num_qo_heads=6, num_kv_heads=4) == skv.ERR_INVALID
    assert call(o=None) == skv.ERR_INVALID
    assert call(q=fake + 2) == skv.ERR_ALIGNMENT
    assert call(o_dtype=7) == skv.ERR_UNSUPPORTED
    bad = skv.PagedParams.from_buffer_copy(p)
    bad.k_stride[1] = 100   # not a multiple of 8 elements
    assert fwd(ctypes.byref(bad), fake, ctypes.byref(info), None) == skv.ERR_ALIGNMENT
    info2 = skv.PlanInfo.from_buffer_copy(info)
    info2.num_partial_rows = 4     # plan splits but no partial buffers given
    assert fwd(ctypes.byref(p), fake, ctypes.byref(info2), None) == skv.ERR_WORKSPACE
    assert fwd(None, fake, ctypes.byref(info), None) == skv.ERR_INVALID
    assert fwd(ctypes.byref(p), None, ctypes.byref(info), None) == skv.ERR_INVALID
    # merge_states validation
    assert skv._merge(fake, fake, None, -1, 4, 8, 64, fake, 1, None, None) == skv.ERR_INVALID
    assert skv._merge(fake, fake, None, 2, 4, 8, 62, fake, 1, None, None) == skv.ERR_UNSUPPORTED
    assert skv._merge(fake, fake, None, 2, 4, 70000, 64, fake, 1, None, None) == skv.ERR_UNSUPPORTED
    assert skv._merge(fake, fake, None, 2, 0, 8, 64, fake, 1, None, None) == skv.OK   # nothing to do


def test_mla_validation():
    info = skv.PlanInfo()
    info.num_work, info.q_tile, info.kernel = 1, 1, 11
    p = skv.MlaParams()
    fake = 1 << 20
    p.q_nope = p.q_pe = p.ckv = p.kpe = p.kv_indptr = p.kv_indices = p.kv_last_page_len = p.o = fake
    p.ckv_stride[0], p.ckv_stride[1] = 64 * 576, 576
    p.kpe_stride[0], p.kpe_stride[1] = 64 * 576, 576
    p.batch, p.q_len, p.num_heads, p.num_pages, p.page_size, p.sm_scale = 1, 1, 16, 4, 64, 0.07
    fwd = skv._mla_fwd

    def call(**kw):
        q = skv.MlaParams.from_buffer_copy(p)
        for k, v in kw.items():
            setattr(q, k, v)
        return fwd(ctypes.byref(q), fake, ctypes.byref(info), None)

    assert call(kv_dtype=5) == skv.ERR_UNSUPPORTED
    assert call(kv_dtype=skv.E4M3, kv_scale=0.0) == skv.ERR_INVALID
    assert call(q_len=0) == skv.ERR_INVALID
    assert call(kpe=fake + 8) == skv.ERR_ALIGNMENT
    bad = skv.MlaParams.from_buffer_copy(p)
    bad.ckv_stride[1] = 577
    assert fwd(ctypes.byref(bad), fake, ctypes.byref(info), None) == skv.ERR_ALIGNMENT


def test_empty_plans_launch_nothing():
    """A batch without requests, or without query rows, plans no work; the launches then return OK
    without touching the device (so this runs on a machine without a GPU)."""
    fake = 1 << 20
    for qo, ip, la in (([0], [0], []), ([0, 0, 0], [0, 2, 3], [5, 16])):
        plan = skv.plan_paged(np.array(qo), np.array(ip), np.array(la), 16, 64, 8, 128, "balanced", 148)
        assert plan.info.num_work == 0 and plan.info.num_merge_rows == 0
        p = skv.PagedParams()
        p.q = p.k_cache = p.v_cache = p.kv_indptr = p.kv_indices = p.kv_last_page_len = p.o = fake
        for i in range(3):
            p.k_stride[i] = p.v_stride[i] = [16 * 8 * 128, 8 * 128, 128][i]
        p.batch, p.total_q, p.num_pages, p.page_size = len(ip) - 1, 0, 4, 16
        p.num_qo_heads, p.num_kv_heads, p.head_dim, p.sm_scale = 64, 8, 128, 0.088
        words = np.ascontiguousarray(plan.words)
        assert skv._paged_fwd(ctypes.byref(p), words.ctypes.data, ctypes.byref(plan.info), None) == skv.OK
    plan = skv.plan_mla(1, np.array([0]), np.array([], np.int32), 64, 16, "balanced", 148)
    assert plan.info.num_work == 0
    m = skv.MlaParams()
    m.q_nope = m.q_pe = m.ckv = m.kpe = m.kv_indptr = m.kv_indices = m.kv_last_page_len = m.o = fake
    m.ckv_stride[0], m.ckv_stride[1] = 64 * 576, 576
    m.kpe_stride[0], m.kpe_stride[1] = 64 * 576, 576
    m.batch, m.q_len, m.num_heads, m.num_pages, m.page_size, m.sm_scale = 0, 1, 16, 4, 64, 0.07
    words = np.ascontiguousarray(plan.words)
    assert skv._mla_fwd(ctypes.byref(m), words.ctypes.data, ctypes.byref(plan.info), None) == skv.OK


def test_splice_validation():
    """skv_mla_splice rejects bad arguments before launching (pointers never dereferenced)."""
    fake = 1 << 20
    p = skv.SpliceParams()
    p.src_ckv = p.src_kpe = p.dst_ckv = p.dst_kpe = p.src_pages = p.dst_pages = fake
    p.src_ckv_stride[0], p.src_ckv_stride[1] = 64 * 576, 576
    p.src_kpe_stride[0], p.src_kpe_stride[1] = 64 * 576, 576
    p.dst_ckv_stride[0], p.dst_ckv_stride[1] = 16 * 512, 512
    p.dst_kpe_stride[0], p.dst_kpe_stride[1] = 16 * 64, 64
    p.src_num_pages, p.src_page_size, p.dst_num_pages, p.dst_page_size = 8, 64, 40, 16
    p.rope_theta = 10000.0
    good = [(0, 10, 100, 4096), (100, 300, 50, -7)]

    def call(chunks=good, **kw):
        q = skv.SpliceParams.from_buffer_copy(p)
        for k, v in kw.items():
            setattr(q, k, v)
        arr = skv.splice_chunks(chunks)
        return skv._splice(ctypes.byref(q), arr, arr._n, None)

    assert call([]) == skv.OK                          # nothing to move: no launch
    assert call([(0, 0, 0, 5), (3, 9, 0, 1)]) == skv.OK
    assert call([(0, 0, -1, 0)]) == skv.ERR_INVALID
    assert call([(0, -2, 4, 0)]) == skv.ERR_INVALID
    assert call([(2 ** 62, 0, 4, 0)]) == skv.ERR_INVALID
    assert call(dst_pages=None) == skv.ERR_INVALID
    assert call(src_page_size=0) == skv.ERR_INVALID
    assert call(rope_layout=2) == skv.ERR_INVALID
    assert call(rope_theta=0.0) == skv.ERR_INVALID
    assert call(rope_theta=float("inf")) == skv.ERR_INVALID
    assert call(kv_dtype=skv.E4M3) == skv.ERR_UNSUPPORTED
    assert call(dst_kpe=fake + 8) == skv.ERR_ALIGNMENT
    bad = skv.SpliceParams.from_buffer_copy(p)
    bad.dst_ckv_stride[1] = 516
    arr = skv.splice_chunks(good)
    assert skv._splice(ctypes.byref(bad), arr, 2, None) == skv.ERR_ALIGNMENT
    assert skv._splice(None, arr, 2, None) == skv.ERR_INVALID
    assert skv._splice(ctypes.byref(p), None, 2, None) == skv.ERR_INVALID
    assert skv._splice(ctypes.byref(p), arr, -1, None) == skv.ERR_INVALID


# ----------------------------------------------------------------------------- kernel choice
@pytest.mark.parametrize("hq,hk,q_len,page_size,kernel,q_tile", [
    (64, 8, 1, 16, 3, 1),     # Llama decode: all-KV-heads decode kernel
    (16, 4, 1, 32, 2, 1),     # 4 KV heads: per-head decode kernel (one token per unit)
    (32, 8, 128, 64, 4, 32),  # shared-KV prefill: 128-row prefill kernel, 128 / g tokens per unit
    (8, 8, 40, 128, 4, 128),  # g = 1 prefill with pages larger than a tile
    (32, 2, 9, 32, 4, 8),     # g = 16: 9 tokens x 16 heads > one decode tile
    (32, 8, 128, 4, 1, 4),    # page size 4 is below every tensor-core kernel: CUDA-core kernel
])
def test_paged_planner_kernel_choice(hq, hk, q_len, page_size, kernel, q_tile):
    """The planner's dispatch: which kernel a shape runs on and how many query tokens a unit holds."""
    n_req = 3
    qo = (np.arange(n_req + 1) * q_len).astype(np.int32)
    pages = np.array([5, 1, 9], np.int32)
    kv_indptr = np.concatenate([[0], np.cumsum(pages)]).astype(np.int32)
    last = np.full(n_req, page_size, np.int32)
    plan = skv.plan_paged(qo, kv_indptr, last, page_size, hq, hk, 128, "none", 0)
    assert plan.info.kernel == kernel and plan.info.q_tile == q_tile
    w, _ = _items(plan)
    assert np.all(w[:, 2] <= q_tile)                                    # q_count within the tile
    assert sorted(set(map(tuple, w[:, [0, 1]].tolist()))) == sorted(
        (r, int(qo[r]) + q0) for r in range(n_req) for q0 in range(0, q_len, q_tile))


@pytest.mark.parametrize("H,q_len,kv_dtype,page_size,kernel", [
    (16, 1, "bf16", 64, 12), (16, 4, "bf16", 64, 14), (128, 1, "bf16", 64, 14), (128, 4, "bf16", 64, 14),
    (16, 2, "bf16", 64, 13), (96, 1, "bf16", 64, 13),   # 32 rows; 96 heads are no multiple of 64
    (16, 4, "bf16", 1, 13),                              # page size 1 takes at most 32 rows
    (16, 1, "e4m3", 64, 12), (128, 4, "e4m3", 64, 13),   # native fp8 tensor-core kernel
    (128, 1, "e4m3", 64, 13), (16, 4, "e4m3", 64, 13),   # ... in CTA groups of 4 and 2 per KV slice
    (16, 1, "bf16", 1, 12),                              # page size 1: row gather on the tensor cores
    (16, 1, "e4m3", 1, 11),                              # e4m3 with page size 1: CUDA-core kernel
    (16, 1, "bf16", 4, 11),
])
def test_mla_planner_kernel_choice(H, q_len, kv_dtype, page_size, kernel):
    kv_indptr = np.array([0, 7, 7, 20], np.int32)
    last = np.array([page_size, 1, max(1, page_size // 2)], np.int32)
    plan = skv.plan_mla(q_len, kv_indptr, last, page_size, H, "balanced", 148, kv_dtype=kv_dtype)
    assert plan.info.kernel == kernel
    rows = {12: 16, 13: 32, 14: 64}.get(kernel, 128)
    assert plan.info.q_tile == (skv.mla_fold_ratio(H, q_len, rows) if H <= rows else 1)
    if kernel == 14 or (kernel in (12, 13) and kv_dtype == "e4m3"):
        # a group of (query tiles x head groups) CTAs per KV slice
        group = (q_len // plan.info.q_tile) * (H // rows if H > rows else 1)
        assert plan.info.num_ctas % group == 0 and 1 <= plan.info.num_ctas // group <= 148 // group
        w, _ = _items(plan)
        assert np.all(w[:, 1] % q_len == 0)   # the items stand for query tile 0 of each request


@pytest.mark.parametrize("H,q_len", [(16, 1), (16, 4), (128, 1), (128, 4)])
def test_mla_flat_plan_balances_tiles_and_pieces(H, q_len):
    """The persistent MLA plan charges every work item a fixed cost per query unit (head groups x
    query tiles) on top of its tiles -- two 64-token tiles on the bf16 16 / 32-row kernel, four on
    the 64-row kernel; per CTA, tiles + charges stay within a few tiles of the mean, every page of
    every request is covered once, and no CTA is left with the remainder of a degenerate cut."""
    from workloads import mla_decode_case
    c = mla_decode_case(H, q_len, "bf16")
    plan = skv.plan_mla(q_len, c.kv_indptr, c.kv_last_page_len, 64, H, "balanced", 148, kv_dtype="bf16")
    info = plan.info
    assert info.kernel in (12, 13, 14)
    rows = {12: 16, 13: 32, 14: 64}[info.kernel]
    hg = H // rows if H > rows else 1
    qt = -(-q_len // info.q_tile) * hg                       # query units per piece
    if info.kernel == 14:
        # grouped: each of the `qt` CTAs of a slice's group runs one query unit of every piece, so a
        # slice costs its tiles once per CTA; the items stand for query tile 0
        group, hg, qt = qt, 1, 1
        assert info.num_ctas == 148 // group * group
        q_len_eff = info.q_tile
    else:
        group, q_len_eff = 1, q_len
        assert info.num_ctas == 148
    slices = info.num_ctas // group
    w, _ = _items(plan)
    cta = plan.words[info.cta_offset: info.cta_offset + slices + 1]
    L = c.kv_lengths()
    n = np.diff(c.kv_indptr)
    cost = []
    for i in range(slices):
        items = w[cta[i]:cta[i + 1]]
        # work items of one request piece differ only by query tile: count pieces once
        pieces = {(int(r), int(a), int(b)) for r, _, _, a, b, *_ in items}
        tiles = sum(-(-(min(b * 64, L[r]) - a * 64) // 64) for r, a, b in pieces)
        charge = 4 if info.kernel == 14 else 2
        cost.append(hg * tiles * -(-q_len_eff // info.q_tile) + charge * qt * len(pieces))
    cost = np.array(cost)
    assert cost.max() <= cost.mean() + 8 * qt + 8 * hg, (cost.max(), cost.mean())
    for r in range(c.batch):
        spans = sorted({(int(a), int(b)) for rr, _, _, a, b, *_ in w if rr == r})
        assert spans[0][0] == 0 and spans[-1][1] == n[r]
        assert all(spans[i][1] == spans[i + 1][0] for i in range(len(spans) - 1))
