"""The seeded input generators shared by the oracle and the CUDA path (no GPU): draws independent
of the thread count, distinct streams, page tables that are permutations with the documented
lengths, and bf16 rounding to nearest even (torch's cast as the reference)."""
import numpy as np
import torch

from workloads import build_page_table, f32_to_bf16_bits, fetch_splice_case, normal_f32
from workloads.gen import _CHUNK


def test_draws_do_not_depend_on_the_thread_count():
    n = 2 * _CHUNK + 12345
    a = normal_f32(3, 1, n, threads=1)
    b = normal_f32(3, 1, n, threads=8)
    assert np.array_equal(a, b)
    assert not np.array_equal(a[:1000], normal_f32(3, 2, 1000))        # another stream
    assert not np.array_equal(a[:1000], normal_f32(4, 1, 1000))        # another seed
    assert abs(float(a.mean())) < 0.01 and abs(float(a.std()) - 1.0) < 0.01


def test_page_table_is_a_permutation_with_the_documented_lengths():
    rng = np.random.Generator(np.random.PCG64(9))
    lengths = [0, 1, 15, 16, 17, 1000, 0, 64]
    for P in (1, 16, 64):
        kv_indptr, kv_indices, last, num_pages = build_page_table(rng, lengths, P, extra_pages=5)
        n = np.diff(kv_indptr)
        assert np.array_equal(n, [(L + P - 1) // P for L in lengths])
        assert num_pages == int(n.sum()) + 5
        assert len(np.unique(kv_indices)) == len(kv_indices) and kv_indices.min() >= 0
        assert kv_indices.max() < num_pages
        for L, nr, lr in zip(lengths, n, last):
            assert (lr == 0) if nr == 0 else (1 <= lr <= P and (nr - 1) * P + lr == L)


def test_bf16_rounding_is_nearest_even():
    rng = np.random.Generator(np.random.PCG64(10))
    x = np.concatenate([rng.standard_normal(100000) * 10.0 ** rng.integers(-6, 6, 100000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.0e38, -2.5e-38]]).astype(np.float32)
    # 1.00390625 and 1.01171875 are ties between two bf16 neighbours (round to the even one)
    got = f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).bfloat16().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


def test_fetch_splice_case_moves_every_chunk_once():
    c = fetch_splice_case(num_chunks=5, chunk_tokens=100, src_page_size=16, dst_page_size=32, context=7, seed=3)
    assert sorted(c.dst_start.tolist()) == [7 + 100 * i for i in range(5)]
    assert np.array_equal(c.src_start, np.arange(5) * 100)
    assert np.array_equal(c.delta, c.dst_start - c.src_start)
    assert len(np.unique(c.src_pages)) == len(c.src_pages) == c.src.shape[0]
    assert len(np.unique(c.dst_pages)) == len(c.dst_pages) and c.dst_pages.max() < c.dst_num_pages
    assert len(c.dst_pages) * c.dst_page_size >= 7 + 500
