"""Pins for the splice oracle (the fetch primitive's local compute), checked against things
other than itself:

* closed forms: quarter and half turns (a table of angles pi/2, pi, 0), and rotations by exactly
  one radian at the frequencies base^(-2i/64) whose period is a power of ten, checked against the
  printed textbook values of cos 1 and sin 1;
* the defining property of rotary position encodings: a query-key dot product depends only on
  the difference of their positions, so moving both by the same offset changes nothing;
* group structure: rotations compose, undo each other and keep every pair's length;
* the row move against a dense reshape of the pages built by the test itself, with token ids
  written into the rows;
* mutation tests: plausible mistakes planted in the oracle (on the CPU) must each fail a pin.
"""
import ast
import contextlib
import inspect
import math
import textwrap

import numpy as np
import pytest

import oracle.splice as OS
from workloads import f32_to_bf16_bits, normal_bf16

COS1 = 0.5403023058681398   # cos(1)
SIN1 = 0.8414709848078965   # sin(1)


def _rand(seed, shape):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape)


# ----------------------------------------------------------------------------- pins
def pin_quarter_half_turns():
    """Per-pair angle table: pair 5 turns by pi (both entries negate), pair 9 by pi/2
    ((a, b) -> (-b, a)), every other pair by 0.  Pair 5 is elements (10, 11) interleaved and
    (5, 37) in halves; pair 9 is (18, 19) and (9, 41)."""
    x = np.arange(1.0, 65.0)
    freq = np.zeros(32)
    freq[5] = math.pi
    freq[9] = math.pi / 2
    for layout, (a5, b5), (a9, b9) in (("interleaved", (10, 11), (18, 19)), ("halves", (5, 37), (9, 41))):
        want = x.copy()
        want[a5], want[b5] = -x[a5], -x[b5]
        want[a9], want[b9] = -x[b9], x[a9]
        np.testing.assert_allclose(OS.rerotate(x, 1, freq, layout), want, rtol=0, atol=1e-13)
        # three quarter turns the other way round equal one quarter turn
        got = OS.rerotate(x, -3, freq, layout)
        np.testing.assert_allclose(got[[a9, b9]], want[[a9, b9]], rtol=0, atol=1e-13)


def pin_one_radian():
    """base 10000: theta_i = 10^(-i/8), so pairs 0, 8, 16, 24 turn by exactly 1 rad when moved by
    1, 10, 100, 1000 positions: (1, 0) -> (cos 1, sin 1), (0, 1) -> (-sin 1, cos 1)."""
    freq = OS.rope_inv_freq(10000.0)
    for layout in ("interleaved", "halves"):
        a_idx, b_idx = (lambda i: 2 * i, lambda i: 2 * i + 1) if layout == "interleaved" else \
            (lambda i: i, lambda i: i + 32)
        for i, delta in ((0, 1), (8, 10), (16, 100), (24, 1000)):
            e_a = np.zeros(64); e_a[a_idx(i)] = 1.0
            e_b = np.zeros(64); e_b[b_idx(i)] = 1.0
            ra, rb = OS.rerotate(e_a, delta, freq, layout), OS.rerotate(e_b, delta, freq, layout)
            np.testing.assert_allclose([ra[a_idx(i)], ra[b_idx(i)]], [COS1, SIN1], rtol=0, atol=1e-12)
            np.testing.assert_allclose([rb[a_idx(i)], rb[b_idx(i)]], [-SIN1, COS1], rtol=0, atol=1e-12)
            assert np.count_nonzero(np.abs(ra) > 1e-15) == 2


def pin_relative_position():
    """q at position a and k at position b score the same as q at a + c and k at b + c, and
    differently once a - b changes (so the rotation is not the identity)."""
    freq = OS.rope_inv_freq(10000.0)
    q, k = _rand(1, 64), _rand(2, 64)
    for layout in ("interleaved", "halves"):
        for a, b, c in ((0, 0, 17), (5, 123, 4096), (70000, 3, -65000)):
            s0 = OS.rerotate(q, a, freq, layout) @ OS.rerotate(k, b, freq, layout)
            s1 = OS.rerotate(q, a + c, freq, layout) @ OS.rerotate(k, b + c, freq, layout)
            assert abs(s0 - s1) <= 1e-10 * (1 + abs(s0))
            s2 = OS.rerotate(q, a + 1, freq, layout) @ OS.rerotate(k, b, freq, layout)
            assert abs(s2 - s0) > 1e-6


def pin_group():
    """rotate(rotate(x, a), b) = rotate(x, a + b); rotate(., -d) undoes rotate(., d); pair
    lengths are kept."""
    x = _rand(3, (5, 64))
    for layout, freq in (("interleaved", OS.rope_inv_freq(10000.0)), ("halves", OS.rope_inv_freq(500000.0))):
        a_idx, b_idx = OS.rope_pairs(layout)
        r = OS.rerotate(x, 777, freq, layout)
        np.testing.assert_allclose(OS.rerotate(r, -1234, freq, layout), OS.rerotate(x, -457, freq, layout),
                                   rtol=0, atol=1e-12)
        np.testing.assert_allclose(OS.rerotate(r, -777, freq, layout), x, rtol=0, atol=1e-12)
        np.testing.assert_allclose(np.hypot(r[:, a_idx], r[:, b_idx]), np.hypot(x[:, a_idx], x[:, b_idx]),
                                   rtol=1e-13, atol=0)
        assert np.max(np.abs(r - x)) > 0.1


def _ids_cache(num_pages, P, seed):
    """Latent cache whose ckv[..., 0] holds (page * P + slot) exactly (bf16 integers < 256)."""
    ckv = normal_bf16(seed, 1, (num_pages, P, 512)).copy()
    kpe = normal_bf16(seed, 2, (num_pages, P, 64))
    ids = np.arange(num_pages * P, dtype=np.float32).reshape(num_pages, P)
    ckv[..., 0] = f32_to_bf16_bits(ids)
    return ckv, kpe


def pin_row_move():
    """Source tokens [3, 24) of a 4-token-page list land at positions [5, 26) of an 8-token-page
    list; the test forms the logical rows by reshaping the gathered pages itself."""
    Ps, Pd, n, s0, d0 = 4, 8, 21, 3, 5
    ckv, kpe = _ids_cache(12, Ps, 7)
    rng = np.random.Generator(np.random.PCG64(8))
    src_pages = rng.permutation(12)[:7]
    dst_pages = rng.permutation(9)[:4] + 100
    freq = OS.rope_inv_freq(10000.0)
    dp, ds, c, kr = OS.splice_rows(ckv, kpe, src_pages, s0, dst_pages, Pd, d0, n, 0, freq)
    dense_ckv = ckv[src_pages].reshape(-1, 512)[s0:s0 + n]
    dense_kpe = kpe[src_pages].reshape(-1, 64)[s0:s0 + n]
    ids = (src_pages[:, None] * Ps + np.arange(Ps)).reshape(-1)[s0:s0 + n]
    np.testing.assert_array_equal(c[:, 0], ids)
    np.testing.assert_array_equal(f32_to_bf16_bits(c.astype(np.float32)), dense_ckv)
    np.testing.assert_array_equal(f32_to_bf16_bits(kr.astype(np.float32)), dense_kpe)  # delta 0: unchanged
    pos = np.arange(d0, d0 + n)
    np.testing.assert_array_equal(dp, dst_pages[pos // Pd])
    np.testing.assert_array_equal(ds, pos % Pd)
    # a moved chunk: rope rows are the dense rows turned by delta, the latent untouched
    dp2, ds2, c2, kr2 = OS.splice_rows(ckv, kpe, src_pages, s0, dst_pages, Pd, d0, n, 4096, freq, "halves")
    np.testing.assert_array_equal(c2, c)
    np.testing.assert_array_equal(dp2, dp)
    np.testing.assert_array_equal(ds2, ds)
    x = dense_kpe.astype(np.uint32) << np.uint32(16)
    x = x.view(np.float32).astype(np.float64)
    back = OS.rerotate(kr2, -4096, freq, "halves")
    np.testing.assert_allclose(back, x, rtol=0, atol=1e-12)
    assert np.max(np.abs(kr2 - x)) > 0.1


PINS = [pin_quarter_half_turns, pin_one_radian, pin_relative_position, pin_group, pin_row_move]


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
    """Re-define oracle.splice.<func_name> with ``old`` replaced by ``new`` in its source."""
    fn = getattr(OS, func_name)
    src = textwrap.dedent(inspect.getsource(fn))
    assert old in src, (func_name, old)
    ns = OS.__dict__
    exec(compile(src.replace(old, new, 1), OS.__file__, "exec"), ns)
    try:
        assert _code_signature(src.replace(old, new, 1)) != _code_signature(src), \
            f"mutation of {func_name} changes no code"
        yield
    finally:
        ns[func_name] = fn


MUTATIONS = [
    ("rope_inv_freq", "-2.0 * i / rope_dim", "-1.0 * i / rope_dim"),
    ("rope_inv_freq", "-2.0 * i / rope_dim", "-2.0 * (i + 1) / rope_dim"),
    ("rope_pairs", "return 2 * i, 2 * i + 1", "return i, i + half"),
    ("rope_pairs", "return i, i + half", "return 2 * i, 2 * i + 1"),
    ("rerotate", "a * c - b * s", "a * c + b * s"),
    ("rerotate", "a * s + b * c", "-a * s + b * c"),
    ("rerotate", "np.float64(delta) *", "np.float64(-delta) *"),
    ("rerotate", "c, s = np.cos(ang), np.sin(ang)", "s, c = np.cos(ang), np.sin(ang)"),
    ("splice_rows", "ld % dst_page_size", "ld % ps"),
    ("splice_rows", "ls, ld = src_start + t, dst_start + t", "ls, ld = src_start + t, dst_start + t + 1"),
    ("splice_rows", "sp, ss = int(src_pages[ls // ps]), ls % ps", "sp, ss = int(src_pages[ls // ps]), t % ps"),
]


@pytest.mark.parametrize("mut", MUTATIONS, ids=lambda m: f"{m[0]}:{m[2][:24]}")
def test_mutation_is_caught(mut):
    caught = []
    with _mutated(*mut):
        for pin in PINS:
            try:
                pin()
            except (AssertionError, ValueError, IndexError):
                caught.append(pin.__name__)
    assert caught, f"no pin catches mutation {mut}"
