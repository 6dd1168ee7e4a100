"""The e4m3 MLA kernel multiplies bf16 queries by the fp8 cache as two e4m3 terms: after a
power-of-two scaling that puts the unit's largest |q| in [128, 256), hi = e4m3(q) and
lo = e4m3(q - hi), both rounded to nearest even (in the kernel, fp32 values and the hardware's
satfinite conversion; here torch's float8_e4m3fn cast).  This pins the accuracy claim the kernel
design rests on:

* hi + lo reproduces q exactly whenever |q| >= 2^-9 of the unit's maximum (q's last bit is then no
  finer than the e4m3 subnormal step 2^-9 that lo can hold), and
* for every q the error is at most 2^-10 in scaled units (half that subnormal step), i.e. below
  2^-17 of the unit's maximum.

The bound 2^-9 is tight: 2^-10 of the maximum is not enough (checked below)."""
import numpy as np
import torch


def _split(q):
    """q: float64 bf16 values of one unit -> (scaled q, hi + lo), with the kernel's scaling."""
    m = float(np.max(np.abs(q)))
    e = 7 - int(np.floor(np.log2(m)))
    qs = torch.from_numpy(q * 2.0 ** e).float()                 # exact: bf16 x 2^e fits fp32
    hi = qs.to(torch.float8_e4m3fn).float()
    lo = (qs - hi).to(torch.float8_e4m3fn).float()              # qs - hi is exact in fp32
    return qs.double().numpy(), (hi.double() + lo.double()).numpy(), m, e


def _bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).bfloat16().double().numpy()


def test_every_bf16_value_below_the_unit_maximum():
    """All finite bf16 values of magnitude <= 255, in a unit whose maximum is 255 (scale 2^0)."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    v = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    v = v[np.isfinite(v) & (np.abs(v) <= 255.0)]
    q = np.concatenate([[255.0], v])
    qs, back, m, e = _split(q)
    assert e == 0
    big = np.abs(q) >= 2.0 ** -9 * m
    assert np.array_equal(back[big], qs[big])
    assert np.max(np.abs(back - qs)) <= 2.0 ** -10
    # the threshold cannot be lowered to 2^-10 of the maximum: some value there is not exact
    mid = (np.abs(q) >= 2.0 ** -10 * m) & ~big
    assert np.any(back[mid] != qs[mid])


def test_random_units_at_many_scales():
    rng = np.random.Generator(np.random.PCG64(7))
    for _ in range(500):
        x = rng.standard_normal(576) * 2.0 ** int(rng.integers(-30, 30))
        q = _bf16(x)
        qs, back, m, e = _split(q)
        assert 128.0 <= np.max(np.abs(qs)) < 256.0
        big = np.abs(q) >= 2.0 ** -9 * m
        assert np.array_equal(back[big], qs[big])
        assert np.max(np.abs(back - qs)) <= 2.0 ** -10
        assert np.max(np.abs(back - qs)) / np.max(np.abs(qs)) <= 2.0 ** -17


def test_softmax_weights_keep_eight_bits():
    """Softmax weights p in [0, 2^8] (fp32, not scaled) split the same way: relative error at most
    2^-8 from 2^-2 up (lo normal), absolute error at most 2^-10 below (lo on the subnormal grid)."""
    rng = np.random.Generator(np.random.PCG64(8))
    p = torch.from_numpy(np.concatenate([rng.random(200000) * 256.0, 2.0 ** rng.uniform(-20, 8, 200000),
                                         [0.0, 1.0, 256.0]]).astype(np.float32))
    hi = p.to(torch.float8_e4m3fn).float()
    lo = (p - hi).to(torch.float8_e4m3fn).float()
    err = (hi.double() + lo.double() - p.double()).abs()
    normal = p >= 0.25
    assert bool(torch.all(err[normal] <= 2.0 ** -8 * p[normal].double()))
    assert float(err[~normal].max()) <= 2.0 ** -10
