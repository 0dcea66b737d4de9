"""Two pieces of arithmetic the CUDA path relies on, checked on the host.

* The folded search adds |c~|^2 inside the MMAs as three bf16 parts (h, m, l):
  h = bf16(c), m = bf16(c - h), l = bf16(c - h - m), each remainder computed in
  fp32. The claim is that h + m + l equals the fp32 value c exactly, because each
  subtraction is exact (its operands are within a factor of two) and the last
  remainder has at most 8 significant bits. Checked here with torch's
  round-to-nearest-even bf16 conversion over fp32 values of every binade the
  norms can take.
* The donor draw compares non-negative doubles through their IEEE 754 encodings
  as signed 64-bit integers, and replaces a target on (or rounded past) the total
  W by the largest double below W: min(bits(tg), bits(W) - 1). Checked here: the
  encodings order as the values, bits(W) - 1 is the predecessor of W, and the min
  keeps tg whenever tg < W.
"""

import numpy as np
import torch


def _split3(c32: torch.Tensor):
    """The norms operand's three parts, as the kernel forms them (fp32 remainders)."""
    h = c32.to(torch.bfloat16)
    r1 = c32 - h.float()
    m = r1.to(torch.bfloat16)
    r2 = r1 - m.float()
    lo = r2.to(torch.bfloat16)
    return h, m, lo


def test_three_bf16_parts_carry_an_fp32_norm_exactly():
    g = torch.Generator().manual_seed(7)
    # magnitudes from 2^-100 to 2^100 (norms of real data sit far inside), plus
    # every mantissa pattern's neighbourhood of a few binades
    e = torch.randint(-100, 100, (200_000,), generator=g).float()
    mant = 1.0 + torch.rand(200_000, generator=g)
    c = (mant * torch.pow(2.0, e)).float()
    extra = torch.tensor([1.0, 1.0 + 2.0 ** -23, 2.0 - 2.0 ** -23, 3.0, 1e-30, 1e30, 0.0], dtype=torch.float32)
    c = torch.cat([c, extra])
    h, m, lo = _split3(c)
    total = h.double() + m.double() + lo.double()
    assert torch.equal(total, c.double())
    # each part is an exact bf16 value and the remainders shrink by 2^8 or more
    assert torch.all((m.double().abs() <= h.double().abs() * 2.0 ** -8) | (h == 0))
    assert torch.all((lo.double().abs() <= m.double().abs() * 2.0 ** -8) | (m == 0))


def test_non_finite_norm_goes_into_the_first_part():
    c = torch.tensor([float("inf")], dtype=torch.float32)
    h = c.to(torch.bfloat16)
    assert torch.isinf(h.float()).all()


def _bits(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).view(np.int64)


def test_ieee_encodings_order_non_negative_doubles():
    rng = np.random.default_rng(3)
    x = np.concatenate([
        rng.uniform(0.0, 1e6, 100_000),
        np.ldexp(rng.uniform(1.0, 2.0, 100_000), rng.integers(-1074, 1000, 100_000)),
        [0.0, 5e-324, 1e-308, 2.2250738585072014e-308, 1.0, np.inf],
    ])
    order_v = np.argsort(x, kind="stable")
    order_b = np.argsort(_bits(x), kind="stable")
    assert np.array_equal(x[order_v], x[order_b])
    a, b = x[:-1], x[1:]
    assert np.array_equal(a <= b, _bits(a) <= _bits(b))


def test_target_clamp_is_the_predecessor_of_the_total():
    rng = np.random.default_rng(5)
    W = np.concatenate([rng.uniform(1e-3, 1e9, 50_000), [5e-324, 1.0, 65536.0]])
    pred = (_bits(W) - 1).view(np.float64)
    assert np.array_equal(pred, np.nextafter(W, 0.0))
    u = rng.random(W.shape[0])
    tg = u * W
    clamped = np.minimum(_bits(tg), _bits(W) - 1)
    # tg < W: the clamp leaves the target as it is; tg >= W: the largest double below W
    keep = tg < W
    assert np.array_equal(clamped[keep], _bits(tg)[keep])
    assert np.array_equal(clamped[~keep], (_bits(W) - 1)[~keep])
    # "first position whose cumulative weight exceeds the clamped target" is then
    # the first that reaches W when the target was on the total
    cum = np.array([0.5, 1.0, 1.0, 3.0])
    Wc = cum[-1]
    t_on = Wc
    tb = min(_bits(np.array([t_on]))[0], _bits(np.array([Wc]))[0] - 1)
    first = int(np.sum(_bits(cum) <= tb))
    assert first == 3 and cum[first] == Wc
