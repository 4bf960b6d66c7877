"""Pins for the oracle's residual add x = RN16(h + d) (the binary16 addition
that produces the preparation operator's input in a pre-norm layer): every
finite binary16 round-trips through the oracle's nearest-binary16 encoder;
random operand bit patterns (subnormals, overflow) agree with numpy's float16
addition; hand-made ties go to the even neighbour and the overflow threshold
is exact."""
import numpy as np


def test_every_finite_half_round_trips(orc):
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    f = h.view(np.float16)
    fin = np.isfinite(f)
    for b in h[fin][::7].tolist() + [0x0000, 0x8000, 0x0001, 0x8001, 0x03FF, 0x0400, 0x7BFF, 0xFBFF]:
        assert orc.double_to_half(orc.half_to_double(b)) == b


def test_random_adds_match_numpy_float16(orc):
    rng = np.random.default_rng(11)
    h = rng.integers(0, 1 << 16, 400000, dtype=np.uint32).astype(np.uint16)
    d = rng.integers(0, 1 << 16, 400000, dtype=np.uint32).astype(np.uint16)
    # small magnitudes too: subnormal sums and cancellations
    h[:50000] &= 0x83FF
    d[:50000] &= 0x87FF
    ok = np.isfinite(h.view(np.float16)) & np.isfinite(d.view(np.float16))
    h, d = h[ok], d[ok]
    x = orc.add_fp16(h, d)
    with np.errstate(over="ignore"):
        ref = (h.view(np.float16) + d.view(np.float16)).view(np.uint16)
    assert np.array_equal(x, ref)


def test_ties_and_overflow(orc):
    f16 = lambda v: np.float16(v).view(np.uint16)
    cases = [  # (h, d, expected x)
        (2048.0, 1.0, 2048.0),      # 2049 is halfway between 2048 and 2050: even mantissa
        (2050.0, 1.0, 2052.0),      # 2051: halfway, the even neighbour is 2052
        (65504.0, 16.0, np.inf),    # 65520: halfway to 2^16, rounds to even = overflow
        (65504.0, 15.5, 65504.0),   # below the overflow threshold
        (-65504.0, -16.0, -np.inf),
        (2.0 ** -24, 2.0 ** -24, 2.0 ** -23),  # subnormals add exactly
        (1.0, -1.0, 0.0),           # +0 from exact cancellation
        (-0.0, -0.0, -0.0),
    ]
    for h, d, want in cases:
        x = orc.add_fp16(np.array([f16(h)]), np.array([f16(d)]))[0]
        assert x == f16(want), (h, d, want, hex(x))
