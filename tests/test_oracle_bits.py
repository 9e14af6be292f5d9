"""Pins of the 16-bit conversions every oracle comparison rests on.

The oracle reads the stored fp16/bf16 bit patterns as exact float64 values
(``oracle.bits_to_f64``), and the seeded generators round float32 draws to
those bit patterns (``workloads.f32_to_bits``).  Both sides of every parity
test see the same bits, so a wrong conversion would cancel out in the
brute-force pins, which upcast their inputs with the same function.  These
tests tie both conversions to things outside them:

* the IEEE-754 binary16 and bfloat16 field layouts, decoded here in plain
  Python integers (sign, biased exponent, fraction; subnormals, infinities,
  NaN) for all 65,536 patterns of each type;
* bit patterns whose values are fixed by those formats (1.0, -2.0, the
  smallest subnormals, the largest finite values, infinities);
* round to nearest, ties to even, written out from its definition on the
  two neighbouring 16-bit values, and torch's own float32 -> bfloat16 /
  float16 casts as an independent library routine;
* planted mistakes in copies of the conversions, each of which must fail one
  of the pins above.

The attention arithmetic itself follows the vLLM blog §"关键细节" 2): the
scores and weighted sums are taken on the stored 16-bit values, read exactly.
"""

import math

import numpy as np
import pytest

from oracle import bits_to_f64
from workloads import f32_to_bits

# overflow to infinity and NaN reinterpretations are part of what is tested
pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")

# ---------------------------------------------------------------------------
# the formats, decoded field by field
# ---------------------------------------------------------------------------

FORMATS = {
    # name: (exponent bits, fraction bits)
    "fp16": (5, 10),
    "bf16": (8, 7),
}


def field_value(bits: int, dtype: str) -> float:
    """Value of one 16-bit pattern from its fields: (-1)^s * 1.f * 2^(e-bias)
    for normal numbers, (-1)^s * 0.f * 2^(1-bias) for e = 0, infinities and
    NaN for the all-ones exponent."""
    ebits, fbits = FORMATS[dtype]
    bias = (1 << (ebits - 1)) - 1
    sign = -1.0 if (bits >> 15) & 1 else 1.0
    e = (bits >> fbits) & ((1 << ebits) - 1)
    f = bits & ((1 << fbits) - 1)
    if e == (1 << ebits) - 1:
        return sign * math.inf if f == 0 else math.nan
    if e == 0:
        return sign * math.ldexp(f, 1 - bias - fbits)
    return sign * math.ldexp((1 << fbits) + f, e - bias - fbits)


def upcast_mismatches(fn, dtype: str) -> int:
    """How many of the 65,536 patterns fn(bits, dtype) maps to another value
    than the field decoding (NaN must map to NaN, zeros keep their sign)."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = np.asarray(fn(bits, dtype), dtype=np.float64)
    bad = 0
    for b in range(1 << 16):
        want = field_value(b, dtype)
        g = float(got[b])
        if math.isnan(want):
            bad += not math.isnan(g)
        elif g != want or math.copysign(1.0, g) != math.copysign(1.0, want):
            bad += 1
    return bad


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_upcast_matches_field_decoding_for_every_pattern(dtype):
    assert upcast_mismatches(bits_to_f64, dtype) == 0


KNOWN = [
    # (dtype, bits, value) fixed by the formats
    ("fp16", 0x3C00, 1.0),
    ("fp16", 0xC000, -2.0),
    ("fp16", 0x3555, 0.333251953125),
    ("fp16", 0x0001, 2.0 ** -24),
    ("fp16", 0x03FF, 1023 * 2.0 ** -24),
    ("fp16", 0x0400, 2.0 ** -14),
    ("fp16", 0x7BFF, 65504.0),
    ("fp16", 0x7C00, math.inf),
    ("fp16", 0xFC00, -math.inf),
    ("fp16", 0x8000, -0.0),
    ("bf16", 0x3F80, 1.0),
    ("bf16", 0xC000, -2.0),
    ("bf16", 0x3EAB, 0.333984375),
    ("bf16", 0x0001, 2.0 ** -133),
    ("bf16", 0x0080, 2.0 ** -126),
    ("bf16", 0x7F7F, (2 - 2.0 ** -7) * 2.0 ** 127),
    ("bf16", 0x7F80, math.inf),
    ("bf16", 0xFF80, -math.inf),
    ("bf16", 0x8000, -0.0),
]


@pytest.mark.parametrize("dtype,bits,value", KNOWN, ids=lambda x: hex(x) if isinstance(x, int) else str(x))
def test_upcast_of_known_patterns(dtype, bits, value):
    got = float(bits_to_f64(np.array([bits], np.uint16), dtype)[0])
    assert got == value
    assert math.copysign(1.0, got) == math.copysign(1.0, value)


@pytest.mark.parametrize("dtype,bits", [("fp16", 0x7E00), ("fp16", 0x7C01), ("bf16", 0x7FC0), ("bf16", 0xFF81)])
def test_upcast_of_nan_patterns(dtype, bits):
    assert math.isnan(float(bits_to_f64(np.array([bits], np.uint16), dtype)[0]))


# ---------------------------------------------------------------------------
# rounding float32 to 16 bits: nearest, ties to even
# ---------------------------------------------------------------------------


def round_nearest_even(x: float, dtype: str) -> int:
    """The 16-bit pattern of finite float32 x rounded to nearest, ties to the
    pattern with an even last fraction bit, from the definition: find the
    two representable neighbours by search over the ordered patterns and
    compare exact float64 distances (float32 and 16-bit values and their
    differences are exact in float64)."""
    if x == 0.0:
        return 0x8000 if math.copysign(1.0, x) < 0 else 0
    sign = 0x8000 if x < 0 else 0
    a = abs(x)
    finite_max = 0x7BFF if dtype == "fp16" else 0x7F7F
    lo, hi = 0, finite_max
    if a >= field_value(finite_max, dtype):
        lo = finite_max
    else:
        # largest magnitude pattern whose value is <= a (patterns 0..max are ordered)
        while lo < hi:
            mid = (lo + hi + 1) // 2
            if field_value(mid, dtype) <= a:
                lo = mid
            else:
                hi = mid - 1
    below = field_value(lo, dtype)
    if below == a:
        return sign | lo
    above_bits = lo + 1
    if lo == finite_max:
        # past the largest finite value: overflow to infinity once a reaches
        # halfway to the next power of two (the value one more ulp would have)
        ebits, fbits = FORMATS[dtype]
        bias = (1 << (ebits - 1)) - 1
        above = math.ldexp(1.0, (1 << ebits) - 1 - bias)
        above_bits = finite_max + 1
    else:
        above = field_value(above_bits, dtype)
    d_lo, d_hi = a - below, above - a
    if d_lo < d_hi:
        r = lo
    elif d_hi < d_lo:
        r = above_bits
    else:
        r = lo if lo % 2 == 0 else above_bits
    return sign | r


def _samples(n: int, seed: int) -> np.ndarray:
    """float32 test values: normal draws like the workloads', wide-range
    magnitudes, exact ties and their neighbours for both formats, and values
    near the overflow and subnormal edges."""
    rng = np.random.default_rng(seed)
    parts = [
        rng.standard_normal(n).astype(np.float32),
        (rng.standard_normal(n) * np.exp2(rng.integers(-140, 128, n))).astype(np.float32),
    ]
    u = rng.integers(0, 0x7F800000, n, dtype=np.uint32)  # finite positive float32 patterns
    for low in (0x8000, 0x7FFF, 0x8001, 0x0000):  # bf16 ties and their neighbours
        parts.append(((u & np.uint32(0xFFFF0000)) | np.uint32(low)).view(np.float32))
    # fp16 ties: float32 whose 13 dropped fraction bits are exactly 1000..0
    v = rng.integers(0x38800000, 0x477FE000, n, dtype=np.uint32)  # fp16 normal range
    parts.append(((v & np.uint32(0xFFFFE000)) | np.uint32(0x1000)).view(np.float32))
    parts.append(np.array([65504.0, 65519.0, 65520.0, 65536.0, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26,
                           3.3895314e38, 3.3961775e38, 2.0 ** -133, 2.0 ** -134, 1.5 * 2.0 ** -134],
                          np.float32))
    x = np.concatenate(parts)
    sign = np.where(rng.random(x.shape[0]) < 0.5, -1, 1).astype(np.float32)
    x = x * sign
    return x[np.isfinite(x)]


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_rounding_matches_torch_cast(dtype):
    torch = pytest.importorskip("torch")
    x = _samples(20000, 5)
    want = torch.from_numpy(x).to(torch.float16 if dtype == "fp16" else torch.bfloat16)
    want = want.view(torch.int16).numpy().view(np.uint16)
    got = f32_to_bits(x, dtype)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, [(float(x[i]), hex(int(got[i])), hex(int(want[i]))) for i in bad[:5]]


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_rounding_matches_definition(dtype):
    x = _samples(600, 6)
    got = f32_to_bits(x, dtype)
    for xi, gi in zip(x.tolist(), got.tolist()):
        assert gi == round_nearest_even(xi, dtype), (xi, hex(gi), hex(round_nearest_even(xi, dtype)))


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_round_trip_is_the_nearest_16_bit_value(dtype):
    x = _samples(20000, 7)
    y = bits_to_f64(f32_to_bits(x, dtype), dtype)
    xd = x.astype(np.float64)
    fin = np.isfinite(y)
    # a finite result is within half a unit in the last place of the format
    ebits, fbits = FORMATS[dtype]
    bias = (1 << (ebits - 1)) - 1
    e = np.floor(np.log2(np.maximum(np.abs(y[fin]), 2.0 ** (1 - bias))))
    half_ulp = np.exp2(e - fbits - 1)
    assert (np.abs(y[fin] - xd[fin]) <= half_ulp).all()
    # an infinite one only where x is at least halfway past the largest finite value
    big = field_value(0x7BFF if dtype == "fp16" else 0x7F7F, dtype)
    assert (np.abs(xd[~fin]) > big).all()


# ---------------------------------------------------------------------------
# planted mistakes must fail a pin
# ---------------------------------------------------------------------------


def _mutant_upcast(kind):
    def f(bits, dtype):
        bits = np.asarray(bits, dtype=np.uint16)
        if kind == "bf16_read_as_fp16" and dtype == "bf16":
            return bits.view(np.float16).astype(np.float64)
        if kind == "fp16_read_as_bf16" and dtype == "fp16":
            return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
        if kind == "bf16_shift_15" and dtype == "bf16":
            return (bits.astype(np.uint32) << np.uint32(15)).view(np.float32).astype(np.float64)
        if kind == "subnormals_flushed":
            v = bits_to_f64(bits, dtype)
            tiny = 2.0 ** -14 if dtype == "fp16" else 2.0 ** -126
            return np.where(np.abs(v) < tiny, 0.0, v)
        if kind == "sign_dropped":
            return np.abs(bits_to_f64(bits, dtype))
        return bits_to_f64(bits, dtype)

    return f


@pytest.mark.parametrize("kind,dtype", [("bf16_read_as_fp16", "bf16"), ("fp16_read_as_bf16", "fp16"),
                                        ("bf16_shift_15", "bf16"), ("subnormals_flushed", "fp16"),
                                        ("subnormals_flushed", "bf16"), ("sign_dropped", "bf16")])
def test_planted_upcast_mistakes_are_caught(kind, dtype):
    assert upcast_mismatches(_mutant_upcast(kind), dtype) > 0


def _mutant_round(kind):
    def f(x, dtype):
        x = np.ascontiguousarray(x, dtype=np.float32)
        if dtype != "bf16":
            return f32_to_bits(x, dtype)
        u = x.view(np.uint32).astype(np.uint64)
        if kind == "truncate":
            return (u >> np.uint64(16)).astype(np.uint16)
        if kind == "ties_away":
            return ((u + np.uint64(0x8000)) >> np.uint64(16)).astype(np.uint16)
        if kind == "ties_to_odd":
            lsb = (u >> np.uint64(16)) & np.uint64(1)
            return ((u + np.uint64(0x8000) - lsb) >> np.uint64(16)).astype(np.uint16)
        return f32_to_bits(x, dtype)

    return f


@pytest.mark.parametrize("kind", ["truncate", "ties_away", "ties_to_odd"])
def test_planted_rounding_mistakes_are_caught(kind):
    x = _samples(300, 8)
    got = _mutant_round(kind)(x, "bf16")
    want = [round_nearest_even(v, "bf16") for v in x.tolist()]
    assert any(int(g) != w for g, w in zip(got.tolist(), want))
