"""Pins of the oracle's element and scale codecs against what the pages fix.

E2M1: the code table, the midpoint rule and the self-check outputs of
"NVFP4 与 MXFP4 格式" (charlestar.github.io) §1.  E4M3: the value table of
torch's float8_e4m3fn (an independent library) and exact rational rounding
with Python's fractions; §2 and §4 of the same page fix max 448, min
subnormal 2^-9 and the E4M3 scale 0.6 -> 0.625.
"""
import math
import struct
import sys
from fractions import Fraction

import numpy as np
import pytest
import torch

from conftest import golden

pytestmark = pytest.mark.filterwarnings("ignore")


def f32(v):
    return struct.unpack("f", struct.pack("f", v))[0]


def nextafter32(v, toward):
    return float(np.nextafter(np.float32(v), np.float32(toward)))


# ---------------------------------------------------------------- E2M1 ----

def test_codebook_values_and_negative_zero(oracle_mod):
    gd = golden("e2m1_codebook.json")
    for code, want in enumerate(gd["values"]):
        got = oracle_mod.e2m1_decode(code)
        assert got == want and math.copysign(1, got) == math.copysign(1, want), code
    assert math.copysign(1.0, oracle_mod.e2m1_decode(8)) == -1.0


def test_all_codes_round_trip(oracle_mod):
    assert [oracle_mod.e2m1_encode(oracle_mod.e2m1_decode(c)) for c in range(16)] == list(range(16))


def test_midpoints_go_to_even_code(oracle_mod):
    gd = golden("e2m1_codebook.json")
    got = [oracle_mod.e2m1_decode(oracle_mod.e2m1_encode(m)) for m in gd["midpoints"]]
    assert got == gd["midpoints_round_to"]
    neg = [oracle_mod.e2m1_decode(oracle_mod.e2m1_encode(-m)) for m in gd["midpoints"]]
    assert neg == [-v for v in gd["midpoints_round_to"]]


def test_saturation(oracle_mod):
    dec = lambda v: oracle_mod.e2m1_decode(oracle_mod.e2m1_encode(v))
    assert dec(100.0) == 6.0 and dec(-100.0) == -6.0
    assert dec(sys.float_info.max) == 6.0 and dec(-sys.float_info.max) == -6.0
    fmax = float(np.finfo(np.float32).max)
    assert dec(fmax) == 6.0 and dec(-fmax) == -6.0


@pytest.mark.parametrize("bad", [float("nan"), float("inf"), -float("inf")])
def test_nonfinite_rejected(oracle_mod, bad):
    with pytest.raises(ValueError):
        oracle_mod.e2m1_encode(bad)
    assert oracle_mod.e2m1_encode_f32(np.array([bad], np.float32))[0] == 0xFF


def test_pack_bytes_and_odd_length(oracle_mod):
    gd = golden("e2m1_codebook.json")
    packed = oracle_mod.pack4(list(range(16)))
    assert packed.hex(" ") == gd["packed_codes_0_to_15_hex"]
    assert oracle_mod.unpack4(packed) == list(range(16))
    with pytest.raises(ValueError):
        oracle_mod.pack4([1, 2, 3])
    with pytest.raises(ValueError):
        oracle_mod.pack4([1, 16])


def test_signed_zero_and_tiny_negatives(oracle_mod):
    assert oracle_mod.e2m1_encode(-0.0) == 8
    assert oracle_mod.e2m1_encode(0.0) == 0
    assert oracle_mod.e2m1_encode(-1e-30) == 8
    assert oracle_mod.e2m1_encode(-0.25) == 8   # midpoint 0.25 -> 0, sign kept
    assert oracle_mod.e2m1_encode(-0.2500001) == 9


def test_encode_is_monotone_symmetric_and_switches_only_at_midpoints(oracle_mod):
    """The seven midpoints and the tie rule pinned above, plus monotonicity and
    sign symmetry, determine the encoder completely; check both on a dense
    fp32 sweep of [0, 8] and on the neighbours of every midpoint."""
    gd = golden("e2m1_codebook.json")
    v = np.linspace(0.0, 8.0, 400_001, dtype=np.float32)
    c = oracle_mod.e2m1_encode_f32(v).astype(np.int64)
    assert np.all(np.diff(c) >= 0) and c[0] == 0 and c[-1] == 7
    cn = oracle_mod.e2m1_encode_f32(-v).astype(np.int64)
    assert np.array_equal(cn, c | 8)
    # the code changes only across a midpoint
    mids = np.array(gd["midpoints"], np.float32)
    jumps = np.nonzero(np.diff(c))[0]
    assert len(jumps) == 7
    for j, m in zip(jumps, mids):
        assert v[j] <= m <= v[j + 1]
    for k, m in enumerate(gd["midpoints"]):
        below, above = nextafter32(m, 0.0), nextafter32(m, 10.0)
        assert oracle_mod.e2m1_encode(below) == k
        assert oracle_mod.e2m1_encode(above) == k + 1
        at = oracle_mod.e2m1_encode(m)
        assert at in (k, k + 1) and at % 2 == 0


# ---------------------------------------------------------------- E4M3 ----

def _torch_e4m3_table():
    vals = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().tolist()
    return vals


def test_e4m3_values_match_torch_float8(oracle_mod):
    tab = _torch_e4m3_table()
    for code in range(127):
        assert oracle_mod.e4m3_value(code) == tab[code], code
    for byte in range(256):
        want, got = tab[byte], oracle_mod.e4m3_decode_byte(byte)
        if math.isnan(want):
            assert math.isnan(got) and byte & 0x7F == 0x7F
        else:
            assert got == want, byte
    assert oracle_mod.e4m3_value(126) == 448.0
    assert oracle_mod.e4m3_value(1) == 2.0 ** -9 and oracle_mod.e4m3_value(8) == 2.0 ** -6


def _exact_e4m3_round(t: Fraction, tab) -> int:
    """Correctly rounded (ties to even code) E4M3 code of an exact rational,
    saturated at 448, by exhaustive comparison in exact arithmetic."""
    t = min(t, tab[126])
    return min(range(127), key=lambda c: (abs(tab[c] - t), c & 1))


@pytest.fixture(scope="module")
def e4m3_fracs():
    return [Fraction(v) for v in _torch_e4m3_table()[:127]]


def test_e4m3_encode_page_values(oracle_mod):
    assert oracle_mod.e4m3_value(oracle_mod.e4m3_encode(0.6)) == 0.625
    assert oracle_mod.e4m3_value(oracle_mod.e4m3_encode(0.875)) == 0.875
    assert oracle_mod.e4m3_encode(464.0) == 126 and oracle_mod.e4m3_encode(1e6) == 126
    assert oracle_mod.e4m3_encode(2.0 ** -10) == 0           # tie -> even code 0
    assert oracle_mod.e4m3_encode(nextafter32(2.0 ** -10, 1)) == 1


def test_e4m3_encode_matches_torch_on_fp32_inputs(oracle_mod):
    g = torch.Generator().manual_seed(7)
    t = torch.cat([torch.rand(20000, generator=g) * 448,
                   torch.rand(20000, generator=g) * 2.0 ** -5,
                   torch.exp2(torch.rand(20000, generator=g) * 18 - 10)]).clamp(max=448)
    want = t.to(torch.float8_e4m3fn).view(torch.uint8).tolist()
    got = [oracle_mod.e4m3_encode(float(v)) for v in t.tolist()]
    assert got == want


def test_e4m3_midpoints_ties_even(oracle_mod, e4m3_fracs):
    for c in range(126):
        m = (e4m3_fracs[c] + e4m3_fracs[c + 1]) / 2
        got = oracle_mod.e4m3_encode(float(m))          # dyadic, exact in double
        assert got == (c if c % 2 == 0 else c + 1), c


def test_block_scale_code_is_exact_rational_rounding(oracle_mod, e4m3_fracs):
    """A_b / (6 g) rounded once to E4M3 from the exact rational: random
    (A_b, g) pairs plus pairs built to sit exactly on, and one fp32 step
    either side of, every E4M3 midpoint."""
    rng = np.random.default_rng(11)
    cases = []
    for _ in range(3000):
        g = f32(float(2.0 ** rng.uniform(-40, 40)))
        t = float(rng.choice([rng.uniform(0, 500), 2.0 ** rng.uniform(-12, 9)]))
        ab = f32(t * 6 * g)
        cases.append((ab, g))
    for g in (1.0, f32(0.0123), f32(3.7e-20)):
        for c in range(126):
            m = (e4m3_fracs[c] + e4m3_fracs[c + 1]) / 2
            ab = f32(float(m * 6 * Fraction(g)))
            for a in (ab, nextafter32(ab, 0), nextafter32(ab, float("inf"))):
                cases.append((a, g))
    for ab, g in cases:
        want = _exact_e4m3_round(Fraction(ab) / (6 * Fraction(g)), e4m3_fracs)
        assert oracle_mod.nv_block_scale_code(ab, g) == want, (ab, g)


def test_e8m0_values(oracle_mod):
    assert oracle_mod.e8m0_value(127) == 1.0
    assert oracle_mod.e8m0_value(0) == 2.0 ** -127
    assert oracle_mod.e8m0_value(254) == 2.0 ** 127
    assert math.isnan(oracle_mod.e8m0_value(255))


def test_bf16_rounding_matches_torch(oracle_mod):
    g = torch.Generator().manual_seed(3)
    x = torch.cat([torch.randn(50000, generator=g) * 10.0 ** torch.randint(-40, 38, (50000,), generator=g),
                   torch.tensor([0.0, -0.0, 3.4e38, -3.4e38, 1e-45, 2.0 ** -130, float("inf")])])
    want = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle_mod.f32_to_bf16_fast(x.numpy()), want)
    assert np.array_equal(oracle_mod.f32_to_bf16(x.numpy()[:2000]), want[:2000])
