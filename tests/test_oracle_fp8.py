"""Pins for the fp8 (e4m3) input variant on the oracle side, and for the input
encoder the tests and the bench use.

The reading (the FlashDreams SANA-WM streaming runner page lists fp8 precision
modes without a scheme): q, k, v arrive as OCP e4m3 bytes, v with one float scale,
v = v_scale * e4m3(v8), and the layer is the gated delta rule on those values.
So the pins are

* the e4m3 format itself: hand-derived special values, the whole 256-code table
  against the e4m3 dtype of torch (a library routine), monotonicity and sign
  symmetry;
* the encoder: round trip of every finite code, ties to even, saturation, and
  agreement with torch's cast on random values;
* a hand-derived two-token example given as e4m3 codes with a scale
  (tests/golden/worked_example_fp8.txt), through every oracle form;
* the scale enters linearly: scaling v by 2 scales the output and the state
  produced from a zero state by 2.

A planted mistake in the decoder (a wrong exponent bias, a dropped subnormal
branch, the scale on q instead of v) fails at least one pin (last test).
"""

import math
import os

import numpy as np
import pytest

from oracle import gdn_reference as R
from workloads import draw, e4m3_encode, to_fp8, v_scale_for

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *rest = line.split()
            vals[key] = [float(x) for x in rest]
    return vals


class _X8:
    """e4m3 inputs in the shape the oracle's widening reads."""

    def __init__(self, q8, k8, v8, v_scale, gate, beta, state, frame_len):
        self.q8, self.k8, self.v8, self.v_scale = q8, k8, v8, v_scale
        self.gate, self.beta, self.state, self.frame_len = gate, beta, state, frame_len
        self.gate_mode = 0


# ---------------------------------------------------------------- the format

def check_decoder_special_values(dec):
    cases = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x0F: 1.875 * 2.0 ** -6,
             0x38: 1.0, 0x39: 1.125, 0x3F: 1.875, 0x40: 2.0, 0x44: 3.0, 0x48: 4.0, 0x50: 8.0,
             0x77: 1.875 * 2.0 ** 7, 0x78: 256.0, 0x7E: 448.0, 0xB8: -1.0, 0xC0: -2.0, 0xFE: -448.0,
             0x81: -(2.0 ** -9)}
    got = dec(np.array(list(cases), dtype=np.uint8))
    np.testing.assert_array_equal(got, np.array(list(cases.values())))
    z = dec(np.array([0x80], dtype=np.uint8))[0]
    assert z == 0.0 and math.copysign(1.0, z) == -1.0
    assert np.isnan(dec(np.array([0x7F, 0xFF], dtype=np.uint8))).all()


def check_decoder_monotone_symmetric(dec):
    pos = dec(np.arange(0x00, 0x7F, dtype=np.uint8))
    assert np.all(np.diff(pos) > 0)
    neg = dec(np.arange(0x80, 0xFF, dtype=np.uint8))
    np.testing.assert_array_equal(neg, -pos)


def check_decoder_vs_library(dec):
    torch = pytest.importorskip("torch")
    c = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(c).view(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(dec(c), ref)


def test_decoder_special_values():
    check_decoder_special_values(R.decode_e4m3)


def test_decoder_monotone_and_symmetric():
    check_decoder_monotone_symmetric(R.decode_e4m3)


def test_decoder_matches_library_dtype():
    check_decoder_vs_library(R.decode_e4m3)


# ---------------------------------------------------------------- the encoder

def test_encoder_round_trips_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = R.decode_e4m3(codes).astype(np.float32)
    back = e4m3_encode(vals)
    # -0 and +0 keep their sign
    np.testing.assert_array_equal(back, codes)


def test_encoder_ties_to_even_and_saturates():
    x = np.array([1.0625, 1.1875, -1.0625, 3 * 2.0 ** -10, 5 * 2.0 ** -10, 464.0, 500.0, -1e6, 449.0],
                 dtype=np.float32)
    # 1.0625 lies between 1 (m 0) and 1.125 (m 1): even -> 1; 1.1875 between m 1 and m 2 -> m 2;
    # 3 * 2^-10 between the subnormals 1 and 2 (units of 2^-9) -> 2; 5 * 2^-10 between 2 and 3 -> 2;
    # beyond 448 everything saturates to 448
    want = R.decode_e4m3(np.array([0x38, 0x3A, 0xB8, 0x02, 0x02, 0x7E, 0x7E, 0xFE, 0x7E], dtype=np.uint8))
    np.testing.assert_array_equal(R.decode_e4m3(e4m3_encode(x)), want)


def test_encoder_matches_library_cast():
    torch = pytest.importorskip("torch")
    x = (np.random.default_rng(5).standard_normal(100_000) * 40).astype(np.float32)
    x = np.clip(x, -448, 448)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(e4m3_encode(x), ref)


def test_v_scale_is_a_power_of_two_covering_the_range():
    v = np.array([[0.1, -3000.0, 7.0]], dtype=np.float32)
    s = v_scale_for(v)
    assert s == 8.0 and 3000.0 / s <= 448.0 < 3000.0 / (s / 2)
    assert v_scale_for(np.zeros(3, np.float32)) == 1.0


# ---------------------------------------------------------------- the layer on e4m3 inputs

def golden_fp8():
    g = read_golden("worked_example_fp8.txt")
    x8 = _X8(np.array(g["q8"], np.uint8).reshape(1, 2, 1, 2), np.array(g["k8"], np.uint8).reshape(1, 2, 1, 2),
             np.array(g["v8"], np.uint8).reshape(1, 2, 1, 2), g["v_scale"][0],
             np.array(g["gate"], np.float32).reshape(1, 2, 1), np.array(g["beta"], np.float32).reshape(1, 2, 1),
             None, 1)
    return g, x8


def check_golden(widen):
    g, x8 = golden_fp8()
    w = widen(x8)
    np.testing.assert_array_equal(np.ravel(w.q), g["decoded_q"])
    np.testing.assert_array_equal(np.ravel(w.k), g["decoded_k"])
    np.testing.assert_array_equal(np.ravel(w.v), g["decoded_v"])
    s0 = np.array(g["state_in"], np.float64).reshape(1, 1, 2, 2)
    for form in (lambda i, s: R.token_recurrence(i, s, eps=0.0), lambda i, s: R.c_forward(i, s, eps=0.0),
                 lambda i, s: R.chunked(i, s, chunk_len=64, eps=0.0)):
        out, S = form(w, s0)
        np.testing.assert_allclose(np.ravel(out), g["out"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(np.ravel(S), g["state_out"], rtol=0, atol=1e-12)


def test_golden_two_tokens_fp8():
    check_golden(R.widen_fp8)


def check_scale_linear(widen):
    rng = np.random.Generator(np.random.PCG64(3))
    inp = draw(rng, 1, 2, 40, 8, 8, 5, "f32", 0.0, 1.0)
    x8 = to_fp8(inp, v_scale=0.25)
    o1, s1 = R.token_recurrence(widen(x8), None)
    x8.v_scale = 0.5
    o2, s2 = R.token_recurrence(widen(x8), None)
    np.testing.assert_allclose(o2, 2 * o1, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(s2, 2 * s1, rtol=1e-13, atol=1e-15)


def test_scale_enters_linearly():
    check_scale_linear(R.widen_fp8)


def test_encoded_inputs_stay_close_to_the_draws():
    """The encoder's rounding is within e4m3's half-ulp (2^-4 relative for normals)."""
    rng = np.random.Generator(np.random.PCG64(4))
    inp = draw(rng, 1, 3, 50, 16, 16, 7, "f32", 0.0, 1.0)
    x8 = to_fp8(inp)
    w = R.widen_fp8(x8)
    for a, b, scale in ((w.q, inp.q, 1.0), (w.k, inp.k, 1.0), (w.v, inp.v, x8.v_scale)):
        b = b.astype(np.float64)
        big = np.abs(b) >= 2.0 ** -6 * scale          # the normal range after scaling
        assert big.sum() > 0.9 * b.size
        assert np.all(np.abs(a - b)[big] <= np.abs(b)[big] * 2.0 ** -4)


# ---------------------------------------------------------------- the pins catch planted mistakes

def _mutant_bias8(codes):
    c = np.asarray(codes, np.uint8).astype(np.int64)
    e, m = (c >> 3) & 0xF, (c & 7).astype(np.float64)
    mag = np.where(e == 0, m / 8 * 2.0 ** -6, (1 + m / 8) * np.exp2(e - 8.0))
    return np.where(c >> 7, -1.0, 1.0) * np.where((e == 15) & (m == 7), np.nan, mag)


def _mutant_no_subnormals(codes):
    c = np.asarray(codes, np.uint8).astype(np.int64)
    e, m = (c >> 3) & 0xF, (c & 7).astype(np.float64)
    mag = (1 + m / 8) * np.exp2(e - 7.0)
    return np.where(c >> 7, -1.0, 1.0) * np.where((e == 15) & (m == 7), np.nan, mag)


def _mutant_nan_at_inf(codes):
    c = np.asarray(codes, np.uint8).astype(np.int64)
    out = R.decode_e4m3(codes)
    return np.where(((c >> 3) & 0xF) == 15, np.nan, out)


class _WidenScaleOnQ(R.Widened):
    def __init__(self, x8):
        super().__init__(x8)
        self.q = float(x8.v_scale) * R.decode_e4m3(x8.q8)
        self.v = R.decode_e4m3(x8.v8)


@pytest.mark.parametrize("mutant", [_mutant_bias8, _mutant_no_subnormals, _mutant_nan_at_inf])
def test_decoder_mutants_fail_a_pin(mutant):
    failed = 0
    for check in (check_decoder_special_values, check_decoder_monotone_symmetric, check_decoder_vs_library):
        try:
            check(mutant)
        except AssertionError:
            failed += 1
    assert failed >= 1


def test_scale_on_the_wrong_operand_fails_a_pin():
    with pytest.raises(AssertionError):
        check_golden(_WidenScaleOnQ)
