"""Pins for the oracle's FP8 (E4M3) decoder, used by the FP8 forward parity tests.

The FP8 forward's oracle is the exact attention (already pinned) of the
dequantized inputs code * scale, so what needs its own pin is the decoding of
the codes.  Checked against values fixed by the E4M3 definition, torch's own
float8_e4m3fn widening cast on all 256 codes (a library routine), and
monotonicity; planted mistakes (wrong exponent bias, subnormals treated as
normals, a mantissa of 4 bits) must fail.
"""

import numpy as np
import pytest
import torch

import oracle
import oracle.exact_attention as oa
import synth


def pin_e4m3_definition_values():
    dec = oracle.e4m3_bits_to_f64
    cases = {0x00: 0.0, 0x38: 1.0, 0x40: 2.0, 0x3C: 1.5, 0x7E: 448.0, 0x08: 2.0 ** -6,
             0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0xB8: -1.0, 0xFE: -448.0, 0x30: 0.5}
    for code, val in cases.items():
        assert dec(np.array([code], dtype=np.uint8))[0] == val, hex(code)
    assert np.isnan(dec(np.array([0x7F, 0xFF], dtype=np.uint8))).all()


def pin_e4m3_library_routine():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_bits_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    keep = ~np.isnan(ref)
    assert np.array_equal(ours[keep], ref[keep])


def pin_e4m3_monotone():
    pos = oracle.e4m3_bits_to_f64(np.arange(0, 0x7F, dtype=np.uint8))
    assert np.all(np.diff(pos) > 0)
    neg = oracle.e4m3_bits_to_f64(np.arange(0x80, 0xFF, dtype=np.uint8))
    assert np.array_equal(neg, -pos)


FP8_PINS = [pin_e4m3_definition_values, pin_e4m3_library_routine, pin_e4m3_monotone]


@pytest.mark.parametrize("pin", FP8_PINS, ids=[p.__name__ for p in FP8_PINS])
def test_fp8_pin(pin):
    pin()


def test_quantized_inputs_round_trip():
    """The synthetic FP8 inputs decode to within half an E4M3 step of the
    float32 draws they quantize (relative 2^-4 for normal values)."""
    (q8, k8, v8), (sq, sk, sv) = synth.draw_qkv_fp8(1, 2, 64, 128, seed=9)
    g = torch.Generator(device="cpu")
    g.manual_seed(9)
    q = torch.randn((1, 2, 64, 128), generator=g, dtype=torch.float32).double().numpy()
    deq = oracle.e4m3_bits_to_f64(q8.numpy()) * sq
    err = np.abs(deq - q)
    normal = np.abs(q) >= 2.0 ** -6 * sq
    assert np.all(err[normal] <= 2.0 ** -4 * np.abs(q[normal]) + 1e-15)
    assert np.all(err[~normal] <= 2.0 ** -10 * sq + 1e-15)
    assert abs(np.abs(deq).max() - 448.0 * sq) <= 1e-12


def _mut_bias8(bits):
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 0x7) / 8.0
    return sign * np.where(e == 0, np.ldexp(m, -6), np.ldexp(1.0 + m, e - 8))


def _mut_no_subnormal(bits):
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 0x7) / 8.0
    return sign * np.ldexp(1.0 + m, e - 7)


def _mut_mantissa4(bits):
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 0x7) / 16.0
    return sign * np.where(e == 0, np.ldexp(m, -6), np.ldexp(1.0 + m, e - 7))


@pytest.mark.parametrize("fn", [_mut_bias8, _mut_no_subnormal, _mut_mantissa4])
def test_fp8_mutant_is_caught(fn, monkeypatch):
    monkeypatch.setattr(oa, "e4m3_bits_to_f64", fn)
    monkeypatch.setattr(oracle, "e4m3_bits_to_f64", fn)
    failed = []
    with np.errstate(all="ignore"):
        for pin in FP8_PINS:
            try:
                pin()
            except (AssertionError, ValueError):
                failed.append(pin.__name__)
    assert failed
