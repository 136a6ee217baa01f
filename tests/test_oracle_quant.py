"""Pins for the oracle's quantisers (CPU only)."""
import numpy as np
import pytest
import torch

from oracle.quant import absmax_quantize, e4m3_decode, e4m3_encode, e4m3_value_table
from oracle.paged_attention import quantize_row_int8, quantize_rows_fp8


def _example(golden):
    rec = {r[0]: r[1:] for r in golden("absmax_4bit_example.txt")}
    return rec


def test_absmax_4bit_worked_example_float64(golden):
    rec = _example(golden)
    bits = int(rec["bits"][0])
    values = np.array([float(x) for x in rec["values"]])
    codes, scale, restored = absmax_quantize(values, bits, np.float64)
    assert codes.tolist() == [int(x) for x in rec["codes"]]
    assert np.round(restored, 3).tolist() == [float(x) for x in rec["restored_3dp"]]
    assert [len(values) * 16, len(values) * bits] == [int(x) for x in rec["payload_bits"]]


def test_absmax_4bit_worked_example_float32_same_codes(golden):
    # the cache writer runs the same rule in IEEE float32
    rec = _example(golden)
    values = np.array([float(x) for x in rec["values"]], dtype=np.float32)
    codes, scale, _ = absmax_quantize(values, 4, np.float32)
    assert codes.tolist() == [int(x) for x in rec["codes"]]
    assert scale.dtype == np.float32


@pytest.mark.parametrize("bits,largest", [(4, 7), (8, 127)])
def test_absmax_ties_round_to_even(bits, largest):
    # absmax == largest code makes the scale exactly 1, so quotients are exact
    vals = np.array([largest, 0.5, 1.5, 2.5, -0.5, -2.5, -3.5], dtype=np.float64)
    codes, scale, _ = absmax_quantize(vals, bits, np.float32)
    assert scale == 1.0
    assert codes.tolist() == [largest, 0, 2, 2, 0, -2, -4]


def test_absmax_int8_properties():
    rng = np.random.default_rng(7)
    for _ in range(200):
        x = (rng.standard_normal(128) * rng.uniform(0.01, 50)).astype(np.float32)
        codes, scale = quantize_row_int8(x)
        assert codes.dtype == np.int8
        assert codes.min() >= -127 and codes.max() <= 127
        i = int(np.argmax(np.abs(x)))
        assert abs(int(codes[i])) == 127 and np.sign(codes[i]) == np.sign(x[i])
        err = np.abs(x.astype(np.float64) - codes.astype(np.float64) * float(scale))
        assert err.max() <= float(scale) * (0.5 + 1e-5)
        # symmetric: negating the row negates the codes
        c2, s2 = quantize_row_int8(-x)
        assert s2 == scale and (c2 == -codes).all()
        # power-of-two rescaling changes the scale exactly and keeps the codes
        c3, s3 = quantize_row_int8(x * np.float32(4))
        assert s3 == scale * 4 and (c3 == codes).all()


def test_absmax_zero_row():
    codes, scale = quantize_row_int8(np.zeros(64, dtype=np.float32))
    assert scale == 0 and not codes.any()


def test_e4m3_table_closed_forms():
    t = e4m3_value_table()
    assert t[0x7E] == 448.0 and t[0xFE] == -448.0
    assert t[0x38] == 1.0 and t[0x08] == 2.0 ** -6 and t[0x01] == 2.0 ** -9
    assert t[0x00] == 0.0 and np.signbit(t[0x80])
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    assert np.isnan(t).sum() == 2


def test_e4m3_table_matches_torch_float8():
    # an independent implementation of the same OCP format
    raw = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = raw.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = e4m3_value_table()
    both_nan = np.isnan(ref) & np.isnan(mine)
    assert (both_nan | (ref == mine)).all()


def test_e4m3_encode_roundtrip_every_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    assert (e4m3_encode(e4m3_decode(codes)) == codes).all()


def test_e4m3_encode_midpoints_go_to_even_code():
    t = e4m3_value_table()
    for c in range(0, 0x7E):
        mid = (t[c] + t[c + 1]) / 2
        want = c if c % 2 == 0 else c + 1
        assert e4m3_encode(np.array([mid]))[0] == want, hex(c)
        assert e4m3_encode(np.array([-mid]))[0] == want | 0x80
        # just off the midpoint goes to the nearer neighbour
        eps = (t[c + 1] - t[c]) * 1e-3
        assert e4m3_encode(np.array([mid - eps]))[0] == c
        assert e4m3_encode(np.array([mid + eps]))[0] == c + 1


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(3)
    y = np.concatenate(
        [
            rng.uniform(-448, 448, 200000),
            rng.standard_normal(200000) * 0.01,
            rng.standard_normal(200000),
            np.linspace(-448, 448, 100001),
        ]
    ).astype(np.float32)
    ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert (e4m3_encode(y) == ref).all()


def test_e4m3_encode_saturates():
    assert e4m3_encode(np.array([448.0, 460.0, 1e4, np.inf]))[:3].tolist() == [0x7E, 0x7E, 0x7E]
    assert e4m3_encode(np.array([-1e9]))[0] == 0xFE
    assert e4m3_encode(np.array([-0.0]))[0] == 0x80


def test_fp8_row_writer_uses_float32_division():
    x = np.array([[1.0, -3.0, 0.1]], dtype=np.float32)
    scale = np.array([0.25], dtype=np.float32)
    assert quantize_rows_fp8(x, scale).tolist() == [e4m3_encode(np.array([4.0, -12.0, np.float32(0.1) / np.float32(0.25)])).tolist()]
    assert not quantize_rows_fp8(x, np.zeros(1, np.float32)).any()
