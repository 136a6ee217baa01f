"""Pins for the oracle's further cache formats (CPU only): FP8 E5M2 and the
packed 4-bit cache ("KV Cache Engineering for LLM Serving", section 8;
"Chapter 18 - KV-Cache Optimization Strategies", the fp8_e5m2 cache option)."""
import numpy as np
import torch

import oracle.paged_attention as pa
import oracle.quant as oq
from test_oracle_attention import sdpa_reference


def test_e5m2_table_closed_forms():
    t = oq.e5m2_value_table()
    assert t[0x00] == 0.0 and np.signbit(t[0x80])
    assert t[0x01] == 2.0 ** -16  # smallest subnormal: 2^-14 * 1/4
    assert t[0x03] == 3 * 2.0 ** -16
    assert t[0x04] == 2.0 ** -14  # smallest normal
    assert t[0x3C] == 1.0 and t[0x3D] == 1.25 and t[0x40] == 2.0
    assert t[0x7B] == 57344.0
    assert np.isinf(t[0x7C]) and t[0x7C] > 0 and np.isinf(t[0xFC]) and t[0xFC] < 0
    assert np.isnan(t[[0x7D, 0x7E, 0x7F, 0xFD, 0xFE, 0xFF]]).all()
    fin = np.isfinite(t[:0x80])
    np.testing.assert_array_equal(t[0x80:][fin], -t[:0x80][fin])
    assert (np.diff(t[:0x7C]) > 0).all()


def test_e5m2_table_is_the_top_byte_of_float16():
    # E5M2 keeps float16's sign and exponent and its two top mantissa bits
    halves = (np.arange(256, dtype=np.uint16) << 8).view(np.float16).astype(np.float64)
    t = oq.e5m2_value_table()
    same = np.isnan(t) == np.isnan(halves)
    assert same.all()
    np.testing.assert_array_equal(t[~np.isnan(t)], halves[~np.isnan(halves)])


def test_e5m2_table_matches_torch_float8():
    raw = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = raw.view(torch.float8_e5m2).to(torch.float64).numpy()
    mine = oq.e5m2_value_table()
    assert (np.isnan(ref) == np.isnan(mine)).all()
    np.testing.assert_array_equal(ref[~np.isnan(ref)], mine[~np.isnan(mine)])


def test_e5m2_encode_roundtrip_and_midpoints():
    codes = np.arange(0x7C, dtype=np.uint8)
    assert (oq.e5m2_encode(oq.e5m2_decode(codes)) == codes).all()
    assert (oq.e5m2_encode(-oq.e5m2_decode(codes[1:])) == (codes[1:] | 0x80)).all()
    t = oq.e5m2_value_table()
    for c in range(0x7B):
        mid = (t[c] + t[c + 1]) / 2
        want = c if c % 2 == 0 else c + 1
        assert oq.e5m2_encode(np.array([mid]))[0] == want, hex(c)
        eps = (t[c + 1] - t[c]) * 1e-3
        assert oq.e5m2_encode(np.array([mid - eps]))[0] == c
        assert oq.e5m2_encode(np.array([mid + eps]))[0] == c + 1


def test_e5m2_encode_matches_torch_in_range():
    rng = np.random.default_rng(11)
    y = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.uniform(-6, 4, 20000),
                        rng.uniform(-57344, 57344, 2000)]).astype(np.float32)
    ref = torch.from_numpy(y).to(torch.float8_e5m2).view(torch.uint8).numpy()
    assert (oq.e5m2_encode(y) == ref).all()


def test_e5m2_encode_saturates():
    assert oq.e5m2_encode(np.array([57344.0, 61000.0, 1e9, np.inf])).tolist() == [0x7B] * 4
    assert oq.e5m2_encode(np.array([-np.inf]))[0] == 0xFB
    assert oq.e5m2_encode(np.array([np.nan]))[0] == 0x7F


def test_int4_nibble_order():
    assert oq.pack_int4([1, 2]).tolist() == [0x21]
    assert oq.pack_int4([-1, 0]).tolist() == [0x0F]
    assert oq.pack_int4([0, -8]).tolist() == [0x80]
    assert oq.pack_int4([7, -7, 3, -3]).tolist() == [0x97, 0xD3]


def test_int4_pack_unpack_inverse():
    every = np.array(np.meshgrid(np.arange(-8, 8), np.arange(-8, 8))).reshape(2, -1).T  # all 256 pairs
    packed = oq.pack_int4(every)
    assert sorted(packed[:, 0].tolist()) == list(range(256))
    np.testing.assert_array_equal(oq.unpack_int4(packed), every)


def test_int4_row_quantiser_worked_example(golden):
    rec = {r[0]: r[1:] for r in golden("absmax_4bit_example.txt")}
    values = np.array([float(x) for x in rec["values"]], dtype=np.float32)
    packed, scale = pa.quantize_row_int4(values)
    assert packed.shape == (3,)
    assert oq.unpack_int4(packed).tolist() == [int(x) for x in rec["codes"]]
    assert np.round(oq.unpack_int4(packed) * np.float64(scale), 3).tolist() == [float(x) for x in rec["restored_3dp"]]


def test_int4_row_quantiser_properties():
    rng = np.random.default_rng(12)
    for _ in range(200):
        x = (rng.standard_normal(128) * rng.uniform(0.01, 50)).astype(np.float32)
        packed, scale = pa.quantize_row_int4(x)
        codes = oq.unpack_int4(packed)
        assert codes.min() >= -7 and codes.max() <= 7
        i = int(np.argmax(np.abs(x)))
        assert abs(int(codes[i])) == 7
        err = np.abs(x.astype(np.float64) - codes * float(scale))
        assert err.max() <= float(scale) * (0.5 + 1e-5)


def _nibble(byte, hi):
    v = (int(byte) >> 4) if hi else (int(byte) & 0xF)
    return v - 16 if v >= 8 else v


def test_int4_cache_decode_is_attention_over_restored_values():
    """Cache written through the oracle's writer; the expected output restores
    every element bit by bit here and runs the textbook attention."""
    rng = np.random.default_rng(13)
    L, n_kv, d, n_q = 37, 2, 16, 8
    K = rng.standard_normal((L, n_kv, d))
    V = rng.standard_normal((L, n_kv, d))
    q = rng.standard_normal((n_q, d))
    nb = 3
    kc = np.zeros((nb, 16, n_kv, d // 2), np.uint8)
    vc = np.zeros_like(kc)
    ks = np.zeros((nb, 16, n_kv), np.float32)
    vs = np.zeros_like(ks)
    table = np.array([2, 0, 1])
    slots = table[np.arange(L) // 16] * 16 + np.arange(L) % 16
    pa.kv_cache_write(K, V, kc, vc, slots, "int4", ks, vs)
    Kr = np.zeros((L, n_kv, d))
    Vr = np.zeros((L, n_kv, d))
    for p in range(L):
        b, r = table[p // 16], p % 16
        for h in range(n_kv):
            for i in range(d):
                Kr[p, h, i] = _nibble(kc[b, r, h, i // 2], i % 2) * float(ks[b, r, h])
                Vr[p, h, i] = _nibble(vc[b, r, h, i // 2], i % 2) * float(vs[b, r, h])
    assert np.abs(Kr - K).max() <= np.abs(K).max() / 7 * 0.5 + 1e-6
    out, _ = pa.paged_attention_decode(q[None], kc, vc, table[None], [L], 0.25, "int4", ks, vs)
    np.testing.assert_allclose(out[0], sdpa_reference(q, Kr, Vr, 0.25), atol=1e-12)


def test_e5m2_cache_writer_matches_torch_conversion():
    rng = np.random.default_rng(14)
    x = rng.standard_normal((5, 4, 32)).astype(np.float32) * 30
    sc = np.array([0.5, 2.0, 1e-3, 7.0], np.float32)
    for t in range(5):
        got = pa.quantize_rows_fp8(x[t], sc, "fp8_e5m2")
        y = torch.from_numpy(x[t]) / torch.from_numpy(sc)[:, None]
        ref = y.to(torch.float8_e5m2).view(torch.uint8).numpy()
        finite = np.abs(y.numpy()) <= 57344
        assert (got[finite] == ref[finite]).all()
