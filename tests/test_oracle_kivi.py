"""Pins for the KIVI-style grouped 2-bit quantisation in the oracle (CPU only)."""
import numpy as np

import oracle.kivi as ok
import oracle.quant as oq
from test_oracle_attention import sdpa_reference


def _block(seed, n_kv=2, d=16, outlier=None):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((16, n_kv, d)).astype(np.float32)
    v = rng.standard_normal((16, n_kv, d)).astype(np.float32)
    if outlier is not None:
        k[:, outlier[0], outlier[1]] *= np.float32(50)
    return k, v


def test_two_bit_codes_closed_form():
    """At 2 bits the largest code is 1 and the scale is the group's max |x|, so
    a value maps to sign(x) when |x| / max|x| > 1/2 and to 0 otherwise (ties at
    exactly 1/2 go to the even code 0)."""
    k, v = _block(0)
    kc, ksc, vc, vsc = ok.kivi_quantize_block(k, v)
    amax_k = np.abs(k).max(axis=0)
    assert np.array_equal(ksc, amax_k)
    expect = np.sign(k) * (np.abs(k) / amax_k[None] > 0.5)
    assert np.array_equal(kc, expect.astype(np.int8))
    amax_v = np.abs(v).max(axis=2)
    assert np.array_equal(vsc, amax_v)
    expect_v = np.sign(v) * (np.abs(v) / amax_v[:, :, None] > 0.5)
    assert np.array_equal(vc, expect_v.astype(np.int8))
    # ties: a channel [2, 1, -1, 0, ...] has codes [1, 0, 0, 0, ...]
    k2 = np.zeros((16, 1, 4), np.float32)
    k2[:4, 0, 0] = [2, 1, -1, 0]
    kc2, ksc2, _, _ = ok.kivi_quantize_block(k2, k2)
    assert ksc2[0, 0] == 2 and list(kc2[:4, 0, 0]) == [1, 0, 0, 0]
    assert ksc2[0, 1] == 0 and not kc2[:, 0, 1].any()  # all-zero group: scale 0, codes 0


def test_int2_packing_layout():
    """Element 4j + m sits in bits [2m, 2m+1] of byte j, two's complement."""
    assert oq.pack_int2([-1, 0, 1, -1]).tolist() == [0b11010011]
    assert oq.pack_int2([1, 1, 1, 1, -2, 0, 0, 0]).tolist() == [0b01010101, 0b00000010]
    c = np.random.default_rng(1).integers(-2, 2, (3, 5, 32))
    assert np.array_equal(oq.unpack_int2(oq.pack_int2(c)), c)


def test_key_groups_are_channels():
    """Permuting the tokens of a block permutes the key codes alike and keeps
    the key scales; a channel's scale is the section-8 quantiser's over that
    channel's 16 values."""
    k, v = _block(1)
    kc, ksc, vc, vsc = ok.kivi_quantize_block(k, v)
    perm = np.random.default_rng(2).permutation(16)
    kc2, ksc2, vc2, vsc2 = ok.kivi_quantize_block(k[perm], v[perm])
    assert np.array_equal(kc2, kc[perm]) and np.array_equal(ksc2, ksc)
    assert np.array_equal(vc2, vc[perm]) and np.array_equal(vsc2, vsc[perm])
    codes, scale, _ = oq.absmax_quantize(k[:, 1, 5], 2, np.float32)
    assert ksc[1, 5] == scale and np.array_equal(kc[:, 1, 5], codes)


def test_value_groups_are_tokens():
    k, v = _block(3)
    _, _, vc, vsc = ok.kivi_quantize_block(k, v)
    codes, scale, _ = oq.absmax_quantize(v[7, 0, :], 2, np.float32)
    assert vsc[7, 0] == scale and np.array_equal(vc[7, 0], codes)


def test_an_outlier_channel_leaves_other_channels_exact():
    """Per-channel keys: a x50 channel changes only its own scale and codes."""
    k, v = _block(4)
    k_out, _ = _block(4, outlier=(0, 3))
    kc, ksc, _, _ = ok.kivi_quantize_block(k, v)
    kc2, ksc2, _, _ = ok.kivi_quantize_block(k_out, v)
    other = np.ones((2, 16), bool)
    other[0, 3] = False
    assert np.array_equal(ksc2[other], ksc[other])
    assert np.array_equal(kc2[:, other], kc[:, other])
    assert ksc2[0, 3] == np.float32(50) * ksc[0, 3]


def test_round_trip_bounds():
    """|x - restored| <= scale / 2 in every group; each nonzero channel and
    token keeps its largest magnitude exactly."""
    k, v = _block(5)
    kc, ksc, vc, vsc = ok.kivi_quantize_block(k, v)
    kd, vd = ok.kivi_dequantize_block(kc, ksc, vc, vsc)
    assert (np.abs(kd - k) <= ksc[None] * (0.5 + 1e-6)).all()
    assert (np.abs(vd - v) <= vsc[:, :, None] * (0.5 + 1e-6)).all()
    assert (np.abs(kc).max(axis=0) == 1).all()
    i = np.abs(k).argmax(axis=0)
    assert np.allclose(np.take_along_axis(np.abs(kd), i[None], 0)[0], ksc)


def test_cache_state_splits_full_blocks_and_residual():
    rng = np.random.default_rng(7)
    for L in (0, 5, 16, 37, 48):
        k = rng.standard_normal((L, 2, 16)).astype(np.float32)
        v = rng.standard_normal((L, 2, 16)).astype(np.float32)
        blocks, rk, rv = ok.kivi_cache_state(k, v)
        assert len(blocks) == L // 16 and rk.shape[0] == L % 16
        assert np.array_equal(rk, k[16 * (L // 16):]) and np.array_equal(rv, v[16 * (L // 16):])
        for b, blk in enumerate(blocks):
            ref = ok.kivi_quantize_block(k[16 * b:16 * b + 16], v[16 * b:16 * b + 16])
            assert all(np.array_equal(x, y) for x, y in zip(blk, ref))


def test_decode_is_attention_over_restored_rows():
    """Full blocks dequantised element by element here, then the residual rows;
    with no full block the decode is plain attention over the residual."""
    rng = np.random.default_rng(6)
    q = rng.standard_normal((8, 16))
    blocks, rows_k, rows_v = [], [], []
    for b in range(2):
        k, v = _block(10 + b)
        blk = ok.kivi_quantize_block(k, v)
        blocks.append(blk)
        kc, ksc, vc, vsc = blk
        rk = np.zeros((16, 2, 16))
        rv = np.zeros((16, 2, 16))
        for t in range(16):
            for h in range(2):
                for i in range(16):
                    rk[t, h, i] = float(kc[t, h, i]) * float(ksc[h, i])
                    rv[t, h, i] = float(vc[t, h, i]) * float(vsc[t, h])
        rows_k.append(rk)
        rows_v.append(rv)
    res_k = rng.standard_normal((5, 2, 16))
    res_v = rng.standard_normal((5, 2, 16))
    out, lse = ok.kivi_decode(q, blocks, res_k, res_v, 0.25)
    K = np.concatenate(rows_k + [res_k])
    V = np.concatenate(rows_v + [res_v])
    np.testing.assert_allclose(out, sdpa_reference(q, K, V, 0.25), atol=1e-12)
    only, _ = ok.kivi_decode(q, [], res_k, res_v, 0.25)
    np.testing.assert_allclose(only, sdpa_reference(q, res_k, res_v, 0.25), atol=1e-12)
    none, lse0 = ok.kivi_decode(q, [], res_k[:0], res_v[:0], 0.25)
    assert not none.any() and np.isneginf(lse0).all()
