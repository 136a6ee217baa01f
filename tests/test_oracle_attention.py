"""Pins for the oracle's gather, attention and cache append (CPU only)."""
import math

import numpy as np
import pytest
import torch

import oracle
import oracle.paged_attention as pa
from oracle.paged_attention import (
    attention_one_sequence,
    gather_sequence,
    kv_cache_write,
    kv_head_of,
    logical_to_physical,
    paged_attention_decode,
)
from paged_kv_cache_467_b200 import accounting, workloads
from bruteforce import brute_decode


# ------------------------------------------------------------------ helpers
def build_cache(w, poison=np.nan):
    """Fill oracle caches for workload w through the oracle's own writer.

    Unwritten rows (free blocks, tails of last blocks) hold ``poison``.
    Returns (key_cache, value_cache, k_scale, v_scale, q).
    """
    shape = (w.num_blocks, w.block_size, w.n_kv, w.head_dim)
    if w.cache_dtype == "int8":
        kc = np.full(shape, 77, dtype=np.int8)
        vc = np.full(shape, -77, dtype=np.int8)
        ks = np.full(shape[:3], poison, dtype=np.float32)
        vs = np.full(shape[:3], poison, dtype=np.float32)
    elif w.cache_dtype == "fp8_e4m3":
        kc = np.full(shape, 0x7F, dtype=np.uint8)  # NaN code
        vc = np.full(shape, 0x7F, dtype=np.uint8)
        ks, vs = w.fp8_head_scales()
    else:
        kc = np.full(shape, poison, dtype=np.float64)
        vc = np.full(shape, poison, dtype=np.float64)
        ks = vs = None
    if w.shared_prefix_tokens:
        pk, pv = w.prefix_kv()
        kv_cache_write(pk, pv, kc, vc, w.prefix_slots(), w.cache_dtype, ks, vs)
    for s in range(w.num_seqs):
        hk, hv = w.history_kv(s)
        kv_cache_write(hk, hv, kc, vc, w.history_slots(s), w.cache_dtype, ks, vs)
    nk, nv = w.new_kv()
    kv_cache_write(nk, nv, kc, vc, w.new_token_slots(), w.cache_dtype, ks, vs)
    return kc, vc, ks, vs, w.query()


def decode(w, caches=None):
    kc, vc, ks, vs, q = caches or build_cache(w)
    return paged_attention_decode(q, kc, vc, w.block_tables, w.context_lens, w.sm_scale, w.cache_dtype, ks, vs)


def sdpa_reference(q, K, V, sm_scale):
    """torch's scaled_dot_product_attention in float64 on contiguous K/V.

    GQA is expressed by repeating each KV head for its consecutive group of
    query heads (repeat_interleave), independently of ``kv_head_of``.
    """
    n_q = q.shape[0]
    n_kv = K.shape[1]
    qt = torch.from_numpy(np.asarray(q, dtype=np.float64))[None, :, None, :]
    kt = torch.from_numpy(np.asarray(K, dtype=np.float64)).permute(1, 0, 2).repeat_interleave(n_q // n_kv, 0)[None]
    vt = torch.from_numpy(np.asarray(V, dtype=np.float64)).permute(1, 0, 2).repeat_interleave(n_q // n_kv, 0)[None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=sm_scale)
    return o[0, :, 0, :].numpy()


TINY_SHAPES = [
    # (lengths, n_q, n_kv, d, block_size)
    ([40, 17, 64, 5], 8, 2, 8, 16),
    ([1, 16, 33], 4, 4, 6, 16),  # MHA
    ([7, 20], 6, 1, 5, 4),  # MQA
    ([9], 3, 3, 4, 8),
    ([31, 2, 18], 8, 2, 4, 16),
]


# ------------------------------------------------------------------ golden pins
def test_block_table_example(golden):
    rec = {r[0]: r[1:] for r in golden("block_table_40_tokens.txt")}
    L, bs = int(rec["length"][0]), int(rec["block_size"][0])
    table = np.array([int(x) for x in rec["table"]])
    assert [logical_to_physical(table, p, bs)[0] for p in (0, 15, 16, 31, 32, 39)] == [7, 7, 2, 2, 14, 14]
    # a cache whose rows carry their own (block, row) coordinates
    nb = 16
    cache = np.zeros((nb, bs, 1, 2))
    cache[:, :, 0, 0] = np.arange(nb)[:, None]
    cache[:, :, 0, 1] = np.arange(bs)[None, :]
    g = gather_sequence(cache, table, L, bs)
    assert g.shape[0] == L
    assert g[:, 0, 0].tolist() == [7] * 16 + [2] * 16 + [14] * int(rec["tokens_in_last_block"][0])
    assert g[:, 0, 1].tolist() == list(range(16)) * 2 + list(range(8))


def test_gqa_mapping_example(golden):
    rows = golden("gqa_mapping.txt")
    hdr = {r[0]: int(r[1]) for r in rows[:3]}
    for r in rows[3:]:
        kv = int(r[2])
        mapping = [int(x) for x in r[4:12]]
        assert [pa.kv_head_of(h, hdr["query_heads"], kv) for h in range(hdr["query_heads"])] == mapping
        assert accounting.cached_scalars(kv, hdr["tokens"], hdr["head_size"]) == int(r[13])


# ------------------------------------------------------------------ brute force
def _tiny(lengths, n_q, n_kv, d, bs, seed, cache_dtype="f32"):
    return workloads.make_workload(
        "t", seed=seed, context_lens=lengths, n_q=n_q, n_kv=n_kv, head_dim=d, block_size=bs,
        act_dtype="f32", cache_dtype=cache_dtype, extra_blocks=3,
    )


def check_against_brute(decode_fn=decode):
    for i, (lengths, n_q, n_kv, d, bs) in enumerate(TINY_SHAPES):
        w = _tiny(lengths, n_q, n_kv, d, bs, seed=10 + i)
        caches = build_cache(w)
        out, _ = decode_fn(w, caches)
        kc, vc, _, _, q = caches
        ref = brute_decode(q.tolist(), kc.tolist(), vc.tolist(), w.block_tables.tolist(), w.context_lens, w.sm_scale, n_kv)
        np.testing.assert_allclose(out, np.array(ref), rtol=0, atol=1e-12)


def test_oracle_matches_brute_force():
    check_against_brute()


def test_tiny_config_matches_brute_force():
    w = workloads.tiny()
    caches = build_cache(w)
    out, lse = decode(w, caches)
    kc, vc, _, _, q = caches
    ref = brute_decode(q.tolist(), kc.tolist(), vc.tolist(), w.block_tables.tolist(), w.context_lens, w.sm_scale, w.n_kv)
    np.testing.assert_allclose(out, np.array(ref), rtol=0, atol=1e-12)
    assert np.isfinite(out).all() and np.isfinite(lse).all()


# ------------------------------------------------------------------ invariants
def check_contiguous_equals_sdpa(decode_fn=decode):
    """Paged result == torch SDPA on the un-paged rows the workload generated."""
    for i, (lengths, n_q, n_kv, d, bs) in enumerate(TINY_SHAPES + [([300, 129, 48], 16, 4, 32, 16)]):
        w = _tiny(lengths, n_q, n_kv, d, bs, seed=20 + i)
        out, _ = decode_fn(w, build_cache(w))
        q = w.query()
        for s in range(w.num_seqs):
            K, V = w.sequence_kv(s)
            np.testing.assert_allclose(out[s], sdpa_reference(q[s], K, V, w.sm_scale), rtol=0, atol=1e-12)


def test_paged_equals_contiguous_sdpa():
    check_contiguous_equals_sdpa()


def test_pool_permutation_invariance_bitwise():
    for cache_dtype in ("f32", "int8", "fp8_e4m3"):
        w = _tiny([40, 17, 64, 5], 8, 2, 16, 16, seed=3, cache_dtype=cache_dtype)
        kc, vc, ks, vs, q = build_cache(w)
        out, lse = decode(w, (kc, vc, ks, vs, q))
        perm = np.random.default_rng(1).permutation(w.num_blocks)  # new position of old block b is perm[b]
        kc2, vc2 = np.empty_like(kc), np.empty_like(vc)
        kc2[perm], vc2[perm] = kc, vc
        ks2, vs2 = ks, vs
        if cache_dtype == "int8":
            ks2, vs2 = np.empty_like(ks), np.empty_like(vs)
            ks2[perm], vs2[perm] = ks, vs
        tables = np.where(w.block_tables >= 0, perm[np.maximum(w.block_tables, 0)], -1)
        out2, lse2 = paged_attention_decode(q, kc2, vc2, tables, w.context_lens, w.sm_scale, cache_dtype, ks2, vs2)
        assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def test_softmax_rows_sum_to_one():
    rng = np.random.default_rng(0)
    for L in (1, 2, 17, 500):
        q = rng.standard_normal((8, 32))
        K = rng.standard_normal((L, 2, 32)) * 3
        V = rng.standard_normal((L, 2, 32))
        _, lse, weights = attention_one_sequence(q, K, V, 1 / math.sqrt(32), return_weights=True)
        for h, wts in enumerate(weights):
            assert abs(wts.sum() - 1.0) < 1e-12 and (wts >= 0).all()
            s = (K[:, h // 4, :] @ q[h]) / math.sqrt(32)
            assert abs(lse[h] - np.log(np.exp(s).sum())) < 1e-9


def test_closed_forms():
    rng = np.random.default_rng(1)
    K = rng.standard_normal((1, 2, 16))
    V = rng.standard_normal((1, 2, 16))
    q = rng.standard_normal((4, 16))
    out, lse = attention_one_sequence(q, K, V, 0.25)
    for h in range(4):
        assert np.array_equal(out[h], V[0, h // 2])  # one token: the output is its value row
        assert abs(lse[h] - 0.25 * K[0, h // 2] @ q[h]) < 1e-15
    K = rng.standard_normal((37, 2, 16))
    V = rng.standard_normal((37, 2, 16))
    out, lse = attention_one_sequence(np.zeros((4, 16)), K, V, 0.25)  # q = 0: uniform weights
    for h in range(4):
        np.testing.assert_allclose(out[h], V[:, h // 2].mean(axis=0), atol=1e-14)
        assert abs(lse[h] - math.log(37)) < 1e-14
    Keq = np.repeat(K[:1], 37, axis=0)  # all keys equal: uniform weights
    out, _ = attention_one_sequence(q, Keq, V, 0.25)
    for h in range(4):
        np.testing.assert_allclose(out[h], V[:, h // 2].mean(axis=0), atol=1e-14)


def test_empty_sequence_reading():
    out, lse = attention_one_sequence(np.ones((2, 4)), np.zeros((0, 1, 4)), np.zeros((0, 1, 4)), 1.0)
    assert not out.any() and np.isneginf(lse).all()


def test_identical_tables_identical_outputs():
    w = workloads.make_workload("p", seed=5, context_lens=[48 + 5, 48 + 20], n_q=4, n_kv=2, head_dim=8,
                                act_dtype="f32", cache_dtype="f32", shared_prefix_tokens=48)
    kc, vc, ks, vs, q = build_cache(w)
    # both sequences share the 3 prefix blocks
    assert (w.block_tables[0, :3] == w.block_tables[1, :3]).all()
    tables = np.stack([w.block_tables[0], w.block_tables[0]])
    lens = np.array([w.context_lens[0]] * 2)
    out, _ = paged_attention_decode(np.stack([q[0], q[0]]), kc, vc, tables, lens, w.sm_scale)
    assert np.array_equal(out[0], out[1])


# ------------------------------------------------------------------ quantised caches
@pytest.mark.parametrize("cache_dtype", ["int8", "fp8_e4m3"])
def test_quantized_decode_is_attention_over_dequantized_rows(cache_dtype):
    w = workloads.make_workload("q", seed=8, context_lens=[70, 33, 16], n_q=8, n_kv=2, head_dim=32,
                                act_dtype="bf16", cache_dtype=cache_dtype, outlier_fraction=0.05)
    kc, vc, ks, vs, q = build_cache(w)
    out, _ = decode(w, (kc, vc, ks, vs, q))
    t8 = torch.float8_e4m3fn
    for s in range(w.num_seqs):
        L = int(w.context_lens[s])
        rows = [(w.block_tables[s][p // 16], p % 16) for p in range(L)]
        if cache_dtype == "int8":
            K = np.stack([kc[b, r].astype(np.float64) * ks[b, r][:, None].astype(np.float64) for b, r in rows])
            V = np.stack([vc[b, r].astype(np.float64) * vs[b, r][:, None].astype(np.float64) for b, r in rows])
        else:
            dec = lambda a: torch.from_numpy(np.ascontiguousarray(a)).view(t8).to(torch.float64).numpy()
            K = np.stack([dec(kc[b, r]) * ks[:, None].astype(np.float64) for b, r in rows])
            V = np.stack([dec(vc[b, r]) * vs[:, None].astype(np.float64) for b, r in rows])
        np.testing.assert_allclose(out[s], sdpa_reference(q[s], K, V, w.sm_scale), atol=1e-12)
        # and it stays close to attention over the unquantised rows
        K0, V0 = w.sequence_kv(s)
        assert np.abs(out[s] - sdpa_reference(q[s], K0, V0, w.sm_scale)).max() < 0.2


def test_cache_write_slot_roundtrip():
    w = _tiny([40, 17, 64, 5], 8, 2, 8, 16, seed=4)
    kc, vc, _, _, _ = build_cache(w)
    for s in range(w.num_seqs):
        K, V = w.sequence_kv(s)
        g = gather_sequence(kc, w.block_tables[s], int(w.context_lens[s]), 16)
        assert np.array_equal(g, K)
        assert np.array_equal(gather_sequence(vc, w.block_tables[s], int(w.context_lens[s]), 16), V)
    # slot -1 writes nothing
    before = kc.copy()
    kv_cache_write(np.ones((1, 2, 8)), np.ones((1, 2, 8)), kc, vc, np.array([-1]))
    assert np.array_equal(before, kc, equal_nan=True)


def test_oracle_exports():
    assert oracle.paged_attention_decode is paged_attention_decode
