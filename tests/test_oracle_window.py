"""Pins for sliding-window + attention-sink decode in the oracle (CPU only)."""
import numpy as np

import oracle.paged_attention as pa
from oracle.paged_attention import attended_positions, kv_cache_write, paged_attention_decode
from test_oracle_attention import sdpa_reference


def test_sliding_window_example(golden):
    rows = golden("sliding_window_example.txt")
    window = int(rows[0][1])
    for r in rows[1:-1]:
        t = int(r[1])
        want = [int(x) for x in r[3:]]
        assert pa.attended_positions(t + 1, window).tolist() == want
    assert max(len(pa.attended_positions(L, window)) for L in range(1, 40)) == int(rows[-1][1])


def test_attention_sink_layout(golden):
    rec = {r[0]: int(r[1]) for r in golden("attention_sinks_layout.txt")}
    for L in (4096, 4097, 10000):
        keep = pa.attended_positions(L, rec["window"], rec["sinks"])
        assert len(keep) == rec["entries"]
        assert keep[: rec["sinks"]].tolist() == list(range(rec["sinks"]))
        assert keep[rec["sinks"] :].tolist() == list(range(L - rec["window"], L))
    # shorter than sinks + window: nothing is dropped
    assert pa.attended_positions(3000, rec["window"], rec["sinks"]).tolist() == list(range(3000))


def test_window_zero_and_wide_window_are_full_attention():
    assert attended_positions(37, 0).tolist() == list(range(37))
    assert attended_positions(37, 37).tolist() == list(range(37))
    assert attended_positions(37, 36, 1).tolist() == list(range(37))


def _pool(seed, L, n_kv=2, d=8, nb_extra=3):
    rng = np.random.default_rng(seed)
    nb = -(-L // 16) + nb_extra
    kc = np.full((nb, 16, n_kv, d), np.nan)
    vc = np.full_like(kc, np.nan)
    table = rng.permutation(nb)[: -(-L // 16)]
    K, V = rng.standard_normal((L, n_kv, d)), rng.standard_normal((L, n_kv, d))
    kv_cache_write(K, V, kc, vc, table[np.arange(L) // 16] * 16 + np.arange(L) % 16)
    return kc, vc, table, K, V, rng.standard_normal((1, 4, d))


def test_windowed_decode_is_attention_over_kept_rows():
    for L, W, S in [(100, 20, 4), (100, 20, 0), (50, 10, 30), (17, 5, 4), (64, 16, 16), (33, 1, 0)]:
        kc, vc, table, K, V, q = _pool(L, L)
        out, lse = paged_attention_decode(q, kc, vc, table[None], [L], 0.35, window=W, sinks=S)
        keep = attended_positions(L, W, S)
        np.testing.assert_allclose(out[0], sdpa_reference(q[0], K[keep], V[keep], 0.35), atol=1e-12)
        full, _ = paged_attention_decode(q, kc, vc, table[None], [L], 0.35)
        assert not np.allclose(out, full)


def test_evicted_blocks_are_never_read():
    L, W, S = 200, 40, 4
    kc, vc, table, K, V, q = _pool(7, L)
    out, _ = paged_attention_decode(q, kc, vc, table[None], [L], 0.35, window=W, sinks=S)
    # blocks holding neither sinks nor window positions are freed: table entry -1, content poisoned
    keep_blocks = set((attended_positions(L, W, S) // 16).tolist())
    t2 = table.copy()
    for j in range(len(t2)):
        if j not in keep_blocks:
            kc[t2[j]] = np.nan
            vc[t2[j]] = np.nan
            t2[j] = -1
    out2, _ = paged_attention_decode(q, kc, vc, t2[None], [L], 0.35, window=W, sinks=S)
    assert np.array_equal(out, out2)
