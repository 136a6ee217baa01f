"""Byte accounting against the pages' figures, and the seeded input builders (CPU only)."""
import numpy as np

from paged_kv_cache_467_b200 import accounting, workloads


def test_capacity_figures(golden):
    for r in golden("capacity_figures.txt"):
        kv = dict(zip(r[1::2], (float(x) for x in r[2::2])))
        if r[0] == "block":
            assert accounting.block_bytes(int(kv["block_size"]), int(kv["kv_heads"]), int(kv["head_dim"]), kv["bytes"]) == kv["total_bytes"]
        elif r[0].startswith("llama70b"):
            b = accounting.cache_bytes(int(kv["layers"]), int(kv["kv_heads"]), int(kv["head_dim"]), int(kv["tokens"]), kv["bytes"])
            assert b == kv["approx_gib"] * 2 ** 30
            per_token = accounting.cache_bytes(int(kv["layers"]), int(kv["kv_heads"]), int(kv["head_dim"]), 1, kv["bytes"])
            if kv["kv_heads"] == 8:
                assert per_token == 320 * 1024
                assert accounting.cache_bytes(80, 8, 128, 1, 1) == 160 * 1024  # FP8: one byte per value
        elif r[0] == "pool":
            assert accounting.tokens_in_pool(kv["pool_gib"] * 2 ** 30, kv["per_token_kib"] * 1024) == kv["tokens"]


def test_free_list_example(golden):
    rows = golden("free_list_example.txt")
    pool = workloads.BlockPool([int(x) for x in rows[0][1:]])
    a = pool.allocate(int(rows[1][1]))
    b = pool.allocate(int(rows[2][1]))
    assert a == [int(x) for x in rows[1][3:]] and b == [int(x) for x in rows[2][3:]]
    pool.release(a)
    assert pool.free == [int(x) for x in rows[3][1:]]
    assert pool.allocate(int(rows[4][1])) == [int(x) for x in rows[4][3:]]


def _check_tables(w):
    used = []
    for s, L in enumerate(w.context_lens):
        n = workloads.blocks_for(L, w.block_size)
        row = w.block_tables[s]
        assert (row[:n] >= 0).all() and (row[:n] < w.num_blocks).all() and (row[n:] == -1).all()
        used.append(row[:n])
    return np.concatenate(used)


def test_tiny_config():
    w = workloads.tiny()
    assert w.context_lens.tolist() == [40, 17, 64, 5]
    assert (w.n_q, w.n_kv, w.head_dim, w.block_size, w.num_blocks) == (8, 2, 64, 16, 32)
    used = _check_tables(w)
    assert len(used) == 10 and len(set(used.tolist())) == 10
    slots = w.new_token_slots()
    rows = slots % 16
    assert rows.tolist() == [7, 0, 15, 4]  # partial block, fresh block, block filled exactly, first block
    assert (slots // 16).tolist() == [w.block_tables[0, 2], w.block_tables[1, 1], w.block_tables[2, 3], w.block_tables[3, 0]]
    again = workloads.tiny()
    assert np.array_equal(again.block_tables, w.block_tables) and np.array_equal(again.query(), w.query())


def test_llama_config_pool_fits_exactly():
    w = workloads.llama3_8b()
    assert w.num_seqs == 64 and w.context_lens.min() >= 512 and w.context_lens.max() <= 4096
    used = _check_tables(w)
    assert len(used) == w.num_blocks and len(np.unique(used)) == w.num_blocks
    assert w.kv_bytes_read() == int(w.context_lens.sum()) * 8 * 128 * 2 * 2


def test_prefix_config_shares_blocks():
    w = workloads.prefix_sharing()
    assert w.num_seqs == 128
    suffix = w.context_lens - 2048
    assert suffix.min() >= 64 and suffix.max() <= 512
    assert (w.block_tables[:, :128] == w.block_tables[0, :128]).all()
    private = np.concatenate([w.block_tables[s, 128 : workloads.blocks_for(L, 16)] for s, L in enumerate(w.context_lens)])
    assert len(np.unique(private)) == len(private) and not np.isin(private, w.block_tables[0, :128]).any()
    assert w.num_blocks == 128 + len(private)
    # the appended token lands in a private block
    assert np.isin(w.new_token_slots() // 16, private).all()
    logical = accounting.decode_kv_bytes(w, unique=False)
    unique = accounting.decode_kv_bytes(w, unique=True)
    assert logical - unique == 127 * 2048 * 8 * 128 * 2 * 2


def test_quantized_config_outliers():
    w = workloads.quantized("int8")
    assert w.num_seqs == 256 and len(w.k_outlier_channels) == 10
    assert w.kv_bytes_read() == int(w.context_lens.sum()) * (8 * 128 * 2 + 8 * 2 * 4)
    k, _ = w.new_kv()
    flat = np.abs(k.reshape(256, -1))
    assert flat[:, w.k_outlier_channels].mean() > 5 * flat.mean()


def test_sequence_rows_cover_context():
    w = workloads.make_workload("x", seed=1, context_lens=[33, 1, 64], n_q=4, n_kv=2, head_dim=8, act_dtype="f32", cache_dtype="f32")
    for s, L in enumerate(w.context_lens):
        k, v = w.sequence_kv(s)
        assert k.shape == (L, 2, 8) and v.shape == (L, 2, 8)
        assert len(w.history_slots(s)) == L - 1
    assert w.query().dtype == np.float32


def test_kivi_bytes_and_bench_oracle_step():
    """KIVI step bytes: 1600 B per full block and KV head (codes, K channel
    scales, V token scales) plus the BF16 residual rows; the bench's oracle
    step appends, quantises a completed block and decodes like the oracle's
    own sequence decode."""
    import numpy as np

    import bench
    import oracle
    from paged_kv_cache_467_b200 import accounting, workloads

    assert accounting.kivi_block_bytes(1, 128) == 1600
    w = workloads.make_workload("kivi_cpu", seed=5, context_lens=[16, 21, 32, 3], n_q=4, n_kv=2, head_dim=128,
                                cache_dtype="kivi2")
    want = sum((L // 16) * 2 * 1600 + (L % 16) * 2 * 128 * 2 * 2 for L in (16, 21, 32, 3))
    assert accounting.decode_kv_bytes(w) == want
    rows = bench.prepare_oracle_rows(w, range(4))
    assert bench.oracle_step_sample(w, range(4), rows) == want
    q = w.query()
    for s in range(4):
        blocks, rk, rv, K, V, _ = rows[s]
        L = int(w.context_lens[s])
        assert len(blocks) == (L - 1) // 16 and rk.shape[0] == (L - 1) % 16
        out, _ = oracle.kivi_decode_sequence(q[s], K[:L], V[:L], w.sm_scale)
        assert np.isfinite(out).all()
