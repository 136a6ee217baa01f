"""Pins for the oracle's block movers (CPU only)."""
import numpy as np

from oracle.block_ops import copy_blocks, swap_blocks
from oracle.paged_attention import kv_cache_write, paged_attention_decode
from test_oracle_attention import sdpa_reference


def _marked_block(value, shape=(16, 2, 8)):
    return np.full(shape, float(value))


def test_offload_example(golden):
    """The page's two-session GPU pool: C arrives, A moves out; A returns, B moves out."""
    rec = {r[0]: r[1:] for r in golden("offload_example.txt")}
    data = {"cache-a": 1.0, "cache-b": 2.0, "cache-c": 3.0}  # one block per session cache
    gpu = np.zeros((2, 16, 2, 8))
    cpu = np.zeros((2, 16, 2, 8))
    gpu_order, cpu_order = [], []  # session names, oldest first, with their block slots
    for slot, name in enumerate(rec["gpu_initial"]):
        gpu[slot] = _marked_block(data[name])
        gpu_order.append((name, slot))

    def move_out(cpu_slot):
        name, slot = gpu_order.pop(0)
        swap_blocks([gpu], [cpu], [(slot, cpu_slot)])
        cpu_order.append((name, cpu_slot))
        return slot

    # cache C needs GPU space, so the oldest cache moves to CPU memory
    free = move_out(cpu_slot=0)
    gpu[free] = _marked_block(data["cache-c"])
    gpu_order.append(("cache-c", free))
    assert [n for n, _ in gpu_order] == rec["gpu_after_c"] and [n for n, _ in cpu_order] == rec["cpu_after_c"]
    # cache A is needed again: the oldest GPU cache moves out, A comes back into the freed slot
    a_cpu = dict(cpu_order)["cache-a"]
    cpu_order = [e for e in cpu_order if e[0] != "cache-a"]
    free = move_out(cpu_slot=1)
    swap_blocks([cpu], [gpu], [(a_cpu, free)])
    gpu_order.append(("cache-a", free))
    assert [n for n, _ in gpu_order] == rec["gpu_after_a_returns"]
    assert [n for n, _ in cpu_order] == rec["cpu_after_a_returns"]
    # the data moved with the names
    for name, slot in gpu_order:
        assert (gpu[slot] == data[name]).all()
    for name, slot in cpu_order:
        assert (cpu[slot] == data[name]).all()


def test_copy_on_write_divergence():
    """Two sequences share 40 tokens (blocks p0, p1 and a partly filled p2); each
    then appends a different token.  B copies p2 before writing, so both see
    their own history plus their own new token."""
    rng = np.random.default_rng(0)
    n_kv, d, bs = 2, 8, 16
    kc = np.full((6, bs, n_kv, d), np.nan)
    vc = np.full_like(kc, np.nan)
    hist_k, hist_v = rng.standard_normal((40, n_kv, d)), rng.standard_normal((40, n_kv, d))
    shared = np.array([4, 1, 3])
    kv_cache_write(hist_k, hist_v, kc, vc, shared[np.arange(40) // bs] * bs + np.arange(40) % bs)
    new_a = rng.standard_normal((2, 1, n_kv, d))
    new_b = rng.standard_normal((2, 1, n_kv, d))
    # divergence: B takes a private copy of the shared last block, then both append row 8
    copy_blocks([kc, vc], [(3, 5)])
    table_a, table_b = shared, np.array([4, 1, 5])
    kv_cache_write(new_a[0], new_a[1], kc, vc, [3 * bs + 8])
    kv_cache_write(new_b[0], new_b[1], kc, vc, [5 * bs + 8])
    q = rng.standard_normal((2, 4, d))
    out, _ = paged_attention_decode(q, kc, vc, np.stack([table_a, table_b]), np.array([41, 41]), 0.3)
    for i, new in enumerate((new_a, new_b)):
        K = np.concatenate([hist_k, new[0]])
        V = np.concatenate([hist_v, new[1]])
        np.testing.assert_allclose(out[i], sdpa_reference(q[i], K, V, 0.3), atol=1e-12)
    # the shared full blocks were never copied or written
    assert np.array_equal(kc[4], np.concatenate([hist_k[:16]])) and np.array_equal(kc[1], hist_k[16:32])


def test_copy_reads_all_sources_first():
    pool = np.arange(4, dtype=np.float64)[:, None] * np.ones((4, 3))
    copy_blocks([pool], [(0, 1), (1, 2)])
    assert pool[:, 0].tolist() == [0.0, 0.0, 1.0, 3.0]


def test_copy_moves_int8_scales_with_codes():
    codes = np.arange(3 * 2 * 4, dtype=np.int8).reshape(3, 2, 4)
    scales = np.arange(3 * 2, dtype=np.float32).reshape(3, 2)
    copy_blocks([codes, scales], [(2, 0)])
    assert np.array_equal(codes[0], codes[2]) and np.array_equal(scales[0], scales[2])


def test_swap_round_trip_keeps_attention_bitwise():
    rng = np.random.default_rng(1)
    kc = rng.standard_normal((5, 16, 2, 8))
    vc = rng.standard_normal((5, 16, 2, 8))
    table = np.array([[3, 0, 4]])
    q = rng.standard_normal((1, 4, 8))
    before, lse = paged_attention_decode(q, kc, vc, table, np.array([40]), 0.5)
    host_k, host_v = np.zeros((3, 16, 2, 8)), np.zeros((3, 16, 2, 8))
    swap_blocks([kc, vc], [host_k, host_v], [(3, 0), (0, 1), (4, 2)])  # offload
    kc[:] = np.nan
    vc[:] = np.nan
    swap_blocks([host_k, host_v], [kc, vc], [(0, 1), (1, 2), (2, 0)])  # restore elsewhere
    after, lse2 = paged_attention_decode(q, kc, vc, np.array([[1, 2, 0]]), np.array([40]), 0.5)
    assert np.array_equal(before, after) and np.array_equal(lse, lse2)
