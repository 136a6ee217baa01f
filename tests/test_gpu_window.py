"""GPU parity of sliding-window + attention-sink decode against the oracle."""
import numpy as np
import pytest
import torch

from paged_kv_cache_467_b200 import workloads
from gpu_harness import assert_close, fill_gpu, oracle_sequence

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from paged_kv_cache_467_b200 import build

    build.build()


def run_window(w, st, window, sinks, tables=None):
    from paged_kv_cache_467_b200 import ops

    dt = torch.float32 if w.act_dtype == "f32" else torch.bfloat16
    out = torch.full((w.num_seqs, w.n_q, w.head_dim), float("nan"), dtype=dt, device="cuda")
    lse = torch.full((w.num_seqs, w.n_q), float("nan"), dtype=torch.float32, device="cuda")
    ops.paged_attention_decode_window(out, st.query, st.key_cache, st.value_cache,
                                      st.block_tables if tables is None else tables, st.context_lens,
                                      w.max_context_len, window, sinks, w.sm_scale, st.k_scale, st.v_scale, lse,
                                      device_error=st.device_error)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def check(w, st, out, lse, window, sinks):
    for s in range(w.num_seqs):
        o, l, _ = oracle_sequence(w, s, st.fp8_scales, window=window, sinks=sinks)
        assert_close(out[s], o, w.cache_dtype, f"seq {s} (window {window}, sinks {sinks})")
        if int(w.context_lens[s]) > 0:
            np.testing.assert_allclose(lse[s], l, rtol=0, atol=2e-3 if w.cache_dtype != "f32" else 1e-5)


LENGTHS = [1000, 17, 64, 5, 300, 1, 1201, 129]


@pytest.mark.parametrize("window,sinks", [(256, 4), (100, 0), (64, 16), (33, 40), (1, 0), (500, 300), (4092, 4),
                                          (10, 7)])
def test_window_bf16(window, sinks):
    w = workloads.make_workload("w", seed=61, context_lens=LENGTHS, n_q=32, n_kv=8, head_dim=128, extra_blocks=3)
    st = fill_gpu(w)
    out, lse = run_window(w, st, window, sinks)
    check(w, st, out, lse, window, sinks)
    assert int(st.device_error.item()) == 0


@pytest.mark.parametrize("cache,act,d", [("int8", "bf16", 128), ("fp8_e4m3", "bf16", 128), ("f32", "f32", 64)])
def test_window_other_caches(cache, act, d):
    w = workloads.make_workload("w", seed=62, context_lens=LENGTHS, n_q=16, n_kv=4, head_dim=d, act_dtype=act,
                                cache_dtype=cache, extra_blocks=3, outlier_fraction=0.01 if cache != "f32" else 0.0)
    st = fill_gpu(w)
    for window, sinks in [(256, 4), (33, 40), (1, 0)]:
        out, lse = run_window(w, st, window, sinks)
        check(w, st, out, lse, window, sinks)
    assert int(st.device_error.item()) == 0


def test_freed_blocks_are_not_read():
    """Blocks outside the sinks and the window are freed: table entry -1 and
    poisoned content.  No range error, same result."""
    window, sinks = 200, 4
    w = workloads.make_workload("w", seed=63, context_lens=[1000, 700, 1201], n_q=32, n_kv=8, head_dim=128)
    st = fill_gpu(w)
    out, lse = run_window(w, st, window, sinks)
    tables = w.block_tables.copy()
    for s, L in enumerate(w.context_lens):
        keep = set()
        for p in list(range(min(sinks, L))) + list(range(max(L - window, 0), L)):
            keep.add(p // 16)
        for j in range(workloads.blocks_for(L, 16)):
            if j not in keep:
                st.key_cache[int(tables[s, j])] = float("nan")
                st.value_cache[int(tables[s, j])] = float("nan")
                tables[s, j] = -1
    out2, lse2 = run_window(w, st, window, sinks, torch.from_numpy(tables).cuda())
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)
    assert int(st.device_error.item()) == 0


def test_window_covering_everything_equals_full_decode():
    from gpu_harness import run_decode

    w = workloads.make_workload("w", seed=64, context_lens=LENGTHS, n_q=32, n_kv=8, head_dim=128)
    st = fill_gpu(w)
    full, lse_full = run_decode(w, st)
    out, lse = run_window(w, st, max(LENGTHS), 0)
    assert np.array_equal(out, full) and np.array_equal(lse, lse_full)
    out0, lse0 = run_window(w, st, 0, 5)
    assert np.array_equal(out0, full) and np.array_equal(lse0, lse_full)


@pytest.mark.parametrize("cache,act,d", [("bf16", "bf16", 128), ("int8", "bf16", 128), ("fp8_e5m2", "bf16", 128),
                                         ("f32", "f32", 64)])
def test_fused_window_step(cache, act, d):
    """Append token L-1 and attend over the window and sinks in one call: the
    appended rows are bit-exact and the outputs match the oracle."""
    from paged_kv_cache_467_b200 import ops
    from gpu_harness import assert_rows_bit_exact, named, new_rows

    window, sinks = 200, 4
    w = workloads.make_workload("w", seed=64, context_lens=LENGTHS, n_q=16, n_kv=4, head_dim=d, act_dtype=act,
                                cache_dtype=cache, extra_blocks=3, outlier_fraction=0.01 if cache != "f32" else 0.0)
    st = fill_gpu(w, append_new=False)
    k, v = new_rows(w)
    dt = torch.float32 if act == "f32" else torch.bfloat16
    out = torch.full((w.num_seqs, w.n_q, w.head_dim), float("nan"), dtype=dt, device="cuda")
    lse = torch.full((w.num_seqs, w.n_q), float("nan"), dtype=torch.float32, device="cuda")
    ops.paged_decode_step_window(out, st.query, k, v, st.key_cache, st.value_cache, st.block_tables, st.context_lens,
                                 w.max_context_len, window, sinks, w.sm_scale, st.k_scale, st.v_scale, lse,
                                 device_error=st.device_error, cache_dtype=named(w))
    torch.cuda.synchronize()
    assert int(st.device_error.item()) == 0
    got = out.float().cpu().numpy().astype(np.float64)
    gl = lse.cpu().numpy().astype(np.float64)
    check(w, st, got, gl, window, sinks)
    for s in range(w.num_seqs):
        _, _, rows = oracle_sequence(w, s, st.fp8_scales, window=window, sinks=sinks)
        assert_rows_bit_exact(w, st, s, rows)
