"""pkv_paged_attention_decode_static: decode for callers that cannot allocate.

Such a caller (for example a plug-in whose host runtime owns all device memory,
or a loop that must not call cudaMalloc) gets its scratch from a fixed array
inside libpkv.  These tests call that entry point through the C ABI and check
it against the oracle and against pkv_paged_attention_decode, which takes a
caller-owned workspace, on two calls in a row: the second call finds the array
as the first one left it.  The file is named to be collected last.
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_467_b200 import workloads
from gpu_harness import TOL, assert_close, fill_gpu, oracle_sequence, run_decode

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from paged_kv_cache_467_b200 import build

    build.build()


def _static_decode(w, st):
    from paged_kv_cache_467_b200 import ops

    out = torch.full((w.num_seqs, w.n_q, w.head_dim), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((w.num_seqs, w.n_q), float("nan"), dtype=torch.float32, device="cuda")
    ops.paged_attention_decode_static(out, st.query, st.key_cache, st.value_cache, st.block_tables, st.context_lens,
                                      w.max_context_len, w.sm_scale, st.k_scale, st.v_scale, lse, st.device_error)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def _compare(got, want, cache_dtype):
    mx_tol, mean_tol = TOL[cache_dtype]
    assert np.isfinite(got).all()
    d = np.abs(got - want)
    assert d.max() <= mx_tol and d.mean() <= mean_tol, (d.max(), d.mean())


def test_static_scratch_matches_workspace_entry_point_two_calls_in_a_row():
    # two different shapes back to back: many short units, then few long ones
    first = workloads.make_workload("a", seed=31, context_lens=[300 + 37 * i for i in range(48)], n_q=32, n_kv=8,
                                    head_dim=128)
    second = workloads.make_workload("b", seed=32, context_lens=[9000, 4100, 17, 6000], n_q=64, n_kv=8, head_dim=128,
                                     cache_dtype="int8")
    for w in (first, second):
        st = fill_gpu(w)
        want, want_lse = run_decode(w, st)
        got, got_lse = _static_decode(w, st)
        _compare(got, want, w.cache_dtype)
        np.testing.assert_allclose(got_lse, want_lse, rtol=0, atol=2e-3)
        assert int(st.device_error.item()) == 0
        for s in range(w.num_seqs):  # and against the oracle directly
            o, l, _ = oracle_sequence(w, s)
            assert_close(got[s], o, w.cache_dtype, f"{w.name} seq {s}")
            np.testing.assert_allclose(got_lse[s], l, rtol=0, atol=2e-3)


def test_static_scratch_rejects_shapes_beyond_its_size():
    from paged_kv_cache_467_b200 import ops

    # 64 query heads on one KV head: the partial results need ~39 MB, more than the 16 MiB array
    w = workloads.make_workload("c", seed=33, context_lens=[500, 70], n_q=64, n_kv=1, head_dim=128)
    st = fill_gpu(w)
    out = torch.full((w.num_seqs, w.n_q, w.head_dim), 7.0, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ops.PkvError) as e:
        ops.paged_attention_decode_static(out, st.query, st.key_cache, st.value_cache, st.block_tables,
                                          st.context_lens, w.max_context_len, w.sm_scale)
    assert e.value.status == 3 and "bytes of scratch" in str(e.value)
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())  # nothing was launched
