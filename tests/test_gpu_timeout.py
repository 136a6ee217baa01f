"""Bounded waits: a wait inside a kernel that runs out sets PKV_DEVERR_TIMEOUT
and the kernel returns instead of hanging, with no copy or tensor-core
operation left in flight; the stream and the context stay usable and the next
call matches the oracle.

The waits are made to run out by the test-only launch override
wait_limit_cycles = 1 (a wait not satisfied at once gives up): nothing faults
or hangs a GPU here.
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_467_b200 import workloads
from gpu_harness import assert_close, fill_gpu, oracle_sequence, run_decode

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from paged_kv_cache_467_b200 import build

    build.build()


def _ops():
    from paged_kv_cache_467_b200 import ops

    return ops


def _check_all(w, out, lse):
    for s in range(w.num_seqs):
        o, l, _ = oracle_sequence(w, s)
        assert_close(out[s], o, w.cache_dtype, f"seq {s}")
        np.testing.assert_allclose(lse[s], l, rtol=0, atol=2e-3)


@pytest.mark.parametrize("cache_dtype", ["bf16", "int8"])
def test_decode_waits_give_up_then_next_call_is_exact(cache_dtype):
    ops = _ops()
    w = workloads.make_workload("t", seed=91, context_lens=[700 + 37 * i for i in range(24)], n_q=32, n_kv=8,
                                head_dim=128, cache_dtype=cache_dtype)
    st = fill_gpu(w)
    short = ops.DecodeTuning(0, 0, 0, 0, 0, 0, 1)
    for _ in range(2):
        run_decode(w, st, tuning=short)
        assert int(st.device_error.item()) & ops.DEVERR_TIMEOUT
        st.device_error.zero_()
    out, lse = run_decode(w, st)
    assert int(st.device_error.item()) == 0
    _check_all(w, out, lse)


def test_shared_prefix_waits_give_up_then_next_call_is_exact():
    ops = _ops()
    w = workloads.make_workload("t", seed=92, context_lens=[600 + 29 * i for i in range(20)], n_q=32, n_kv=8,
                                head_dim=128, extra_blocks=3, shared_prefix_tokens=512)
    st = fill_gpu(w)

    def run(tuning):
        out = torch.full((w.num_seqs, w.n_q, w.head_dim), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((w.num_seqs, w.n_q), float("nan"), dtype=torch.float32, device="cuda")
        ops.paged_attention_decode_shared_prefix(out, st.query, st.key_cache, st.value_cache, st.block_tables,
                                                 st.context_lens, w.max_context_len, 32, sm_scale=w.sm_scale,
                                                 lse_out=lse, device_error=st.device_error, tuning=tuning)
        torch.cuda.synchronize()
        return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)

    run(ops.DecodeTuning(0, 0, 0, 0, 0, 0, 1))
    assert int(st.device_error.item()) & ops.DEVERR_TIMEOUT
    st.device_error.zero_()
    out, lse = run(None)
    assert int(st.device_error.item()) == 0
    _check_all(w, out, lse)


def test_wait_limit_must_not_be_negative():
    ops = _ops()
    w = workloads.make_workload("t", seed=93, context_lens=[40, 17], n_q=8, n_kv=2, head_dim=128)
    st = fill_gpu(w)
    with pytest.raises(ops.PkvError) as e:
        run_decode(w, st, tuning=ops.DecodeTuning(0, 0, 0, 0, 0, 0, -5))
    assert e.value.status == 1
