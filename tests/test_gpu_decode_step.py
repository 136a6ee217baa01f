"""The fused decode step (append token L-1 + attention in one launch) against
the oracle and against the two-call path (pkv_kv_cache_write, then decode)."""
import numpy as np
import pytest
import torch

from paged_kv_cache_467_b200 import workloads
from gpu_harness import fill_gpu, run_decode, run_decode_step
from test_gpu_parity import check_all

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from paged_kv_cache_467_b200 import build

    build.build()


CASES = [
    # lengths, n_q, n_kv, d, act, cache
    ([40, 17, 64, 5, 1, 16, 33, 700], 32, 8, 128, "bf16", "bf16"),
    ([300, 129, 48, 1000, 0, 17], 64, 8, 128, "bf16", "bf16"),
    ([200, 3, 511], 16, 1, 64, "bf16", "bf16"),
    ([40, 17, 64, 5, 1, 16, 33, 700], 32, 8, 128, "bf16", "int8"),
    ([300, 129, 48, 1000], 64, 8, 128, "f32", "int8"),
    ([40, 17, 64, 5, 1, 16, 33, 700], 32, 8, 128, "bf16", "fp8_e4m3"),
    ([40, 17, 64, 5, 0], 8, 2, 64, "f32", "f32"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[4]}-{c[5]}-q{c[1]}kv{c[2]}d{c[3]}")
def test_decode_step_matches_oracle_and_two_call_path(case):
    lengths, n_q, n_kv, d, act, cache = case
    w = workloads.make_workload("s", seed=41, context_lens=lengths, n_q=n_q, n_kv=n_kv, head_dim=d, act_dtype=act,
                                cache_dtype=cache, extra_blocks=4, outlier_fraction=0.01 if cache != "f32" else 0.0)
    st = fill_gpu(w, append_new=False)
    out, lse = run_decode_step(w, st)
    assert int(st.device_error.item()) == 0
    # every row, the appended one included, is bit-exact and the outputs match the oracle
    check_all(w, st, out, lse, fp8_scales=st.fp8_scales)
    # the two-call path on the same cache gives the same bits
    ref = fill_gpu(w, fp8_scales=st.fp8_scales)
    out2, lse2 = run_decode(w, ref)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def test_decode_step_full_llama_config():
    w = workloads.llama3_8b()
    st = fill_gpu(w, append_new=False)
    out, lse = run_decode_step(w, st)
    assert int(st.device_error.item()) == 0
    check_all(w, st, out, lse, seqs=range(0, 64, 7))
