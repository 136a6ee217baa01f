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
    ([40, 17, 64, 5, 1, 16, 33, 700], 32, 8, 128, "bf16", "fp8_e5m2"),
    ([40, 17, 64, 5, 1, 16, 33, 700], 32, 8, 128, "bf16", "int4"),
    ([300, 129, 48, 1000], 64, 8, 128, "f32", "int4"),
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


def test_overlapped_prologue_in_a_step_loop():
    """PKV_TUNE_OVERLAP_PROLOGUE: each step's query and new rows come from a
    torch kernel launched just before the decode, so a decode that read them
    before its wait would see the previous step's values."""
    from paged_kv_cache_467_b200 import ops

    w = workloads.make_workload("o", seed=43, context_lens=[900 + 61 * i for i in range(24)], n_q=32, n_kv=8,
                                head_dim=128)
    a = fill_gpu(w, append_new=False)
    b = fill_gpu(w, append_new=False)
    over = ops.DecodeTuning(0, 0, 0, ops.TUNE_OVERLAP_PROLOGUE)
    gen = torch.Generator(device="cuda").manual_seed(5)
    S, nq, nkv, d = w.num_seqs, w.n_q, w.n_kv, w.head_dim
    q = torch.empty((S, nq, d), dtype=torch.bfloat16, device="cuda")
    k = torch.empty((S, nkv, d), dtype=torch.bfloat16, device="cuda")
    v = torch.empty_like(k)
    out_a, out_b = torch.empty_like(q), torch.empty_like(q)
    for step in range(6):
        k.copy_(torch.randn((S, nkv, d), device="cuda", generator=gen))
        v.copy_(torch.randn((S, nkv, d), device="cuda", generator=gen))
        q.copy_(torch.randn((S, nq, d), device="cuda", generator=gen))  # the kernel right before the decode
        ops.paged_decode_step(out_a, q, k, v, a.key_cache, a.value_cache, a.block_tables, a.context_lens,
                              w.max_context_len, w.sm_scale, tuning=over, device_error=a.device_error)
        ops.paged_decode_step(out_b, q, k, v, b.key_cache, b.value_cache, b.block_tables, b.context_lens,
                              w.max_context_len, w.sm_scale, device_error=b.device_error)
        torch.cuda.synchronize()
        assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16)), f"step {step}"
    assert torch.equal(a.key_cache.view(torch.int16), b.key_cache.view(torch.int16))
    assert int(a.device_error.item()) == 0 and int(b.device_error.item()) == 0
