"""GPU parity of the shared-prefix decode (a dense pass over the blocks every
sequence shares, then each sequence's own blocks) against the oracle's plain
decode ("Chapter 18 - KV-Cache Optimization Strategies", Prefix Caching)."""
import numpy as np
import pytest
import torch

from paged_kv_cache_467_b200 import workloads
from gpu_harness import assert_close, assert_rows_bit_exact, fill_gpu, new_rows, oracle_sequence, run_decode

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


def run_shared(w, st, append=False):
    ops = _ops()
    out = torch.full((w.num_seqs, w.n_q, w.head_dim), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((w.num_seqs, w.n_q), float("nan"), dtype=torch.float32, device="cuda")
    k = v = None
    if append:
        k, v = new_rows(w)
    ops.paged_attention_decode_shared_prefix(out, st.query, st.key_cache, st.value_cache, st.block_tables,
                                             st.context_lens, w.max_context_len, w.shared_prefix_tokens // 16,
                                             key=k, value=v, sm_scale=w.sm_scale, lse_out=lse,
                                             device_error=st.device_error)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def check(w, st, out, lse, seqs=None, rows=False):
    for s in range(w.num_seqs) if seqs is None else seqs:
        o, l, orows = oracle_sequence(w, s)
        assert_close(out[s], o, "bf16", f"seq {s}")
        np.testing.assert_allclose(lse[s], l, rtol=0, atol=2e-3)
        if rows:
            assert_rows_bit_exact(w, st, s, orows)


CASES = [
    # lengths, shared prefix tokens, n_q, n_kv, d
    ([100, 80, 65, 200, 17 + 64], 64, 32, 8, 128),  # G 4, 20 query rows per KV head (a ragged tile)
    ([300, 290, 1000, 600], 256, 64, 8, 128),  # G 8
    ([40, 33, 90], 32, 8, 8, 128),  # MHA
    ([500, 260, 300], 240, 32, 2, 128),  # G 16 (two warps per KV head in the decode)
    ([70, 90, 19, 200, 33, 48], 16, 16, 4, 64),  # d 64, one prefix block
    ([17, 33, 49], 16, 32, 8, 128),  # one private token past a one-block prefix
    ([1025, 2048 + 7, 1500], 1024, 32, 8, 128),  # long prefix: several splits
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"P{c[1]}-q{c[2]}kv{c[3]}d{c[4]}")
def test_shared_prefix_matches_oracle(case):
    lengths, prefix, n_q, n_kv, d = case
    w = workloads.make_workload("p", seed=81, context_lens=lengths, n_q=n_q, n_kv=n_kv, head_dim=d, extra_blocks=3,
                                shared_prefix_tokens=prefix)
    st = fill_gpu(w)
    out, lse = run_shared(w, st)
    check(w, st, out, lse)
    assert int(st.device_error.item()) == 0
    # the plain decode on the same cache agrees within the bf16 tolerance
    plain, _ = run_decode(w, st)
    assert np.abs(plain - out).max() <= 2e-2


def test_shared_prefix_with_fused_append():
    w = workloads.make_workload("p", seed=82, context_lens=[100, 81, 200, 65], n_q=32, n_kv=8, head_dim=128,
                                extra_blocks=3, shared_prefix_tokens=64)
    st = fill_gpu(w, append_new=False)
    out, lse = run_shared(w, st, append=True)
    assert int(st.device_error.item()) == 0
    check(w, st, out, lse, rows=True)


def test_prefix_config_sampled():
    w = workloads.prefix_sharing()
    st = fill_gpu(w)
    shared = torch.from_numpy(w.shared_prefix_blocks.astype(np.int64)).cuda()
    before = st.key_cache.index_select(0, shared).clone()
    out, lse = run_shared(w, st)
    assert int(st.device_error.item()) == 0
    assert torch.equal(before.view(torch.int16), st.key_cache.index_select(0, shared).view(torch.int16))
    check(w, st, out, lse, seqs=range(0, 128, 11))
    again, lse2 = run_shared(w, st)
    assert np.array_equal(out, again) and np.array_equal(lse, lse2)  # deterministic
