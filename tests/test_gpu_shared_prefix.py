"""GPU parity of the shared-prefix decode (a dense tensor-core pass over the
blocks every sequence shares, beside the paged decode of each sequence's own
blocks, then the merge of both) against the oracle's plain decode ("Chapter 18
- KV-Cache Optimization Strategies", Prefix Caching), and the device checks of
the prefix contract."""
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


def run_shared(w, st, append=False, tuning=None, prefix_blocks=None):
    ops = _ops()
    out = torch.full((w.num_seqs, w.n_q, w.head_dim), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((w.num_seqs, w.n_q), float("nan"), dtype=torch.float32, device="cuda")
    k = v = None
    if append:
        k, v = new_rows(w)
    pb = w.shared_prefix_tokens // 16 if prefix_blocks is None else prefix_blocks
    ops.paged_attention_decode_shared_prefix(out, st.query, st.key_cache, st.value_cache, st.block_tables,
                                             st.context_lens, w.max_context_len, pb, key=k, value=v,
                                             sm_scale=w.sm_scale, lse_out=lse, device_error=st.device_error,
                                             tuning=tuning)
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


def test_prefix_pass_beside_and_after_the_decode_agree():
    """The prefix pass running beside the decode, or before it, and any number
    of splits along the prefix: the same pieces, merged in the same order."""
    ops = _ops()
    w = workloads.make_workload("p", seed=83, context_lens=[1100 + 61 * i for i in range(40)], n_q=32, n_kv=8,
                                head_dim=128, extra_blocks=3, shared_prefix_tokens=1024)
    st = fill_gpu(w)
    results = {}
    for splits in (0, 1, 3, 16):
        for serial in (False, True):
            tun = ops.DecodeTuning(0, 0, 0, ops.TUNE_PREFIX_SERIAL if serial else 0, splits)
            out, lse = run_shared(w, st, tuning=tun)
            assert int(st.device_error.item()) == 0
            check(w, st, out, lse, seqs=range(0, 40, 7))
            results[(splits, serial)] = (out, lse)
        # the order of the two passes does not change a bit
        assert np.array_equal(results[(splits, False)][0], results[(splits, True)][0])
        assert np.array_equal(results[(splits, False)][1], results[(splits, True)][1])


def test_repeated_calls_are_bitwise_equal():
    """The same call, repeated, gives the same bits (every piece is written by
    one CTA at a fixed place and merged in a fixed order): per split setting
    and order of the passes, four calls, outputs compared byte for byte."""
    ops = _ops()
    w = workloads.make_workload("p", seed=83, context_lens=[1100 + 61 * i for i in range(40)], n_q=32, n_kv=8,
                                head_dim=128, extra_blocks=3, shared_prefix_tokens=1024)
    st = fill_gpu(w)
    for splits in (0, 1, 3):
        for serial in (False, True):
            tun = ops.DecodeTuning(0, 0, 0, ops.TUNE_PREFIX_SERIAL if serial else 0, splits)
            first, first_lse = run_shared(w, st, tuning=tun)
            for _ in range(3):
                out, lse = run_shared(w, st, tuning=tun)
                assert np.array_equal(out, first) and np.array_equal(lse, first_lse), (splits, serial)
            assert int(st.device_error.item()) == 0


def test_sequence_shorter_than_prefix_is_flagged():
    """A context that does not reach past the shared prefix sets the context-length
    bit; the other sequences are unaffected."""
    ops = _ops()
    w = workloads.make_workload("p", seed=84, context_lens=[200, 150, 90, 300], n_q=32, n_kv=8, head_dim=128,
                                extra_blocks=3, shared_prefix_tokens=64)
    st = fill_gpu(w)
    lens = st.context_lens.clone()
    lens[2] = 50  # inside the 64-token prefix
    st.context_lens = lens
    out, lse = run_shared(w, st)
    assert int(st.device_error.item()) & ops.DEVERR_CONTEXT_LEN
    assert not int(st.device_error.item()) & ops.DEVERR_PREFIX
    check(w, st, out, lse, seqs=[0, 1, 3])


def test_table_that_leaves_the_prefix_is_flagged():
    """A block table whose first entries are not row 0's sets PKV_DEVERR_PREFIX.
    Here the diverging block is a byte copy of the shared one, so every output
    still matches the oracle."""
    ops = _ops()
    w = workloads.make_workload("p", seed=85, context_lens=[200, 150, 90, 300], n_q=32, n_kv=8, head_dim=128,
                                extra_blocks=3, shared_prefix_tokens=64)
    st = fill_gpu(w)
    used = set(int(b) for b in w.block_tables.reshape(-1) if b >= 0)
    spare = next(b for b in range(w.num_blocks) if b not in used)
    src = int(w.block_tables[2, 1])
    pairs = torch.tensor([[src, spare]], dtype=torch.int64, device="cuda")
    ops.copy_blocks(st.key_cache, st.value_cache, pairs)
    tables = st.block_tables.clone()
    tables[2, 1] = spare
    st.block_tables = tables
    out, lse = run_shared(w, st)
    assert int(st.device_error.item()) == ops.DEVERR_PREFIX
    check(w, st, out, lse)
