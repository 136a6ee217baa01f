"""GPU parity of the CUDA path (through the C ABI) against the CPU oracle."""
import numpy as np
import pytest
import torch

from paged_kv_cache_467_b200 import workloads
from gpu_harness import assert_close, assert_rows_bit_exact, fill_gpu, oracle_sequence, run_decode

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


def _wl(lengths, n_q, n_kv, d, act="bf16", cache="bf16", seed=0, **kw):
    return workloads.make_workload("t", seed=seed, context_lens=lengths, n_q=n_q, n_kv=n_kv, head_dim=d,
                                   act_dtype=act, cache_dtype=cache, extra_blocks=5, **kw)


def check_all(w, st, out, lse, seqs=None, fp8_scales=None, rows=True):
    errs = []
    for s in range(w.num_seqs) if seqs is None else seqs:
        o, l, orows = oracle_sequence(w, s, fp8_scales)
        if rows:
            assert_rows_bit_exact(w, st, s, orows)
        errs.append(assert_close(out[s], o, w.cache_dtype, f"seq {s}"))
        if int(w.context_lens[s]) > 0:
            np.testing.assert_allclose(lse[s], l, rtol=0, atol=2e-3 if w.cache_dtype != "f32" else 1e-5)
        else:
            assert np.isneginf(lse[s]).all() and not out[s].any()
    return errs


# ------------------------------------------------------------------ cache writer
@pytest.mark.parametrize("act,cache", [("f32", "f32"), ("bf16", "bf16"), ("bf16", "int8"), ("f32", "int8"),
                                       ("bf16", "fp8_e4m3"), ("f32", "fp8_e4m3"), ("bf16", "fp8_e5m2"),
                                       ("f32", "fp8_e5m2"), ("bf16", "int4"), ("f32", "int4")])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_cache_write_bit_exact(act, cache, d):
    w = _wl([40, 17, 64, 5, 33], 8, 2, d, act, cache, seed=d, outlier_fraction=0.02 if cache != "f32" else 0.0)
    st = fill_gpu(w)
    assert int(st.device_error.item()) == 0
    for s in range(w.num_seqs):
        _, _, orows = oracle_sequence(w, s, st.fp8_scales)
        assert_rows_bit_exact(w, st, s, orows)
    # free blocks were never written
    used = set(w.block_tables[w.block_tables >= 0].tolist())
    free = [b for b in range(w.num_blocks) if b not in used]
    kc = st.key_cache[free].cpu()
    if cache in ("f32", "bf16"):
        assert torch.isnan(kc.float()).all()
    elif cache == "int8":
        assert (kc == 77).all()
    elif cache == "int4":
        assert (kc == 0x77).all()
    else:
        assert (kc.view(torch.uint8) == 0x7F).all()


def test_cache_write_skip_and_range_flag():
    ops = _ops()
    kc = torch.zeros((4, 16, 2, 128), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    k = torch.randn((4, 2, 128), device="cuda").to(torch.bfloat16)
    v = torch.randn_like(k)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    slots = torch.tensor([3, -1, 64, 17], dtype=torch.int64, device="cuda")  # 64 = 4 blocks * 16: out of range
    ops.kv_cache_write(k, v, kc, vc, slots, device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == ops.DEVERR_SLOT_RANGE
    flat_k = kc.view(64, 2, 128)
    assert torch.equal(flat_k[3], k[0]) and torch.equal(flat_k[17], k[3])
    assert torch.count_nonzero(flat_k.float()).item() == torch.count_nonzero(k[0].float()) + torch.count_nonzero(k[3].float())


# ------------------------------------------------------------------ decode
def test_tiny_fp32_config():
    w = workloads.tiny()
    st = fill_gpu(w)
    out, lse = run_decode(w, st)
    check_all(w, st, out, lse)
    assert int(st.device_error.item()) == 0


SHAPES = [
    # lengths, n_q, n_kv, d
    ([40, 17, 64, 5, 1, 16, 33, 700], 32, 8, 128),  # G 4
    ([300, 129, 48, 1000], 64, 8, 128),  # G 8
    ([77, 16, 15, 250], 8, 8, 128),  # MHA
    ([90, 31, 400], 32, 1, 128),  # MQA, G 32
    ([200, 3, 511], 16, 1, 64),  # G 16, d 64
    ([129, 64, 2], 16, 4, 64),  # G 4, d 64
    ([517, 9], 12, 4, 128),  # G 3
    ([260, 70], 64, 1, 128),  # G 64
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"q{s[1]}kv{s[2]}d{s[3]}")
def test_decode_bf16_shapes(shape):
    lengths, n_q, n_kv, d = shape
    w = _wl(lengths, n_q, n_kv, d, seed=n_q + n_kv + d)
    st = fill_gpu(w)
    out, lse = run_decode(w, st)
    check_all(w, st, out, lse)
    assert int(st.device_error.item()) == 0


@pytest.mark.parametrize("shape", [([40, 17, 64, 5, 1, 16, 33, 700], 32, 8, 128), ([300, 129, 48, 1000], 64, 8, 128)])
@pytest.mark.parametrize("cache", ["int8", "fp8_e4m3", "fp8_e5m2", "int4"])
def test_decode_quantized_shapes(shape, cache):
    lengths, n_q, n_kv, d = shape
    w = _wl(lengths, n_q, n_kv, d, cache=cache, seed=7, outlier_fraction=0.01)
    st = fill_gpu(w)
    out, lse = run_decode(w, st)
    check_all(w, st, out, lse, fp8_scales=st.fp8_scales)
    assert int(st.device_error.item()) == 0


@pytest.mark.parametrize("ctas,stages,hpc", [(1, 2, 0), (2, 3, 0), (5, 2, 2), (37, 3, 1), (148, 0, 0), (400, 0, 4),
                                             (1000, 2, 8)])
def test_decode_launch_shapes(ctas, stages, hpc):
    ops = _ops()
    w = _wl([700, 33, 1, 256, 17, 1200, 64, 5], 32, 8, 128, seed=11)
    st = fill_gpu(w)
    tuning = ops.DecodeTuning(ctas, stages, hpc)
    out, lse = run_decode(w, st, tuning=tuning)
    check_all(w, st, out, lse, rows=False)
    again, lse2 = run_decode(w, st, tuning=tuning)
    assert np.array_equal(out, again) and np.array_equal(lse, lse2)  # the merge order is fixed


@pytest.mark.parametrize("cache", ["bf16", "int8", "fp8_e4m3", "f32"])
def test_pool_permutation_is_bitwise_invisible(cache):
    act = "f32" if cache == "f32" else "bf16"
    d = 64 if cache == "f32" else 128
    w = _wl([300, 17, 64, 129, 1], 16, 4, d, act=act, cache=cache, seed=5)
    st = fill_gpu(w)
    out, lse = run_decode(w, st)
    perm = torch.randperm(w.num_blocks, generator=torch.Generator().manual_seed(3))  # block b moves to perm[b]
    inv = torch.argsort(perm).cuda()
    st.key_cache = st.key_cache[inv].contiguous()
    st.value_cache = st.value_cache[inv].contiguous()
    if cache == "int8":
        st.k_scale = st.k_scale[inv].contiguous()
        st.v_scale = st.v_scale[inv].contiguous()
    tables = torch.from_numpy(np.where(w.block_tables >= 0, perm.numpy()[np.maximum(w.block_tables, 0)], -1).astype(np.int32)).cuda()
    out2, lse2 = run_decode(w, st, block_tables=tables)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def test_workspace_reused_across_shapes():
    ops = _ops()
    # one zero-filled workspace, big enough for both shapes, used by both in turn
    w1 = _wl([3000, 2500, 40], 64, 8, 128, seed=21)  # few units, long
    w2 = _wl([300 + 13 * i for i in range(40)], 32, 8, 128, seed=22)  # many units
    n = max(ops.paged_attention_workspace_size(w.num_seqs, w.n_q, w.n_kv, 128, 16, ops.PKV_BF16) for w in (w1, w2))
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    for w in (w1, w2, w1):
        st = fill_gpu(w)
        out, lse = run_decode(w, st, workspace=ws)
        check_all(w, st, out, lse, rows=False)


def test_empty_sequences():
    w = _wl([0, 40, 0, 17, 0], 16, 4, 128, seed=2)
    st = fill_gpu(w)
    out, lse = run_decode(w, st)
    check_all(w, st, out, lse, rows=False)
    wf = _wl([0, 40, 0], 8, 2, 64, act="f32", cache="f32", seed=2)
    stf = fill_gpu(wf)
    outf, lsef = run_decode(wf, stf)
    check_all(wf, stf, outf, lsef, rows=False)


@pytest.mark.parametrize("cache", ["bf16", "int8", "f32"])
def test_out_of_range_block_is_flagged_not_read(cache):
    ops = _ops()
    act = "f32" if cache == "f32" else "bf16"
    d = 64 if cache == "f32" else 128
    w = _wl([40, 50, 33], 16, 4, d, act=act, cache=cache, seed=9)
    st = fill_gpu(w)
    tables = w.block_tables.copy()
    tables[1, 1] = w.num_blocks + 1000  # outside the pool
    out, _ = run_decode(w, st, block_tables=torch.from_numpy(tables).cuda())
    assert int(st.device_error.item()) & ops.DEVERR_BLOCK_RANGE
    for s in (0, 2):  # other sequences are unaffected
        o, _, _ = oracle_sequence(w, s)
        assert_close(out[s], o, cache, f"seq {s}")


def test_context_len_beyond_bound_is_flagged():
    ops = _ops()
    w = _wl([40, 50], 16, 4, 128, seed=4)
    st = fill_gpu(w)
    out = torch.empty((2, 16, 128), dtype=torch.bfloat16, device="cuda")
    ops.paged_attention_decode(out, st.query, st.key_cache, st.value_cache, st.block_tables, st.context_lens, 45,
                               w.sm_scale, device_error=st.device_error)
    torch.cuda.synchronize()
    assert int(st.device_error.item()) & ops.DEVERR_CONTEXT_LEN


# ------------------------------------------------------------------ full-size configs
def test_llama3_8b_config_full():
    w = workloads.llama3_8b()
    st = fill_gpu(w)
    out, lse = run_decode(w, st)
    errs = check_all(w, st, out, lse, rows=False)
    for s in (0, 31, 63):
        _, _, orows = oracle_sequence(w, s)
        assert_rows_bit_exact(w, st, s, orows)
    assert int(st.device_error.item()) == 0
    print("llama3_8b max/mean abs err", max(e[0] for e in errs), np.mean([e[1] for e in errs]))


def test_long_70b_config_sampled():
    w = workloads.long_70b()
    st = fill_gpu(w)
    out, lse = run_decode(w, st)
    lens = w.context_lens
    seqs = sorted({int(np.argmax(lens)), int(np.argmin(lens)), 3})
    check_all(w, st, out, lse, seqs=seqs)
    assert np.isfinite(out).all()
    assert int(st.device_error.item()) == 0


def test_prefix_sharing_config():
    w = workloads.prefix_sharing()
    st = fill_gpu(w)
    shared = torch.from_numpy(w.shared_prefix_blocks.astype(np.int64)).cuda()
    before = st.key_cache.index_select(0, shared).clone(), st.value_cache.index_select(0, shared).clone()
    # the step's own append: one token per sequence, into private blocks
    ops = _ops()
    nk, nv = w.new_kv()
    ops.kv_cache_write(torch.from_numpy(nk).cuda().to(torch.bfloat16), torch.from_numpy(nv).cuda().to(torch.bfloat16),
                       st.key_cache, st.value_cache, torch.from_numpy(w.new_token_slots()).cuda(),
                       device_error=st.device_error)
    out, lse = run_decode(w, st)
    assert torch.equal(before[0].view(torch.int16), st.key_cache.index_select(0, shared).view(torch.int16))
    assert torch.equal(before[1].view(torch.int16), st.value_cache.index_select(0, shared).view(torch.int16))
    check_all(w, st, out, lse, seqs=range(0, 128, 9))
    assert int(st.device_error.item()) == 0


@pytest.mark.parametrize("cache", ["int8", "fp8_e4m3", "fp8_e5m2", "int4"])
def test_quantized_config_sampled(cache):
    w = workloads.quantized(cache, seed={"int8": 4, "fp8_e4m3": 5, "fp8_e5m2": 6, "int4": 7}[cache])
    scales = w.fp8_head_scales() if cache.startswith("fp8") else None
    st = fill_gpu(w, fp8_scales=scales)
    out, lse = run_decode(w, st)
    errs = check_all(w, st, out, lse, seqs=range(0, 256, 37), fp8_scales=scales)
    assert np.isfinite(out).all()
    assert int(st.device_error.item()) == 0
    # quantisation error against the unquantised rows: reported, not gated
    q = w.query()
    from test_oracle_attention import sdpa_reference

    K, V = w.sequence_kv(0)
    qerr = np.abs(out[0] - sdpa_reference(q[0], K, V, w.sm_scale)).max()
    print(f"{cache}: max/mean abs err vs dequantised oracle {max(e[0] for e in errs):.3e}/{np.mean([e[1] for e in errs]):.3e}; "
          f"vs unquantised seq 0 {qerr:.3e}")


@pytest.mark.parametrize("cache", ["int8", "fp8_e4m3", "fp8_e5m2", "int4"])
def test_decode_quantized_f32_queries(cache):
    """float32 queries and outputs over a quantised cache (queries rounded to
    f16 for the tensor cores: the quantised tolerance covers it)."""
    w = _wl([40, 17, 64, 5, 1, 300], 32, 8, 128, act="f32", cache=cache, seed=8, outlier_fraction=0.01)
    st = fill_gpu(w)
    out, lse = run_decode(w, st)
    check_all(w, st, out, lse, fp8_scales=st.fp8_scales)
    assert int(st.device_error.item()) == 0
