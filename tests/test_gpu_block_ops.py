"""GPU parity of the block movers (pkv_copy_blocks, pkv_swap_blocks) against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_467_b200 import workloads
from gpu_harness import fill_gpu, oracle_sequence, run_decode
from test_gpu_parity import check_all

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


def _pairs(nb, n, seed):
    rng = np.random.default_rng(seed)
    perm = rng.permutation(nb)
    return np.stack([perm[:n], perm[n : 2 * n]], axis=1).astype(np.int64)  # sources and destinations disjoint


def _host(t):
    """Host copy of a pool as numpy; bf16 travels as its int16 bit pattern."""
    t = t.cpu()
    if t.dtype == torch.bfloat16:
        t = t.view(torch.int16)
    elif t.dtype in (torch.float8_e4m3fn, torch.float8_e5m2):
        t = t.view(torch.uint8)
    return t.numpy().copy()


@pytest.mark.parametrize("cache", ["bf16", "int8", "fp8_e4m3", "f32", "fp8_e5m2", "int4"])
def test_copy_blocks_bit_exact(cache):
    ops = _ops()
    act = "f32" if cache == "f32" else "bf16"
    w = workloads.make_workload("c", seed=3, context_lens=[300, 129, 48, 700], n_q=16, n_kv=4, head_dim=128,
                                act_dtype=act, cache_dtype=cache, extra_blocks=20)
    st = fill_gpu(w)
    pairs = _pairs(w.num_blocks, 17, seed=9)
    row_scaled = cache in ("int8", "int4")
    pools = [_host(st.key_cache), _host(st.value_cache)]
    if row_scaled:
        pools += [_host(st.k_scale), _host(st.v_scale)]
    oracle.copy_blocks(pools, pairs)
    scales = (st.k_scale, st.v_scale) if row_scaled else (None, None)  # fp8 scales are per head, not per block
    ops.copy_blocks(st.key_cache, st.value_cache, torch.from_numpy(pairs).cuda(), *scales, st.device_error,
                    cache_dtype="int4" if cache == "int4" else None)
    torch.cuda.synchronize()
    got = [_host(st.key_cache), _host(st.value_cache)] + ([_host(st.k_scale), _host(st.v_scale)] if row_scaled else [])
    for g, want in zip(got, pools):
        assert np.array_equal(g.view(np.uint8), want.view(np.uint8))
    assert int(st.device_error.item()) == 0


def test_copy_on_write_divergence_on_gpu():
    """Sequences A and B share their whole history; B diverges: it copies the
    shared partial last block, then each appends its own token with the fused
    step.  Both must match the oracle run through the same operations."""
    ops = _ops()
    n_kv, d = 4, 128
    w = workloads.make_workload("cow", seed=12, context_lens=[201, 201], n_q=16, n_kv=n_kv, head_dim=d,
                                extra_blocks=3)
    # make B's table point at A's blocks (shared history), keeping a spare block for the copy
    tables = w.block_tables.copy()
    nb_used = workloads.blocks_for(201, 16)
    tables[1, :nb_used] = tables[0, :nb_used]
    spare = int(sorted(set(range(w.num_blocks)) - set(tables[0, :nb_used].tolist()))[0])
    last = int(tables[0, nb_used - 1])
    gen = np.random.default_rng(4)
    hist_k = workloads.round_to_bf16(gen.standard_normal((200, n_kv, d)).astype(np.float32))
    hist_v = workloads.round_to_bf16(gen.standard_normal((200, n_kv, d)).astype(np.float32))
    new_k = workloads.round_to_bf16(gen.standard_normal((2, n_kv, d)).astype(np.float32))
    new_v = workloads.round_to_bf16(gen.standard_normal((2, n_kv, d)).astype(np.float32))
    q = workloads.round_to_bf16(gen.standard_normal((2, 16, d)).astype(np.float32))
    slots = (tables[0, np.arange(200) // 16].astype(np.int64) * 16 + np.arange(200) % 16)

    # device: shared history, CoW copy, B's table points at its private block, fused step appends token 200
    kc = torch.full((w.num_blocks, 16, n_kv, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    vc = torch.full_like(kc, float("nan"))
    bf = lambda a: torch.from_numpy(a).cuda().to(torch.bfloat16)  # noqa: E731
    ops.kv_cache_write(bf(hist_k), bf(hist_v), kc, vc, torch.from_numpy(slots).cuda())
    ops.copy_blocks(kc, vc, torch.tensor([[last, spare]], dtype=torch.int64, device="cuda"))
    tables_b = tables.copy()
    tables_b[1, nb_used - 1] = spare
    out = torch.empty((2, 16, d), dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.paged_decode_step(out, bf(q), bf(new_k), bf(new_v), kc, vc, torch.from_numpy(tables_b).cuda(),
                          torch.tensor([201, 201], dtype=torch.int32, device="cuda"), 201, w.sm_scale,
                          device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0

    # oracle: the same operations on a host pool
    okc = np.full((w.num_blocks, 16, n_kv, d), np.nan)
    ovc = np.full_like(okc, np.nan)
    oracle.kv_cache_write(hist_k, hist_v, okc, ovc, slots)
    oracle.copy_blocks([okc, ovc], [(last, spare)])
    new_slots = tables_b[np.arange(2), (200 // 16)].astype(np.int64) * 16 + 200 % 16
    oracle.kv_cache_write(new_k, new_v, okc, ovc, new_slots)
    ref, _ = oracle.paged_attention_decode(q, okc, ovc, tables_b, np.array([201, 201]), w.sm_scale)
    got = out.float().cpu().numpy()
    assert np.abs(got - ref).max() < 2e-2 and np.abs(got - ref).mean() < 2e-3
    # A and B differ only in their last token, so their outputs differ
    assert not np.allclose(got[0], got[1])


@pytest.mark.parametrize("cache", ["bf16", "int8"])
def test_swap_to_host_and_back(cache):
    ops = _ops()
    w = workloads.make_workload("s", seed=5, context_lens=[300, 17, 64, 129, 1], n_q=16, n_kv=4, head_dim=128,
                                cache_dtype=cache, extra_blocks=8)
    st = fill_gpu(w)
    out0, lse0 = run_decode(w, st)
    used = np.unique(w.block_tables[w.block_tables >= 0])
    # offload every used block to a page-locked host pool
    hk = torch.empty((len(used),) + tuple(st.key_cache.shape[1:]), dtype=st.key_cache.dtype).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    hks = hvs = None
    if cache == "int8":
        hks = torch.empty((len(used),) + tuple(st.k_scale.shape[1:]), dtype=torch.float32).pin_memory()
        hvs = torch.empty_like(hks).pin_memory()
    out_pairs = np.stack([used, np.arange(len(used))], axis=1).astype(np.int64)
    ops.swap_blocks(st.key_cache, st.value_cache, hk, hv, torch.from_numpy(out_pairs).cuda(), st.k_scale, st.v_scale,
                    hks, hvs, st.device_error)
    torch.cuda.synchronize()
    assert np.array_equal(hk.view(torch.uint8).numpy(), st.key_cache[torch.from_numpy(used).cuda()].cpu().view(torch.uint8).numpy())
    # wipe the device pool, then restore the blocks into other slots and remap the tables
    st.key_cache.fill_(float("nan") if cache == "bf16" else 0)
    st.value_cache.fill_(float("nan") if cache == "bf16" else 0)
    new_slot = np.random.default_rng(2).permutation(w.num_blocks)[: len(used)]
    in_pairs = np.stack([np.arange(len(used)), new_slot], axis=1).astype(np.int64)
    ops.swap_blocks(hk, hv, st.key_cache, st.value_cache, torch.from_numpy(in_pairs).cuda(), hks, hvs, st.k_scale,
                    st.v_scale, st.device_error, device=st.key_cache.device)
    remap = np.full(w.num_blocks, -1, dtype=np.int64)
    remap[used] = new_slot
    tables = np.where(w.block_tables >= 0, remap[np.maximum(w.block_tables, 0)], -1).astype(np.int32)
    out1, lse1 = run_decode(w, st, block_tables=torch.from_numpy(tables).cuda())
    assert np.array_equal(out0, out1) and np.array_equal(lse0, lse1)
    assert int(st.device_error.item()) == 0


def test_block_mover_flags_out_of_range_ids():
    ops = _ops()
    kc = torch.zeros((4, 16, 2, 128), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    kc[1] = 1.0
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.copy_blocks(kc, vc, torch.tensor([[1, 2], [0, 9], [-3, 0]], dtype=torch.int64, device="cuda"),
                    device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) & ops.DEVERR_BLOCK_RANGE
    assert bool((kc[2] == 1.0).all()) and bool((kc[0] == 0).all())


def test_swap_rejects_unmapped_host_memory():
    ops = _ops()
    kc = torch.zeros((4, 16, 2, 128), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    host_k = torch.zeros((4, 16, 2, 128), dtype=torch.bfloat16)  # pageable: not addressable by the device
    host_v = torch.zeros_like(host_k)
    with pytest.raises(ops.PkvError) as e:
        ops.swap_blocks(kc, vc, host_k, host_v, torch.tensor([[0, 1]], dtype=torch.int64, device="cuda"))
    assert e.value.status == 1
