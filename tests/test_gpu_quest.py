"""GPU parity of the Quest operations (page summaries, page selection, decode
over listed pages) against the oracle ("KV Cache Engineering for LLM
Serving", section 7)."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_467_b200 import workloads
from gpu_harness import TOL, assert_close, fill_gpu, oracle_sequence

pytestmark = pytest.mark.gpu

LENGTHS = [1000, 17, 64, 5, 300, 1, 1201, 129, 0, 640]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from paged_kv_cache_467_b200 import build

    build.build()


def _ops():
    from paged_kv_cache_467_b200 import ops

    return ops


def _wl(cache="bf16", d=128, n_q=32, n_kv=8, seed=71, lengths=LENGTHS):
    act = "f32" if cache == "f32" else "bf16"
    return workloads.make_workload("q", seed=seed, context_lens=lengths, n_q=n_q, n_kv=n_kv, head_dim=d,
                                   act_dtype=act, cache_dtype=cache, extra_blocks=3,
                                   outlier_fraction=0.01 if cache in ("int8", "fp8_e4m3") else 0.0)


def _summaries(w, st):
    ops = _ops()
    shape = (w.num_blocks, w.n_kv, w.head_dim)
    mn = torch.full(shape, float("nan"), dtype=st.key_cache.dtype, device="cuda")
    mx = torch.full(shape, float("nan"), dtype=st.key_cache.dtype, device="cuda")
    ops.quest_page_summaries(st.key_cache, mn, mx, st.block_tables, st.context_lens, st.device_error)
    torch.cuda.synchronize()
    return mn, mx


def _oracle_keys(w, s, st):
    """Sequence s's cached keys as the oracle's writer stores them, [L, n_kv, d] float64."""
    L = int(w.context_lens[s])
    nb = max(workloads.blocks_for(L, w.block_size), 1)
    kc = np.zeros((nb, w.block_size, w.n_kv, w.head_dim))
    vc = np.zeros_like(kc)
    K, V = w.sequence_kv(s)
    oracle.kv_cache_write(K, V, kc, vc, np.arange(L, dtype=np.int64), w.cache_dtype)
    return kc.reshape(-1, w.n_kv, w.head_dim)[:L]


def _bits(x, cache):
    """float64 host values (exact in the cache dtype) -> their stored bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if cache == "bf16":
        return t.to(torch.bfloat16).view(torch.int16).numpy()
    return t.view(torch.int32).numpy()


def _gpu_bits(t, cache):
    t = t.cpu()
    return t.view(torch.int16).numpy() if cache == "bf16" else t.view(torch.int32).numpy()


@pytest.mark.parametrize("cache,d", [("bf16", 128), ("bf16", 64), ("f32", 128), ("f32", 64)])
def test_page_summaries_bit_exact(cache, d):
    w = _wl(cache, d, n_q=16, n_kv=4)
    st = fill_gpu(w)
    mn, mx = _summaries(w, st)
    for s in range(w.num_seqs):
        L = int(w.context_lens[s])
        if L == 0:
            continue
        mins, maxs = oracle.page_summaries(_oracle_keys(w, s, st), w.block_size)
        blocks = torch.from_numpy(w.block_tables[s, : mins.shape[0]].astype(np.int64)).cuda()
        assert np.array_equal(_gpu_bits(mn.index_select(0, blocks), cache), _bits(mins, cache)), f"seq {s} min"
        assert np.array_equal(_gpu_bits(mx.index_select(0, blocks), cache), _bits(maxs, cache)), f"seq {s} max"
    assert int(st.device_error.item()) == 0


def test_last_page_refresh_after_append():
    """Summaries of L-1 tokens, then append token L-1 and refresh only each
    sequence's last page: every page equals the oracle's summary of L tokens."""
    ops = _ops()
    w = _wl("bf16", 128, n_q=16, n_kv=4, seed=79, lengths=[1000, 17, 64, 5, 300, 1, 129, 33])
    st = fill_gpu(w, append_new=False)
    shape = (w.num_blocks, w.n_kv, w.head_dim)
    mn = torch.full(shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    mx = torch.full(shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    ops.quest_page_summaries(st.key_cache, mn, mx, st.block_tables, st.context_lens - 1, st.device_error)
    nk, nv = w.new_kv()
    dt = torch.bfloat16
    ops.kv_cache_write(torch.from_numpy(nk.astype(np.float32)).to("cuda", dt),
                       torch.from_numpy(nv.astype(np.float32)).to("cuda", dt), st.key_cache, st.value_cache,
                       torch.from_numpy(w.new_token_slots()).cuda(), None, None, st.device_error)
    ops.quest_page_summaries(st.key_cache, mn, mx, st.block_tables, st.context_lens, st.device_error,
                             last_page_only=True)
    torch.cuda.synchronize()
    for s in range(w.num_seqs):
        mins, maxs = oracle.page_summaries(_oracle_keys(w, s, st), w.block_size)
        blocks = torch.from_numpy(w.block_tables[s, : mins.shape[0]].astype(np.int64)).cuda()
        assert np.array_equal(_gpu_bits(mn.index_select(0, blocks), "bf16"), _bits(mins, "bf16")), f"seq {s} min"
        assert np.array_equal(_gpu_bits(mx.index_select(0, blocks), "bf16"), _bits(maxs, "bf16")), f"seq {s} max"
    assert int(st.device_error.item()) == 0


def _select(w, st, mn, mx, k):
    ops = _ops()
    max_pages = -(-min(w.max_context_len, w.max_blocks_per_seq * w.block_size) // w.block_size)
    sel = torch.full((w.num_seqs, w.n_kv, k), -7, dtype=torch.int32, device="cuda")
    scores = torch.full((w.num_seqs, w.n_kv, max_pages), float("nan"), dtype=torch.float32, device="cuda")
    ops.quest_select(st.query, mn, mx, st.block_tables, st.context_lens, w.max_context_len, k, sel, scores,
                     st.device_error)
    torch.cuda.synchronize()
    return sel.cpu().numpy(), scores.cpu().numpy().astype(np.float64)


def _oracle_group_scores(w, s, st):
    mins, maxs = oracle.page_summaries(_oracle_keys(w, s, st), w.block_size)
    return oracle.group_scores(oracle.page_scores(w.query()[s], mins, maxs), w.n_kv)


def _assert_valid_topk(sel_row, sc, k):
    """sel_row: the kernel's choice; sc: the kernel's own page scores.  The
    choice is the k best of sc, ascending, ties to the lower page."""
    P = len(sc)
    K = min(k, P)
    chosen = sel_row[:K]
    assert (sel_row[K:] == -1).all()
    assert (np.diff(chosen) > 0).all() and chosen[0] >= 0 and chosen[-1] < P
    rest = np.setdiff1d(np.arange(P), chosen)
    if len(rest):
        worst = sc[chosen].min()
        assert sc[rest].max() <= worst
        tied_out = rest[sc[rest] == worst]
        tied_in = chosen[sc[chosen] == worst]
        if len(tied_out):
            assert tied_in.max() < tied_out.min(), "ties must go to the lower page"


LONG = [20000, 16000, 35000, 5, 12345, 40000, 1, 23456]


@pytest.mark.parametrize("cache,d,n_q,n_kv,lengths", [("bf16", 128, 32, 8, LENGTHS), ("bf16", 64, 16, 16, LENGTHS),
                                                      ("bf16", 128, 32, 2, LENGTHS), ("f32", 128, 8, 2, LENGTHS),
                                                      ("f32", 64, 12, 4, LENGTHS), ("bf16", 128, 64, 8, LONG),
                                                      ("bf16", 64, 20, 4, LONG)])
@pytest.mark.parametrize("k", [1, 4, 16, 200])
def test_select_matches_oracle(cache, d, n_q, n_kv, lengths, k):
    """bf16 with up to 8 query heads per KV head runs the tensor-core scorer
    (the long lengths give every warp several tiles); f32 and wider groups the
    CUDA-core one."""
    w = _wl(cache, d, n_q=n_q, n_kv=n_kv, seed=72, lengths=lengths)
    st = fill_gpu(w)
    mn, mx = _summaries(w, st)
    sel, scores = _select(w, st, mn, mx, k)
    for s in range(w.num_seqs):
        L = int(w.context_lens[s])
        P = -(-L // w.block_size)
        if P == 0:
            assert (sel[s] == -1).all()
            continue
        want = _oracle_group_scores(w, s, st)
        for kv in range(w.n_kv):
            got = scores[s, kv, :P]
            np.testing.assert_allclose(got, want[kv], rtol=1e-5, atol=1e-4 * (1 + np.abs(want[kv]).max()))
            _assert_valid_topk(sel[s, kv], got, k)
            # where the oracle's k-th and (k+1)-th best are well apart, the pick is the oracle's
            order = np.sort(want[kv])[::-1]
            if k < P and order[k - 1] - order[k] > 1e-2:
                assert np.array_equal(sel[s, kv, :k], oracle.select_pages(want[kv], k)), (s, kv)
            if k >= P:
                assert np.array_equal(sel[s, kv, :P], np.arange(P))
    assert int(st.device_error.item()) == 0


def test_select_ties_to_lower_page():
    """Every page of a sequence summarised by the same key: all scores tie, so
    the k lowest pages are kept."""
    w = _wl("bf16", 128, n_q=8, n_kv=2, seed=73, lengths=[160, 47])
    st = fill_gpu(w)
    mn, mx = _summaries(w, st)
    # overwrite every used page's summary with the same vectors
    one_min, one_max = mn[int(w.block_tables[0, 0])].clone(), mx[int(w.block_tables[0, 0])].clone()
    for s, L in enumerate(w.context_lens):
        for j in range(-(-int(L) // 16)):
            mn[int(w.block_tables[s, j])] = one_min
            mx[int(w.block_tables[s, j])] = one_max
    sel, scores = _select(w, st, mn, mx, 4)
    assert sel[0].tolist() == [[0, 1, 2, 3]] * 2
    assert sel[1].tolist() == [[0, 1, 2, -1]] * 2
    assert int(st.device_error.item()) == 0


def _run_pages(w, st, pages, lse=True):
    ops = _ops()
    dt = torch.float32 if w.act_dtype == "f32" else torch.bfloat16
    out = torch.full((w.num_seqs, w.n_q, w.head_dim), float("nan"), dtype=dt, device="cuda")
    lse_t = torch.full((w.num_seqs, w.n_q), float("nan"), dtype=torch.float32, device="cuda")
    ops.paged_attention_decode_pages(out, st.query, st.key_cache, st.value_cache, st.block_tables, st.context_lens,
                                     w.max_context_len, torch.from_numpy(pages).cuda(), w.sm_scale, st.k_scale,
                                     st.v_scale, lse_t, device_error=st.device_error)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64), lse_t.cpu().numpy().astype(np.float64)


def _random_pages(w, k, seed):
    """Seeded page lists: for each (sequence, KV head) a random ascending subset
    of up to k pages (sometimes all, sometimes none), -1 after."""
    rng = np.random.default_rng(seed)
    pages = np.full((w.num_seqs, w.n_kv, k), -1, dtype=np.int32)
    for s, L in enumerate(w.context_lens):
        P = -(-int(L) // w.block_size)
        for kv in range(w.n_kv):
            n = min(P, k) if rng.random() < 0.3 else int(rng.integers(0, min(P, k) + 1))
            pages[s, kv, :n] = np.sort(rng.choice(P, size=n, replace=False))
    return pages


def _oracle_pages(w, st, s, pages):
    L = int(w.context_lens[s])
    _, _, (kc, vc, ks, vs) = oracle_sequence(w, s, st.fp8_scales)
    table = np.arange(kc.shape[0], dtype=np.int32)
    return oracle.decode_over_pages(w.query()[s], kc, vc, table, L, w.sm_scale, pages[s], w.cache_dtype, ks, vs)


def _check_pages(w, st, pages, out, lse):
    for s in range(w.num_seqs):
        o, l = _oracle_pages(w, st, s, pages)
        assert_close(out[s], o, w.cache_dtype, f"seq {s}")
        fin = np.isfinite(l)
        assert (np.isneginf(lse[s]) == ~fin).all(), f"seq {s}: lse -inf pattern"
        np.testing.assert_allclose(lse[s][fin], l[fin], rtol=0, atol=2e-3 if w.cache_dtype != "f32" else 1e-5)


@pytest.mark.parametrize("cache,d", [("bf16", 128), ("bf16", 64), ("int8", 128), ("fp8_e4m3", 128), ("f32", 64),
                                     ("f32", 128)])
@pytest.mark.parametrize("k", [3, 24, 80])
def test_decode_pages_matches_oracle(cache, d, k):
    w = _wl(cache, d, n_q=16, n_kv=4, seed=74)
    st = fill_gpu(w)
    pages = _random_pages(w, k, seed=75 + k)
    out, lse = _run_pages(w, st, pages)
    _check_pages(w, st, pages, out, lse)
    assert int(st.device_error.item()) == 0


def test_decode_pages_all_listed_is_full_decode():
    w = _wl("bf16", 128, seed=76)
    st = fill_gpu(w)
    k = max(-(-int(L) // 16) for L in w.context_lens)
    pages = np.full((w.num_seqs, w.n_kv, k), -1, dtype=np.int32)
    for s, L in enumerate(w.context_lens):
        P = -(-int(L) // 16)
        pages[s, :, :P] = np.arange(P)
    out, lse = _run_pages(w, st, pages)
    for s in range(w.num_seqs):
        o, l, _ = oracle_sequence(w, s)
        assert_close(out[s], o, "bf16", f"seq {s}")
    assert int(st.device_error.item()) == 0


def test_page_past_sequence_is_flagged():
    ops = _ops()
    w = _wl("bf16", 128, n_q=16, n_kv=4, seed=77, lengths=[100, 40, 70])
    st = fill_gpu(w)
    pages = np.full((3, 4, 4), -1, dtype=np.int32)
    pages[0, :, :2] = [1, 3]
    pages[1, 0, :2] = [0, 5]  # sequence 1 has 3 pages
    pages[2, :, :3] = [0, 2, 4]
    out, _ = _run_pages(w, st, pages)
    assert int(st.device_error.item()) & ops.DEVERR_BLOCK_RANGE
    for s in (0, 2):
        o, _ = _oracle_pages(w, st, s, pages)
        assert_close(out[s], o, "bf16", f"seq {s}")


@pytest.mark.parametrize("cache", ["bf16", "f32"])
def test_quest_pipeline_end_to_end(cache):
    """Summaries, selection and sparse decode chained on the device equal the
    oracle's Quest decode where the oracle's choice is unambiguous."""
    d = 128 if cache == "bf16" else 64
    w = _wl(cache, d, n_q=16, n_kv=4, seed=78)
    st = fill_gpu(w)
    k = 6
    mn, mx = _summaries(w, st)
    sel, _ = _select(w, st, mn, mx, k)
    out, lse = _run_pages(w, st, sel)
    for s in range(w.num_seqs):
        L = int(w.context_lens[s])
        _, _, (kc, vc, ks, vs) = oracle_sequence(w, s, st.fp8_scales)
        table = np.arange(kc.shape[0], dtype=np.int32)
        o, l, want_sel = oracle.quest_decode(w.query()[s], kc, vc, table, L, w.sm_scale, k, w.cache_dtype, ks, vs)
        if L == 0:
            assert (out[s] == 0).all()
            continue
        grp = _oracle_group_scores(w, s, st)
        for kv in range(w.n_kv):
            P = grp.shape[1]
            order = np.sort(grp[kv])[::-1]
            if k >= P or order[k - 1] - order[k] > 1e-2:
                g = w.n_q // w.n_kv
                assert np.array_equal(sel[s, kv, : min(k, P)], want_sel[kv])
                mx_tol, _ = TOL[cache]
                assert np.abs(out[s, kv * g : (kv + 1) * g] - o[kv * g : (kv + 1) * g]).max() <= mx_tol
    assert int(st.device_error.item()) == 0
