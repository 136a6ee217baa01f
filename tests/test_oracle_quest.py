"""Pins for the Quest page selection in the oracle (CPU only)."""
import numpy as np

import oracle.quest as oq
from oracle.paged_attention import kv_cache_write, paged_attention_decode
from test_oracle_attention import sdpa_reference


def _example(golden):
    rows = golden("quest_example.txt")
    pages = []
    rec = {}
    for r in rows:
        if r[0] == "page":
            a, b = " ".join(r[3:]).split(",")
            pages.append([[float(x) for x in a.split()], [float(x) for x in b.split()]])
        else:
            rec[r[0]] = r[1:]
    return np.array(pages), rec


def test_quest_worked_example(golden):
    pages, rec = _example(golden)
    keys = pages.reshape(-1, 1, 2)  # 8 keys of one KV head, pages of 2
    mins, maxs = oq.page_summaries(keys, page_size=2)
    q = np.array([[float(x) for x in rec["query"]]])
    scores = oq.page_scores(q, mins, maxs)[0]
    np.testing.assert_allclose(scores, [float(x) for x in rec["scores"]], atol=1e-12)
    sel = oq.select_pages(scores, int(rec["select"][0]))
    assert sel.tolist() == [int(x) for x in rec["selected"]]
    assert len(sel) * 2 == int(rec["entries_read"][0]) and keys.shape[0] == int(rec["entries_stored"][0])


def check_upper_bound(seed=0):
    """Every key of a page scores at most the page score, for any query."""
    rng = np.random.default_rng(seed)
    for L in (16, 37, 200):
        K = rng.standard_normal((L, 2, 16)) * rng.uniform(0.1, 5)
        q = rng.standard_normal((4, 16))
        mins, maxs = oq.page_summaries(K, 16)
        head = oq.page_scores(q, mins, maxs)
        grp = oq.group_scores(head, 2)
        for h in range(4):
            kv = h // 2
            dots = K[:, kv, :] @ q[h]
            for j in range(mins.shape[0]):
                assert dots[j * 16 : (j + 1) * 16].max() <= head[h, j] + 1e-12
                assert head[h, j] <= grp[kv, j]
        # the bound is reached when a page holds a single key
        m1, x1 = oq.page_summaries(K[:1], 16)
        np.testing.assert_allclose(oq.page_scores(q, m1, x1)[0, 0], K[0, 0] @ q[0], atol=1e-12)


def test_page_score_is_an_upper_bound():
    check_upper_bound()


def test_ties_go_to_the_lower_page():
    assert oq.select_pages([1.0, 3.0, 3.0, 2.0], 1).tolist() == [1]
    assert oq.select_pages([1.0, 3.0, 3.0, 2.0], 3).tolist() == [1, 2, 3]
    assert oq.select_pages([1.0, 3.0], 5).tolist() == [0, 1]


def _pool(seed, L, n_kv=2, d=16):
    rng = np.random.default_rng(seed)
    nb = -(-L // 16)
    kc = np.full((nb + 2, 16, n_kv, d), np.nan)
    vc = np.full_like(kc, np.nan)
    table = rng.permutation(nb + 2)[:nb]
    K, V = rng.standard_normal((L, n_kv, d)), rng.standard_normal((L, n_kv, d))
    kv_cache_write(K, V, kc, vc, table[np.arange(L) // 16] * 16 + np.arange(L) % 16)
    return kc, vc, table, K, V, rng.standard_normal((8, d))


def test_enough_pages_is_full_attention():
    kc, vc, table, K, V, q = _pool(1, 150)
    out, lse, sel = oq.quest_decode(q, kc, vc, table, 150, 0.25, k_pages=10)
    full, lse_full = paged_attention_decode(q[None], kc, vc, table[None], [150], 0.25)
    np.testing.assert_allclose(out, full[0], atol=1e-12)
    np.testing.assert_allclose(lse, lse_full[0], atol=1e-12)
    assert sel.shape == (2, 10)


def test_quest_decode_attends_over_selected_rows():
    kc, vc, table, K, V, q = _pool(2, 300)
    out, _, sel = oq.quest_decode(q, kc, vc, table, 300, 0.25, k_pages=5)
    assert sel.shape == (2, 5)
    for kv in range(2):
        rows = np.concatenate([np.arange(j * 16, min(j * 16 + 16, 300)) for j in sel[kv]])
        ref = sdpa_reference(q[kv * 4 : kv * 4 + 4], K[rows][:, kv : kv + 1], V[rows][:, kv : kv + 1], 0.25)
        np.testing.assert_allclose(out[kv * 4 : kv * 4 + 4], ref, atol=1e-12)
    # the chosen pages are the best-scoring ones of each group
    mins, maxs = oq.page_summaries(K, 16)
    grp = oq.group_scores(oq.page_scores(q, mins, maxs), 2)
    for kv in range(2):
        worst_chosen = grp[kv, sel[kv]].min()
        rest = np.delete(grp[kv], sel[kv])
        assert (rest <= worst_chosen).all()


def test_decode_over_listed_pages():
    """Listing every page is full attention; -1 ends a list; an empty list is
    the empty sum (zero output, lse -inf); each head sees only its own list."""
    kc, vc, table, K, V, q = _pool(3, 90)  # 6 pages, the last one partial
    full, lse_full = paged_attention_decode(q[None], kc, vc, table[None], [90], 0.25)
    out, lse = oq.decode_over_pages(q, kc, vc, table, 90, 0.25, np.array([[0, 1, 2, 3, 4, 5], [0, 1, 2, 3, 4, 5]]))
    np.testing.assert_allclose(out, full[0], atol=1e-12)
    np.testing.assert_allclose(lse, lse_full[0], atol=1e-12)
    out, lse = oq.decode_over_pages(q, kc, vc, table, 90, 0.25, np.array([[1, 5, -1, 3], [-1, -1, -1, -1]]))
    rows = np.r_[16:32, 80:90]
    np.testing.assert_allclose(out[:4], sdpa_reference(q[:4], K[rows][:, :1], V[rows][:, :1], 0.25), atol=1e-12)
    assert (out[4:] == 0).all() and np.isneginf(lse[4:]).all()


def test_empty_sequence_has_no_pages():
    """Length 0: no page, nothing selected, zero output and lse -inf (the
    empty-sum reading of the decode)."""
    kc, vc, table, K, V, q = _pool(4, 40)
    mins, maxs = oq.page_summaries(K[:0], 16)
    assert mins.shape == (0, 2, 16) and maxs.shape == (0, 2, 16)
    out, lse, sel = oq.quest_decode(q, kc, vc, table, 0, 0.25, k_pages=3)
    assert sel.shape == (2, 0) and (out == 0).all() and np.isneginf(lse).all()
