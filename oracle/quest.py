"""Quest: query-aware selection of cache pages, written out plainly.

Test infrastructure (see ``oracle/__init__.py``).  "KV Cache Engineering for
LLM Serving", section 7 (Query-aware sparse reads): the cache is divided into
pages of neighbouring tokens; each page keeps the element-wise minimum and
maximum of its keys; a query scores every page by
sum_i max(q_i * min_i, q_i * max_i), an upper bound of q . k for any key k of
the page, and only the highest-scoring pages are read.

Readings (the page shows one head and one query):
  * a page is one cache block (block_size tokens); the last page covers only the
    sequence's rows below its length;
  * grouped-query attention: pages are chosen per (sequence, KV head), and a
    page's score is the largest score of the query heads of that group (still
    an upper bound for each of them);
  * the k best pages are kept, ties broken toward the lower page index; with k
    at least the page count every page is kept.
"""
from __future__ import annotations

import numpy as np

from .paged_attention import attention_one_sequence, gather_dequantized, kv_head_of


def page_summaries(keys, page_size: int):
    """keys [L, n_kv, d] -> (min, max), each [ceil(L / page_size), n_kv, d]."""
    keys = np.asarray(keys, dtype=np.float64)
    L = keys.shape[0]
    pages = -(-L // page_size)
    if pages == 0:  # an empty sequence has no pages
        return np.zeros((0,) + keys.shape[1:]), np.zeros((0,) + keys.shape[1:])
    mins = np.stack([keys[j * page_size : min((j + 1) * page_size, L)].min(axis=0) for j in range(pages)])
    maxs = np.stack([keys[j * page_size : min((j + 1) * page_size, L)].max(axis=0) for j in range(pages)])
    return mins, maxs


def page_scores(q, mins, maxs):
    """q [n_q, d], mins/maxs [P, n_kv, d] -> scores [n_q, P] of each query head on its KV head's pages."""
    q = np.asarray(q, dtype=np.float64)
    n_q = q.shape[0]
    n_kv = mins.shape[1]
    out = np.zeros((n_q, mins.shape[0]))
    for h in range(n_q):
        kv = kv_head_of(h, n_q, n_kv)
        out[h] = np.maximum(q[h] * mins[:, kv, :], q[h] * maxs[:, kv, :]).sum(axis=1)
    return out


def group_scores(head_scores, n_kv: int):
    """[n_q, P] -> [n_kv, P]: the largest score among each KV head's query heads."""
    n_q = head_scores.shape[0]
    g = n_q // n_kv
    return head_scores.reshape(n_kv, g, -1).max(axis=1)


def select_pages(scores, k: int):
    """Indices of the k highest scores (ties: lower index first), in increasing order."""
    scores = np.asarray(scores, dtype=np.float64)
    order = sorted(range(len(scores)), key=lambda j: (-scores[j], j))
    return np.array(sorted(order[: min(k, len(scores))]), dtype=np.int64)


def decode_over_pages(q, key_cache, value_cache, block_row, length: int, sm_scale: float, pages,
                      cache_dtype: str = "f32", k_scale=None, v_scale=None):
    """Decode one sequence, KV head kv attending only to the rows of logical pages ``pages[kv]``.

    ``pages`` [n_kv, k]: page indices below ceil(length / block_size); a -1 entry
    and all after it are ignored.  Returns (out [n_q, d], lse [n_q]); a head with
    no page gets a zero output and lse -inf.
    """
    block_size = key_cache.shape[1]
    K = gather_dequantized(key_cache, k_scale, block_row, length, block_size, cache_dtype)
    V = gather_dequantized(value_cache, v_scale, block_row, length, block_size, cache_dtype)
    q = np.asarray(q, dtype=np.float64)
    n_q, d = q.shape
    n_kv = K.shape[1]
    g = n_q // n_kv
    out = np.zeros((n_q, d))
    lse = np.full(n_q, -np.inf)
    for kv in range(n_kv):
        listed = []
        for j in pages[kv]:
            if j < 0:
                break
            assert j * block_size < length, "page past the sequence"
            listed.append(int(j))
        if not listed:
            continue
        rows = np.concatenate([np.arange(j * block_size, min((j + 1) * block_size, length)) for j in listed])
        o, l = attention_one_sequence(q[kv * g : (kv + 1) * g], K[rows][:, kv : kv + 1], V[rows][:, kv : kv + 1],
                                      sm_scale)
        out[kv * g : (kv + 1) * g], lse[kv * g : (kv + 1) * g] = o, l
    return out, lse


def quest_decode(q, key_cache, value_cache, block_row, length: int, sm_scale: float, k_pages: int,
                 cache_dtype: str = "f32", k_scale=None, v_scale=None):
    """Decode one sequence reading only each KV head's k best pages.

    Returns (out [n_q, d], lse [n_q], selected pages [n_kv, k']).
    """
    block_size = key_cache.shape[1]
    K = gather_dequantized(key_cache, k_scale, block_row, length, block_size, cache_dtype)
    n_kv = K.shape[1]
    mins, maxs = page_summaries(K, block_size)
    chosen = group_scores(page_scores(q, mins, maxs), n_kv)
    selected = np.stack([select_pages(chosen[kv], k_pages) for kv in range(n_kv)]).reshape(n_kv, -1)
    out, lse = decode_over_pages(q, key_cache, value_cache, block_row, length, sm_scale, selected, cache_dtype,
                                 k_scale, v_scale)
    return out, lse, selected
