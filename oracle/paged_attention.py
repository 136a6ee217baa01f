"""Paged decode attention and the cache append, written out plainly in float64.

Test infrastructure (see ``oracle/__init__.py``).  Paging changes where K/V
rows live, not the arithmetic ("Chapter 18 - KV-Cache Optimization
Strategies", comparison table: PagedAttention has no quality impact), so the
oracle gathers each sequence's rows through its block table into contiguous
arrays and then applies the textbook attention definition.

Cache layout (reading of the Physical KV Block figure in Chapter 18): separate
key and value pools, each ``[num_blocks, block_size, n_kv, d]``.
Dtype names: "f32", "bf16" (values held as float), "int8" (codes with a float32
scale per (block, row, head)), "int4" (two codes per byte, pools
``[num_blocks, block_size, n_kv, d/2]``, a float32 scale per (block, row,
head)), "fp8_e4m3" and "fp8_e5m2" (bytes with a float32 scale per head).
"""
from __future__ import annotations

import math

import numpy as np

from .quant import absmax_quantize, e4m3_decode, e4m3_encode, e5m2_decode, e5m2_encode, pack_int4, unpack_int4

FP8_CODECS = {"fp8_e4m3": (e4m3_encode, e4m3_decode), "fp8_e5m2": (e5m2_encode, e5m2_decode)}
ROW_SCALED = ("int8", "int4")


def kv_head_of(h: int, n_q: int, n_kv: int) -> int:
    """KV head read by query head h under grouped-query attention.

    "KV Cache Engineering for LLM Serving", section 1 (GQA and MQA): query
    heads are split into consecutive groups of n_q / n_kv, one KV pair per
    group; the printed mapping for 8 query / 2 KV heads is [0,0,0,0,1,1,1,1].
    """
    return h // (n_q // n_kv)


def logical_to_physical(block_row, position: int, block_size: int) -> tuple[int, int]:
    """(physical block, row inside it) holding a logical token position.

    KV-cache overview page (t13_4), block-table paragraph: logical block
    position // block_size maps through the sequence's block table; the row is
    the position inside the block.
    """
    return int(block_row[position // block_size]), position % block_size


def gather_sequence(cache, block_row, length: int, block_size: int):
    """Rows 0..length-1 of one sequence, in logical order: [length, n_kv, d].

    Only the first ceil(length / block_size) table entries are read; rows of
    the last block past ``length`` are not part of the sequence (KV-cache
    overview page: the last block may be partially filled).
    """
    n_blocks = -(-length // block_size)
    blocks = [cache[int(block_row[j])] for j in range(n_blocks)]
    if not blocks:
        return cache[:0, 0]
    return np.concatenate(blocks, axis=0)[:length]


def dequantize_rows(rows, cache_dtype: str, row_scales=None, head_scales=None):
    """Stored rows -> float64 values.

    int8 / int4: code * scale of that (token, head) ("KV Cache Engineering",
    section 8: multiplying the codes by the scale restores the values); int4
    codes are unpacked from their nibbles first.  fp8_e4m3 / fp8_e5m2: FP8
    value * per-head scale.  f32 / bf16: the stored values.
    """
    if cache_dtype == "int8":
        return rows.astype(np.float64) * np.asarray(row_scales, dtype=np.float64)[..., None]
    if cache_dtype == "int4":
        return unpack_int4(rows).astype(np.float64) * np.asarray(row_scales, dtype=np.float64)[..., None]
    if cache_dtype in FP8_CODECS:
        return FP8_CODECS[cache_dtype][1](rows) * np.asarray(head_scales, dtype=np.float64)[None, :, None]
    return rows.astype(np.float64)


def gather_dequantized(cache, scales, block_row, length, block_size, cache_dtype):
    rows = gather_sequence(cache, block_row, length, block_size)
    if cache_dtype in ROW_SCALED:
        row_scales = gather_sequence(scales, block_row, length, block_size)
        return dequantize_rows(rows, cache_dtype, row_scales=row_scales)
    if cache_dtype in FP8_CODECS:
        return dequantize_rows(rows, cache_dtype, head_scales=scales)
    return dequantize_rows(rows, cache_dtype)


def attention_one_sequence(q, K, V, sm_scale: float, return_weights: bool = False):
    """Single-token attention of every query head over one sequence.

    q: [n_q, d]; K, V: [L, n_kv, d].  For query head h with KV head
    kv = kv_head_of(h): scores s_p = sm_scale * <q_h, K[p, kv]>, weights are
    the softmax of the scores (computed after subtracting their maximum), and
    the output is the weighted sum of V[p, kv] ("KV Cache Engineering",
    section 1: the query is compared with the cached keys, the comparisons give
    attention weights, and the weights combine the cached values).

    Also returns lse_h = log(sum_p exp(s_p)).  Reading for L == 0: output 0
    and lse = -inf.
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    n_q, d = q.shape
    L, n_kv, _ = K.shape
    out = np.zeros((n_q, d), dtype=np.float64)
    lse = np.full(n_q, -np.inf, dtype=np.float64)
    weights = []
    for h in range(n_q):
        kv = kv_head_of(h, n_q, n_kv)
        if L == 0:
            weights.append(np.zeros(0))
            continue
        s = sm_scale * (K[:, kv, :] @ q[h])
        m = s.max()
        e = np.exp(s - m)
        total = e.sum()
        w = e / total
        out[h] = w @ V[:, kv, :]
        lse[h] = m + math.log(total)
        weights.append(w)
    if return_weights:
        return out, lse, weights
    return out, lse


def attended_positions(length: int, window: int = 0, sinks: int = 0) -> np.ndarray:
    """Positions a new token attends to under a sliding window with sinks.

    Sliding window ("KV Cache Engineering for LLM Serving", section 3): only the
    latest ``window`` positions are kept; each new entry removes the oldest
    once the window is full.  Attention sinks ("Chapter 18 - KV-Cache
    Optimization Strategies", Token Eviction and Pruning, StreamingLLM): the
    first ``sinks`` positions are always kept as well.  window == 0 keeps
    every position.
    """
    pos = np.arange(length)
    if window <= 0:
        return pos
    keep = (pos >= length - window) | (pos < sinks)
    return pos[keep]


def paged_attention_decode(
    q,
    key_cache,
    value_cache,
    block_tables,
    context_lens,
    sm_scale: float,
    cache_dtype: str = "f32",
    k_scale=None,
    v_scale=None,
    window: int = 0,
    sinks: int = 0,
):
    """Decode attention of S sequences over a paged cache.

    For each sequence: gather its K and V rows through its block table
    (dequantising where the cache is quantised), keep the attended positions
    (all of them, or a sliding window plus sinks), then attend.  Returns
    (out [S, n_q, d], lse [S, n_q]) in float64.
    """
    q = np.asarray(q)
    S, n_q, d = q.shape
    block_size = key_cache.shape[1]
    out = np.zeros((S, n_q, d), dtype=np.float64)
    lse = np.full((S, n_q), -np.inf, dtype=np.float64)
    for s in range(S):
        L = int(context_lens[s])
        K = gather_dequantized(key_cache, k_scale, block_tables[s], L, block_size, cache_dtype)
        V = gather_dequantized(value_cache, v_scale, block_tables[s], L, block_size, cache_dtype)
        if window > 0:
            keep = attended_positions(L, window, sinks)
            K, V = K[keep], V[keep]
        out[s], lse[s] = attention_one_sequence(q[s], K, V, sm_scale)
    return out, lse


# ------------------------------------------------------------ cache append
def quantize_row_int8(x):
    """One (token, head) row -> (int8 codes, float32 scale).

    The section-8 absmax quantiser of "KV Cache Engineering" at 8 bits, one
    scale per (token, head), arithmetic in IEEE float32.
    """
    codes, scale, _ = absmax_quantize(np.asarray(x, dtype=np.float32), 8, np.float32)
    return codes.astype(np.int8), np.float32(scale)


def quantize_row_int4(x):
    """One (token, head) row -> (packed int4 bytes, float32 scale).

    The section-8 absmax quantiser of "KV Cache Engineering" at 4 bits (codes
    -7..7, the page's own example), one scale per (token, head), arithmetic in
    IEEE float32, codes packed two per byte.
    """
    codes, scale, _ = absmax_quantize(np.asarray(x, dtype=np.float32), 4, np.float32)
    return pack_int4(codes), np.float32(scale)


def quantize_rows_fp8(x, head_scales, cache_dtype: str = "fp8_e4m3"):
    """[..., n_kv, d] rows -> FP8 bytes of x / scale_h (division in float32).

    Reading for scale_h == 0: codes 0 (no division).
    """
    x = np.asarray(x, dtype=np.float32)
    sc = np.asarray(head_scales, dtype=np.float32)[:, None]
    safe = np.where(sc == 0, np.float32(1), sc).astype(np.float32)
    y = (x / safe).astype(np.float32)
    codes = FP8_CODECS[cache_dtype][0](y)
    return np.where(sc == 0, np.uint8(0), codes).astype(np.uint8)


def kv_cache_write(key, value, key_cache, value_cache, slot_mapping, cache_dtype: str = "f32", k_scale=None, v_scale=None):
    """Write new tokens' K/V rows into their slots (in place).

    Chapter 18, How PagedAttention Works: new tokens fill the current block.
    Slot sigma addresses row sigma % block_size of block sigma // block_size;
    slot -1 means "no write".  int8 / int4 also write the per-(token, head)
    scales into ``k_scale``/``v_scale`` [num_blocks, block_size, n_kv]; the FP8
    formats read per-head scales from them.
    """
    block_size = key_cache.shape[1]
    key = np.asarray(key)
    value = np.asarray(value)
    for t, slot in enumerate(np.asarray(slot_mapping, dtype=np.int64)):
        if slot < 0:
            continue
        b, r = int(slot) // block_size, int(slot) % block_size
        if cache_dtype in ROW_SCALED:
            quantize = quantize_row_int8 if cache_dtype == "int8" else quantize_row_int4
            for h in range(key.shape[1]):
                key_cache[b, r, h], k_scale[b, r, h] = quantize(key[t, h])
                value_cache[b, r, h], v_scale[b, r, h] = quantize(value[t, h])
        elif cache_dtype in FP8_CODECS:
            key_cache[b, r] = quantize_rows_fp8(key[t], k_scale, cache_dtype)
            value_cache[b, r] = quantize_rows_fp8(value[t], v_scale, cache_dtype)
        else:
            key_cache[b, r] = key[t]
            value_cache[b, r] = value[t]
