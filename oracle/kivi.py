"""KIVI-style grouped 2-bit quantisation of a paged cache, written out plainly.

Test infrastructure (see ``oracle/__init__.py``).  "KV Cache Engineering for
LLM Serving", section 8 (Quantization): KIVI groups key values by channel (the
same feature across tokens) and value-cache numbers by token, each group with
its own scale, and keeps a 2-bit cache; "Chapter 18 - KV-Cache Optimization
Strategies" (KV-Cache Quantization, methods table): per-channel K, per-token V,
2-bit.

Readings (the pages give neither a layout nor a quantiser of their own for it):
  * the quantiser is the section-8 symmetric absmax one at b = 2 bits: largest
    code 1, scale = max |x| (float32), codes in {-1, 0, 1};
  * a key group is one channel of one KV head over the 16 tokens of a full
    cache block; a value group is the head_dim values of one token of one KV
    head;
  * only full blocks are quantised (a channel group needs all 16 tokens); the
    rows of a sequence's last, partial block stay in BF16 ("residual" rows)
    until the block is full, then the whole block is quantised at once;
  * decoding attends over the dequantised full blocks followed by the residual
    rows, with the plain attention definition.
"""
from __future__ import annotations

import numpy as np

from .paged_attention import attention_one_sequence
from .quant import absmax_quantize

KIVI_BITS = 2
BLOCK = 16


def kivi_quantize_block(k_rows, v_rows, bits: int = KIVI_BITS):
    """One full block: K, V rows [16, n_kv, d] ->
    (K codes int8 [16, n_kv, d], K scales float32 [n_kv, d],
     V codes int8 [16, n_kv, d], V scales float32 [16, n_kv])."""
    k_rows = np.asarray(k_rows, dtype=np.float32)
    v_rows = np.asarray(v_rows, dtype=np.float32)
    T, n_kv, d = k_rows.shape
    k_codes = np.zeros((T, n_kv, d), np.int8)
    k_scales = np.zeros((n_kv, d), np.float32)
    v_codes = np.zeros((T, n_kv, d), np.int8)
    v_scales = np.zeros((T, n_kv), np.float32)
    for h in range(n_kv):
        for i in range(d):  # key group: one channel over the block's tokens
            codes, scale, _ = absmax_quantize(k_rows[:, h, i], bits, np.float32)
            k_codes[:, h, i] = codes
            k_scales[h, i] = scale
        for t in range(T):  # value group: one token
            codes, scale, _ = absmax_quantize(v_rows[t, h, :], bits, np.float32)
            v_codes[t, h, :] = codes
            v_scales[t, h] = scale
    return k_codes, k_scales, v_codes, v_scales


def kivi_dequantize_block(k_codes, k_scales, v_codes, v_scales):
    """Inverse mapping of one block: codes times their group's scale, float64."""
    k = np.asarray(k_codes, np.float64) * np.asarray(k_scales, np.float64)[None, :, :]
    v = np.asarray(v_codes, np.float64) * np.asarray(v_scales, np.float64)[:, :, None]
    return k, v


def kivi_cache_state(k_rows, v_rows):
    """The cache of one sequence after its rows [L, n_kv, d] were written in
    order: (list of its L // 16 quantised full blocks, residual K rows,
    residual V rows), the residual holding the last L % 16 rows as written."""
    k_rows = np.asarray(k_rows)
    v_rows = np.asarray(v_rows)
    full = k_rows.shape[0] // BLOCK
    blocks = [kivi_quantize_block(k_rows[b * BLOCK:(b + 1) * BLOCK], v_rows[b * BLOCK:(b + 1) * BLOCK])
              for b in range(full)]
    return blocks, k_rows[full * BLOCK:].astype(np.float64), v_rows[full * BLOCK:].astype(np.float64)


def kivi_decode(q, blocks, residual_k, residual_v, sm_scale: float):
    """Decode one sequence: ``blocks`` is the list of its full quantised blocks
    in logical order (each a tuple from kivi_quantize_block), ``residual_k`` /
    ``residual_v`` [r, n_kv, d] the rows of its partial last block (r < 16).
    Returns (out [n_q, d], lse [n_q]); no row at all gives out 0, lse -inf."""
    ks, vs = [], []
    for blk in blocks:
        k, v = kivi_dequantize_block(*blk)
        ks.append(k)
        vs.append(v)
    ks.append(np.asarray(residual_k, np.float64))
    vs.append(np.asarray(residual_v, np.float64))
    K = np.concatenate(ks, axis=0)
    V = np.concatenate(vs, axis=0)
    return attention_one_sequence(q, K, V, sm_scale)


def kivi_decode_sequence(q, k_rows, v_rows, sm_scale: float):
    """Decode over the KIVI cache that holds a sequence's rows [L, n_kv, d]
    (the decode step appends its new row first: pass L + 1 rows)."""
    return kivi_decode(q, *kivi_cache_state(k_rows, v_rows), sm_scale)
