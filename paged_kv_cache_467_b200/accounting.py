"""Byte accounting for a paged KV cache.

The cache-size rule is stated in words on the KV-cache overview page (t13_4,
cache-size paragraph): keys and values (the leading 2), times layers, KV heads,
head dimension, retained tokens and bytes per element.  "KV Cache Engineering
for LLM Serving", The cache formula, gives the same rule (its own copy of the
formula did not survive extraction) and notes 2 bytes for BF16, 1 for FP8.
"""
from __future__ import annotations

BYTES_PER_VALUE = {"f32": 4, "bf16": 2, "int8": 1, "fp8_e4m3": 1, "fp8_e5m2": 1, "int4": 0.5, "kivi2": 0.25}


def cache_bytes(layers: int, kv_heads: int, head_dim: int, tokens: int, bytes_per_value: float) -> float:
    """Raw K+V cache bytes for one sequence."""
    return 2 * layers * kv_heads * head_dim * tokens * bytes_per_value


def block_bytes(block_size: int, kv_heads: int, head_dim: int, bytes_per_value: float) -> float:
    """K+V bytes of one physical block of one layer (Chapter 18, Physical KV Block)."""
    return cache_bytes(1, kv_heads, head_dim, block_size, bytes_per_value)


def cached_scalars(kv_heads: int, tokens: int, head_size: int) -> int:
    """K+V scalars held for ``tokens`` tokens of one layer ("KV Cache Engineering", section 1)."""
    return 2 * kv_heads * tokens * head_size


def tokens_in_pool(pool_bytes: float, bytes_per_token: float) -> int:
    """Whole tokens that fit in a fixed pool ("KV Cache Engineering", section 10)."""
    return int(pool_bytes // bytes_per_token)


def scale_bytes_per_token(cache_dtype: str, kv_heads: int) -> int:
    """Per-token scale metadata read with the codes: one fp32 per (token, head) for K and V with int8 / int4."""
    return 2 * kv_heads * 4 if cache_dtype in ("int8", "int4") else 0


def decode_kv_bytes(w, unique: bool = True) -> int:
    """K+V bytes one decode step must read from HBM for workload ``w``.

    ``unique=True`` counts each physical block once (a shared prefix block is
    read from DRAM once per step at best); ``unique=False`` counts the logical
    bytes every sequence attends to.  Per-token scale bytes are included.
    """
    if w.cache_dtype == "kivi2":
        return kivi_decode_bytes(w)
    per_token = cache_bytes(1, w.n_kv, w.head_dim, 1, BYTES_PER_VALUE[w.cache_dtype])
    per_token += scale_bytes_per_token(w.cache_dtype, w.n_kv)
    lens = w.context_lens.astype("int64")
    if getattr(w, "window", 0) > 0:
        # attended positions only: [0, sinks) and [L - window, L)
        lens = lens.clip(max=w.window + w.sinks)
    tokens = int(lens.sum())
    if unique and w.shared_prefix_tokens:
        tokens -= (w.num_seqs - 1) * w.shared_prefix_tokens
    return int(tokens * per_token)


def kivi_block_bytes(kv_heads: int, head_dim: int, block_size: int = 16) -> int:
    """Bytes of one full block of the 2-bit KIVI cache: K and V codes (a quarter
    byte each), one fp32 K scale per (head, channel), one fp32 V scale per
    (token, head)."""
    codes = cache_bytes(1, kv_heads, head_dim, block_size, 0.25)
    return int(codes + kv_heads * head_dim * 4 + block_size * kv_heads * 4)


def kivi_decode_bytes(w) -> int:
    """Bytes one KIVI decode step reads: the full blocks of every sequence and
    its L % 16 BF16 residual rows (K and V)."""
    lens = w.context_lens.astype("int64")
    full = int((lens // w.block_size).sum())
    resid = int((lens % w.block_size).sum())
    return full * kivi_block_bytes(w.n_kv, w.head_dim, w.block_size) + int(cache_bytes(1, w.n_kv, w.head_dim, resid, 2))
