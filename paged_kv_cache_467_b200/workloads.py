"""Seeded synthetic inputs for paged decode attention.

This module only *builds inputs*: context lengths, block tables drawn from a
shuffled block pool, slot numbers, queries and key/value rows. It performs none
of the attention or quantisation arithmetic, so both the CUDA path and the CPU
oracle can consume the same arrays.

Shapes follow the pages' statement of the problem:
  * a physical block holds ``block_size`` tokens x ``n_kv`` heads x ``d`` values
    ("Chapter 18 - KV-Cache Optimization Strategies", How PagedAttention Works,
    Physical KV Block figure);
  * a per-sequence block table maps logical block j to a physical block
    (KV-cache overview page, t13_4, block-table paragraph and its
    ``[7, 2, 14]`` example);
  * new tokens fill the current block and a fresh block is taken when it is full
    (Chapter 18, How PagedAttention Works).

Reading used for every workload: ``context_lens[s]`` is the number of tokens
attended *after* the append, and the appended token sits at position
``context_lens[s] - 1``.

Random draws use numpy's PCG64 ``default_rng`` with a fixed key per stream:
``[seed, 0]`` lengths then pool permutation, ``[seed, 1, s]`` history of
sequence ``s``, ``[seed, 2]`` queries, ``[seed, 3]`` appended rows,
``[seed, 4]`` the shared prefix, ``[seed, 5]`` outlier channels.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

DTYPES = ("f32", "bf16", "int8", "fp8_e4m3", "fp8_e5m2", "int4", "kivi2")
FP8_MAX = {"fp8_e4m3": 448.0, "fp8_e5m2": 57344.0}  # largest finite value of each format


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Return float32 values that are exactly representable in bfloat16.

    Input preparation only (round-to-nearest-even through torch's cast), so a
    bf16 tensor built from the result holds exactly these values.
    """
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


class BlockPool:
    """FIFO free list of physical block ids.

    Requests take blocks from the head of the free list and finished requests
    return theirs to the tail, as in the allocation example of
    "KV Cache Engineering for LLM Serving", section 10 (Paging).
    """

    def __init__(self, blocks):
        self.free = list(blocks)

    def allocate(self, n: int) -> list[int]:
        if n > len(self.free):
            raise MemoryError(f"pool has {len(self.free)} free blocks, {n} requested")
        taken, self.free = self.free[:n], self.free[n:]
        return taken

    def release(self, blocks) -> None:
        self.free.extend(blocks)


def blocks_for(tokens: int, block_size: int) -> int:
    return (int(tokens) + block_size - 1) // block_size


def slots_for_positions(block_row: np.ndarray, positions: np.ndarray, block_size: int) -> np.ndarray:
    """Slot numbers (physical block * block_size + row) of logical positions."""
    positions = np.asarray(positions, dtype=np.int64)
    phys = block_row[positions // block_size].astype(np.int64)
    return phys * block_size + positions % block_size


@dataclass
class DecodeWorkload:
    name: str
    seed: int
    n_q: int
    n_kv: int
    head_dim: int
    block_size: int
    num_blocks: int
    act_dtype: str
    cache_dtype: str
    context_lens: np.ndarray  # int32 [S]
    block_tables: np.ndarray  # int32 [S, max_blocks_per_seq], -1 padded
    sm_scale: float
    shared_prefix_tokens: int = 0
    shared_prefix_blocks: np.ndarray | None = None
    k_outlier_channels: np.ndarray | None = None  # flat (head * d + dim) indices
    outlier_factor: float = 10.0
    window: int = 0  # sliding window (0 = attend to every position)
    sinks: int = 0  # attention sinks kept with the window
    _prefix_cache: tuple | None = field(default=None, repr=False)

    # ----------------------------------------------------------------- sizes
    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0

    @property
    def group_size(self) -> int:
        return self.n_q // self.n_kv

    # -------------------------------------------------------------- slots
    def new_token_slots(self) -> np.ndarray:
        """int64 [S]: slot of the appended token (position L-1), -1 if L == 0."""
        out = np.full(self.num_seqs, -1, dtype=np.int64)
        for s, L in enumerate(self.context_lens):
            if L > 0:
                out[s] = slots_for_positions(self.block_tables[s], np.array([L - 1]), self.block_size)[0]
        return out

    def history_positions(self, s: int) -> np.ndarray:
        """Logical positions of sequence s written before the append.

        Positions covered by a shared prefix are written once for the pool (see
        ``prefix_positions``) and are excluded here.
        """
        L = int(self.context_lens[s])
        return np.arange(min(self.shared_prefix_tokens, max(L - 1, 0)), max(L - 1, 0), dtype=np.int64)

    def history_slots(self, s: int) -> np.ndarray:
        return slots_for_positions(self.block_tables[s], self.history_positions(s), self.block_size)

    def prefix_slots(self) -> np.ndarray:
        if not self.shared_prefix_tokens:
            return np.zeros(0, dtype=np.int64)
        pos = np.arange(self.shared_prefix_tokens, dtype=np.int64)
        return slots_for_positions(self.shared_prefix_blocks, pos, self.block_size)

    # -------------------------------------------------------------- values
    def _finish(self, x: np.ndarray, is_key: bool) -> np.ndarray:
        if is_key and self.k_outlier_channels is not None:
            flat = x.reshape(x.shape[0], self.n_kv * self.head_dim)
            flat[:, self.k_outlier_channels] *= np.float32(self.outlier_factor)
            x = flat.reshape(x.shape)
        if self.act_dtype == "bf16":
            x = round_to_bf16(x)
        return np.ascontiguousarray(x, dtype=np.float32)

    def _normal(self, key, shape) -> np.ndarray:
        rng = np.random.default_rng(key)
        return rng.standard_normal(shape, dtype=np.float32)

    def query(self) -> np.ndarray:
        q = self._normal([self.seed, 2], (self.num_seqs, self.n_q, self.head_dim))
        if self.act_dtype == "bf16":
            q = round_to_bf16(q)
        return q

    def new_kv(self) -> tuple[np.ndarray, np.ndarray]:
        """Key and value rows of the appended tokens, [S, n_kv, d] each."""
        rng = np.random.default_rng([self.seed, 3])
        shape = (self.num_seqs, self.n_kv, self.head_dim)
        k = rng.standard_normal(shape, dtype=np.float32)
        v = rng.standard_normal(shape, dtype=np.float32)
        return self._finish(k, True), self._finish(v, False)

    def prefix_kv(self) -> tuple[np.ndarray, np.ndarray]:
        """Rows of the shared prefix, [P, n_kv, d] each (P = shared tokens)."""
        if self._prefix_cache is None:
            rng = np.random.default_rng([self.seed, 4])
            shape = (self.shared_prefix_tokens, self.n_kv, self.head_dim)
            k = rng.standard_normal(shape, dtype=np.float32)
            v = rng.standard_normal(shape, dtype=np.float32)
            self._prefix_cache = (self._finish(k, True), self._finish(v, False))
        return self._prefix_cache

    def history_kv(self, s: int) -> tuple[np.ndarray, np.ndarray]:
        """Rows of sequence s at ``history_positions(s)``, [n, n_kv, d] each."""
        n = self.history_positions(s).shape[0]
        rng = np.random.default_rng([self.seed, 1, s])
        shape = (n, self.n_kv, self.head_dim)
        k = rng.standard_normal(shape, dtype=np.float32)
        v = rng.standard_normal(shape, dtype=np.float32)
        return self._finish(k, True), self._finish(v, False)

    def sequence_kv(self, s: int) -> tuple[np.ndarray, np.ndarray]:
        """All L rows of sequence s in logical order (prefix, history, new)."""
        L = int(self.context_lens[s])
        parts_k, parts_v = [], []
        if self.shared_prefix_tokens and L > 0:
            pk, pv = self.prefix_kv()
            n = min(self.shared_prefix_tokens, L - 1)
            parts_k.append(pk[:n])
            parts_v.append(pv[:n])
        hk, hv = self.history_kv(s)
        parts_k.append(hk)
        parts_v.append(hv)
        if L > 0:
            nk, nv = self.new_kv()
            parts_k.append(nk[s : s + 1])
            parts_v.append(nv[s : s + 1])
        shape0 = (0, self.n_kv, self.head_dim)
        k = np.concatenate(parts_k, axis=0) if parts_k else np.zeros(shape0, np.float32)
        v = np.concatenate(parts_v, axis=0) if parts_v else np.zeros(shape0, np.float32)
        assert k.shape[0] == L
        return k, v

    def fp8_head_scales(self) -> tuple[np.ndarray, np.ndarray]:
        """Static per-KV-head scales for an FP8 cache: absmax of the head / the
        format's largest finite value (448 for E4M3, 57344 for E5M2).

        Calibration input handed to the cache writer; computed over every row
        the workload will ever write (prefix, histories, appended rows).
        """
        amax_k = np.zeros(self.n_kv, dtype=np.float32)
        amax_v = np.zeros(self.n_kv, dtype=np.float32)
        parts = []
        if self.shared_prefix_tokens:
            parts.append(self.prefix_kv())
        parts.append(self.new_kv())
        for k, v in parts:
            amax_k = np.maximum(amax_k, np.abs(k).max(axis=(0, 2)) if k.size else 0)
            amax_v = np.maximum(amax_v, np.abs(v).max(axis=(0, 2)) if v.size else 0)
        for s in range(self.num_seqs):
            k, v = self.history_kv(s)
            if k.size:
                amax_k = np.maximum(amax_k, np.abs(k).max(axis=(0, 2)))
                amax_v = np.maximum(amax_v, np.abs(v).max(axis=(0, 2)))
        top = np.float32(FP8_MAX.get(self.cache_dtype, 448.0))
        return (amax_k / top).astype(np.float32), (amax_v / top).astype(np.float32)

    # --------------------------------------------------------------- bytes
    def kv_bytes_read(self) -> int:
        """Algorithmic K+V bytes one decode step reads, counting each block once."""
        from .accounting import decode_kv_bytes

        return decode_kv_bytes(self)


def _tables_from_lengths(lengths, block_size, rng, extra_blocks=0, prefix_blocks=0):
    """Shuffled pool sized to fit exactly; blocks handed out in table order."""
    need = [blocks_for(L, block_size) for L in lengths]
    private = [max(n - prefix_blocks, 0) for n in need]
    num_blocks = int(sum(private)) + prefix_blocks + extra_blocks
    perm = rng.permutation(num_blocks).astype(np.int32)
    pool = BlockPool(perm.tolist())
    shared = np.array(pool.allocate(prefix_blocks), dtype=np.int32)
    max_blocks = max(need) if need else 1
    tables = np.full((len(lengths), max(max_blocks, 1)), -1, dtype=np.int32)
    for s, n in enumerate(need):
        row = list(shared[: min(prefix_blocks, n)]) + pool.allocate(private[s])
        tables[s, : len(row)] = row
    return tables, num_blocks, shared


def make_workload(
    name: str,
    *,
    seed: int,
    context_lens,
    n_q: int,
    n_kv: int,
    head_dim: int,
    block_size: int = 16,
    act_dtype: str = "bf16",
    cache_dtype: str = "bf16",
    sm_scale: float | None = None,
    extra_blocks: int = 0,
    shared_prefix_tokens: int = 0,
    outlier_fraction: float = 0.0,
    window: int = 0,
    sinks: int = 0,
) -> DecodeWorkload:
    """Generic workload from explicit lengths (used by the parity tests)."""
    assert act_dtype in DTYPES[:2] and cache_dtype in DTYPES
    lengths = np.asarray(context_lens, dtype=np.int32)
    rng = np.random.default_rng([seed, 0])
    assert shared_prefix_tokens % block_size == 0
    pblocks = shared_prefix_tokens // block_size
    if pblocks:
        assert (lengths > shared_prefix_tokens).all()
    tables, num_blocks, shared = _tables_from_lengths(lengths, block_size, rng, extra_blocks, pblocks)
    outliers = None
    if outlier_fraction:
        n_ch = n_kv * head_dim
        k = int(round(outlier_fraction * n_ch))
        outliers = np.sort(np.random.default_rng([seed, 5]).choice(n_ch, size=k, replace=False))
    return DecodeWorkload(
        name=name,
        seed=seed,
        n_q=n_q,
        n_kv=n_kv,
        head_dim=head_dim,
        block_size=block_size,
        num_blocks=num_blocks,
        act_dtype=act_dtype,
        cache_dtype=cache_dtype,
        context_lens=lengths,
        block_tables=tables,
        sm_scale=float(sm_scale if sm_scale is not None else 1.0 / math.sqrt(head_dim)),
        shared_prefix_tokens=shared_prefix_tokens,
        shared_prefix_blocks=shared if pblocks else None,
        k_outlier_channels=outliers,
        window=window,
        sinks=sinks,
    )


def _uniform_lengths(seed, n, lo, hi):
    return np.random.default_rng([seed, 0, 99]).integers(lo, hi + 1, size=n).astype(np.int32)


# ------------------------------------------------------------------ configs
def tiny(seed: int = 0) -> DecodeWorkload:
    """4 sequences {40, 17, 64, 5}, 8 q / 2 KV heads, d 64, fp32, 32-block pool."""
    lengths = np.array([40, 17, 64, 5], dtype=np.int32)
    rng = np.random.default_rng([seed, 0])
    perm = rng.permutation(32).astype(np.int32)
    pool = BlockPool(perm.tolist())
    tables = np.full((4, 4), -1, dtype=np.int32)
    for s, L in enumerate(lengths):
        row = pool.allocate(blocks_for(L, 16))
        tables[s, : len(row)] = row
    return DecodeWorkload(
        name="tiny_fp32_4seq_8q2kv_d64",
        seed=seed,
        n_q=8,
        n_kv=2,
        head_dim=64,
        block_size=16,
        num_blocks=32,
        act_dtype="f32",
        cache_dtype="f32",
        context_lens=lengths,
        block_tables=tables,
        sm_scale=1.0 / 8.0,
    )


def llama3_8b(seed: int = 1) -> DecodeWorkload:
    """Batch 64, 32 q / 8 KV heads, d 128, bf16, L ~ U[512, 4096]."""
    lengths = _uniform_lengths(seed, 64, 512, 4096)
    return make_workload("llama3_8b_b64_32q8kv_d128_bf16", seed=seed, context_lens=lengths, n_q=32, n_kv=8, head_dim=128)


def long_70b(seed: int = 2) -> DecodeWorkload:
    """Batch 8, 64 q / 8 KV heads, d 128, bf16, L ~ U[32768, 131072]."""
    lengths = _uniform_lengths(seed, 8, 32768, 131072)
    return make_workload("long_70b_b8_64q8kv_d128_bf16", seed=seed, context_lens=lengths, n_q=64, n_kv=8, head_dim=128)


def prefix_sharing(seed: int = 3) -> DecodeWorkload:
    """Batch 128, 32 q / 8 KV heads: 2048 shared tokens + U[64, 512] own tokens."""
    suffix = _uniform_lengths(seed, 128, 64, 512)
    return make_workload(
        "prefix_b128_2048shared_32q8kv_d128_bf16",
        seed=seed,
        context_lens=2048 + suffix,
        n_q=32,
        n_kv=8,
        head_dim=128,
        shared_prefix_tokens=2048,
    )


def quantized(cache_dtype: str = "int8", seed: int = 4) -> DecodeWorkload:
    """Batch 256, 32 q / 8 KV heads, L ~ U[1024, 8192], a quantised cache, 1% K outliers x10."""
    lengths = _uniform_lengths(seed, 256, 1024, 8192)
    return make_workload(
        f"quantized_b256_32q8kv_d128_{cache_dtype}",
        seed=seed,
        context_lens=lengths,
        n_q=32,
        n_kv=8,
        head_dim=128,
        cache_dtype=cache_dtype,
        outlier_fraction=0.01,
    )


def sliding_window(seed: int = 1) -> DecodeWorkload:
    """The Llama-3-8B-shaped step on a local layer: 1024-token window plus 4 sinks."""
    w = llama3_8b(seed)
    w.name = "window1024_sinks4_b64_32q8kv_d128_bf16"
    w.window, w.sinks = 1024, 4
    return w


def first_sequences(w: DecodeWorkload, n: int) -> DecodeWorkload:
    """The same workload cut to its first n sequences (a smaller case of the
    same shapes, lengths and pool recipe, for profiling)."""
    if n >= w.num_seqs:
        return w
    out = make_workload(
        f"{w.name}_first{n}", seed=w.seed, context_lens=w.context_lens[:n], n_q=w.n_q, n_kv=w.n_kv,
        head_dim=w.head_dim, block_size=w.block_size, act_dtype=w.act_dtype, cache_dtype=w.cache_dtype,
        sm_scale=w.sm_scale, shared_prefix_tokens=w.shared_prefix_tokens,
        outlier_fraction=0.01 if w.k_outlier_channels is not None else 0.0, window=w.window, sinks=w.sinks)
    return out


CONFIGS = {
    "tiny": tiny,
    "llama3_8b": llama3_8b,
    "long_70b": long_70b,
    "prefix": prefix_sharing,
    "int8": lambda: quantized("int8"),
    "fp8": lambda: quantized("fp8_e4m3", seed=5),
    "fp8_e5m2": lambda: quantized("fp8_e5m2", seed=6),
    "int4": lambda: quantized("int4", seed=7),
    "kivi2": lambda: quantized("kivi2", seed=8),
    "window": sliding_window,
}
