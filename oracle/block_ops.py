"""Whole-block movers of a paged cache, written out plainly.

Test infrastructure (see ``oracle/__init__.py``).

* copy_blocks: duplicate physical blocks inside one pool.  Shared prefix blocks
  are copied on write: several block tables point at one physical block, and
  only when a sequence diverges is the affected block duplicated
  ("Chapter 18 - KV-Cache Optimization Strategies", Prefix Caching; KV-cache
  overview page t13_4, copy-on-write paragraph).
* swap_blocks: move blocks between two pools, e.g. GPU memory and CPU memory,
  and back when they are needed again ("KV Cache Engineering for LLM Serving",
  section 12, Cache Offloading from GPU).

Reading for both: all sources are read before any destination is written (a
parallel copy), so a block that is both a source and a destination in one call
contributes its old content.
"""
from __future__ import annotations

import numpy as np


def copy_blocks(pools, pairs):
    """For each (src, dst) in ``pairs``: block dst of every pool <- block src.

    ``pools`` is a list of arrays indexed by physical block on axis 0 (K pool,
    V pool, and the int8 scale arrays when present); every pool is updated the
    same way.
    """
    pairs = np.asarray(pairs, dtype=np.int64).reshape(-1, 2)
    for pool in pools:
        if pool is None:
            continue
        src = pool[pairs[:, 0]].copy()
        pool[pairs[:, 1]] = src


def swap_blocks(src_pools, dst_pools, pairs):
    """For each (src, dst): block dst of dst_pools[i] <- block src of src_pools[i]."""
    pairs = np.asarray(pairs, dtype=np.int64).reshape(-1, 2)
    for sp, dp in zip(src_pools, dst_pools):
        if sp is None:
            continue
        dp[pairs[:, 1]] = sp[pairs[:, 0]].copy()
