"""CPU float64 oracle for paged decode attention and the cache append.

Test infrastructure, not product code.  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` import
it; the CUDA path never calls it and shares no code with it.

Every function cites the passage it follows.  Pages:
  * "Chapter 18 - KV-Cache Optimization Strategies" (karam-nus.github.io)
  * "KV Cache Engineering for LLM Serving, clearly explained" (readless.cn)
  * the untitled KV-cache overview page (learning-ai.frontdeskbot.net, topic t13_4)

Pins (tests marked ``not gpu``) tie each function to the pages' worked
examples, closed forms, invariants and independent library routines; see
``tests/test_oracle_*.py``.  No function here is "parity unpinned".
"""
from .quant import (absmax_quantize, e4m3_decode, e4m3_encode, e4m3_value_table, e5m2_decode,  # noqa: F401
                    e5m2_encode, e5m2_value_table, pack_int2, pack_int4, unpack_int2, unpack_int4)
from .paged_attention import (  # noqa: F401
    attention_one_sequence,
    dequantize_rows,
    gather_sequence,
    kv_cache_write,
    kv_head_of,
    paged_attention_decode,
)
from .block_ops import copy_blocks, swap_blocks  # noqa: F401,E402
from .quest import (decode_over_pages, group_scores, page_scores, page_summaries, quest_decode,  # noqa: F401,E402
                    select_pages)
from .kivi import (KIVI_BITS, kivi_cache_state, kivi_decode, kivi_decode_sequence,  # noqa: F401,E402
                   kivi_dequantize_block, kivi_quantize_block)
