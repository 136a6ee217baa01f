"""ctypes binding of libpkv.so: same names as the C ABI in include/pkv.h.

Only argument marshalling happens here (dtype codes, raw pointers, the current
CUDA stream); every step of the computation runs in the library's kernels.
Importing this module raises when the library has not been built, so no caller
can end up on a silent fallback.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpkv.so")

PKV_F32, PKV_BF16, PKV_INT8, PKV_FP8_E4M3, PKV_FP8_E5M2, PKV_INT4, PKV_KIVI2 = 0, 1, 2, 3, 4, 5, 6
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape or dtype", 3: "workspace missing or too small", 4: "CUDA error"}
DEVERR_SLOT_RANGE, DEVERR_BLOCK_RANGE, DEVERR_CONTEXT_LEN, DEVERR_TIMEOUT, DEVERR_PREFIX = 0x1, 0x2, 0x4, 0x8, 0x10

_CACHE_DTYPES = {
    "f32": PKV_F32,
    "bf16": PKV_BF16,
    "int8": PKV_INT8,
    "fp8_e4m3": PKV_FP8_E4M3,
    "fp8_e5m2": PKV_FP8_E5M2,
    "int4": PKV_INT4,  # pools hold uint8 bytes, two codes each: pass cache_dtype="int4"
    "kivi2": PKV_KIVI2,  # uint8 pools, four 2-bit codes a byte (block movers only; decode via kivi_decode)
}


class PkvError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        msg = f"{where}: {STATUS.get(status, status)}"
        if detail:
            msg += f" ({detail})"
        super().__init__(msg)


class DecodeTuning(ctypes.Structure):
    """pkv_decode_tuning: launch overrides (0 = automatic); see include/pkv.h."""

    _fields_ = [("num_ctas", ctypes.c_int), ("stages", ctypes.c_int), ("heads_per_cta", ctypes.c_int),
                ("flags", ctypes.c_int), ("prefix_splits", ctypes.c_int), ("reserved", ctypes.c_int),
                ("wait_limit_cycles", ctypes.c_int64)]


TUNE_OVERLAP_PROLOGUE = 0x1
TUNE_PREFIX_SERIAL = 0x2


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_467_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    lib.pkv_kv_cache_write.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i32, i32, i32, i64, i32, i32, vp, vp]
    lib.pkv_kv_cache_write.restype = i32
    lib.pkv_paged_attention_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32]
    lib.pkv_paged_attention_workspace_size.restype = sz
    lib.pkv_paged_attention_workspace_size_ex.argtypes = [i32, i32, i32, i32, i32, i32, ctypes.POINTER(DecodeTuning)]
    lib.pkv_paged_attention_workspace_size_ex.restype = sz
    decode_args = [vp, vp, vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, i32, i32, i64, f32, i32, i32, vp, vp, sz, vp]
    lib.pkv_paged_attention_decode.argtypes = decode_args + [vp]
    lib.pkv_paged_attention_decode.restype = i32
    lib.pkv_paged_attention_decode_ex.argtypes = decode_args + [ctypes.POINTER(DecodeTuning), vp]
    lib.pkv_paged_attention_decode_ex.restype = i32
    lib.pkv_paged_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, i32, i32, i64,
                                          f32, i32, i32, vp, vp, sz, vp, vp]
    lib.pkv_paged_decode_step.restype = i32
    lib.pkv_paged_decode_step_ex.argtypes = lib.pkv_paged_decode_step.argtypes[:-1] + [ctypes.POINTER(DecodeTuning), vp]
    lib.pkv_paged_decode_step_ex.restype = i32
    lib.pkv_paged_attention_decode_static.argtypes = decode_args[:20] + [vp, vp]
    lib.pkv_paged_attention_decode_static.restype = i32
    lib.pkv_paged_attention_decode_window.argtypes = decode_args[:17] + [i32, i32] + decode_args[17:] + [vp]
    lib.pkv_paged_attention_decode_window.restype = i32
    lib.pkv_copy_blocks.argtypes = [vp, vp, vp, vp, vp, i64, i32, i32, i32, i64, i32, vp, vp]
    lib.pkv_copy_blocks.restype = i32
    lib.pkv_swap_blocks.argtypes = [vp, vp, vp, vp, i64, vp, vp, vp, vp, i64, vp, i64, i32, i32, i32, i32, vp, vp]
    lib.pkv_swap_blocks.restype = i32
    lib.pkv_quest_page_summaries.argtypes = [vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, i64, i32, i32, vp, vp]
    lib.pkv_quest_page_summaries.restype = i32
    lib.pkv_quest_select.argtypes = [vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, i32, i32, i64, i32, i32, i32, vp, vp,
                                     vp, vp]
    lib.pkv_quest_select.restype = i32
    lib.pkv_paged_attention_decode_pages.argtypes = decode_args[:17] + [vp, i32] + decode_args[17:] + [vp]
    lib.pkv_paged_attention_decode_pages.restype = i32
    lib.pkv_paged_attention_decode_pages_ex.argtypes = (lib.pkv_paged_attention_decode_pages.argtypes[:-1]
                                                        + [ctypes.POINTER(DecodeTuning), vp])
    lib.pkv_paged_attention_decode_pages_ex.restype = i32
    lib.pkv_paged_decode_step_window.argtypes = (lib.pkv_paged_decode_step.argtypes[:19] + [i32, i32]
                                                 + lib.pkv_paged_decode_step.argtypes[19:])
    lib.pkv_paged_decode_step_window.restype = i32
    lib.pkv_shared_prefix_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32]
    lib.pkv_shared_prefix_workspace_size.restype = sz
    lib.pkv_shared_prefix_workspace_size_ex.argtypes = [i32, i32, i32, i32, i32, i32, ctypes.POINTER(DecodeTuning)]
    lib.pkv_shared_prefix_workspace_size_ex.restype = sz
    lib.pkv_paged_attention_decode_shared_prefix.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32,
                                                             i32, i32, i64, f32, i32, i32, i32, vp, vp, sz, vp, vp]
    lib.pkv_paged_attention_decode_shared_prefix.restype = i32
    lib.pkv_paged_attention_decode_shared_prefix_ex.argtypes = (
        lib.pkv_paged_attention_decode_shared_prefix.argtypes[:-1] + [ctypes.POINTER(DecodeTuning), vp])
    lib.pkv_paged_attention_decode_shared_prefix_ex.restype = i32
    lib.pkv_kivi_workspace_size.argtypes = [i32, i32, i32, i32, i32]
    lib.pkv_kivi_workspace_size.restype = sz
    lib.pkv_kivi_quantize_blocks.argtypes = [vp, vp, vp, i64, vp, vp, vp, vp, i32, i32, i32, i64, i32, vp, vp]
    lib.pkv_kivi_quantize_blocks.restype = i32
    lib.pkv_kivi_decode.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, i32, i32,
                                    i64, f32, i32, vp, vp, sz, vp, vp]
    lib.pkv_kivi_decode.restype = i32
    lib.pkv_status_string.argtypes = [i32]
    lib.pkv_status_string.restype = ctypes.c_char_p
    lib.pkv_last_cuda_error.argtypes = []
    lib.pkv_last_cuda_error.restype = ctypes.c_char_p
    lib.pkv_version.argtypes = []
    lib.pkv_version.restype = i32
    return lib


lib = _load()


def _check(status: int, where: str) -> None:
    if status != 0:
        detail = lib.pkv_last_cuda_error().decode() if status == 4 else ""
        raise PkvError(status, where, detail)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libpkv must be contiguous")
    return t.data_ptr()


def _stream(device=None) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _default_scale(sm_scale, head_dim: int) -> float:
    """The softmax scale to pass: the caller's, else 1 / sqrt(head_dim)."""
    return 1.0 / math.sqrt(head_dim) if sm_scale is None else sm_scale


def act_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return PKV_F32
    if t.dtype == torch.bfloat16:
        return PKV_BF16
    raise TypeError(f"unsupported activation dtype {t.dtype}")


def cache_code(t: torch.Tensor, cache_dtype: str | None = None) -> int:
    """Cache dtype code from an explicit name, else from the pool's torch dtype
    (uint8 pools are E4M3 unless named; an INT4 pool must be named "int4")."""
    if cache_dtype is not None:
        return _CACHE_DTYPES[cache_dtype]
    if t.dtype == torch.float32:
        return PKV_F32
    if t.dtype == torch.bfloat16:
        return PKV_BF16
    if t.dtype == torch.int8:
        return PKV_INT8
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return PKV_FP8_E4M3
    if t.dtype == torch.float8_e5m2:
        return PKV_FP8_E5M2
    raise TypeError(f"unsupported cache dtype {t.dtype}")


def kv_cache_write(key, value, key_cache, value_cache, slot_mapping, k_scale=None, v_scale=None, device_error=None,
                   cache_dtype: str | None = None):
    """Append rows of ``key``/``value`` [T, n_kv, d] at ``slot_mapping`` [T] (int64)."""
    T, n_kv, d = key.shape
    num_blocks, block_size = key_cache.shape[0], key_cache.shape[1]
    st = lib.pkv_kv_cache_write(
        _ptr(key), _ptr(value), _ptr(key_cache), _ptr(value_cache), _ptr(k_scale), _ptr(v_scale), _ptr(slot_mapping),
        T, n_kv, d, block_size, num_blocks, act_code(key), cache_code(key_cache, cache_dtype), _ptr(device_error),
        _stream(key.device),
    )
    _check(st, "pkv_kv_cache_write")


def paged_attention_workspace_size(num_seqs, n_q, n_kv, head_dim, block_size, cache_dtype: int, tuning=None) -> int:
    if tuning is None:
        n = lib.pkv_paged_attention_workspace_size(num_seqs, n_q, n_kv, head_dim, block_size, cache_dtype)
    else:
        n = lib.pkv_paged_attention_workspace_size_ex(num_seqs, n_q, n_kv, head_dim, block_size, cache_dtype, ctypes.byref(tuning))
    if n == ctypes.c_size_t(-1).value:
        raise PkvError(2, "pkv_paged_attention_workspace_size")
    return int(n)


_ws_lock = threading.Lock()
_workspaces: dict = {}


def workspace_for(nbytes: int, device) -> torch.Tensor:
    """Zero-filled scratch reused per (device, stream); grows when needed."""
    key = (torch.device(device).index, _stream(device))
    with _ws_lock:
        ws = _workspaces.get(key)
        if ws is None or ws.numel() < nbytes:
            ws = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)
            _workspaces[key] = ws
        return ws


def paged_attention_decode(
    out,
    query,
    key_cache,
    value_cache,
    block_tables,
    context_lens,
    max_context_len: int,
    sm_scale: float | None = None,
    k_scale=None,
    v_scale=None,
    lse_out=None,
    workspace=None,
    device_error=None,
    tuning: DecodeTuning | None = None,
    cache_dtype: str | None = None,
):
    """Decode attention of ``query`` [S, n_q, d] over a paged cache into ``out``."""
    S, n_q, d = query.shape
    num_blocks, block_size, n_kv = key_cache.shape[0], key_cache.shape[1], key_cache.shape[2]
    ccode = cache_code(key_cache, cache_dtype)
    sm_scale = _default_scale(sm_scale, d)
    if workspace is None:
        nbytes = paged_attention_workspace_size(S, n_q, n_kv, d, block_size, ccode, tuning)
        workspace = workspace_for(nbytes, query.device) if nbytes else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    args = [
        _ptr(out), _ptr(query), _ptr(key_cache), _ptr(value_cache), _ptr(k_scale), _ptr(v_scale), _ptr(block_tables),
        block_tables.shape[1], _ptr(context_lens), int(max_context_len), S, n_q, n_kv, d, block_size, num_blocks,
        float(sm_scale), act_code(query), ccode, _ptr(lse_out), _ptr(workspace), ws_bytes, _ptr(device_error),
    ]
    if tuning is None:
        st = lib.pkv_paged_attention_decode(*args, _stream(query.device))
    else:
        st = lib.pkv_paged_attention_decode_ex(*args, ctypes.byref(tuning), _stream(query.device))
    _check(st, "pkv_paged_attention_decode")
    return out


def paged_decode_step(out, query, key, value, key_cache, value_cache, block_tables, context_lens, max_context_len: int,
                      sm_scale: float | None = None, k_scale=None, v_scale=None, lse_out=None, workspace=None,
                      device_error=None, tuning: DecodeTuning | None = None, cache_dtype: str | None = None):
    """One fused decode step: append ``key``/``value`` [S, n_kv, d] as token L-1 of each sequence, then attend."""
    S, n_q, d = query.shape
    num_blocks, block_size, n_kv = key_cache.shape[0], key_cache.shape[1], key_cache.shape[2]
    ccode = cache_code(key_cache, cache_dtype)
    sm_scale = _default_scale(sm_scale, d)
    if workspace is None:
        nbytes = paged_attention_workspace_size(S, n_q, n_kv, d, block_size, ccode, tuning)
        workspace = workspace_for(nbytes, query.device) if nbytes else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    args = [
        _ptr(out), _ptr(query), _ptr(key), _ptr(value), _ptr(key_cache), _ptr(value_cache), _ptr(k_scale),
        _ptr(v_scale), _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), int(max_context_len), S, n_q,
        n_kv, d, block_size, num_blocks, float(sm_scale), act_code(query), ccode, _ptr(lse_out), _ptr(workspace),
        ws_bytes, _ptr(device_error),
    ]
    if tuning is None:
        st = lib.pkv_paged_decode_step(*args, _stream(query.device))
    else:
        st = lib.pkv_paged_decode_step_ex(*args, ctypes.byref(tuning), _stream(query.device))
    _check(st, "pkv_paged_decode_step")
    return out


def paged_attention_decode_static(out, query, key_cache, value_cache, block_tables, context_lens, max_context_len: int,
                                  sm_scale: float | None = None, k_scale=None, v_scale=None, lse_out=None,
                                  device_error=None, cache_dtype: str | None = None):
    """pkv_paged_attention_decode_static: decode with the library's own scratch (no workspace argument)."""
    S, n_q, d = query.shape
    num_blocks, block_size, n_kv = key_cache.shape[0], key_cache.shape[1], key_cache.shape[2]
    sm_scale = _default_scale(sm_scale, d)
    st = lib.pkv_paged_attention_decode_static(
        _ptr(out), _ptr(query), _ptr(key_cache), _ptr(value_cache), _ptr(k_scale), _ptr(v_scale), _ptr(block_tables),
        block_tables.shape[1], _ptr(context_lens), int(max_context_len), S, n_q, n_kv, d, block_size, num_blocks,
        float(sm_scale), act_code(query), cache_code(key_cache, cache_dtype), _ptr(lse_out), _ptr(device_error),
        _stream(query.device),
    )
    if st != 0:
        raise PkvError(st, "pkv_paged_attention_decode_static", lib.pkv_last_cuda_error().decode())
    return out


def copy_blocks(key_cache, value_cache, block_mapping, k_scale=None, v_scale=None, device_error=None, stream=None,
                cache_dtype: str | None = None):
    """Copy-on-write block copies inside one pool; ``block_mapping`` int64 [P, 2] = (src, dst)."""
    nb, bs, n_kv, d = key_cache.shape
    code = cache_code(key_cache, cache_dtype)
    if code == PKV_INT4:
        d *= 2
    elif code == PKV_KIVI2:  # pools [nb, n_kv, 16, d / 4]
        bs, n_kv, d = n_kv, bs, d * 4
    st = lib.pkv_copy_blocks(_ptr(key_cache), _ptr(value_cache), _ptr(k_scale), _ptr(v_scale), _ptr(block_mapping),
                             block_mapping.shape[0], n_kv, d, bs, nb, code, _ptr(device_error),
                             stream if stream is not None else _stream(key_cache.device))
    _check(st, "pkv_copy_blocks")


def swap_blocks(src_key, src_value, dst_key, dst_value, block_mapping, src_k_scale=None, src_v_scale=None,
                dst_k_scale=None, dst_v_scale=None, device_error=None, device=None, cache_dtype: str | None = None):
    """Move blocks between two pools (either may be pinned host memory); (src, dst) pairs."""
    snb, bs, n_kv, d = src_key.shape
    code = cache_code(src_key, cache_dtype)
    if code == PKV_INT4:
        d *= 2
    elif code == PKV_KIVI2:  # pools [nb, n_kv, 16, d / 4]
        bs, n_kv, d = n_kv, bs, d * 4
    dev = device if device is not None else (src_key.device if src_key.is_cuda else dst_key.device)
    st = lib.pkv_swap_blocks(_ptr(src_key), _ptr(src_value), _ptr(src_k_scale), _ptr(src_v_scale), snb,
                             _ptr(dst_key), _ptr(dst_value), _ptr(dst_k_scale), _ptr(dst_v_scale), dst_key.shape[0],
                             _ptr(block_mapping), block_mapping.shape[0], n_kv, d, bs, code,
                             _ptr(device_error), _stream(dev))
    _check(st, "pkv_swap_blocks")


def paged_attention_decode_window(out, query, key_cache, value_cache, block_tables, context_lens, max_context_len: int,
                                  window: int, sinks: int = 0, sm_scale: float | None = None, k_scale=None,
                                  v_scale=None, lse_out=None, workspace=None, device_error=None,
                                  cache_dtype: str | None = None):
    """Decode attention over positions [0, sinks) and [L - window, L) of each sequence."""
    S, n_q, d = query.shape
    num_blocks, block_size, n_kv = key_cache.shape[0], key_cache.shape[1], key_cache.shape[2]
    ccode = cache_code(key_cache, cache_dtype)
    sm_scale = _default_scale(sm_scale, d)
    if workspace is None:
        nbytes = paged_attention_workspace_size(S, n_q, n_kv, d, block_size, ccode)
        workspace = workspace_for(nbytes, query.device) if nbytes else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib.pkv_paged_attention_decode_window(
        _ptr(out), _ptr(query), _ptr(key_cache), _ptr(value_cache), _ptr(k_scale), _ptr(v_scale), _ptr(block_tables),
        block_tables.shape[1], _ptr(context_lens), int(max_context_len), S, n_q, n_kv, d, block_size, num_blocks,
        float(sm_scale), int(window), int(sinks), act_code(query), ccode, _ptr(lse_out), _ptr(workspace), ws_bytes,
        _ptr(device_error), _stream(query.device),
    )
    _check(st, "pkv_paged_attention_decode_window")
    return out


def quest_page_summaries(key_cache, page_min, page_max, block_tables, context_lens, device_error=None,
                         last_page_only: bool = False):
    """Element-wise min / max of each page's keys into ``page_min`` / ``page_max`` [num_blocks, n_kv, d]."""
    nb, bs, n_kv, d = key_cache.shape
    st = lib.pkv_quest_page_summaries(_ptr(key_cache), _ptr(page_min), _ptr(page_max), _ptr(block_tables),
                                      block_tables.shape[1], _ptr(context_lens), block_tables.shape[0], n_kv, d, bs,
                                      nb, cache_code(key_cache), int(bool(last_page_only)), _ptr(device_error),
                                      _stream(key_cache.device))
    _check(st, "pkv_quest_page_summaries")


def quest_select(query, page_min, page_max, block_tables, context_lens, max_context_len: int, k_pages: int,
                 selected, scores=None, device_error=None):
    """Each (sequence, KV head)'s ``k_pages`` best pages into ``selected`` [S, n_kv, k_pages] (ascending, -1 after)."""
    S, n_q, d = query.shape
    nb, n_kv = page_min.shape[0], page_min.shape[1]
    if scores is None:
        cap = min(int(max_context_len), block_tables.shape[1] * 16)
        scores = torch.empty((S, n_kv, max(1, -(-cap // 16))), dtype=torch.float32, device=query.device)
    st = lib.pkv_quest_select(_ptr(query), _ptr(page_min), _ptr(page_max), _ptr(block_tables), block_tables.shape[1],
                              _ptr(context_lens), int(max_context_len), S, n_q, n_kv, d, 16, nb, act_code(query),
                              cache_code(page_min), int(k_pages), _ptr(selected), _ptr(scores), _ptr(device_error),
                              _stream(query.device))
    _check(st, "pkv_quest_select")
    return selected


def paged_attention_decode_pages(out, query, key_cache, value_cache, block_tables, context_lens, max_context_len: int,
                                 pages, sm_scale: float | None = None, k_scale=None, v_scale=None, lse_out=None,
                                 workspace=None, device_error=None, tuning: DecodeTuning | None = None,
                                 cache_dtype: str | None = None):
    """Decode attention over the logical pages listed in ``pages`` [S, n_kv, k] for each KV head."""
    S, n_q, d = query.shape
    num_blocks, block_size, n_kv = key_cache.shape[0], key_cache.shape[1], key_cache.shape[2]
    ccode = cache_code(key_cache, cache_dtype)
    sm_scale = _default_scale(sm_scale, d)
    if workspace is None:
        t1 = None if tuning is None else DecodeTuning(tuning.num_ctas, tuning.stages, 1, tuning.flags)
        nbytes = paged_attention_workspace_size(S, n_q, n_kv, d, block_size, ccode, t1)
        workspace = workspace_for(nbytes, query.device) if nbytes else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    args = [
        _ptr(out), _ptr(query), _ptr(key_cache), _ptr(value_cache), _ptr(k_scale), _ptr(v_scale), _ptr(block_tables),
        block_tables.shape[1], _ptr(context_lens), int(max_context_len), S, n_q, n_kv, d, block_size, num_blocks,
        float(sm_scale), _ptr(pages), pages.shape[-1], act_code(query), ccode, _ptr(lse_out), _ptr(workspace),
        ws_bytes, _ptr(device_error),
    ]
    if tuning is None:
        st = lib.pkv_paged_attention_decode_pages(*args, _stream(query.device))
    else:
        st = lib.pkv_paged_attention_decode_pages_ex(*args, ctypes.byref(tuning), _stream(query.device))
    _check(st, "pkv_paged_attention_decode_pages")
    return out


def shared_prefix_workspace_size(num_seqs, n_q, n_kv, head_dim, block_size, prefix_blocks, tuning=None) -> int:
    if tuning is None:
        n = lib.pkv_shared_prefix_workspace_size(num_seqs, n_q, n_kv, head_dim, block_size, prefix_blocks)
    else:
        n = lib.pkv_shared_prefix_workspace_size_ex(num_seqs, n_q, n_kv, head_dim, block_size, prefix_blocks,
                                                    ctypes.byref(tuning))
    if n == ctypes.c_size_t(-1).value:
        raise PkvError(2, "pkv_shared_prefix_workspace_size")
    return int(n)


def paged_attention_decode_shared_prefix(out, query, key_cache, value_cache, block_tables, context_lens,
                                         max_context_len: int, prefix_blocks: int, key=None, value=None,
                                         sm_scale: float | None = None, lse_out=None, workspace=None,
                                         device_error=None, tuning: DecodeTuning | None = None):
    """Decode with the first ``prefix_blocks`` blocks shared by every sequence: one dense pass over the
    prefix for all queries beside the decode of each sequence's own blocks, then their merge;
    ``key``/``value`` append token L-1 first."""
    S, n_q, d = query.shape
    num_blocks, block_size, n_kv = key_cache.shape[0], key_cache.shape[1], key_cache.shape[2]
    sm_scale = _default_scale(sm_scale, d)
    if workspace is None:
        nbytes = shared_prefix_workspace_size(S, n_q, n_kv, d, block_size, prefix_blocks, tuning)
        workspace = workspace_for(nbytes, query.device) if nbytes else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    args = [
        _ptr(out), _ptr(query), _ptr(key), _ptr(value), _ptr(key_cache), _ptr(value_cache), _ptr(block_tables),
        block_tables.shape[1], _ptr(context_lens), int(max_context_len), S, n_q, n_kv, d, block_size, num_blocks,
        float(sm_scale), int(prefix_blocks), act_code(query), cache_code(key_cache), _ptr(lse_out), _ptr(workspace),
        ws_bytes, _ptr(device_error),
    ]
    if tuning is None:
        st = lib.pkv_paged_attention_decode_shared_prefix(*args, _stream(query.device))
    else:
        st = lib.pkv_paged_attention_decode_shared_prefix_ex(*args, ctypes.byref(tuning), _stream(query.device))
    _check(st, "pkv_paged_attention_decode_shared_prefix")
    return out


def paged_decode_step_window(out, query, key, value, key_cache, value_cache, block_tables, context_lens,
                             max_context_len: int, window: int, sinks: int = 0, sm_scale: float | None = None,
                             k_scale=None, v_scale=None, lse_out=None, workspace=None, device_error=None,
                             cache_dtype: str | None = None):
    """The fused step (append token L-1, attend) over positions [0, sinks) and [L - window, L)."""
    S, n_q, d = query.shape
    num_blocks, block_size, n_kv = key_cache.shape[0], key_cache.shape[1], key_cache.shape[2]
    ccode = cache_code(key_cache, cache_dtype)
    sm_scale = _default_scale(sm_scale, d)
    if workspace is None:
        nbytes = paged_attention_workspace_size(S, n_q, n_kv, d, block_size, ccode)
        workspace = workspace_for(nbytes, query.device) if nbytes else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib.pkv_paged_decode_step_window(
        _ptr(out), _ptr(query), _ptr(key), _ptr(value), _ptr(key_cache), _ptr(value_cache), _ptr(k_scale),
        _ptr(v_scale), _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), int(max_context_len), S, n_q,
        n_kv, d, block_size, num_blocks, float(sm_scale), int(window), int(sinks), act_code(query), ccode,
        _ptr(lse_out), _ptr(workspace), ws_bytes, _ptr(device_error), _stream(query.device),
    )
    _check(st, "pkv_paged_decode_step_window")
    return out


def _check_kivi_tensors(S, n_kv, d, num_blocks, block_size, residual_k, residual_v, key_cache, value_cache,
                        k_scale, v_scale):
    """Shapes and dtypes the C ABI cannot see: the pools are head-major uint8 [num_blocks, n_kv, 16, d / 4]."""
    want = {
        "residual_k": (residual_k, torch.bfloat16, (S, block_size, n_kv, d)),
        "residual_v": (residual_v, torch.bfloat16, (S, block_size, n_kv, d)),
        "key_cache": (key_cache, torch.uint8, (num_blocks, n_kv, block_size, d // 4)),
        "value_cache": (value_cache, torch.uint8, (num_blocks, n_kv, block_size, d // 4)),
        "k_scale": (k_scale, torch.float32, (num_blocks, n_kv, d)),
        "v_scale": (v_scale, torch.float32, (num_blocks, n_kv, block_size)),
    }
    for name, (t, dtype, shape) in want.items():
        if t is None or t.dtype != dtype or tuple(t.shape) != shape:
            got = None if t is None else (t.dtype, tuple(t.shape))
            raise ValueError(f"kivi_decode: {name} must be {dtype} {shape}, got {got}")


def kivi_workspace_size(num_seqs, n_q, n_kv, head_dim, block_size) -> int:
    n = lib.pkv_kivi_workspace_size(num_seqs, n_q, n_kv, head_dim, block_size)
    if n == ctypes.c_size_t(-1).value:
        raise PkvError(2, "pkv_kivi_workspace_size")
    return int(n)


def kivi_quantize_blocks(key_rows, value_rows, dst_blocks, key_cache, value_cache, k_scale, v_scale,
                         device_error=None):
    """Quantise whole blocks ``key_rows``/``value_rows`` [n, 16, n_kv, d] (bf16) into the 2-bit pools
    (uint8 [num_blocks, n_kv, 16, d / 4]) at physical blocks ``dst_blocks`` [n] (int32, -1 skips)."""
    n, block_size, n_kv, d = key_rows.shape
    st = lib.pkv_kivi_quantize_blocks(
        _ptr(key_rows), _ptr(value_rows), _ptr(dst_blocks), n, _ptr(key_cache), _ptr(value_cache), _ptr(k_scale),
        _ptr(v_scale), n_kv, d, block_size, key_cache.shape[0], act_code(key_rows), _ptr(device_error),
        _stream(key_rows.device),
    )
    _check(st, "pkv_kivi_quantize_blocks")


def kivi_decode(out, query, residual_k, residual_v, key_cache, value_cache, k_scale, v_scale, block_tables,
                context_lens, max_context_len: int, key=None, value=None, sm_scale: float | None = None,
                lse_out=None, workspace=None, device_error=None):
    """Decode over a 2-bit KIVI cache (full blocks in the pools, the partial last block in the BF16
    residual [S, 16, n_kv, d]; pools uint8 [num_blocks, n_kv, 16, d / 4], k_scale [num_blocks, n_kv, d],
    v_scale [num_blocks, n_kv, 16]); ``key``/``value`` [S, n_kv, d] append token L-1 first."""
    S, n_q, d = query.shape
    block_size, n_kv = residual_k.shape[1], residual_k.shape[2]  # residual [S, 16, n_kv, d]
    num_blocks = key_cache.shape[0]
    _check_kivi_tensors(S, n_kv, d, num_blocks, block_size, residual_k, residual_v, key_cache, value_cache, k_scale,
                        v_scale)
    sm_scale = _default_scale(sm_scale, d)
    if workspace is None:
        nbytes = kivi_workspace_size(S, n_q, n_kv, d, block_size)
        workspace = workspace_for(nbytes, query.device) if nbytes else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib.pkv_kivi_decode(
        _ptr(out), _ptr(query), _ptr(key), _ptr(value), _ptr(residual_k), _ptr(residual_v), _ptr(key_cache),
        _ptr(value_cache), _ptr(k_scale), _ptr(v_scale), _ptr(block_tables), block_tables.shape[1],
        _ptr(context_lens), int(max_context_len), S, n_q, n_kv, d, block_size, num_blocks, float(sm_scale),
        act_code(query), _ptr(lse_out), _ptr(workspace), ws_bytes, _ptr(device_error), _stream(query.device),
    )
    _check(st, "pkv_kivi_decode")
    return out
