"""Shared helpers of the GPU parity tests.

The device cache is filled through the library's own cache writer from the
seeded host rows; the oracle gets the same host rows and runs its own writer
and decode on a compact per-sequence pool (the result is invariant to where
blocks sit in the pool, which the oracle pins check).  Nothing computed on the
GPU is ever fed to the oracle.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

import oracle
from paged_kv_cache_467_b200 import workloads

TOL = {
    "f32": (1e-4, 1e-5),
    "bf16": (2e-2, 2e-3),
    "int8": (3e-2, 3e-3),
    "fp8_e4m3": (3e-2, 3e-3),
    "fp8_e5m2": (3e-2, 3e-3),
    "int4": (3e-2, 3e-3),
}

_TORCH_CACHE = {"f32": torch.float32, "bf16": torch.bfloat16, "int8": torch.int8, "fp8_e4m3": torch.uint8,
                "fp8_e5m2": torch.float8_e5m2, "int4": torch.uint8}
FP8 = ("fp8_e4m3", "fp8_e5m2")
ROW_SCALED = ("int8", "int4")


def named(w):
    """cache_dtype keyword for the binding: pools whose torch dtype does not name the format."""
    return "int4" if w.cache_dtype == "int4" else None


def row_width(w):
    """Last dimension of a pool: head_dim values, or head_dim / 2 bytes for int4."""
    return w.head_dim // 2 if w.cache_dtype == "int4" else w.head_dim
_TORCH_ACT = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclass
class GpuState:
    key_cache: torch.Tensor
    value_cache: torch.Tensor
    k_scale: torch.Tensor | None
    v_scale: torch.Tensor | None
    query: torch.Tensor
    block_tables: torch.Tensor
    context_lens: torch.Tensor
    device_error: torch.Tensor
    fp8_scales: tuple | None


def _poisoned_cache(w, device):
    shape = (w.num_blocks, w.block_size, w.n_kv, row_width(w))
    dt = _TORCH_CACHE[w.cache_dtype]
    if w.cache_dtype in ("f32", "bf16"):
        kc = torch.full(shape, float("nan"), dtype=dt, device=device)
        vc = torch.full(shape, float("nan"), dtype=dt, device=device)
    elif w.cache_dtype == "int8":
        kc = torch.full(shape, 77, dtype=dt, device=device)
        vc = torch.full(shape, -77, dtype=dt, device=device)
    elif w.cache_dtype == "int4":
        kc = torch.full(shape, 0x77, dtype=dt, device=device)  # codes 7, 7
        vc = torch.full(shape, 0x99, dtype=dt, device=device)  # codes -7, -7
    else:
        kc = torch.full(shape, 0x7F, dtype=torch.uint8, device=device).view(dt)  # a NaN code of both FP8 formats
        vc = torch.full(shape, 0x7F, dtype=torch.uint8, device=device).view(dt)
    return kc, vc


def _rows(x, w, device):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device=device, dtype=_TORCH_ACT[w.act_dtype])


def fill_gpu(w: workloads.DecodeWorkload, device="cuda", fp8_scales=None, chunk_tokens=1 << 20,
             append_new: bool = True) -> GpuState:
    """Allocate a poisoned pool and append rows through pkv_kv_cache_write.

    With ``append_new=False`` the new token (position L-1) is left out, for
    the fused decode step to append.
    """
    from paged_kv_cache_467_b200 import ops

    kc, vc = _poisoned_cache(w, device)
    ks = vs = None
    if w.cache_dtype in ROW_SCALED:
        ks = torch.full((w.num_blocks, w.block_size, w.n_kv), float("nan"), dtype=torch.float32, device=device)
        vs = torch.full_like(ks, float("nan"))
    elif w.cache_dtype in FP8:
        if fp8_scales is None:
            fp8_scales = w.fp8_head_scales()
        ks = torch.from_numpy(fp8_scales[0]).to(device)
        vs = torch.from_numpy(fp8_scales[1]).to(device)
    err = torch.zeros(1, dtype=torch.int32, device=device)

    def write(k, v, slots):
        if len(slots) == 0:
            return
        ops.kv_cache_write(_rows(k, w, device), _rows(v, w, device), kc, vc,
                           torch.from_numpy(np.asarray(slots, dtype=np.int64)).to(device), ks, vs, err,
                           cache_dtype=named(w))

    if w.shared_prefix_tokens:
        pk, pv = w.prefix_kv()
        write(pk, pv, w.prefix_slots())
    bk, bv, bslots, n = [], [], [], 0
    for s in range(w.num_seqs):
        hk, hv = w.history_kv(s)
        bk.append(hk), bv.append(hv), bslots.append(w.history_slots(s))
        n += len(hk)
        if n >= chunk_tokens or s == w.num_seqs - 1:
            write(np.concatenate(bk), np.concatenate(bv), np.concatenate(bslots))
            bk, bv, bslots, n = [], [], [], 0
    if append_new:
        nk, nv = w.new_kv()
        write(nk, nv, w.new_token_slots())
    torch.cuda.synchronize()
    return GpuState(
        key_cache=kc,
        value_cache=vc,
        k_scale=ks,
        v_scale=vs,
        query=_rows(w.query(), w, device),
        block_tables=torch.from_numpy(w.block_tables).to(device),
        context_lens=torch.from_numpy(w.context_lens).to(device),
        device_error=err,
        fp8_scales=fp8_scales,
    )


def run_decode(w, st: GpuState, tuning=None, workspace=None, block_tables=None):
    from paged_kv_cache_467_b200 import ops

    out = torch.full((w.num_seqs, w.n_q, w.head_dim), float("nan"), dtype=_TORCH_ACT[w.act_dtype], device=st.query.device)
    lse = torch.full((w.num_seqs, w.n_q), float("nan"), dtype=torch.float32, device=st.query.device)
    ops.paged_attention_decode(
        out, st.query, st.key_cache, st.value_cache, st.block_tables if block_tables is None else block_tables,
        st.context_lens, w.max_context_len, w.sm_scale, st.k_scale, st.v_scale, lse, workspace, st.device_error, tuning,
        cache_dtype=named(w),
    )
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


# ------------------------------------------------------------------ oracle side
def oracle_sequence(w, s, fp8_scales=None, window=0, sinks=0):
    """Oracle (out [n_q, d], lse [n_q], written rows) for sequence s.

    The sequence's rows are appended by ``oracle.kv_cache_write`` into a compact
    pool whose block table is 0, 1, 2, ..., then decoded by
    ``oracle.paged_attention_decode``.
    """
    L = int(w.context_lens[s])
    nb = max(workloads.blocks_for(L, w.block_size), 1)
    shape = (nb, w.block_size, w.n_kv, row_width(w))
    if w.cache_dtype == "int8":
        kc, vc = np.zeros(shape, np.int8), np.zeros(shape, np.int8)
        ks, vs = np.zeros(shape[:3], np.float32), np.zeros(shape[:3], np.float32)
    elif w.cache_dtype == "int4":
        kc, vc = np.zeros(shape, np.uint8), np.zeros(shape, np.uint8)
        ks, vs = np.zeros(shape[:3], np.float32), np.zeros(shape[:3], np.float32)
    elif w.cache_dtype in FP8:
        kc, vc = np.zeros(shape, np.uint8), np.zeros(shape, np.uint8)
        ks, vs = fp8_scales if fp8_scales is not None else w.fp8_head_scales()
    else:
        kc, vc = np.zeros(shape, np.float64), np.zeros(shape, np.float64)
        ks = vs = None
    K, V = w.sequence_kv(s)
    oracle.kv_cache_write(K, V, kc, vc, np.arange(L, dtype=np.int64), w.cache_dtype, ks, vs)
    table = np.arange(nb, dtype=np.int32)[None]
    out, lse = oracle.paged_attention_decode(w.query()[s : s + 1], kc, vc, table, np.array([L]), w.sm_scale,
                                             w.cache_dtype, ks, vs, window=window, sinks=sinks)
    return out[0], lse[0], (kc, vc, ks, vs)


def gpu_sequence_rows(w, st: GpuState, s):
    """The device cache's rows (and int8 scales) of sequence s, in logical order, as host arrays."""
    L = int(w.context_lens[s])
    nb = workloads.blocks_for(L, w.block_size)
    blocks = torch.from_numpy(w.block_tables[s, :nb].astype(np.int64)).to(st.key_cache.device)
    kc, vc = st.key_cache, st.value_cache
    if kc.dtype in (torch.float8_e4m3fn, torch.float8_e5m2):
        kc, vc = kc.view(torch.uint8), vc.view(torch.uint8)
    k = kc.index_select(0, blocks).reshape(-1, w.n_kv, row_width(w))[:L]
    v = vc.index_select(0, blocks).reshape(-1, w.n_kv, row_width(w))[:L]
    res = [k.cpu(), v.cpu()]
    if w.cache_dtype in ROW_SCALED:
        res += [st.k_scale.index_select(0, blocks).reshape(-1, w.n_kv)[:L].cpu(),
                st.v_scale.index_select(0, blocks).reshape(-1, w.n_kv)[:L].cpu()]
    return res


def assert_rows_bit_exact(w, st, s, oracle_rows):
    """Device cache rows of sequence s equal the oracle writer's, bit for bit."""
    kc, vc, ks, vs = oracle_rows
    L = int(w.context_lens[s])
    got = gpu_sequence_rows(w, st, s)
    want_k = kc.reshape(-1, w.n_kv, row_width(w))[:L]
    want_v = vc.reshape(-1, w.n_kv, row_width(w))[:L]
    if w.cache_dtype == "bf16":
        gk = got[0].view(torch.int16).numpy()
        wk = torch.from_numpy(want_k.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
        gv = got[1].view(torch.int16).numpy()
        wv = torch.from_numpy(want_v.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
        assert np.array_equal(gk, wk) and np.array_equal(gv, wv)
    elif w.cache_dtype == "f32":
        assert np.array_equal(got[0].numpy().view(np.int32), want_k.astype(np.float32).view(np.int32))
        assert np.array_equal(got[1].numpy().view(np.int32), want_v.astype(np.float32).view(np.int32))
    else:
        assert np.array_equal(got[0].numpy().view(np.uint8), want_k.view(np.uint8))
        assert np.array_equal(got[1].numpy().view(np.uint8), want_v.view(np.uint8))
        if w.cache_dtype in ROW_SCALED:
            assert np.array_equal(got[2].numpy().view(np.int32), ks.reshape(-1, w.n_kv)[:L].view(np.int32))
            assert np.array_equal(got[3].numpy().view(np.int32), vs.reshape(-1, w.n_kv)[:L].view(np.int32))


def errors(got, want):
    d = np.abs(got - want)
    return float(d.max()), float(d.mean())


def assert_close(got, want, cache_dtype, what=""):
    mx_tol, mean_tol = TOL[cache_dtype]
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    mx, mean = errors(got, want)
    assert mx <= mx_tol and mean <= mean_tol, f"{what}: max abs {mx:.3e} (tol {mx_tol}), mean abs {mean:.3e} (tol {mean_tol})"
    return mx, mean


def new_rows(w, device="cuda"):
    nk, nv = w.new_kv()
    return _rows(nk, w, device), _rows(nv, w, device)


def run_decode_step(w, st: GpuState, workspace=None):
    """The fused step (append token L-1, then attend) through pkv_paged_decode_step."""
    from paged_kv_cache_467_b200 import ops

    k, v = new_rows(w, st.query.device)
    out = torch.full((w.num_seqs, w.n_q, w.head_dim), float("nan"), dtype=_TORCH_ACT[w.act_dtype], device=st.query.device)
    lse = torch.full((w.num_seqs, w.n_q), float("nan"), dtype=torch.float32, device=st.query.device)
    ops.paged_decode_step(out, st.query, k, v, st.key_cache, st.value_cache, st.block_tables, st.context_lens,
                          w.max_context_len, w.sm_scale, st.k_scale, st.v_scale, lse, workspace, st.device_error,
                          cache_dtype=named(w))
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)
