"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments on the host before touching a GPU (CPU only)."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_467_b200 import build

    build.build()
    from paged_kv_cache_467_b200 import ops

    return ops.lib


def declared_functions():
    text = open(os.path.join(ROOT, "include", "pkv.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pkv_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert "pkv_kv_cache_write" in names and "pkv_paged_attention_decode" in names
    raw = ctypes.CDLL(os.path.join(ROOT, "paged_kv_cache_467_b200", "libpkv.so"))
    for n in names:
        assert hasattr(raw, n), n


def test_status_strings_and_version(lib):
    assert lib.pkv_status_string(0) == b"ok"
    assert lib.pkv_status_string(3) == b"workspace missing or too small"
    assert lib.pkv_version() >= 100


FAKE = 0x10000  # an aligned, never dereferenced address: validation fails before any launch


def _write(lib, **kw):
    args = dict(key=FAKE, value=FAKE, key_cache=FAKE, value_cache=FAKE, k_scale=None, v_scale=None, slots=FAKE,
                T=4, n_kv=2, d=128, bs=16, nb=8, act=1, cache=1, err=None)
    args.update(kw)
    return lib.pkv_kv_cache_write(args["key"], args["value"], args["key_cache"], args["value_cache"], args["k_scale"],
                                  args["v_scale"], args["slots"], args["T"], args["n_kv"], args["d"], args["bs"],
                                  args["nb"], args["act"], args["cache"], args["err"], None)


def test_cache_write_host_validation(lib):
    assert _write(lib, T=0) == 0  # nothing to do
    assert _write(lib, key=None) == 1
    assert _write(lib, key=FAKE + 4) == 1  # misaligned
    assert _write(lib, d=96) == 2
    assert _write(lib, act=0, cache=1) == 2  # F32 rows into a BF16 cache
    assert _write(lib, act=2) == 1  # int8 rows are not an activation dtype
    assert _write(lib, cache=2) == 1  # INT8 cache needs scale arrays
    assert _write(lib, k_scale=FAKE, v_scale=FAKE) == 1  # BF16 cache takes no scales
    assert _write(lib, cache=7) == 1
    assert _write(lib, n_kv=0) == 1


def _decode(lib, **kw):
    a = dict(out=FAKE, q=FAKE, kc=FAKE, vc=FAKE, ks=None, vs=None, bt=FAKE, mb=8, cl=FAKE, mcl=100, S=2, nq=8, nkv=2,
             d=128, bs=16, nb=16, scale=0.1, act=1, cache=1, lse=None, ws=FAKE, wsb=1 << 20, err=None)
    a.update(kw)
    return lib.pkv_paged_attention_decode(a["out"], a["q"], a["kc"], a["vc"], a["ks"], a["vs"], a["bt"], a["mb"],
                                          a["cl"], a["mcl"], a["S"], a["nq"], a["nkv"], a["d"], a["bs"], a["nb"],
                                          a["scale"], a["act"], a["cache"], a["lse"], a["ws"], a["wsb"], a["err"], None)


def test_decode_host_validation(lib):
    assert _decode(lib, S=0) == 0
    assert _decode(lib, nq=6, nkv=4) == 1  # query heads not a multiple of KV heads
    assert _decode(lib, bs=32) == 2
    assert _decode(lib, d=96) == 2
    assert _decode(lib, nq=130, nkv=2) == 2  # group of 65
    assert _decode(lib, out=None) == 1
    assert _decode(lib, kc=FAKE + 8) == 1
    assert _decode(lib, ks=FAKE, vs=FAKE) == 1  # BF16 cache takes no scales
    assert _decode(lib, cache=2) == 1  # INT8 without scales
    assert _decode(lib, act=0, cache=1) == 2  # F32 query with a BF16 cache
    assert _decode(lib, act=1, cache=0, d=64) == 2  # BF16 query with an F32 cache
    assert _decode(lib, cache=2, ks=FAKE, vs=FAKE, d=64) == 2  # quantised caches need head_dim 128
    assert _decode(lib, nb=1 << 28) == 2  # pool rows beyond int32
    assert _decode(lib, mcl=-1) == 1
    assert _decode(lib, mb=0) == 1


def test_workspace_size_host_paths(lib):
    # an F32 cache needs no workspace and no device query
    assert lib.pkv_paged_attention_workspace_size(4, 8, 2, 64, 16, 0) == 0
    # unsupported shapes report (size_t)-1
    assert lib.pkv_paged_attention_workspace_size(4, 8, 2, 96, 16, 1) == ctypes.c_size_t(-1).value
    if not torch.cuda.is_available():
        # sizing the tensor-core path needs the device's SM count
        assert lib.pkv_paged_attention_workspace_size(4, 8, 2, 128, 16, 1) == ctypes.c_size_t(-1).value


def test_new_format_host_validation(lib):
    # INT4 / E5M2 caches: row-scaled and head-scaled scale arrays are required
    assert _write(lib, cache=5) == 1  # INT4 without scales
    assert _write(lib, cache=4) == 1  # E5M2 without scales
    assert _write(lib, cache=6) == 1  # no such dtype
    assert _decode(lib, cache=5, ks=FAKE, vs=FAKE, d=64) == 2  # quantised caches need head_dim 128
    assert _decode(lib, cache=4) == 1


def test_window_pages_and_prefix_host_validation(lib):
    a = dict(out=FAKE, q=FAKE, kc=FAKE, vc=FAKE, ks=None, vs=None, bt=FAKE, mb=8, cl=FAKE, mcl=100, S=2, nq=8, nkv=2,
             d=128, bs=16, nb=16, scale=0.1)
    common = [a[k] for k in ("out", "q", "kc", "vc", "ks", "vs", "bt", "mb", "cl", "mcl", "S", "nq", "nkv", "d", "bs",
                             "nb", "scale")]
    # window / sinks must be >= 0
    assert lib.pkv_paged_attention_decode_window(*common, -1, 0, 1, 1, None, FAKE, 1 << 20, None, None) == 1
    # a page list needs at least one entry per (sequence, KV head)
    assert lib.pkv_paged_attention_decode_pages(*common, FAKE, 0, 1, 1, None, FAKE, 1 << 20, None, None) == 1
    assert lib.pkv_paged_attention_decode_pages(*common, None, 4, 1, 1, None, FAKE, 1 << 20, None, None) == 1
    # shared prefix: at least one block, shorter than every context, BF16 only
    sp = lib.pkv_paged_attention_decode_shared_prefix

    def shared(prefix, mcl=100, cache=1, key=None, value=None):
        return sp(FAKE, FAKE, key, value, FAKE, FAKE, FAKE, 8, FAKE, mcl, 2, 8, 2, 128, 16, 16, 0.1, prefix, 1, cache,
                  None, FAKE, 1 << 20, None, None)

    assert shared(0) == 1
    assert shared(7, mcl=100) == 1  # 7 blocks = 112 tokens: no private token left
    assert shared(2, key=FAKE) == 1  # key without value
    assert shared(2, cache=2) == 1  # INT8 without scales is rejected first
    assert lib.pkv_shared_prefix_workspace_size(2, 8, 2, 128, 16, 0) == ctypes.c_size_t(-1).value


def test_quest_host_validation(lib):
    # summaries: BF16 / F32 caches, head_dim 64 or 128, block size 16
    summ = lib.pkv_quest_page_summaries
    assert summ(FAKE, FAKE, FAKE, FAKE, 8, FAKE, 2, 2, 96, 16, 16, 1, 0, None, None) == 2
    assert summ(FAKE, FAKE, FAKE, FAKE, 8, FAKE, 2, 2, 128, 16, 16, 2, 0, None, None) == 2
    assert summ(FAKE, FAKE, FAKE, FAKE, 8, FAKE, 0, 2, 128, 16, 16, 1, 0, None, None) == 0  # nothing to do
    sel = lib.pkv_quest_select
    # k_pages >= 1, the score buffer is required, query heads a multiple of KV heads
    assert sel(FAKE, FAKE, FAKE, FAKE, 8, FAKE, 100, 2, 8, 2, 128, 16, 16, 1, 1, 0, FAKE, FAKE, None, None) == 1
    assert sel(FAKE, FAKE, FAKE, FAKE, 8, FAKE, 100, 2, 8, 2, 128, 16, 16, 1, 1, 4, FAKE, None, None, None) == 1
    assert sel(FAKE, FAKE, FAKE, FAKE, 8, FAKE, 100, 2, 6, 4, 128, 16, 16, 1, 1, 4, FAKE, FAKE, None, None) == 1


def _kivi_decode(lib, **kw):
    a = dict(out=FAKE, q=FAKE, key=None, value=None, rk=FAKE, rv=FAKE, kc=FAKE, vc=FAKE, ks=FAKE, vs=FAKE, bt=FAKE,
             mb=8, cl=FAKE, mcl=100, S=2, nq=8, nkv=2, d=128, bs=16, nb=16, scale=0.1, act=1, lse=None, ws=FAKE,
             wsb=1 << 24, err=None)
    a.update(kw)
    return lib.pkv_kivi_decode(a["out"], a["q"], a["key"], a["value"], a["rk"], a["rv"], a["kc"], a["vc"], a["ks"],
                               a["vs"], a["bt"], a["mb"], a["cl"], a["mcl"], a["S"], a["nq"], a["nkv"], a["d"],
                               a["bs"], a["nb"], a["scale"], a["act"], a["lse"], a["ws"], a["wsb"], a["err"], None)


def test_kivi_host_validation(lib):
    none = ctypes.c_size_t(-1).value
    assert lib.pkv_kivi_workspace_size(0, 8, 2, 128, 16) == 0
    assert lib.pkv_kivi_workspace_size(2, 8, 2, 64, 16) == none  # head_dim 128 only
    assert lib.pkv_kivi_workspace_size(2, 6, 4, 128, 16) == none
    assert _kivi_decode(lib, S=0) == 0
    assert _kivi_decode(lib, key=FAKE) == 1  # key without value
    assert _kivi_decode(lib, key=FAKE, value=FAKE + 8) == 1  # misaligned
    assert _kivi_decode(lib, rk=None) == 1  # the residual is required
    assert _kivi_decode(lib, ks=FAKE + 4) == 1
    assert _kivi_decode(lib, d=64) == 2
    assert _kivi_decode(lib, act=0) == 2  # BF16 activations only
    assert _kivi_decode(lib, act=2) == 1
    assert _kivi_decode(lib, nq=6, nkv=4) == 1
    assert _kivi_decode(lib, bs=32) == 2
    assert _kivi_decode(lib, mb=0) == 1  # context but no table
    q = lib.pkv_kivi_quantize_blocks
    assert q(FAKE, FAKE, FAKE, 0, FAKE, FAKE, FAKE, FAKE, 2, 128, 16, 8, 1, None, None) == 0
    assert q(None, FAKE, FAKE, 3, FAKE, FAKE, FAKE, FAKE, 2, 128, 16, 8, 1, None, None) == 1
    assert q(FAKE, FAKE, FAKE, 3, FAKE, FAKE, None, FAKE, 2, 128, 16, 8, 1, None, None) == 1
    assert q(FAKE + 2, FAKE, FAKE, 3, FAKE, FAKE, FAKE, FAKE, 2, 128, 16, 8, 1, None, None) == 1
    assert q(FAKE, FAKE, FAKE, 3, FAKE, FAKE, FAKE, FAKE, 2, 64, 16, 8, 1, None, None) == 2
    assert q(FAKE, FAKE, FAKE, 3, FAKE, FAKE, FAKE, FAKE, 2, 128, 16, 8, 0, None, None) == 2
    assert q(FAKE, FAKE, FAKE, -1, FAKE, FAKE, FAKE, FAKE, 2, 128, 16, 8, 1, None, None) == 1


def test_kivi_binding_rejects_token_major_pools(lib):
    """The binding checks the shapes the C ABI cannot see before any call."""
    from paged_kv_cache_467_b200 import ops

    S, nq, nkv, d, nb = 2, 8, 2, 128, 4
    q = torch.zeros((S, nq, d), dtype=torch.bfloat16)
    rk = torch.zeros((S, 16, nkv, d), dtype=torch.bfloat16)
    ks = torch.zeros((nb, nkv, d))
    vs = torch.zeros((nb, nkv, 16))
    bt = torch.zeros((S, 1), dtype=torch.int32)
    cl = torch.zeros(S, dtype=torch.int32)
    head_major = torch.zeros((nb, nkv, 16, d // 4), dtype=torch.uint8)
    token_major = torch.zeros((nb, 16, nkv, d // 4), dtype=torch.uint8)
    with pytest.raises(ValueError, match="key_cache"):
        ops.kivi_decode(torch.empty_like(q), q, rk, rk, token_major, token_major, ks, vs, bt, cl, 0)
    with pytest.raises(ValueError, match="residual_k"):
        ops.kivi_decode(torch.empty_like(q), q, rk.float(), rk, head_major, head_major, ks, vs, bt, cl, 0)
    with pytest.raises(ValueError, match="v_scale"):
        ops.kivi_decode(torch.empty_like(q), q, rk, rk, head_major, head_major, ks, vs.transpose(1, 2), bt, cl, 0)
