"""2-bit KIVI cache on the GPU against the oracle, through the C ABI.

Block quantisation is compared code for code and scale for scale (bit-exact);
the decode and the decode step are compared element by element with the
oracle's float64 attention over the same quantised blocks and residual rows.
Tolerances: outputs are BF16 (half an ulp is 2^-9 relative of values of order
1) and the kernel scores with f16 query-times-scale operands (about 2^-11
relative per term), so max abs 3e-2 / mean abs 3e-3 on the outputs and 5e-3
on the natural-log lse.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle.quant import pack_int2, unpack_int2
from paged_kv_cache_467_b200 import workloads

pytestmark = pytest.mark.gpu

D = 128
TOL_OUT = (3e-2, 3e-3)
TOL_LSE = 5e-3


def _ops():
    from paged_kv_cache_467_b200 import ops

    return ops


def _codes(block_bytes):
    """One device block [n_kv, 16, d/4] -> signed codes [16, n_kv, d] (the oracle's order)."""
    return unpack_int2(block_bytes).transpose(1, 0, 2)


def _bf16(x, dev="cuda"):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).to(dev)


def _wl(lens, n_q, n_kv, seed, extra_blocks=3):
    return workloads.make_workload("kivi_test", seed=seed, context_lens=lens, n_q=n_q, n_kv=n_kv, head_dim=D,
                                   cache_dtype="kivi2", extra_blocks=extra_blocks)


class Cache:
    """Device KIVI cache of workload w after n_rows[s] rows of each sequence.

    Pools start as random bytes and scales as random floats (unused blocks
    stay so), residual rows past a sequence's count hold NaN: reading either
    by mistake shows in the outputs."""

    def __init__(self, w, n_rows, source="oracle"):
        ops = _ops()
        S, nb, nkv = w.num_seqs, w.num_blocks, w.n_kv
        g = torch.Generator(device="cuda").manual_seed(7)
        self.kc = torch.randint(0, 256, (nb, nkv, 16, D // 4), device="cuda", dtype=torch.uint8, generator=g)
        self.vc = torch.randint(0, 256, (nb, nkv, 16, D // 4), device="cuda", dtype=torch.uint8, generator=g)
        self.ks = torch.rand((nb, nkv, D), device="cuda", generator=g) * 3
        self.vs = torch.rand((nb, nkv, 16), device="cuda", generator=g) * 3
        self.rk = torch.full((S, 16, nkv, D), float("nan"), device="cuda", dtype=torch.bfloat16)
        self.rv = torch.full((S, 16, nkv, D), float("nan"), device="cuda", dtype=torch.bfloat16)
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")
        for s in range(S):
            K, V = w.sequence_kv(s)
            n = max(int(n_rows[s]), 0)
            full = n // 16
            if full and source == "oracle":
                blocks, _, _ = oracle.kivi_cache_state(K[: 16 * full], V[: 16 * full])
                for b, (kcode, kscale, vcode, vscale) in enumerate(blocks):
                    phys = int(w.block_tables[s, b])
                    # device layout: head-major inside the block
                    self.kc[phys] = torch.from_numpy(pack_int2(kcode.transpose(1, 0, 2))).cuda()
                    self.vc[phys] = torch.from_numpy(pack_int2(vcode.transpose(1, 0, 2))).cuda()
                    self.ks[phys] = torch.from_numpy(kscale).cuda()
                    self.vs[phys] = torch.from_numpy(np.ascontiguousarray(vscale.T)).cuda()
            elif full:
                kr = _bf16(K[: 16 * full].reshape(full, 16, nkv, D))
                vr = _bf16(V[: 16 * full].reshape(full, 16, nkv, D))
                dst = torch.from_numpy(w.block_tables[s, :full].copy()).cuda()
                ops.kivi_quantize_blocks(kr, vr, dst, self.kc, self.vc, self.ks, self.vs, device_error=self.err)
            r = n - 16 * full
            if r:
                self.rk[s, :r] = _bf16(K[16 * full : n])
                self.rv[s, :r] = _bf16(V[16 * full : n])
        torch.cuda.synchronize()

    def run(self, w, key=None, value=None):
        ops = _ops()
        q = _bf16(w.query())
        out = torch.empty_like(q)
        lse = torch.empty(q.shape[:2], device="cuda")
        bt = torch.from_numpy(w.block_tables).cuda()
        cl = torch.from_numpy(w.context_lens).cuda()
        ops.kivi_decode(out, q, self.rk, self.rv, self.kc, self.vc, self.ks, self.vs, bt, cl, w.max_context_len,
                        key=key, value=value, sm_scale=w.sm_scale, lse_out=lse, device_error=self.err)
        torch.cuda.synchronize()
        assert int(self.err.item()) == 0
        return out.float().cpu().numpy(), lse.cpu().numpy()


def _check(w, out, lse, seqs=None):
    q = w.query()
    for s in range(w.num_seqs) if seqs is None else seqs:
        L = int(w.context_lens[s])
        K, V = w.sequence_kv(s)
        want, wl = oracle.kivi_decode_sequence(q[s], K[:L], V[:L], w.sm_scale)
        if L == 0:
            assert not out[s].any() and np.isneginf(lse[s]).all()
            continue
        assert np.isfinite(out[s]).all(), f"seq {s}: non-finite output"
        d = np.abs(out[s] - want)
        assert d.max() <= TOL_OUT[0] and d.mean() <= TOL_OUT[1], f"seq {s} (L={L}): max {d.max():.3e} mean {d.mean():.3e}"
        np.testing.assert_allclose(lse[s], wl, rtol=0, atol=TOL_LSE, err_msg=f"seq {s} lse")


def test_quantize_blocks_bit_exact():
    """Codes and scales of whole blocks equal the oracle's, with an all-zero
    channel, an all-zero token, exact ties at half the scale, and a skipped
    destination (-1) whose block stays untouched."""
    ops = _ops()
    rng = np.random.default_rng([11, 0])
    n, nkv, nb = 6, 2, 9
    K = workloads.round_to_bf16(rng.standard_normal((n, 16, nkv, D), dtype=np.float32) * 2)
    V = workloads.round_to_bf16(rng.standard_normal((n, 16, nkv, D), dtype=np.float32))
    K[1, :, 0, 5] = 0.0                                  # all-zero channel
    V[2, 3, 1, :] = 0.0                                  # all-zero token
    K[3, :, 1, 7] = 0.0
    K[3, :4, 1, 7] = [2.0, 1.0, -1.0, 0.5]               # ties at |x| / max = 1/2
    V[4, 0, 0, :8] = [4.0, 2.0, -2.0, 1.0, 0, 0, 0, 0]
    V[4, 0, 0, 8:] = 0.0
    dst = np.array([7, 0, 3, -1, 5, 8], np.int32)
    kc = torch.randint(0, 256, (nb, nkv, 16, D // 4), device="cuda", dtype=torch.uint8)
    vc = torch.randint(0, 256, (nb, nkv, 16, D // 4), device="cuda", dtype=torch.uint8)
    ks = torch.rand((nb, nkv, D), device="cuda")
    vs = torch.rand((nb, nkv, 16), device="cuda")
    before = [t.clone() for t in (kc, vc, ks, vs)]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.kivi_quantize_blocks(_bf16(K), _bf16(V), torch.from_numpy(dst).cuda(), kc, vc, ks, vs, device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    kc, vc, ks, vs = (t.cpu().numpy() for t in (kc, vc, ks, vs))
    for i, phys in enumerate(dst):
        if phys < 0:
            continue
        kcode, kscale, vcode, vscale = oracle.kivi_quantize_block(K[i], V[i])
        assert np.array_equal(_codes(kc[phys]), kcode), f"block {i}: K codes"
        assert np.array_equal(_codes(vc[phys]), vcode), f"block {i}: V codes"
        assert np.array_equal(ks[phys].view(np.int32), kscale.view(np.int32)), f"block {i}: K scales"
        assert np.array_equal(vs[phys].T.view(np.int32), vscale.view(np.int32)), f"block {i}: V scales"
    untouched = [b for b in range(nb) if b not in set(dst.tolist())]
    for t, b0 in zip((kc, vc, ks, vs), before):
        assert np.array_equal(t[untouched], b0.cpu().numpy()[untouched])


def test_quantize_blocks_flags_bad_destination():
    ops = _ops()
    rows = torch.zeros((2, 16, 1, D), device="cuda", dtype=torch.bfloat16)
    kc = torch.zeros((4, 1, 16, D // 4), device="cuda", dtype=torch.uint8)
    vc, ks, vs = torch.zeros_like(kc), torch.zeros((4, 1, D), device="cuda"), torch.zeros((4, 1, 16), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.kivi_quantize_blocks(rows, rows, torch.tensor([1, 4], dtype=torch.int32, device="cuda"), kc, vc, ks, vs,
                             device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == ops.DEVERR_BLOCK_RANGE


LENS = [0, 1, 15, 16, 17, 40, 64, 100, 333, 1000]


@pytest.mark.parametrize("n_q,n_kv", [(32, 8), (8, 8), (16, 2), (64, 4), (40, 5)])
def test_decode_parity(n_q, n_kv):
    """Plain decode (no new row) over oracle-quantised blocks and residual rows:
    empty, residual-only, block-aligned and ragged lengths, group sizes 1-16."""
    w = _wl(LENS, n_q, n_kv, seed=n_q + n_kv)
    c = Cache(w, w.context_lens)
    out, lse = c.run(w)
    _check(w, out, lse)


@pytest.mark.parametrize("n_q,n_kv", [(32, 8), (16, 2)])
def test_decode_step_parity(n_q, n_kv):
    """The step appends token L-1 first: steps that complete a block quantise it
    (codes bit-exact against the oracle), the others extend the residual."""
    lens = [1, 15, 16, 17, 32, 48, 100, 257, 2048]
    w = _wl(lens, n_q, n_kv, seed=3 + n_q)
    c = Cache(w, w.context_lens - 1)
    nk, nv = w.new_kv()
    out, lse = c.run(w, key=_bf16(nk), value=_bf16(nv))
    _check(w, out, lse)
    kc, vc, ks, vs = (t.cpu().numpy() for t in (c.kc, c.vc, c.ks, c.vs))
    rk = c.rk.float().cpu().numpy()
    for s, L in enumerate(lens):
        K, V = w.sequence_kv(s)
        if L % 16 == 0:  # this step completed block L/16 - 1
            phys = int(w.block_tables[s, L // 16 - 1])
            kcode, kscale, vcode, vscale = oracle.kivi_quantize_block(K[L - 16 : L], V[L - 16 : L])
            assert np.array_equal(_codes(kc[phys]), kcode) and np.array_equal(_codes(vc[phys]), vcode)
            assert np.array_equal(ks[phys], kscale) and np.array_equal(vs[phys].T, vscale)
        else:
            assert np.array_equal(rk[s, (L - 1) % 16], K[L - 1])


def test_decode_after_gpu_quantisation():
    """Blocks quantised by the library's own kernel give the oracle's result."""
    w = _wl([33, 160, 700], 32, 8, seed=21)
    c = Cache(w, w.context_lens, source="gpu")
    out, lse = c.run(w)
    _check(w, out, lse)


def test_full_size_step_sampled():
    """The timed configuration (256 sequences, L ~ U[1024, 8192], 32 q / 8 KV
    heads, 1% key outlier channels x10) in the bench's launch shape: one fused
    step, sampled sequences against the oracle."""
    w = workloads.CONFIGS["kivi2"]()
    c = Cache(w, w.context_lens - 1, source="gpu")
    nk, nv = w.new_kv()
    out, lse = c.run(w, key=_bf16(nk), value=_bf16(nv))
    lens = w.context_lens
    seqs = sorted({int(np.argmin(lens)), int(np.argmax(lens % 16 == 0)), 37})
    _check(w, out, lse, seqs=seqs)
    assert np.isfinite(out).all()


def test_copy_and_swap_blocks():
    """Block movers carry a KIVI block whole: codes, per-channel K scales and
    per-token V scales (copy-on-write in the pool, and offload to pinned host
    memory and back)."""
    ops = _ops()
    nb, nkv = 8, 2
    g = torch.Generator(device="cuda").manual_seed(3)
    kc = torch.randint(0, 256, (nb, nkv, 16, D // 4), device="cuda", dtype=torch.uint8, generator=g)
    vc = torch.randint(0, 256, (nb, nkv, 16, D // 4), device="cuda", dtype=torch.uint8, generator=g)
    ks = torch.rand((nb, nkv, D), device="cuda", generator=g)
    vs = torch.rand((nb, nkv, 16), device="cuda", generator=g)
    ref = [t.cpu().clone() for t in (kc, vc, ks, vs)]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.copy_blocks(kc, vc, torch.tensor([[1, 5], [2, 6]], dtype=torch.int64, device="cuda"), ks, vs,
                    device_error=err, cache_dtype="kivi2")
    for r in ref:
        r[5], r[6] = r[1].clone(), r[2].clone()
    host = [torch.zeros((3,) + tuple(t.shape[1:]), dtype=t.dtype).pin_memory() for t in (kc, vc, ks, vs)]
    ops.swap_blocks(kc, vc, host[0], host[1], torch.tensor([[0, 2], [7, 0]], dtype=torch.int64, device="cuda"),
                    ks, vs, host[2], host[3], device_error=err, cache_dtype="kivi2")
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for t, r, h in zip((kc, vc, ks, vs), ref, host):
        assert torch.equal(t.cpu(), r)
        assert torch.equal(h[2], r[0]) and torch.equal(h[0], r[7]) and not h[1].any()


def test_decode_error_paths():
    """A block-table entry outside the pool sets PKV_DEVERR_BLOCK_RANGE and a
    length past the table sets PKV_DEVERR_CONTEXT_LEN; the other sequences keep
    the oracle's result and nothing outside the buffers is touched."""
    ops = _ops()
    w = _wl([40, 64, 33], 8, 2, seed=31)
    c = Cache(w, w.context_lens)
    q = _bf16(w.query())
    bt = torch.from_numpy(w.block_tables.copy()).cuda()
    bt[1, 1] = w.num_blocks + 5  # sequence 1 reads a block outside the pool
    out = torch.empty_like(q)
    ops.kivi_decode(out, q, c.rk, c.rv, c.kc, c.vc, c.ks, c.vs, bt, torch.from_numpy(w.context_lens).cuda(),
                    w.max_context_len, sm_scale=w.sm_scale, device_error=c.err)
    torch.cuda.synchronize()
    assert int(c.err.item()) & ops.DEVERR_BLOCK_RANGE
    got = out.float().cpu().numpy()
    qh = w.query()
    for s in (0, 2):
        K, V = w.sequence_kv(s)
        L = int(w.context_lens[s])
        want, _ = oracle.kivi_decode_sequence(qh[s], K[:L], V[:L], w.sm_scale)
        assert np.abs(got[s] - want).max() <= TOL_OUT[0]
    c.err.zero_()
    cl = torch.from_numpy(w.context_lens.copy()).cuda()
    cl[0] = w.block_tables.shape[1] * 16 + 7  # longer than its table
    ops.kivi_decode(out, q, c.rk, c.rv, c.kc, c.vc, c.ks, c.vs, torch.from_numpy(w.block_tables).cuda(), cl,
                    int(cl.max().item()), sm_scale=w.sm_scale, device_error=c.err)
    torch.cuda.synchronize()
    assert int(c.err.item()) & ops.DEVERR_CONTEXT_LEN
