"""Benchmark of one paged decode step: cache append + decode attention.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference] [--config NAME]

A step appends one token per sequence and runs decode attention over every
sequence's paged cache, for one layer of the workload: one fused launch
(pkv_paged_decode_step), or with --unfused the two calls pkv_kv_cache_write and
pkv_paged_attention_decode.  Default workload: the largest single-GPU
configuration, the long-context 70B-shaped decode step (batch 8, 64 query / 8
KV heads, head_dim 128, BF16 cache, block 16, context lengths uniform in
[32768, 131072], shuffled pool sized to fit exactly: about 2.7 GB of K/V read
per step).  ``--config`` selects the others.

Under torchrun every rank runs its own replica of the workload (sequences are
independent: weak scaling, no collective on the data path); rank 0 prints one
JSON line.  ``--impl reference`` times the CPU float64 oracle instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attention KV GB/s (% of HBM peak) and decode tokens/s per step"
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--config", default="long_70b")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--unfused", action="store_true", help="append in its own launch before the decode")
    ap.add_argument("--no-overlap", action="store_true", help="launch each step without overlapping its prologue")
    ap.add_argument("--op", default="decode_step", choices=["decode_step", "copy_blocks", "swap_blocks", "quest"],
                    help="what a step runs (the default is the decode step)")
    ap.add_argument("--prefix-splits", type=int, default=0,
                    help="shared-prefix config: splits of the prefix pass along the prefix (0 = automatic)")
    ap.add_argument("--prefix-serial", action="store_true",
                    help="shared-prefix config: run the decode of each sequence's own blocks after the prefix pass "
                         "instead of beside it")
    ap.add_argument("--plain-decode", action="store_true",
                    help="shared-prefix configuration: run the plain decode step, every sequence reading the "
                         "shared blocks itself (through L2), instead of the shared-prefix pass")
    ap.add_argument("--seqs", type=int, default=0,
                    help="run the configuration's first N sequences only (a smaller case for profiling)")
    ap.add_argument("--quest-budget", type=int, default=4096,
                    help="--op quest: tokens each KV head reads (a multiple of the 16-token page)")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def strip_c_comments(text: str) -> str:
    """C/C++ source without comments, trailing blanks and blank lines (string
    and character literals kept as they are)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i : j + 1])
            i = j + 1
        elif text.startswith("//", i):
            while i < n and text[i] != "\n":
                i += 1
        elif text.startswith("/*", i):
            end = text.find("*/", i + 2)
            i = n if end < 0 else end + 2
        else:
            out.append(c)
            i += 1
    lines = (line.rstrip() for line in "".join(out).splitlines())
    return "\n".join(line for line in lines if line)


# Sources each kernel family is built from: a profile of a kernel stays valid
# while these files keep their code (comments aside).
KERNEL_SOURCES = {
    "decode": ("decode_tc.cu", "pkv_device.cuh", "cache_row.cuh", "internal.h"),
    "prefix": ("prefix.cu", "tcgen05.cuh", "pkv_device.cuh", "internal.h"),
    "kivi": ("kivi.cu", "decode_tc.cu", "pkv_device.cuh", "cache_row.cuh", "internal.h"),
    # the shared-prefix step: the prefix pass and the decode of each sequence's own blocks
    "prefix_step": ("decode_tc.cu", "prefix.cu", "tcgen05.cuh", "pkv_device.cuh", "cache_row.cuh", "internal.h"),
}


def kernel_source_hash(files=None) -> str:
    """Hash of the library's sources (all of them, or the named files of csrc/)
    with comments removed: a profile taken on these sources stays valid across
    comment edits, not across code edits."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_467_b200", "csrc")
    for name in sorted(files if files is not None else os.listdir(csrc)):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + strip_c_comments(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(config: str, family: str = "decode"):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, or None when the summary is missing or was taken on different
    sources of that kernel."""
    path = os.path.join(ROOT, "profiles", f"decode_{config}_ncu.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_hash = re.search(r"kernel_source_hash:\s*([0-9a-f]+)", text)
    m_bytes = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m_hash or not m_bytes or m_hash.group(1) != kernel_source_hash(KERNEL_SOURCES[family]):
        return None
    return float(m_bytes.group(1))


class ClockSampler:
    """nvidia-smi clock / throttle samples taken while the timed loop runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {
            "sm_mhz": statistics.median(sm) if sm else None,
            "sm_max_mhz": max(smax) if smax else None,
            "reasons": sorted(reasons),
            "samples": len(sm),
        }


# ----------------------------------------------------------------- oracle
def oracle_step_sample(w, seqs, host_rows):
    """One oracle step (append + decode) over the sampled sequences; returns KV bytes read."""
    import numpy as np

    import oracle

    from paged_kv_cache_467_b200 import accounting

    if w.cache_dtype == "kivi2":
        return oracle_kivi_step_sample(w, seqs, host_rows)
    per_token = accounting.cache_bytes(1, w.n_kv, w.head_dim, 1, accounting.BYTES_PER_VALUE[w.cache_dtype])
    per_token += accounting.scale_bytes_per_token(w.cache_dtype, w.n_kv)
    kv_bytes = 0
    for s in seqs:
        kc, vc, ks, vs, K, V, q = host_rows[s]
        L = int(w.context_lens[s])
        oracle.kv_cache_write(K[L - 1 : L], V[L - 1 : L], kc, vc, np.array([L - 1], dtype=np.int64), w.cache_dtype,
                              ks, vs)
        nb = kc.shape[0]
        oracle.paged_attention_decode(q, kc, vc, np.arange(nb, dtype=np.int32)[None], np.array([L]), w.sm_scale,
                                      w.cache_dtype, ks, vs, window=w.window, sinks=w.sinks)
        att = min(L, w.window + w.sinks) if w.window else L
        kv_bytes += int(att * per_token)
    return kv_bytes


def oracle_kivi_step_sample(w, seqs, host_rows):
    """One oracle KIVI step per sampled sequence: the new row joins the BF16
    residual, a residual that became a full block is quantised, then the decode."""
    import numpy as np

    import oracle

    from paged_kv_cache_467_b200 import accounting

    kv_bytes = 0
    per_block = accounting.kivi_block_bytes(w.n_kv, w.head_dim, w.block_size)
    for s in seqs:
        blocks, rk, rv, K, V, q = host_rows[s]
        L = int(w.context_lens[s])
        rk = np.concatenate([rk, K[L - 1 : L]])
        rv = np.concatenate([rv, V[L - 1 : L]])
        if rk.shape[0] == w.block_size:
            blocks = blocks + [oracle.kivi_quantize_block(rk, rv)]
            rk, rv = rk[:0], rv[:0]
        oracle.kivi_decode(q, blocks, rk, rv, w.sm_scale)
        kv_bytes += len(blocks) * per_block + rk.shape[0] * w.n_kv * w.head_dim * 2 * 2
    return kv_bytes


def prepare_oracle_rows(w, seqs, scales=None):
    import numpy as np

    import oracle

    rows = {}
    q = w.query()
    if w.cache_dtype == "kivi2":
        for s in seqs:
            L = int(w.context_lens[s])
            K, V = w.sequence_kv(s)
            blocks, rk, rv = oracle.kivi_cache_state(K[: L - 1], V[: L - 1])
            rows[s] = (blocks, rk, rv, K, V, q[s])
        return rows
    for s in seqs:
        L = int(w.context_lens[s])
        nb = -(-L // w.block_size)
        K, V = w.sequence_kv(s)
        width = w.head_dim // 2 if w.cache_dtype == "int4" else w.head_dim
        kc = np.zeros((nb, w.block_size, w.n_kv, width),
                      {"int8": np.int8, "int4": np.uint8}.get(w.cache_dtype, np.uint8 if "fp8" in w.cache_dtype
                                                              else np.float64))
        vc = np.zeros_like(kc)
        ks = vs = None
        if w.cache_dtype in ("int8", "int4"):
            ks = np.zeros((nb, w.block_size, w.n_kv), np.float32)
            vs = np.zeros_like(ks)
        elif w.cache_dtype.startswith("fp8"):
            ks, vs = scales
        oracle.kv_cache_write(K[: L - 1], V[: L - 1], kc, vc, np.arange(L - 1, dtype=np.int64), w.cache_dtype, ks, vs)
        rows[s] = (kc, vc, ks, vs, K, V, q[s : s + 1])
    return rows


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:  # noqa: BLE001
        return 1


def time_oracle(w, budget_s: float, max_seqs: int | None = None):
    """Time oracle steps on a bounded sample of the workload's sequences.

    Sequences are prepared one at a time (their host caches are dropped after
    use, so host memory stays bounded).  Without ``max_seqs`` each sequence is
    stepped once until ``budget_s`` of timed work; with it, at most
    ``max_seqs`` sequences are prepared and each is stepped repeatedly for its
    share of the budget.  Returns (KV bytes, seconds, sequences, steps)."""
    seqs, t_total, b_total, steps = [], 0.0, 0, 0
    scales = w.fp8_head_scales() if w.cache_dtype.startswith("fp8") else None
    for s in range(w.num_seqs):
        if max_seqs is not None and len(seqs) >= max_seqs:
            break
        host = prepare_oracle_rows(w, [s], scales)
        seqs.append(s)
        share = budget_s / max_seqs if max_seqs else 0.0
        t_seq = 0.0
        while True:
            t0 = time.perf_counter()
            b = oracle_step_sample(w, [s], host)
            dt = time.perf_counter() - t0
            t_seq += dt
            b_total += b
            steps += 1
            if t_seq >= share:
                break
        t_total += t_seq
        del host
        if max_seqs is None and t_total >= budget_s:
            break
    return b_total, t_total, seqs, steps


def run_reference(args, rank, world):
    from paged_kv_cache_467_b200 import workloads

    if rank != 0:
        return
    w = workloads.CONFIGS[args.config]()
    # every step: the oracle over a bounded sample of the workload (its first sequence)
    per_step = 1
    host = prepare_oracle_rows(w, list(range(per_step)))
    for _ in range(args.warmup):
        oracle_step_sample(w, range(per_step), host)
    t0 = time.perf_counter()
    b = 0
    for _ in range(args.steps):
        b += oracle_step_sample(w, range(per_step), host)
    dt = time.perf_counter() - t0
    gbs = b / dt / 1e9
    cores = blas_threads()
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": gbs,
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": config_block(w, world),
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"{per_step} of {w.num_seqs} sequences per step (append + float64 decode)"},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def replica_workload(base, rank):
    """Rank r's replica: the same shape with its own seed (sequences are independent)."""
    from paged_kv_cache_467_b200 import workloads

    if rank == 0:
        return base
    return workloads.make_workload(
        base.name, seed=base.seed + 1000 * rank, context_lens=base.context_lens, n_q=base.n_q, n_kv=base.n_kv,
        head_dim=base.head_dim, cache_dtype=base.cache_dtype, shared_prefix_tokens=base.shared_prefix_tokens,
        outlier_fraction=0.01 if base.k_outlier_channels is not None else 0.0, window=base.window, sinks=base.sinks)


def max_over_ranks(values, world, device=None):
    """Element-wise max of a list of floats over all ranks (identity at world 1)."""
    if world == 1:
        return list(values)
    import torch
    import torch.distributed as dist

    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def whole_job_gbs(bytes_per_rank, world, ms):
    """Bytes all ranks processed divided by the slowest rank's time, in GB/s."""
    return bytes_per_rank * world / (ms * 1e-3) / 1e9


def config_block(w, world):
    from paged_kv_cache_467_b200 import accounting

    kv = accounting.decode_kv_bytes(w)
    return {
        "workload": w.name,
        "batch": w.num_seqs,
        "n_q": w.n_q,
        "n_kv": w.n_kv,
        "head_dim": w.head_dim,
        "block_size": w.block_size,
        "cache_dtype": w.cache_dtype,
        "context_tokens": int(w.context_lens.astype("int64").sum()),
        "kv_bytes_per_step_per_gpu": kv,
        "l2": f"inputs larger than L2 ({kv / 2**20:.0f} MiB of KV per step vs 126 MiB L2)" if kv > L2_BYTES
        else "L2 flushed between steps",
        "parallelism": f"replicas x{world} (independent sequences per GPU)",
    }


# ----------------------------------------------------------------- GPU arm
def run_b200(args, rank, world, local):
    import numpy as np
    import torch
    import torch.distributed as dist

    from paged_kv_cache_467_b200 import accounting, ops, workloads

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=__import__("datetime").timedelta(seconds=120))

    base = workloads.CONFIGS[args.config]()
    if args.seqs:
        base = workloads.first_sequences(base, args.seqs)
    w = replica_workload(base, rank)
    S, nq, nkv, d, bs = w.num_seqs, w.n_q, w.n_kv, w.head_dim, w.block_size
    named = "int4" if w.cache_dtype == "int4" else None  # an int4 pool's torch dtype (uint8) does not name it
    gen = torch.Generator(device=dev).manual_seed(1234 + rank)
    shape = (w.num_blocks, bs, nkv, d)
    # q/K/V ~ N(0,1) synthetic cache, filled on the device (the writer is exercised by the step's append)
    act = torch.float32 if w.act_dtype == "f32" else torch.bfloat16
    kivi = w.cache_dtype == "kivi2"
    if kivi:
        if args.unfused:
            raise SystemExit("the 2-bit KIVI cache appends inside its residual pass: no unfused step")
        # every pool block quantised from N(0,1) rows by the library's block quantiser,
        # and N(0,1) residual rows (the partial last block of each sequence)
        kc = torch.empty((w.num_blocks, nkv, bs, d // 4), device=dev, dtype=torch.uint8)
        vc = torch.empty_like(kc)
        ks = torch.empty((w.num_blocks, nkv, d), device=dev)
        vs = torch.empty((w.num_blocks, nkv, bs), device=dev)
        for b0 in range(0, w.num_blocks, 4096):
            nblk = min(4096, w.num_blocks - b0)
            kk = torch.randn((nblk, bs, nkv, d), device=dev, generator=gen).to(torch.bfloat16)
            vv = torch.randn((nblk, bs, nkv, d), device=dev, generator=gen).to(torch.bfloat16)
            dst = torch.arange(b0, b0 + nblk, device=dev, dtype=torch.int32)
            ops.kivi_quantize_blocks(kk, vv, dst, kc, vc, ks, vs)
        res_k = torch.randn((S, bs, nkv, d), device=dev, generator=gen).to(torch.bfloat16)
        res_v = torch.randn((S, bs, nkv, d), device=dev, generator=gen).to(torch.bfloat16)
    elif w.cache_dtype in ("bf16", "f32"):
        kc = torch.randn(shape, device=dev, generator=gen).to(act)
        vc = torch.randn(shape, device=dev, generator=gen).to(act)
        ks = vs = None
    else:
        pool_dtype = {"int8": torch.int8, "fp8_e4m3": torch.uint8, "fp8_e5m2": torch.float8_e5m2,
                      "int4": torch.uint8}[w.cache_dtype]
        pool_shape = shape[:3] + (d // 2,) if w.cache_dtype == "int4" else shape
        kc = torch.empty(pool_shape, device=dev, dtype=pool_dtype)
        vc = torch.empty_like(kc)
        if w.cache_dtype in ("int8", "int4"):
            ks = torch.empty(shape[:3], device=dev)
            vs = torch.empty(shape[:3], device=dev)
        else:
            top = 448.0 if w.cache_dtype == "fp8_e4m3" else 57344.0
            ks = torch.full((nkv,), 5.0 / top, device=dev)
            vs = torch.full((nkv,), 5.0 / top, device=dev)
        slots_all = torch.arange(w.num_blocks * bs, device=dev, dtype=torch.int64)
        for c0 in range(0, slots_all.numel(), 1 << 20):
            sl = slots_all[c0 : c0 + (1 << 20)]
            kk = torch.randn((sl.numel(), nkv, d), device=dev, generator=gen).to(torch.bfloat16)
            vv = torch.randn((sl.numel(), nkv, d), device=dev, generator=gen).to(torch.bfloat16)
            ops.kv_cache_write(kk, vv, kc, vc, sl, ks, vs, cache_dtype=named)
    q = torch.randn((S, nq, d), device=dev, generator=gen).to(act)
    k_new = torch.randn((S, nkv, d), device=dev, generator=gen).to(act)
    v_new = torch.randn((S, nkv, d), device=dev, generator=gen).to(act)
    slots = torch.from_numpy(w.new_token_slots()).to(dev)
    bt = torch.from_numpy(w.block_tables).to(dev)
    cl = torch.from_numpy(w.context_lens).to(dev)
    out = torch.empty_like(q)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    # Block tables and lengths are set up before the loop and never written by
    # the kernel launched right before a step, so each step may overlap its
    # prologue with the previous step's tail (programmatic dependent launch).
    tuning = None if args.no_overlap else ops.DecodeTuning(0, 0, 0, ops.TUNE_OVERLAP_PROLOGUE)
    if kivi:
        nws = ops.kivi_workspace_size(S, nq, nkv, d, bs)
    else:
        nws = ops.paged_attention_workspace_size(S, nq, nkv, d, bs, ops.cache_code(kc, named))
    ws = torch.zeros(max(nws, 256), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    kv_bytes = accounting.decode_kv_bytes(w)


    prefix_blocks = 0 if args.plain_decode else w.shared_prefix_tokens // bs
    prefix_tuning = None
    if prefix_blocks:
        # the shared prefix is attended once for all sequences, beside the decode of each sequence's own blocks
        if args.prefix_splits or args.prefix_serial:
            prefix_tuning = ops.DecodeTuning(0, 0, 0, ops.TUNE_PREFIX_SERIAL if args.prefix_serial else 0,
                                             args.prefix_splits)
        nws = max(nws, ops.shared_prefix_workspace_size(S, nq, nkv, d, bs, prefix_blocks, prefix_tuning))
        ws = torch.zeros(max(nws, 256), dtype=torch.uint8, device=dev)

    def fused(out, q, k_new, v_new, bt, cl, tun):
        if kivi:
            ops.kivi_decode(out, q, res_k, res_v, kc, vc, ks, vs, bt, cl, w.max_context_len, key=k_new, value=v_new,
                            sm_scale=w.sm_scale, workspace=ws, device_error=err)
        elif w.window:
            ops.paged_decode_step_window(out, q, k_new, v_new, kc, vc, bt, cl, w.max_context_len, w.window, w.sinks,
                                         w.sm_scale, ks, vs, workspace=ws, device_error=err, cache_dtype=named)
        elif prefix_blocks:
            ops.paged_attention_decode_shared_prefix(out, q, kc, vc, bt, cl, w.max_context_len, prefix_blocks,
                                                     key=k_new, value=v_new, sm_scale=w.sm_scale, workspace=ws,
                                                     device_error=err, tuning=prefix_tuning)
        else:
            ops.paged_decode_step(out, q, k_new, v_new, kc, vc, bt, cl, w.max_context_len, w.sm_scale, ks, vs,
                                  workspace=ws, device_error=err, tuning=tun, cache_dtype=named)

    def decode(out, q, bt, cl):
        if prefix_blocks:
            ops.paged_attention_decode_shared_prefix(out, q, kc, vc, bt, cl, w.max_context_len, prefix_blocks,
                                                     sm_scale=w.sm_scale, workspace=ws, device_error=err,
                                                     tuning=prefix_tuning)
        elif w.window:
            ops.paged_attention_decode_window(out, q, kc, vc, bt, cl, w.max_context_len, w.window, w.sinks,
                                              w.sm_scale, ks, vs, workspace=ws, device_error=err, cache_dtype=named)
        else:
            ops.paged_attention_decode(out, q, kc, vc, bt, cl, w.max_context_len, w.sm_scale, ks, vs, workspace=ws,
                                       device_error=err, cache_dtype=named)

    def step(q=q, k_new=k_new, v_new=v_new, bt=bt, cl=cl, slots=slots, overlap=True):
        if args.unfused:
            ops.kv_cache_write(k_new, v_new, kc, vc, slots, ks, vs, err, cache_dtype=named)
            decode(out, q, bt, cl)
        else:
            fused(out, q, k_new, v_new, bt, cl, tuning if overlap else None)

    def barrier():
        if world > 1:
            dist.barrier()

    # ---------------- device-resident timing
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0")
    sampler.start()
    t_spin = time.perf_counter()
    while time.perf_counter() - t_spin < 0.4:  # keep the GPU busy while the sampler starts
        step()
        torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ev_start, ev_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # Two-launch step: events around each decode launch give the decode
    # kernel's own time.  One-launch step: the kernel is the whole step, and
    # nothing is recorded between launches (an event between two kernels would
    # keep a step's prologue from overlapping the previous step), so its
    # per-launch time is the timed region / K, gaps included.
    att = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps if args.unfused else 0)]
    ev_start.record(stream)
    for k in range(args.steps):
        if args.unfused:
            ops.kv_cache_write(k_new, v_new, kc, vc, slots, ks, vs, err, cache_dtype=named)
            att[k][0].record(stream)
            decode(out, q, bt, cl)
            att[k][1].record(stream)
        else:
            fused(out, q, k_new, v_new, bt, cl, tuning)
    ev_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    ms = ev_start.elapsed_time(ev_end) / args.steps
    att_ms = sum(a.elapsed_time(b) for a, b in att) / args.steps if args.unfused else ms
    ms, att_ms = max_over_ranks([ms, att_ms], world, dev)
    assert int(err.item()) == 0, f"device error flag {int(err.item())}"

    # ---------------- end to end through the public API with host buffers
    # The step's inputs (query, new K/V rows, block tables, lengths, slots) live
    # in one pinned host buffer and cross to the device in one copy per step;
    # the output comes back in one copy, and the host waits for it.
    parts = [q, k_new, v_new, bt, cl] + ([] if kivi else [slots])
    offs, total = [], 0
    for t in parts:
        offs.append(total)
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    h_in = torch.empty(total, dtype=torch.uint8).pin_memory()
    d_in = torch.empty(total, dtype=torch.uint8, device=dev)
    views = []
    for t, o in zip(parts, offs):
        nbytes = t.numel() * t.element_size()
        h_in[o : o + nbytes].copy_(t.contiguous().view(torch.uint8).reshape(-1).cpu())
        views.append(d_in[o : o + nbytes].view(t.dtype).view(t.shape))
    d_q, d_k, d_v, d_bt, d_cl = views[:5]
    d_slots = None if kivi else views[5]
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = total
    d2h = h_out.numel() * h_out.element_size()
    e2e_steps = min(args.steps, 500)

    def e2e_step():
        d_in.copy_(h_in, non_blocking=True)
        # lengths and tables arrive with this copy, so no prologue overlap here
        step(q=d_q, k_new=d_k, v_new=d_v, bt=d_bt, cl=d_cl, slots=d_slots, overlap=False)
        h_out.copy_(out, non_blocking=True)
        stream.synchronize()  # the host reads the step's result

    for _ in range(3):
        e2e_step()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks([e0.elapsed_time(e1) / e2e_steps], world, dev)[0]

    if rank == 0:
        peak, peak_kind = measured_peaks()
        value = whole_job_gbs(kv_bytes, world, ms)
        achieved = kv_bytes / (att_ms * 1e-3) / 1e9
        traffic = None
        if not args.seqs and not args.plain_decode and not args.unfused:
            traffic = profiled_traffic(args.config, "kivi" if kivi else "prefix_step" if prefix_blocks else "decode")
        line = {
            "metric": METRIC,
            "value": value,
            "unit": "GB/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": w.cache_dtype,
            "data": "synthetic",
            "config": config_block(w, world),
            "tokens_per_s": S * world / (ms * 1e-3),
            "pct_of_hbm_peak": 100.0 * value / world / peak,
            "roofline": {
                "bound": "hbm",
                "achieved": achieved,
                "peak": peak,
                "unit": "GB/s",
                "frac": achieved / peak,
                "traffic": traffic,
                "kernel": "kivi_residual_kernel + decode_tc_kernel<KIVI> + decode_merge_kernel (pkv_kivi_decode)"
                if kivi else ("prefix_tc_kernel (tcgen05) + " if prefix_blocks else "")
                + ("decode_f32_kernel" if w.cache_dtype == "f32" else "decode_tc_kernel")
                + ("" if args.unfused else " with fused append")
                + ("" if w.cache_dtype == "f32" else " + decode_merge_kernel")
                + (" (pkv_paged_attention_decode_shared_prefix)" if prefix_blocks
                   else " (pkv_paged_decode_step_window)" if w.window and not args.unfused
                   else " (pkv_paged_attention_decode)" if args.unfused else " (pkv_paged_decode_step)"),
                "peak_source": f"{peak_kind} hbm_gbs",
                "bytes_per_launch": kv_bytes,
                "launch_ms": att_ms,
            },
            "e2e": {"value": whole_job_gbs(kv_bytes, world, e2e_ms), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": e2e_steps},
            # decode kernel + merge of split sequences (+ the prefix pass, + the cache write when unfused)
            "gpu_launches": ((1 if w.cache_dtype == "f32" else 2) + (1 if prefix_blocks or kivi else 0)
                             + (1 if args.unfused else 0)) * args.steps,
            "step": ("residual pass (append, quantise a completed block, attend the BF16 residual rows), then "
                     "decode over the 2-bit blocks + merge of split sequences" if kivi
                     else "append, then decode + merge of split sequences" if args.unfused
                     else "append fused into the decode kernel, then the merge of split sequences")
            + ("" if args.no_overlap or args.unfused or w.window or prefix_blocks
               else "; prologue overlaps the previous step (programmatic launch)"),
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu_baseline:
            # the KIVI oracle quantises a sequence's blocks group by group before its timed
            # step, and a long-context sequence takes seconds to prepare (both untimed): a few
            # sequences, each stepped repeatedly, bound those runs
            long_ctx = int(w.context_lens.max()) > 16384
            b, t, seqs, nsteps = time_oracle(w, budget_s=12.0, max_seqs=3 if kivi else 2 if long_ctx else None)
            line["cpu_baseline"] = {
                "value": b / t / 1e9,
                "unit": "GB/s",
                "cores": blas_threads(),
                "kind": "oracle",
                "sample": f"{len(seqs)} of {w.num_seqs} sequences, {nsteps} oracle steps (append + float64 "
                          f"decode), {t:.1f} s",
            }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_block_ops(args):
    """--op copy_blocks / swap_blocks: throughput of the block movers on the
    default workload's pool (bf16, 8 KV heads, head_dim 128, 64 KiB of K+V per
    block).  A step moves 1024 random blocks: inside the pool (copy-on-write
    copies), or to page-locked host memory and back (offload, restore)."""
    import numpy as np
    import torch

    from paged_kv_cache_467_b200 import ops, workloads

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = workloads.CONFIGS[args.config]()
    shape = (w.num_blocks, w.block_size, w.n_kv, w.head_dim)
    gen = torch.Generator(device=dev).manual_seed(7)
    kc = torch.randn(shape, device=dev, generator=gen).to(torch.bfloat16)
    vc = torch.randn(shape, device=dev, generator=gen).to(torch.bfloat16)
    n = 1024
    perm = np.random.default_rng(3).permutation(w.num_blocks)
    block_bytes = 2 * kc[0].numel() * kc.element_size()
    stream = torch.cuda.current_stream(dev)
    if args.op == "copy_blocks":
        pairs = torch.from_numpy(np.stack([perm[:n], perm[n : 2 * n]], 1).astype(np.int64)).to(dev)
        steps = [lambda: ops.copy_blocks(kc, vc, pairs)]
        moved = 2 * n * block_bytes  # read + write, like the copy peak
        peak, peak_src, bound, what = measured_peaks()[0], "measured hbm_gbs (copy: read + write)", "hbm", "copy"
    else:
        hk = torch.empty((n,) + shape[1:], dtype=torch.bfloat16).pin_memory()
        hv = torch.empty_like(hk).pin_memory()
        out_pairs = torch.from_numpy(np.stack([perm[:n], np.arange(n)], 1).astype(np.int64)).to(dev)
        in_pairs = torch.from_numpy(np.stack([np.arange(n), perm[n : 2 * n]], 1).astype(np.int64)).to(dev)
        steps = [lambda: ops.swap_blocks(kc, vc, hk, hv, out_pairs),
                 lambda: ops.swap_blocks(hk, hv, kc, vc, in_pairs, device=dev)]
        moved = 2 * n * block_bytes  # n blocks out + n blocks back in
        peak, peak_src, bound, what = 64.0, "nominal PCIe Gen5 x16, per direction (no measured host-link peak)", \
            "host link", "offload + restore"
    for _ in range(max(args.warmup, 3)):
        for f in steps:
            f()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        for f in steps:
            f()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    gbs = moved / (ms * 1e-3) / 1e9
    print(json.dumps({
        "metric": f"paged block {what} GB/s", "value": gbs, "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "blocks_per_step": n, "bytes_per_block_kv": block_bytes,
                   "bytes_moved_per_step": moved},
        "roofline": {"bound": bound, "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                     "traffic": None, "peak_source": peak_src},
        "gpu_launches": len(steps) * args.steps,
    }), flush=True)


def run_quest(args):
    """--op quest: one decode step with query-aware page selection.  A step
    appends the new token, refreshes the summary of each sequence's last page,
    scores every page and keeps each KV head's best budget / 16 pages, then
    attends over those pages only.  The full fused decode step on the same
    cache is timed beside it."""
    import numpy as np
    import torch

    from paged_kv_cache_467_b200 import ops, workloads

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = workloads.CONFIGS[args.config]()
    if w.cache_dtype != "bf16" or w.window:
        raise SystemExit("--op quest runs on a bf16 cache without a window")
    S, nq, nkv, d, bs = w.num_seqs, w.n_q, w.n_kv, w.head_dim, w.block_size
    gen = torch.Generator(device=dev).manual_seed(99)
    shape = (w.num_blocks, bs, nkv, d)
    kc = torch.randn(shape, device=dev, generator=gen).to(torch.bfloat16)
    vc = torch.randn(shape, device=dev, generator=gen).to(torch.bfloat16)
    q = torch.randn((S, nq, d), device=dev, generator=gen).to(torch.bfloat16)
    k_new = torch.randn((S, nkv, d), device=dev, generator=gen).to(torch.bfloat16)
    v_new = torch.randn((S, nkv, d), device=dev, generator=gen).to(torch.bfloat16)
    slots = torch.from_numpy(w.new_token_slots()).to(dev)
    bt = torch.from_numpy(w.block_tables).to(dev)
    cl = torch.from_numpy(w.context_lens).to(dev)
    out = torch.empty_like(q)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    k_pages = max(1, args.quest_budget // bs)
    pmin = torch.empty((w.num_blocks, nkv, d), dtype=torch.bfloat16, device=dev)
    pmax = torch.empty_like(pmin)
    sel = torch.empty((S, nkv, k_pages), dtype=torch.int32, device=dev)
    scores = torch.empty((S, nkv, -(-min(w.max_context_len, w.max_blocks_per_seq * bs) // bs)), device=dev)
    ops.quest_page_summaries(kc, pmin, pmax, bt, cl, err)
    nws = ops.paged_attention_workspace_size(S, nq, nkv, d, bs, ops.cache_code(kc))
    ws = torch.zeros(max(nws, 256), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]

    def quest_step(record=False):
        if record:
            ev[0].record(stream)
        ops.kv_cache_write(k_new, v_new, kc, vc, slots, None, None, err)
        ops.quest_page_summaries(kc, pmin, pmax, bt, cl, err, last_page_only=True)
        if record:
            ev[1].record(stream)
        ops.quest_select(q, pmin, pmax, bt, cl, w.max_context_len, k_pages, sel, scores, err)
        if record:
            ev[2].record(stream)
        ops.paged_attention_decode_pages(out, q, kc, vc, bt, cl, w.max_context_len, sel, w.sm_scale, workspace=ws,
                                         device_error=err)
        if record:
            ev[3].record(stream)

    def full_step():
        ops.paged_decode_step(out, q, k_new, v_new, kc, vc, bt, cl, w.max_context_len, w.sm_scale, workspace=ws,
                              device_error=err)

    for _ in range(max(args.warmup, 3)):
        quest_step()
        full_step()
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0")
    sampler.start()
    t_spin = time.perf_counter()
    while time.perf_counter() - t_spin < 0.4:
        quest_step()
        torch.cuda.synchronize()
    parts = np.zeros(3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.steps):
        quest_step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    n_split = min(args.steps, 200)
    for _ in range(n_split):  # per-launch split (events between launches)
        quest_step(record=True)
        torch.cuda.synchronize()
        parts += [ev[0].elapsed_time(ev[1]), ev[1].elapsed_time(ev[2]), ev[2].elapsed_time(ev[3])]
    parts /= n_split
    e0.record(stream)
    for _ in range(args.steps):
        full_step()
    e1.record(stream)
    torch.cuda.synchronize()
    full_ms = e0.elapsed_time(e1) / args.steps
    clocks = sampler.stop()
    assert int(err.item()) == 0, f"device error flag {int(err.item())}"

    # algorithmic bytes: every page summary of every KV head (min and max), the
    # K and V rows of the selected pages, the refreshed last pages
    lens = w.context_lens.astype(np.int64)
    pages = -(-lens // bs)
    summ_bytes = int(pages.sum()) * nkv * 2 * d * 2
    sel_h = sel.cpu().numpy()
    rows = 0
    for s_ in range(S):
        for kv in range(nkv):
            for j in sel_h[s_, kv]:
                if j >= 0:
                    rows += min(bs, int(lens[s_]) - int(j) * bs)
    kv_bytes = rows * d * 2 * 2
    refresh_bytes = S * (bs * nkv * d * 2 + 2 * nkv * d * 2)
    total = summ_bytes + kv_bytes + refresh_bytes
    full_bytes = int(lens.sum()) * nkv * d * 2 * 2
    peak, peak_kind = measured_peaks()
    print(json.dumps({
        "metric": "Quest decode step: tokens/s", "value": S / (ms * 1e-3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "dtype": "bf16",
        "data": "synthetic", "config": {"workload": w.name, "budget_tokens": k_pages * bs, "pages_per_head": k_pages,
                                        "context_tokens": int(lens.sum())},
        "full_decode_ms_per_step": full_ms, "speedup_vs_full_decode": full_ms / ms,
        "split_ms": {"append + last-page refresh": parts[0], "quest_select": parts[1], "decode_pages": parts[2]},
        "bytes_per_step": {"summaries": summ_bytes, "selected_kv": kv_bytes, "refresh": refresh_bytes,
                           "full_decode_kv": full_bytes},
        "roofline": {"bound": "hbm", "achieved": total / (ms * 1e-3) / 1e9, "peak": peak, "unit": "GB/s",
                     "frac": total / (ms * 1e-3) / 1e9 / peak, "traffic": None, "peak_source": f"{peak_kind} hbm_gbs",
                     "select_gbs": summ_bytes / (parts[1] * 1e-3) / 1e9,
                     "decode_pages_gbs": kv_bytes / (parts[2] * 1e-3) / 1e9},
        # append, last-page refresh, page scoring, top-k, decode over pages, merge
        "gpu_launches": 6 * args.steps, "clocks": clocks,
    }), flush=True)


def main():
    args = parse_args()
    rank, world, local = dist_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.op == "quest":
        run_quest(args)
        return
    if args.op != "decode_step":
        run_block_ops(args)
        return
    run_b200(args, rank, world, local)


if __name__ == "__main__":
    main()
