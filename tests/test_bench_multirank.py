"""Multi-rank host logic of bench.py on CPU: world size 2 over gloo."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    from paged_kv_cache_467_b200 import workloads

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, wsz, _ = bench.dist_env()
        base = workloads.make_workload("x", seed=3, context_lens=[40, 17, 64], n_q=8, n_kv=2, head_dim=64)
        w = bench.replica_workload(base, r)
        # the slowest rank decides: rank 1 reports the larger time
        mx = bench.max_over_ranks([1.0 + r, 5.0 - r], wsz)
        tables = torch.from_numpy(w.block_tables.astype(np.int64))
        gathered = [torch.zeros_like(tables) for _ in range(wsz)]
        dist.all_gather(gathered, tables)
        q0 = torch.from_numpy(w.query())
        qs = [torch.zeros_like(q0) for _ in range(wsz)]
        dist.all_gather(qs, q0)
        results[r] = {
            "rank": r,
            "world": wsz,
            "max": mx,
            "same_shape": all(g.shape == tables.shape for g in gathered),
            "same_lengths": bool((w.context_lens == base.context_lens).all()),
            "distinct_data": not torch.equal(qs[0], qs[1]),
            "value": bench.whole_job_gbs(1e9, wsz, mx[0]),
        }
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_and_max_timing():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, 2, port, results)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        res = dict(results)
    assert set(res) == {0, 1}
    for r in (0, 1):
        assert res[r]["world"] == 2
        assert res[r]["max"] == [2.0, 5.0]  # element-wise max over the two ranks
        assert res[r]["same_shape"] and res[r]["same_lengths"] and res[r]["distinct_data"]
        # whole-job value: both ranks' bytes over the slowest rank's time (2 GB in 2 ms)
        assert abs(res[r]["value"] - 1000.0) < 1e-9


def test_single_rank_helpers():
    import bench

    assert bench.max_over_ranks([3.0, 1.0], 1) == [3.0, 1.0]
    assert bench.whole_job_gbs(6e8, 1, 0.1) == 6000.0


def test_source_hash_ignores_comments_only():
    import bench

    code = 'int a = 1;  // note\n/* block\n   comment */\nconst char* s = "// kept"; char q = \'"\';\n\n'
    assert bench.strip_c_comments(code) == 'int a = 1;\nconst char* s = "// kept"; char q = \'"\';'
    edited = code.replace("// note", "// another note").replace("block", "other block")
    assert bench.strip_c_comments(edited) == bench.strip_c_comments(code)
    assert bench.strip_c_comments(code.replace("a = 1", "a = 2")) != bench.strip_c_comments(code)
    assert len(bench.kernel_source_hash()) == 16
