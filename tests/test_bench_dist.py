"""Multi-rank host logic of bench.py on CPU: two gloo ranks, each timing its own layer; the job
time is the max over ranks and the job FLOPs the sum (weak scaling, no data-path collective)."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms, flops = bench.job_totals(10.0 + 5.0 * rank, 1e12 * (rank + 1), world, device="cpu")
        out[rank] = (ms, flops)
    finally:
        dist.destroy_process_group()


def test_job_totals_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
        res = dict(out)
    assert res[0] == res[1] == (15.0, 3e12)


def _shard_worker(rank, world, port, out):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch
    import workload
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        p = workload.qwen2_7b_video_128k()
        sub, qh, kvh = workload.shard_kv_heads(p, rank, world)
        mine = torch.tensor(list(qh) + [-1] * (p.Hq - len(qh)), dtype=torch.int64)
        parts = [torch.empty_like(mine) for _ in range(world)]
        dist.all_gather(parts, mine)
        out[rank] = sorted(int(h) for t in parts for h in t.tolist() if h >= 0), (sub.Hq, sub.Hkv)
    finally:
        dist.destroy_process_group()


def test_kv_head_shards_of_two_gloo_ranks_cover_the_layer():
    """Each of two ranks takes its KV-head groups of the 128K layer (14 query / 2 KV heads); the
    union over ranks is every query head exactly once."""
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        mp.start_processes(_shard_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
        res = dict(out)
    assert res[0][0] == res[1][0] == list(range(28))
    assert res[0][1] == res[1][1] == (14, 2)


def test_job_totals_single_rank_is_identity():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    assert bench.job_totals(7.5, 42.0, 1) == (7.5, 42.0)


def test_kernel_code_hash_ignores_comments_only():
    """The identity under which the recorded DRAM traffic stays valid: comments and layout do not
    change it, code (including inline-PTX strings) does."""
    import importlib.util
    import os
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(os.path.dirname(__file__), "..", "bench.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    src = 'int f(int x) {  // doubles\n  /* a\n block */ return 2 * x;\n}\nasm("add.s32 %0, %1; // not a comment");\n'
    same = 'int f(int x)\n{ return 2 * x; }   // other words\nasm("add.s32 %0, %1; // not a comment");'
    other = 'int f(int x) { return 3 * x; }\nasm("add.s32 %0, %1; // not a comment");'
    ptx = 'int f(int x) { return 2 * x; }\nasm("sub.s32 %0, %1; // not a comment");'
    assert b.code_only(src) == b.code_only(same)
    assert b.code_only(src) != b.code_only(other)
    assert b.code_only(src) != b.code_only(ptx)
