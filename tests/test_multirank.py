"""The multi-rank pieces of bench.py on CPU ranks (gloo, world size 2).

With N > 1 GPUs every rank quantizes and decodes its own batch (weak
scaling; no collective on that data path), and the sequence-sharded leg
decodes one long sequence split over the ranks (all-gather of the
partials, then the merge).  What crosses ranks is the barrier, the max of
the per-rank step time and that all-gather; these tests run that logic on
two gloo processes, the library's calls stood in for by the oracle.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, values, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        dist.barrier()
        got = bench.max_over_ranks(values[rank], torch.device("cpu"), world)
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.rank_seed(rank))
        out.put((rank, got, seeds))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_max_time_and_distinct_batches():
    world, port = 2, _free_port()
    values = [123.5, 456.25]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, values, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, seeds in res:
        assert got == max(values)
        assert len(set(seeds)) == world        # every rank draws its own batch


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.0, torch.device("cpu"), 1) == 7.0


def test_rank_batches_have_the_benched_shape():
    sys.path.insert(0, ROOT)
    import bench
    from bit_kv_cache_16_b200 import synth
    w = synth.make_workload(bench.WORKLOAD, bench.rank_seed(1), [40] * 2, bench.HQ, bench.HKV, 4, bench.G,
                            bench.R)
    assert w.num_q_heads == bench.HQ and w.num_kv_heads == bench.HKV and w.group == bench.G
    assert bench.rank_seed(0) == synth.SEED_BASE + 1     # rank 0 runs config 1 itself


def _rank_main_sharded(rank, world, port, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import numpy as np
    import bench
    import test_seqshard as ts
    from bit_kv_cache_16_b200 import seqshard, synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        bits, G, R = 4, 16, 16
        w = synth.make_workload("shard", 7700, [700, 333], 4, 2, bits, G, R)
        k, v, cu, lens, res = bench.seqshard_part(w, rank, world)
        assert res == (R if rank == world - 1 else 0)
        seqshard.kvq.kvq_merge_partials = ts._merge_into       # the merge kernel's formula, on the CPU
        o = torch.full((w.batch, w.num_q_heads, 128), float("nan"))
        bench.sharded_step(ts._OracleShard(w, world, rank, bits, G, R), None, o, w.softmax_scale, None, 0,
                           int(lens.max()))
        out.put((rank, o.double().numpy()))
    finally:
        dist.destroy_process_group()


def test_bench_sharded_leg_on_two_ranks():
    """The bench's sequence-sharded decode on two gloo ranks: every rank
    ends with the attention over the whole sequences."""
    import numpy as np
    sys.path.insert(0, ROOT)
    import oracle
    from bit_kv_cache_16_b200 import synth
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main_sharded, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = synth.make_workload("shard", 7700, [700, 333], 4, 2, 4, 16, 16)
    oc = oracle.Cache(4, w.batch, w.num_q_heads, w.num_kv_heads, 128, 16, 16, 704)
    oc.prefill(w.k, w.v, w.cu_seqlens)
    ref = oc.decode(w.q, w.softmax_scale)
    for rank, o in res:
        assert np.max(np.abs(o - ref)) < 1e-5
