"""Sequence sharding of long contexts (bit_kv_cache_16_b200/seqshard.py) on
the CPU: the partition of a sequence into per-rank caches, the exchange of
the partials between gloo ranks, and the merge formula, all against the
oracle's unsharded cache and attention."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from bit_kv_cache_16_b200 import seqshard, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _quantized(n, G, R):
    return G * (max(n - R, 0) // G)


@pytest.mark.parametrize("G,R", [(16, 0), (16, 16), (32, 128), (64, 32)])
@pytest.mark.parametrize("parts", [1, 2, 3, 5])
def test_shard_bounds_cover_the_sequence_on_group_boundaries(G, R, parts):
    for n in [0, 1, G - 1, G, R, R + G - 1, R + G, R + G + 1, 7 * G + R + 3, 4097]:
        b = seqshard.shard_bounds(n, G, R, parts)
        assert len(b) == parts and b[0][0] == 0 and b[-1][1] == n
        for (lo, hi), (lo2, _) in zip(b, b[1:]):
            assert hi == lo2 and lo <= hi
        for p, (lo, hi) in enumerate(b):
            assert lo % G == 0
            if p < parts - 1:
                # whole groups only, all of them quantized in the unsharded cache
                assert (hi - lo) % G == 0 and hi <= _quantized(n, G, R)
        lo, hi = b[-1]
        # the last rank's own window state matches the unsharded one
        assert lo + _quantized(hi - lo, G, R) == _quantized(n, G, R)
        # groups are spread as evenly as whole groups allow
        sizes = [(h - l) // G for l, h in b[:-1]] + [_quantized(hi - lo, G, R) // G]
        assert max(sizes) - min(sizes) <= 1


def _shard_units(w, b, h, parts, bits, G, R, cap):
    """Oracle units of every rank's part of sequence b, kv head h."""
    k = w.seq_k(b)[:, h, :]
    v = w.seq_v(b)[:, h, :]
    units = []
    for p, (lo, hi) in enumerate(seqshard.shard_bounds(len(k), G, R, parts)):
        u = oracle.Unit(bits, 128, G, seqshard.shard_residual(p, parts, R), cap)
        u.prefill(k[lo:hi], v[lo:hi])
        units.append((lo, hi, u))
    return units


@pytest.mark.parametrize("bits,G,R", [(4, 32, 128), (2, 16, 16)])
def test_shards_hold_the_unsharded_groups(bits, G, R):
    """Every rank's codes, scales and zeros are the matching slice of the
    unsharded cache's, and the last rank's window holds the same tokens."""
    n = 1000
    w = synth.make_workload("shard", 7100 + G, [n], 4, 1, bits, G, R)
    cap = 1024
    full = oracle.Unit(bits, 128, G, R, cap)
    full.prefill(w.seq_k(0)[:, 0, :], w.seq_v(0)[:, 0, :])
    W = R + G
    for lo, hi, u in _shard_units(w, 0, 0, 3, bits, G, R, cap):
        nq = u.n_q
        assert u.n == hi - lo
        assert np.array_equal(u.k_codes[:nq], full.k_codes[lo:lo + nq])
        assert np.array_equal(u.k_scale[:nq // G], full.k_scale[lo // G:(lo + nq) // G])
        assert np.array_equal(u.k_zero[:nq // G], full.k_zero[lo // G:(lo + nq) // G])
        assert np.array_equal(u.v_codes[:nq], full.v_codes[lo:lo + nq])
        assert np.array_equal(u.v_scale[:nq], full.v_scale[lo:lo + nq])
        assert np.array_equal(u.v_zero[:nq], full.v_zero[lo:lo + nq])
        # window tokens: only the last rank has any (the others hold whole groups)
        for t in range(lo + nq, hi):
            assert np.array_equal(u.k_ring[(t - lo) % W], full.k_ring[t % W])
            assert np.array_equal(u.v_ring[(t - lo) % W], full.v_ring[t % W])
    assert sum(hi - lo for lo, hi, _ in _shard_units(w, 0, 0, 3, bits, G, R, cap)) == n


def _partials(w, b, h, parts, bits, G, R, cap):
    """(out, lse) of every rank's part for the query heads of kv head h, from
    the oracle's dequantized tokens (double)."""
    g = w.num_q_heads // w.num_kv_heads
    q = synth.bf16_bits_to_f32(w.q[b, h * g:(h + 1) * g, :]).astype(np.float64)
    res = []
    for lo, hi, u in _shard_units(w, b, h, parts, bits, G, R, cap):
        if hi == lo:
            res.append((np.zeros((g, 128)), np.full(g, -np.inf)))
            continue
        kh, vh = u.materialize()
        s = q @ kh.T * w.softmax_scale
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        res.append((e @ vh / e.sum(axis=1, keepdims=True), (m[:, 0] + np.log(e.sum(axis=1)))))
    return res


def _merge(outs, lses):
    """The merge formula: softmax over the union of disjoint token sets."""
    outs, lses = np.asarray(outs), np.asarray(lses)
    M = lses.max(axis=0)
    wts = np.where(np.isfinite(lses), np.exp(lses - M), 0.0)
    return np.einsum("pr,prd->rd", wts, outs) / wts.sum(axis=0)[:, None]


def test_merged_partials_equal_unsharded_attention():
    bits, G, R = 4, 32, 128
    w = synth.make_workload("shard", 7200, [1500, 700], 8, 2, bits, G, R)
    cap = 1536
    g = 4
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            full = oracle.Unit(bits, 128, G, R, cap)
            full.prefill(w.seq_k(b)[:, h, :], w.seq_v(b)[:, h, :])
            ref = full.decode(w.q[b, h * g:(h + 1) * g, :], w.softmax_scale)
            for parts in (1, 2, 3):
                p = _partials(w, b, h, parts, bits, G, R, cap)
                got = _merge([o for o, _ in p], [l for _, l in p])
                assert np.max(np.abs(got - ref)) < 1e-9


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        bits, G, R = 2, 32, 64
        w = synth.make_workload("shard", 7300, [900, 400, 50], 4, 2, bits, G, R)
        rows = []
        lse = []
        for b in range(w.batch):
            for h in range(w.num_kv_heads):
                o, l = _partials(w, b, h, world, bits, G, R, 1024)[rank]
                rows.append(o)
                lse.append(l)
        mine = torch.from_numpy(np.concatenate(rows)).float()
        mine_lse = torch.from_numpy(np.concatenate(lse)).float()
        outs, lses = seqshard.gather_partials(mine, mine_lse)
        out.put((rank, outs.numpy().astype(np.float64), lses.numpy().astype(np.float64)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_exchange_partials_in_rank_order():
    """Two gloo ranks each hold one shard of three sequences; after the
    exchange every rank has both partials in rank order, and merging them
    gives the unsharded attention."""
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    bits, G, R = 2, 32, 64
    w = synth.make_workload("shard", 7300, [900, 400, 50], 4, 2, bits, G, R)
    ref = []
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            full = oracle.Unit(bits, 128, G, R, 1024)
            full.prefill(w.seq_k(b)[:, h, :], w.seq_v(b)[:, h, :])
            ref.append(full.decode(w.q[b, 2 * h:2 * h + 2, :], w.softmax_scale))
    ref = np.concatenate(ref)
    for rank, outs, lses in res:
        assert outs.shape == (world, ref.shape[0], 128) and lses.shape == (world, ref.shape[0])
        # fp32 transport of the partials: merged within fp32 rounding
        assert np.max(np.abs(_merge(outs, lses) - ref)) < 1e-5
        # rank order: part p is what rank p computed
        for p in range(world):
            mine = np.concatenate([_partials(w, b, h, world, bits, G, R, 1024)[p][1]
                                   for b in range(w.batch) for h in range(w.num_kv_heads)])
            assert np.array_equal(lses[p], mine.astype(np.float32).astype(np.float64))


class _OracleShard:
    """Stands in for one rank's libkvq cache on the CPU: its lse decode is
    the oracle's attention over the rank's part."""

    def __init__(self, w, parts, rank, bits, G, R):
        self.shape = type("S", (), {"batch": w.batch, "num_q_heads": w.num_q_heads})()
        self.w, self.parts, self.rank = w, parts, rank
        self.bits, self.G, self.R = bits, G, R

    def decode_attention_lse(self, q, out, lse, softmax_scale, workspace, num_splits, max_len, stream=None):
        w = self.w
        rows_o, rows_l = [], []
        for b in range(w.batch):
            for h in range(w.num_kv_heads):
                o, l = _partials(w, b, h, self.parts, self.bits, self.G, self.R, 1024)[self.rank]
                rows_o.append(o)
                rows_l.append(l)
        out.copy_(torch.from_numpy(np.concatenate(rows_o)).float())
        lse.copy_(torch.from_numpy(np.concatenate(rows_l)).float())


def _merge_into(outs, lses, parts, rows, out, lse_out=None, stream=None):
    out.view(rows, 128).copy_(torch.from_numpy(_merge(outs.double().numpy(), lses.double().numpy())).float())


def _rank_main_decode(rank, world, port, out_q):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        bits, G, R = 4, 16, 16
        w = synth.make_workload("shard", 7700, [700, 333], 4, 2, bits, G, R)
        seqshard.kvq.kvq_merge_partials = _merge_into      # the merge kernel's formula, on the CPU
        out = torch.full((w.batch, w.num_q_heads, 128), float("nan"))
        seqshard.decode_sharded(_OracleShard(w, world, rank, bits, G, R), None, out, w.softmax_scale, None, 0, 700)
        out_q.put((rank, out.double().numpy()))
    finally:
        dist.destroy_process_group()


def test_decode_sharded_on_two_ranks():
    """decode_sharded itself on two gloo ranks, its two library calls stood
    in for by the oracle and the merge formula: every rank ends with the
    attention over the whole sequences."""
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main_decode, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    bits, G, R = 4, 16, 16
    w = synth.make_workload("shard", 7700, [700, 333], 4, 2, bits, G, R)
    oc = oracle.Cache(bits, w.batch, w.num_q_heads, w.num_kv_heads, 128, G, R, 704)
    oc.prefill(w.k, w.v, w.cu_seqlens)
    ref = oc.decode(w.q, w.softmax_scale)
    for rank, out in res:
        assert out.shape == ref.shape
        assert np.max(np.abs(out - ref)) < 1e-5
