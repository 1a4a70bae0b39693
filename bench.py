"""Benchmark of the quantized-KV decode path on B200.

Headline (`value`): the decode step of the Llama-3-8B-shaped layer (B=8,
32 query / 8 kv heads, d=128, INT4, G=32, R=128) over a resident cache that
grows by one token per step, as a serving engine runs it:
  1. append each sequence's new token to the bf16 window and, when the
     window holds R + G tokens, quantize its oldest group (one launch:
     kvq_append_flush; the first step and every 32nd one flush),
  2. decode attention of the 32 query heads over all cached tokens
     (8064+ quantized + the window; two launches, split streaming + merge).
The cache is filled once by quantizing a prefill of 8191 tokens per
sequence; that prefill-quantize is timed on its own (`phases.prefill`).
The L2 is flushed before every timed prefill and before every step's append
by writing a 512 MB buffer and reading it back (cold, clean L2); the flush is
outside the timed windows.  Times are CUDA events on the launching stream.

`workloads` adds, on one GPU, the prefill and decode of every named
workload (tiny check, Llama-3-70B 128K at INT4 and INT2, the paged ragged
batch) and the two streaming runs (INT2 and FP8-E4M3: 512 steps of append +
flush + decode, flush steps reported apart), each with its algorithmic bytes
and fraction of the HBM roofline.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                  [--no-workloads] [--no-cpu-baseline]

With N > 1 (torchrun) every rank runs its own batch of the headline
workload (weak scaling; no collective on that data path; times are the max
over ranks), and `seqshard` times one 131072-token Llama-3-70B sequence
split along its tokens over the N ranks: each decodes its shard, the
(output, ln-sum-exp) partials are all-gathered over NCCL and merged.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import ctypes

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantized-KV decode attention: us/step, KV GB/s and % of B200 HBM peak"
WORKLOAD = "llama3_8b_layer_decode_b8_n8192_int4_g32_r128"
B, HQ, HKV, D, N_CTX, G, R = 8, 32, 8, 128, 8192, 32, 128
N_PREFILL = N_CTX - 1
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0          # the ~8 TB/s B200 HBM3e figure the targets are stated against
# libkvq launches per decode step: append + flush (one), decode split + merge (two)
LAUNCHES_PER_STEP = 3



def cudart():
    """The CUDA runtime the process already uses (loaded by torch), with the
    argument types of the few calls the end-to-end loop makes."""
    lib = ctypes.CDLL("libcudart.so.12")
    vp = ctypes.c_void_p
    lib.cudaMemcpyAsync.argtypes = [vp, vp, ctypes.c_size_t, ctypes.c_int, vp]
    lib.cudaEventCreateWithFlags.argtypes = [ctypes.POINTER(vp), ctypes.c_uint]
    lib.cudaEventRecord.argtypes = [vp, vp]
    lib.cudaStreamWaitEvent.argtypes = [vp, vp, ctypes.c_uint]
    lib.cudaEventDestroy.argtypes = [vp]
    return lib


def rt_check(status: int, value=None):
    if status != 0:
        raise RuntimeError("CUDA runtime call failed with status %d" % status)
    return value

def measured_peak_gbs():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------
# Algorithmic bytes (fp16 scale/zero, bf16 window; q counted once per row)
# ---------------------------------------------------------------------------

def quantized_split(n: int, group: int, residual: int):
    """(n_q, r): quantized tokens and window tokens of a sequence of n tokens."""
    nq = group * (max(n - residual, 0) // group)
    return nq, n - nq


def unit_cache_bytes(bits: int, group: int, residual: int, n: int, head_dim: int = D) -> int:
    """Bytes of one (sequence, kv head) cache of n tokens: K and V codes,
    per-group key and per-token value scale/zero, and the bf16 window
    (e4m3 codes only for FP8; INT8 per token: codes and a key and a value
    (scale, zero) per token)."""
    if bits == 8:
        return n * head_dim * 2
    if bits == 16:
        return n * (head_dim * 2 + 8)
    nq, r = quantized_split(n, group, residual)
    return nq * head_dim * bits // 8 * 2 + (nq // group) * 2 * head_dim * 2 + nq * 4 + r * head_dim * 2 * 2


def decode_bytes(bits, group, residual, q_heads, kv_heads, lengths, head_dim: int = D) -> int:
    """Algorithmic bytes of one decode call at these sequence lengths."""
    return (len(lengths) * q_heads * head_dim * 2 +
            sum(kv_heads * unit_cache_bytes(bits, group, residual, int(n), head_dim) for n in lengths))


def prefill_bytes(bits, group, residual, kv_heads, lengths, head_dim: int = D) -> int:
    """Algorithmic bytes of a prefill: read K and V once, write the cache."""
    return sum(kv_heads * (int(n) * head_dim * 2 * 2 + unit_cache_bytes(bits, group, residual, int(n), head_dim))
               for n in lengths)


def append_flush_bytes(bits, group, residual, batch, kv_heads, n_before: int, head_dim: int = D) -> int:
    """Append one token per (sequence, kv head) at n_before tokens (read and
    write a K and a V row), plus, when the window then holds R + G tokens,
    the flush of one group (read G window rows of K and V, write their codes
    and the group's key and value scale/zero)."""
    if bits in (8, 16):     # the token is encoded straight into the cache (no window)
        return batch * kv_heads * (head_dim * 2 * 2 + head_dim * 2 + (8 if bits == 16 else 0))
    per = head_dim * 2 * 2 * 2
    nq, _ = quantized_split(n_before, group, residual)
    if n_before + 1 - nq == residual + group:
        per += group * head_dim * 2 * 2 + group * head_dim * bits // 8 * 2 + 2 * head_dim * 2 + group * 4
    return batch * kv_heads * per


def mixed_unit_bytes(classes, group: int, residual: int, head_dim: int = D) -> int:
    """Bytes of one (sequence, kv head) of a mixed 2/4-bit cache holding
    tokens of these classes: each quantized group at the widest class of its
    tokens (codes at that width, key scale/zero, value scale/zero), then the
    bf16 window."""
    n = len(classes)
    nq, r = quantized_split(n, group, residual)
    total = r * head_dim * 2 * 2
    for g0 in range(0, nq, group):
        bits = 4 if np.any(np.asarray(classes[g0:g0 + group]) == 4) else 2
        total += group * head_dim * bits // 8 * 2 + 2 * head_dim * 2 + group * 4
    return total


def wl_decode_bytes(w, lengths, classes=None) -> int:
    if w.bits == 6:
        cu = np.concatenate([[0], np.cumsum(w.lengths)])
        return (w.batch * w.num_q_heads * w.head_dim * 2 +
                sum(w.num_kv_heads * mixed_unit_bytes(classes[cu[b]:cu[b] + int(n)], w.group, w.residual, w.head_dim)
                    for b, n in enumerate(lengths)))
    return decode_bytes(w.bits, w.group, w.residual, w.num_q_heads, w.num_kv_heads, lengths, w.head_dim)


def sparse_bytes(w) -> int:
    """Extra bytes of a dense-and-sparse cache: a kept key (4 bytes) per
    channel of every quantized group and a kept value (4 bytes) per
    quantized token, for every (sequence, kv head)."""
    total = 0
    for n in w.lengths:
        nq, _ = quantized_split(int(n), w.group, w.residual)
        total += w.num_kv_heads * ((nq // w.group) * w.head_dim * 4 + nq * 4)
    return total


def wl_prefill_bytes(w, classes=None) -> int:
    if w.bits == 6:
        return (w.num_kv_heads * int(np.sum(w.lengths)) * w.head_dim * 2 * 2 +
                wl_decode_bytes(w, w.lengths, classes) - w.batch * w.num_q_heads * w.head_dim * 2)
    return prefill_bytes(w.bits, w.group, w.residual, w.num_kv_heads, w.lengths, w.head_dim)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for nm, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle leg (the reference arm and the cpu_baseline key)
# ---------------------------------------------------------------------------

def host_cores() -> int:
    """Cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_step_sample(w, budget_s: float, threads: int = 1):
    """The oracle's decode step on the headline workload: every (b, kv) unit
    is prefilled with 8191 tokens (untimed), then the append of the 8192nd
    token, the flush it makes due and the decode of the unit's query heads
    are timed.  Units run in waves of `threads` (the units are independent
    and the C oracle releases the interpreter lock, so each thread runs the
    unchanged oracle on its own unit) until budget_s of wall time has passed,
    at least one wave; a wave's timed section lasts as long as its slowest
    unit.  Returns the time per full step (all 64 units) extrapolated from
    the units done, and their number."""
    from concurrent.futures import ThreadPoolExecutor
    import oracle
    from bit_kv_cache_16_b200 import synth
    kn, vn = synth.streaming_token(w, 0)
    order = [(b, h) for b in range(B) for h in range(HKV)]
    g = HQ // HKV

    def prefilled(bh):
        b, h = bh
        u = oracle.Unit(4, D, G, R, N_CTX)
        lo = int(w.cu_seqlens[b])
        u.prefill(w.k[lo:lo + N_PREFILL, h, :], w.v[lo:lo + N_PREFILL, h, :])
        return u

    def step(args):
        (b, h), u = args
        u.append(kn[b, h], vn[b, h])
        u.flush()
        u.decode(w.q[b, h * g:(h + 1) * g, :], w.softmax_scale)

    timed = 0.0
    done = 0
    wall0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=threads) as ex:
        while done < len(order):
            wave = order[done:done + threads]
            units = list(ex.map(prefilled, wave))
            t0 = time.perf_counter()
            list(ex.map(step, zip(wave, units)))
            timed += time.perf_counter() - t0
            done += len(wave)
            if time.perf_counter() - wall0 >= budget_s:
                break
    return timed / done * len(order), done


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from bit_kv_cache_16_b200 import synth
    import oracle
    oracle.build()
    w = synth.make_config(1, lengths=[N_PREFILL] * B)
    cores = host_cores()
    per_step = []
    units = 0
    for i in range(args.warmup + args.steps):
        t, units = oracle_step_sample(w, budget_s=args.ref_budget, threads=cores)
        if i >= args.warmup:
            per_step.append(t)
    us = statistics.median(per_step) * 1e6
    line = {"metric": METRIC, "value": us, "unit": "us/step", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": us / 1e3, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32-encode/f64-attention", "data": "synthetic",
            "config": {"workload": WORKLOAD, "batch": B, "seq_len": N_CTX, "q_heads": HQ, "kv_heads": HKV,
                       "bits": 4, "group": G, "residual": R},
            "impl": "reference",
            "cpu_baseline": {"value": us, "unit": "us/step", "cores": cores, "kind": "oracle",
                             "sample": "append + flush + decode of %d of %d (sequence, kv head) units per step "
                                       "(each prefilled with 8191 tokens, untimed) on %d threads, extrapolated"
                                       % (units, B * HKV, cores)},
            "e2e": {"value": us, "unit": "us/step", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# Cross-rank pieces
# ---------------------------------------------------------------------------

def rank_seed(rank: int) -> int:
    """Seed of rank r's batch: the config-1 seed on rank 0, distinct streams elsewhere."""
    from bit_kv_cache_16_b200 import synth
    return synth.SEED_BASE + 1 + 1000 * rank


def rank_workload(rank: int):
    """Rank r's batch: the shape of the benched workload, its own seeded values."""
    from bit_kv_cache_16_b200 import synth
    if rank == 0:
        return synth.make_config(1, lengths=[N_PREFILL] * B)
    return synth.make_workload(WORKLOAD, rank_seed(rank), [N_PREFILL] * B, HQ, HKV, 4, G, R)


def max_over_ranks(value: float, device, world: int) -> float:
    """The largest per-rank time (the job finishes when its slowest rank does)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def seqshard_part(w, rank: int, world: int):
    """Rank `rank`'s shard of every sequence of w (whole key groups; the last
    rank also takes the window): (k, v, cu_seqlens, lengths, residual) of a
    cache of its own."""
    from bit_kv_cache_16_b200 import seqshard
    ks, vs, lens = [], [], []
    for b in range(w.batch):
        n = int(w.lengths[b])
        lo, hi = seqshard.shard_bounds(n, w.group, w.residual, world)[rank]
        ks.append(w.seq_k(b)[lo:hi])
        vs.append(w.seq_v(b)[lo:hi])
        lens.append(hi - lo)
    cu = np.zeros(w.batch + 1, np.int32)
    cu[1:] = np.cumsum(lens)
    return (np.ascontiguousarray(np.concatenate(ks)), np.ascontiguousarray(np.concatenate(vs)), cu,
            np.asarray(lens, np.int64), seqshard.shard_residual(rank, world, w.residual))


def sharded_step(cache, q, out, softmax_scale, workspace, num_splits, max_len, stream=None):
    """One decode of the sharded sequences on this rank (the bench's
    multi-GPU leg): the rank's decode with ln-sum-exp, the all-gather of the
    partials and their merge (bit_kv_cache_16_b200.seqshard)."""
    from bit_kv_cache_16_b200 import seqshard
    seqshard.decode_sharded(cache, q, out, softmax_scale, workspace, num_splits, max_len, stream=stream)


# ---------------------------------------------------------------------------
# GPU leg
# ---------------------------------------------------------------------------

class Gpu:
    """Device-side helpers shared by the legs: L2 flush, events, uploads."""

    def __init__(self, dev):
        import torch
        self.torch = torch
        self.dev = dev
        self.stream = torch.cuda.current_stream()
        self.l2 = torch.empty(512 * 2 ** 20, dtype=torch.uint8, device=dev)
        self.l2_words = self.l2.view(torch.int64)

    def flush_l2(self):
        # Write 512 MB (evicts everything), then read it back: the read makes
        # the L2 write back its dirty lines here, so the next timed kernel
        # starts on a cold, clean L2 instead of paying for this buffer's
        # write-back.
        self.l2.zero_()
        self.l2_words.sum()

    def ev(self):
        return self.torch.cuda.Event(enable_timing=True)

    def bf16(self, a):
        return self.torch.from_numpy(np.ascontiguousarray(a.view(np.int16))).to(self.dev)

    def timed(self, fn, n: int):
        """Device time (us) of fn, n calls, each after an L2 flush outside its window."""
        evs = []
        for _ in range(n):
            self.flush_l2()
            e0, e1 = self.ev(), self.ev()
            e0.record(self.stream)
            fn()
            e1.record(self.stream)
            evs.append((e0, e1))
        self.torch.cuda.synchronize()
        return [a.elapsed_time(b) * 1e3 for a, b in evs]


def rate(us: float, nbytes: int, peak: float) -> dict:
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"us": round(us, 3), "bytes": int(nbytes), "GB/s": round(gbs, 1), "frac": round(gbs / peak, 4),
            "frac_nominal": round(gbs / NOMINAL_HBM_GBS, 4)}


def run_gpu(args):
    import torch
    import torch.distributed as dist
    from bit_kv_cache_16_b200 import kvq, synth
    from bit_kv_cache_16_b200.build import build_libkvq

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    if rank == 0:
        build_libkvq()
    if world > 1:
        dist.barrier()
    kvq.load()
    gpu = Gpu(dev)
    stream = gpu.stream
    peak, peak_kind = measured_peak_gbs()
    if args.only:
        # the named workloads alone (a short run to profile one kernel): no step line
        only = args.only.split(",")
        unknown = [n for n in only if n not in [x[0] for x in WORKLOADS] + [x[0] for x in STREAMING]]
        if unknown:
            raise SystemExit("unknown workload(s): %s" % ", ".join(unknown))
        res = run_workloads(gpu, peak, args.workload_iters or args.steps, only)
        if rank == 0:
            print(json.dumps({"only": only, "workloads": res}), flush=True)
        return

    W, K = args.warmup, args.steps
    w = rank_workload(rank)
    e2e_steps = K
    n_steps = W + 2 * K + 2 + e2e_steps       # decode steps the cache must hold past the prefill
    toks = [synth.streaming_token(w, s) for s in range(n_steps)]
    to_pinned = lambda a: torch.from_numpy(np.ascontiguousarray(a.view(np.int16))).pin_memory()
    hk, hv = to_pinned(w.k), to_pinned(w.v)
    hq = to_pinned(w.q)
    hkn = [to_pinned(t[0]) for t in toks]
    hvn = [to_pinned(t[1]) for t in toks]
    hcu = torch.from_numpy(w.cu_seqlens.astype(np.int32)).pin_memory()
    dk, dv, dq, dcu = hk.to(dev), hv.to(dev), hq.to(dev), hcu.to(dev)
    dkn = [t.to(dev) for t in hkn]
    dvn = [t.to(dev) for t in hvn]

    cap = (N_PREFILL + n_steps + G - 1) // G * G
    cache = kvq.Cache(kvq.KVQ_FORMAT_INT4, B, HQ, HKV, cap, group=G, residual=R, device=dev)
    splits = args.splits or kvq.kvq_decode_default_splits(cache.desc, N_CTX)
    ws = torch.empty(cache.workspace_bytes(splits, cap), dtype=torch.uint8, device=dev)
    out = torch.empty(B, HQ, D, dtype=torch.float32, device=dev)
    hout = torch.empty(B, HQ, D, dtype=torch.float32).pin_memory()
    scale = 1.0 / np.sqrt(D)

    def prefill():
        cache.quantize_prefill(dk, dv, dcu, N_PREFILL, stream)

    # ---- phase 1: prefill-quantize (each call rewrites the whole state) ----
    for _ in range(W):
        prefill()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    pre_us = gpu.timed(prefill, K)

    # ---- phase 2: decode steps over the resident cache ----
    # state: 8191 tokens after the last prefill; step s appends token s
    def step(s, ev=None):
        if ev:
            ev[0].record(stream)
        cache.append_flush(dkn[s], dvn[s], stream)
        if ev:
            ev[1].record(stream)
        cache.decode_attention(dq, out, scale, ws, splits, N_PREFILL + s + 1, stream)
        if ev:
            ev[2].record(stream)

    step(0)                                   # correctness guard for this launch configuration
    torch.cuda.synchronize()
    assert cache.error() == 0 and bool(torch.isfinite(out).all())
    for s in range(1, W):
        step(s)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    first = max(W, 1)
    # the step as a caller runs it: events around the pair of calls only (the
    # decode may launch behind the append, programmatic dependent launch)
    step_evs = []
    for s in range(first, first + K):
        gpu.flush_l2()
        e = [gpu.ev(), None, gpu.ev()]
        e[0].record(stream)
        step(s)
        e[2].record(stream)
        step_evs.append(e)
    # the two calls apart: an event between them (no overlap), for the split
    evs = []
    for s in range(first + K, first + 2 * K):
        gpu.flush_l2()
        e = [gpu.ev() for _ in range(3)]
        step(s, e)
        evs.append(e)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    assert cache.error() == 0
    af_us = [e[0].elapsed_time(e[1]) * 1e3 for e in evs]
    dec_us = [e[1].elapsed_time(e[2]) * 1e3 for e in evs]
    step_us = max_over_ranks(sum(e[0].elapsed_time(e[2]) * 1e3 for e in step_evs) / K, dev, world)
    # bytes of step s: append (+ flush when due) at N_PREFILL + s tokens, decode over N_PREFILL + s + 1
    steps_idx = list(range(first + K, first + 2 * K))
    af_bytes = [append_flush_bytes(4, G, R, B, HKV, N_PREFILL + s) for s in steps_idx]
    dec_bytes = [decode_bytes(4, G, R, HQ, HKV, [N_PREFILL + s + 1] * B) for s in steps_idx]
    flush_steps = sum(1 for s in range(first, first + K) if append_flush_bytes(4, G, R, 1, 1, N_PREFILL + s) > D * 8)

    # ---- e2e: the same decode step through the public API with host buffers ----
    # Per step: the query and the new token host -> device as one copy from a
    # pinned staging buffer (q | k_new | v_new, as a serving loop packs them),
    # then append + flush and decode, then `out` back to pinned host memory.
    # As a serving loop would, the copies run on their own streams and are
    # double-buffered, so step s + 1's input copy and step s's read-back
    # overlap the kernels; every step still makes both copies, and the timed
    # region ends when the last read-back has landed.
    # Consecutive steps use four resident caches of the benched shape in
    # turn (as consecutive layers would), so that no step finds its 81 MB of
    # cache in the 126 MB L2: 324 MB of caches against the L2, no flush in
    # the timed region.
    e2e_first = first + 2 * K
    extra = [kvq.Cache(kvq.KVQ_FORMAT_INT4, B, HQ, HKV, cap, group=G, residual=R, device=dev) for _ in range(3)]
    for c in extra:
        c.quantize_prefill(dk, dv, dcu, N_PREFILL, stream)
    rot = [cache] + extra
    lens = [N_PREFILL + e2e_first] + [N_PREFILL] * len(extra)     # tokens each holds
    nq_b, nk_b = hq.numel() * 2, hkn[0].numel() * 2
    hin = {s: torch.cat([hq.view(torch.uint8).flatten(), hkn[s].view(torch.uint8).flatten(),
                         hvn[s].view(torch.uint8).flatten()]).pin_memory()
           for s in range(e2e_first, e2e_first + 2 + e2e_steps)}
    din = [torch.empty(nq_b + 2 * nk_b, dtype=torch.uint8, device=dev) for _ in range(2)]
    views = [(d[:nq_b].view(torch.int16).view(hq.shape), d[nq_b:nq_b + nk_b].view(torch.int16).view(hkn[0].shape),
              d[nq_b + nk_b:].view(torch.int16).view(hvn[0].shape)) for d in din]
    outs = [out, torch.empty_like(out)]
    houts = [hout, torch.empty_like(hout).pin_memory()]
    h2d = din[0].numel()
    d2h = hout.numel() * hout.element_size()
    hs, ds = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)   # input copies, read-backs
    # the copies and their ordering go straight to the CUDA runtime (one
    # call each), so that the host keeps ahead of the device on any machine
    rt = cudart()

    def rt_event():
        h = ctypes.c_void_p()
        return rt_check(rt.cudaEventCreateWithFlags(ctypes.byref(h), 2), h)   # 2: no timing

    in_ready, done, read = [rt_event(), rt_event()], [rt_event(), rt_event()], [rt_event(), rt_event()]
    rt_status = [0]
    hs_p, ds_p, ms_p = (ctypes.c_void_p(x.cuda_stream) for x in (hs, ds, stream))
    din_p = [ctypes.c_void_p(d.data_ptr()) for d in din]
    hin_p = {k: ctypes.c_void_p(v.data_ptr()) for k, v in hin.items()}
    out_p = [ctypes.c_void_p(o.data_ptr()) for o in outs]
    hout_p = [ctypes.c_void_p(o.data_ptr()) for o in houts]
    H2D, D2H = 1, 2

    def e2e_step(s, j):
        bf = j % 2
        if j >= 2:
            rt.cudaStreamWaitEvent(hs_p, done[bf], 0)      # step j - 2 has stopped reading din[bf]
        rt_status[0] |= rt.cudaMemcpyAsync(din_p[bf], hin_p[s], h2d, H2D, hs_p)
        rt.cudaEventRecord(in_ready[bf], hs_p)
        rt.cudaStreamWaitEvent(ms_p, in_ready[bf], 0)
        if j >= 2:
            rt.cudaStreamWaitEvent(ms_p, read[bf], 0)      # step j - 2's output has been read back
        dq_j, dkn_j, dvn_j = views[bf]
        m = s % len(rot)
        lens[m] += 1
        rot[m].append_flush(dkn_j, dvn_j, stream)
        rot[m].decode_attention(dq_j, outs[bf], scale, ws, splits, lens[m], stream)
        rt.cudaEventRecord(done[bf], ms_p)
        rt.cudaStreamWaitEvent(ds_p, done[bf], 0)
        rt_status[0] |= rt.cudaMemcpyAsync(hout_p[bf], out_p[bf], d2h, D2H, ds_p)
        rt.cudaEventRecord(read[bf], ds_p)

    for j, s in enumerate(range(e2e_first, e2e_first + 2)):
        e2e_step(s, j)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = gpu.ev(), gpu.ev()
    gpu.flush_l2()
    e0.record(stream)
    hs.wait_event(e0)
    last = 0
    for j, s in enumerate(range(e2e_first + 2, e2e_first + 2 + e2e_steps)):
        e2e_step(s, j)
        last = j
    rt.cudaStreamWaitEvent(ms_p, read[last % 2], 0)
    e1.record(stream)
    torch.cuda.synchronize()
    assert cache.error() == 0
    rt_check(rt_status[0])
    assert all(c.error() == 0 for c in extra)
    assert torch.equal(houts[last % 2], outs[last % 2].cpu())   # the read-back is the step's output
    for e in in_ready + done + read:
        rt.cudaEventDestroy(e)
    e2e_us = max_over_ranks(e0.elapsed_time(e1) * 1e3 / e2e_steps, dev, world)
    del dk, dv, hk, hv

    line = None
    if rank == 0:
        pre_mean = statistics.mean(pre_us)
        phases = {
            "prefill": rate(pre_mean, prefill_bytes(4, G, R, HKV, [N_PREFILL] * B), peak),
            "append_flush": rate(statistics.mean(af_us), round(statistics.mean(af_bytes)), peak),
            "decode": rate(statistics.mean(dec_us), round(statistics.mean(dec_bytes)), peak),
        }
        dec_rate = rate(sum(dec_us) / K, sum(dec_bytes) / K, peak)
        line = {"metric": METRIC, "value": round(step_us, 3), "unit": "us/step", "n_gpus": world,
                "steps": K, "warmup": W, "ms_per_step": round(step_us / 1e3, 6),
                "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
                "dtype": "int4-codes/f16-mma/f32",
                "data": "synthetic (seeded; K outlier channels x20, V heavy tokens x5, q outliers x5)",
                "config": {"workload": WORKLOAD, "batch": B, "seq_len": "8192..%d (prefill 8191, +1 token per step)"
                           % (N_PREFILL + first + 2 * K), "q_heads": HQ, "kv_heads": HKV, "bits": 4, "group": G,
                           "residual": R, "decode_splits": splits, "flush_steps_timed": flush_steps,
                           "l2": "512 MB write then read before every timed prefill and every step's append "
                                 "(cold, clean L2), outside the timed windows",
                           "parallelism": "dp%d (independent batch per GPU)" % world},
                "phases": phases,
                "phases_note": "append_flush and decode timed apart (an event between the calls, K further "
                               "steps); value times the two calls back to back",
                "step_with_prefill_us": round(step_us + pre_mean, 3),
                "decode_tokens_per_s": round(world * B / (step_us * 1e-6), 1),
                "roofline": {"bound": "hbm", "kernel": "decode (kvq_decode_attention: streaming + merge)",
                             "achieved": dec_rate["GB/s"], "peak": peak,
                             "peak_kind": peak_kind + " hbm_gbs (copy), burst", "unit": "GB/s",
                             "frac": dec_rate["frac"], "frac_nominal": dec_rate["frac_nominal"],
                             "nominal_gbs": NOMINAL_HBM_GBS, "traffic": load_traffic("decode")},
                "prefill_roofline": {"bound": "hbm", "achieved": phases["prefill"]["GB/s"], "peak": peak,
                                     "unit": "GB/s", "frac": phases["prefill"]["frac"],
                                     "frac_nominal": phases["prefill"]["frac_nominal"],
                                     "traffic": load_traffic("prefill")},
                "e2e": {"value": round(e2e_us, 3), "unit": "us/step", "h2d_bytes_per_step": h2d,
                        "d2h_bytes_per_step": d2h,
                        "what": "append + flush + decode through the Python API; q and the new token copied "
                                "in from pinned host memory (one packed copy) and the output read back every "
                                "step, the copies on their own streams and double-buffered; consecutive steps "
                                "use four resident caches of this shape in turn (324 MB > L2), no L2 flush"},
                "gpu_launches": K * LAUNCHES_PER_STEP,
                "clocks": clocks}

    # ---- every named workload (one GPU) ----
    if world == 1 and not args.no_workloads:
        line["workloads"] = run_workloads(gpu, peak, args.workload_iters or K)

    # ---- one long sequence split over the ranks ----
    if world > 1 and not args.no_seqshard:
        ss = run_seqshard(gpu, rank, world, K, W, peak)
        if rank == 0:
            line["seqshard"] = ss

    if rank == 0:
        if not args.no_cpu_baseline:
            t, units = oracle_step_sample(w, budget_s=args.cpu_budget)
            line["cpu_baseline"] = {"value": round(t * 1e6, 1), "unit": "us/step", "cores": 1, "kind": "oracle",
                                    "sample": "append + flush + decode of %d of %d (sequence, kv head) units "
                                              "(each prefilled with 8191 tokens, untimed), extrapolated to the step"
                                              % (units, B * HKV)}
            cores = host_cores()
            t, units = oracle_step_sample(w, budget_s=args.cpu_budget, threads=cores)
            line["cpu_baseline"]["all_cores"] = {
                "value": round(t * 1e6, 1), "unit": "us/step", "cores": cores,
                "sample": "%d of %d units on %d threads, extrapolated" % (units, B * HKV, cores)}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# Every named workload: prefill and decode, and the streaming runs step by
# step (flush steps apart from the others)
# ---------------------------------------------------------------------------

WORKLOADS = [  # (key, config id, bits, options: pre_rope = keys rotated at read, sparse = dense-and-sparse)
    ("tiny_b1_n512_int2_g32_r32", 0, 2, {}),
    ("llama3_70b_layer_b1_n131072_int4_g32_r128", 2, 4, {}),
    ("llama3_70b_layer_b1_n131072_int2_g32_r128", 2, 2, {}),
    ("llama3_70b_layer_b1_n131072_int4_g32_r128_pre_rope", 2, 4, {"pre_rope": True}),
    ("llama3_70b_layer_b1_n131072_int2_g32_r128_pre_rope", 2, 2, {"pre_rope": True}),
    ("paged_ragged_b64_n1k_32k_int4_g16_r16", 3, 4, {}),
    ("llama3_8b_layer_b8_n8192_int8_per_token", 1, 16, {}),
    ("llama3_8b_layer_b8_n8192_mixed24_g32_r128", 1, 6, {}),
    ("llama3_8b_layer_b8_n8192_int4_g32_r128_dense_sparse", 1, 4, {"sparse": True}),
    ("llama3_8b_layer_b8_n8192_int2_g32_r128_dense_sparse", 1, 2, {"sparse": True}),
]
STREAMING = [
    ("streaming_b16_n4096_512steps_int2_g32_r128", 4, 2),
    ("streaming_b16_n4096_512steps_fp8_e4m3", 4, 8),
    ("streaming_b16_n4096_512steps_int8_per_token", 4, 16),
]
STREAM_STEPS = 512


def make_bench_cache(w, extra: int, dev, rope_theta: float = 0.0, sparse: bool = False):
    from bit_kv_cache_16_b200 import kvq, synth
    import torch
    if w.page_size:
        table, P = synth.page_table(w, extra)
        c = kvq.Cache(w.bits, w.batch, w.num_q_heads, w.num_kv_heads, table.shape[1] * w.page_size,
                      group=w.group, residual=w.residual, page_size=w.page_size,
                      max_pages_per_seq=table.shape[1], num_pages=P, device=dev)
        c.set_page_table(torch.from_numpy(table).to(dev))
        return c
    step = max(w.group, 16)
    cap = (int(w.lengths.max()) + extra + step - 1) // step * step
    if w.bits in (8, 16):
        return kvq.Cache(w.bits, w.batch, w.num_q_heads, w.num_kv_heads, cap, group=16, residual=0, device=dev)
    # INT2, INT4 and mixed 2/4-bit
    return kvq.Cache(w.bits, w.batch, w.num_q_heads, w.num_kv_heads, cap, group=w.group, residual=w.residual,
                     device=dev, rope_theta=rope_theta, sparse=sparse)


def run_workloads(gpu, peak: float, iters: int, only=None) -> dict:
    import torch
    from bit_kv_cache_16_b200 import kvq, synth
    dev, stream = gpu.dev, gpu.stream
    res = {"iters": iters, "l2": "512 MB write then read before every timed call, outside the timed window",
           "stat": "median"}
    for name, cid, bits, opt in WORKLOADS:
        if only and name not in only:
            continue
        pre_rope, sparse = opt.get("pre_rope", False), opt.get("sparse", False)
        w = synth.make_config(cid, bits=bits, rope=not pre_rope)
        k, v, q = gpu.bf16(w.k), gpu.bf16(w.v), gpu.bf16(w.q)
        cu = torch.from_numpy(w.cu_seqlens.astype(np.int32)).to(dev)
        max_len = int(w.lengths.max())
        c = make_bench_cache(w, 0, dev, synth.ROPE_THETA_70B if pre_rope else 0.0, sparse)
        splits = kvq.kvq_decode_default_splits(c.desc, max_len)
        ws = torch.empty(max(c.workspace_bytes(splits, max_len), 16), dtype=torch.uint8, device=dev)
        out = torch.empty(w.batch, w.num_q_heads, w.head_dim, dtype=torch.float32, device=dev)
        cls = synth.token_classes(w.seed, w.lengths) if bits == 6 else None
        if bits == 6:
            dcls = torch.from_numpy(cls).to(dev)
            pre = lambda: c.quantize_prefill_mixed(k, v, dcls, cu, max_len, stream)
        else:
            pre = lambda: c.quantize_prefill(k, v, cu, max_len, stream)
        dec = lambda: c.decode_attention(q, out, w.softmax_scale, ws, splits, max_len, stream)
        for _ in range(3):
            pre()
            dec()
        torch.cuda.synchronize()
        assert c.error() == 0 and bool(torch.isfinite(out).all())
        tp = statistics.median(gpu.timed(pre, iters))
        td = statistics.median(gpu.timed(dec, iters))
        sp_bytes = sparse_bytes(w) if sparse else 0
        res[name] = {"batch": w.batch, "max_len": max_len, "decode_splits": splits,
                     "prefill": rate(tp, wl_prefill_bytes(w, cls) + sp_bytes, peak),
                     "decode": rate(td, wl_decode_bytes(w, w.lengths, cls) + sp_bytes, peak),
                     "decode_tokens_per_s": round(w.batch / (td * 1e-6), 1)}
        if bits == 6:
            G = w.group
            gb = [4 if np.any(cls[i:i + G] == 4) else 2 for i in range(0, len(cls), G)]
            res[name]["mean_stored_bits"] = round(float(np.mean(gb)), 3)
            res[name]["tokens_in_2bit_classes"] = round(float(np.mean(cls == 2)), 3)
        if cid == 2:
            res[name]["decode_80_layers_ms"] = round(80 * td / 1e3, 3)
        del c, k, v, ws
        torch.cuda.empty_cache()

    for name, cid, bits in STREAMING:
        if only and name not in only:
            continue
        w = synth.make_config(cid, bits=bits)
        k, v, q = gpu.bf16(w.k), gpu.bf16(w.v), gpu.bf16(w.q)
        cu = torch.from_numpy(w.cu_seqlens.astype(np.int32)).to(dev)
        n0 = int(w.lengths.max())
        toks = [synth.streaming_token(w, s) for s in range(STREAM_STEPS)]
        kn = gpu.bf16(np.stack([t[0] for t in toks]))
        vn = gpu.bf16(np.stack([t[1] for t in toks]))
        c = make_bench_cache(w, STREAM_STEPS, dev)
        splits = [kvq.kvq_decode_default_splits(c.desc, n0 + s + 1) for s in range(STREAM_STEPS)]
        ws = torch.empty(max(max(c.workspace_bytes(sp, n0 + STREAM_STEPS) for sp in set(splits)), 16),
                         dtype=torch.uint8, device=dev)
        out = torch.empty(w.batch, w.num_q_heads, w.head_dim, dtype=torch.float32, device=dev)

        def stream_pass(timed_pass):
            c.quantize_prefill(k, v, cu, n0, stream)
            evs = []
            for s in range(STREAM_STEPS):
                if timed_pass:
                    gpu.flush_l2()
                e = [gpu.ev() for _ in range(3)]
                e[0].record(stream)
                c.append_flush(kn[s], vn[s], stream)
                e[1].record(stream)
                c.decode_attention(q, out, w.softmax_scale, ws, splits[s], n0 + s + 1, stream)
                e[2].record(stream)
                evs.append(e)
            torch.cuda.synchronize()
            return [(e[0].elapsed_time(e[1]) * 1e3, e[1].elapsed_time(e[2]) * 1e3) for e in evs]

        stream_pass(False)
        assert c.error() == 0
        t = stream_pass(True)
        assert c.error() == 0 and bool(torch.isfinite(out).all())
        if bits in (8, 16):
            flush_steps = set()
        else:
            flush_steps = {s for s in range(STREAM_STEPS)
                           if quantized_split(n0 + s + 1, w.group, w.residual)[0]
                           != quantized_split(n0 + s, w.group, w.residual)[0]}
        plain = [s for s in range(STREAM_STEPS) if s not in flush_steps]
        mean = lambda xs: statistics.mean(xs) if xs else None
        r3 = lambda x: None if x is None else round(x, 3)
        ends = {"first_32": range(32), "last_32": range(STREAM_STEPS - 32, STREAM_STEPS)}
        decode = {}
        for key, rg in ends.items():
            us = mean([t[s][1] for s in rg])
            nbytes = round(mean([wl_decode_bytes(w, [n0 + s + 1] * w.batch) for s in rg]))
            decode[key] = rate(us, nbytes, peak)
        all_bytes = sum(wl_decode_bytes(w, [n0 + s + 1] * w.batch) for s in range(STREAM_STEPS))
        decode["all_steps"] = rate(mean([x[1] for x in t]), all_bytes / STREAM_STEPS, peak)
        res[name] = {"batch": w.batch, "start_len": n0, "steps": STREAM_STEPS, "flush_steps": len(flush_steps),
                     "append_flush_us": {"flush_steps": r3(mean([t[s][0] for s in flush_steps])),
                                         "other_steps": r3(mean([t[s][0] for s in plain]))},
                     "step_us": {"flush_steps": r3(mean([sum(t[s]) for s in flush_steps])),
                                 "other_steps": r3(mean([sum(t[s]) for s in plain])),
                                 "all": r3(mean([sum(x) for x in t]))},
                     "decode": decode,
                     "l2": "512 MB write then read before every step, outside the timed windows"}
        del c, k, v, ws
        torch.cuda.empty_cache()
    return res


def run_seqshard(gpu, rank: int, world: int, K: int, W: int, peak: float) -> dict:
    """The Llama-3-70B 131072-token INT4 sequence, split along its tokens over
    the ranks: every rank prefills its shard, then K decodes of the whole
    sequence (rank decode + all-gather of the partials + merge), timed with
    CUDA events on the stream, max over ranks."""
    import torch
    import torch.distributed as dist
    from bit_kv_cache_16_b200 import kvq, synth
    dev, stream = gpu.dev, gpu.stream
    w = synth.make_config(2, bits=4)
    k, v, cu, lens, res_r = seqshard_part(w, rank, world)
    mx = int(lens.max())
    cap = max(w.group, (mx + w.group - 1) // w.group * w.group)
    c = kvq.Cache(4, w.batch, w.num_q_heads, w.num_kv_heads, cap, group=w.group, residual=res_r, device=dev)
    c.quantize_prefill(gpu.bf16(k), gpu.bf16(v), torch.from_numpy(cu).to(dev), mx, stream)
    q = gpu.bf16(w.q)
    splits = kvq.kvq_decode_default_splits(c.desc, max(mx, 1))
    ws = torch.empty(max(c.workspace_bytes(splits, max(mx, 1)), 16), dtype=torch.uint8, device=dev)
    out = torch.empty(w.batch, w.num_q_heads, w.head_dim, dtype=torch.float32, device=dev)
    fn = lambda: sharded_step(c, q, out, w.softmax_scale, ws, splits, max(mx, 1), stream)
    for _ in range(max(W, 1)):
        fn()
    torch.cuda.synchronize()
    dist.barrier()
    us = statistics.median(gpu.timed(fn, K))
    us = max_over_ranks(us, dev, world)
    assert c.error() == 0 and bool(torch.isfinite(out).all())
    total = wl_decode_bytes(w, w.lengths)
    return {"workload": "llama3_70b_layer_b1_n131072_int4_g32_r128 split over %d ranks" % world,
            "ranks": world, "decode": rate(us, total, peak * world),
            "exchange_bytes_per_rank": int(w.batch * w.num_q_heads * (w.head_dim + 1) * 4),
            "note": "decode over the whole sequence: each rank its shard, NCCL all-gather of (out, lse), merge; "
                    "frac is against the ranks' summed HBM peak"}


def load_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary (null if absent)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            return json.load(f).get(kernel)
    except Exception:
        return None


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--splits", type=int, default=0)
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--ref-budget", type=float, default=4.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true", help="skip the per-workload section (one GPU)")
    ap.add_argument("--no-seqshard", action="store_true", help="skip the sequence-sharded leg (N > 1)")
    ap.add_argument("--workload-iters", type=int, default=0, help="timed calls per workload (default: --steps)")
    ap.add_argument("--only", default="", help="comma-separated workload keys: run these alone (no step line)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
