"""Benchmark of the quantized-KV decode path on B200.

One step = one pass of the whole path over one batch of the Llama-3-8B-shaped
layer workload (B=8, 32 query / 8 kv heads, d=128, INT4, G=32, R=128):
  1. quantize the prefill of 8191 tokens per sequence (per-channel key
     groups, per-token values, the last tokens into the bf16 window),
  2. append the 8192nd token, which fills the window, and flush the window's
     oldest key/value group (one launch: kvq_append_flush),
  3. decode attention over the 8192 tokens (8064 quantized + 128 window).
The L2 is flushed before phases 1 and 2 by writing a 512 MB buffer and then
reading it back (so the timed kernels start on a cold L2 that holds no dirty
lines); the flush is outside the timed windows.  Times are CUDA events on the launching stream.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
  python bench.py --sweep [--sweep-iters K]

--sweep times, on one GPU, the prefill and the decode of every named
workload (tiny check, Llama-3-8B layer, Llama-3-70B 128K at INT4 and INT2,
paged ragged batch) and the two streaming runs (INT2 and FP8, 512 steps of
append + flush + decode, flush steps reported apart), one JSON line each.

With N > 1 (torchrun) every rank runs its own batch (weak scaling; no
collective on the data path); times are the max over ranks.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantized-KV decode attention: us/step, KV GB/s and % of B200 HBM peak"
WORKLOAD = "llama3_8b_layer_decode_b8_n8192_int4_g32_r128"
B, HQ, HKV, D, N_CTX, G, R = 8, 32, 8, 128, 8192, 32, 128
N_PREFILL = N_CTX - 1
FALLBACK_HBM_GBS = 6650.0
# libkvq launches per step: prefill, append + flush, decode split + combine
LAUNCHES_PER_STEP = 4


def measured_peak_gbs():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def algorithmic_bytes():
    """Bytes the method must move per phase (fp16 scale/zero, bf16 window)."""
    units = B * HKV
    nq_pre = G * ((N_PREFILL - R) // G)                  # 8032
    r_pre = N_PREFILL - nq_pre                           # 159
    prefill_read = units * N_PREFILL * D * 2 * 2
    prefill_write = units * (nq_pre * (D // 2) * 2 + (nq_pre // G) * 2 * D * 2 + nq_pre * 4 + r_pre * D * 2 * 2)
    nq = G * ((N_CTX - R) // G)                          # 8064
    r = N_CTX - nq                                       # 128
    decode = units * (nq * (D // 2) * 2 + (nq // G) * 2 * D * 2 + nq * 4 + r * D * 2 * 2) + B * HQ * D * 2
    append = units * D * 2 * 2 * 2                       # read + write one token of K and V
    flush = units * (G * D * 2 * 2 + G * (D // 2) * 2 + 2 * D * 2 + G * 4)
    return {"prefill": prefill_read + prefill_write, "append_flush": append + flush, "decode": decode}


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
    """Run the oracle's whole step (prefill 8191, append, flush, decode) on
    (b, kv) units until budget_s has elapsed (at least one wave of `threads`
    units); return the time per full step extrapolated from the units done,
    and their number.  The units are independent and the C oracle releases
    the GIL, so `threads` Python threads run that many units at once, each
    through the unchanged oracle."""
    from concurrent.futures import ThreadPoolExecutor
    import oracle
    from bit_kv_cache_16_b200 import synth
    kn, vn = synth.streaming_token(w, 0)
    order = [(b, h) for b in range(B) for h in range(HKV)]
    g = HQ // HKV

    def unit(bh):
        b, h = bh
        u = oracle.Unit(4, D, G, R, N_CTX)
        lo = int(w.cu_seqlens[b])
        u.prefill(w.k[lo:lo + N_PREFILL, h, :], w.v[lo:lo + N_PREFILL, h, :])
        u.append(kn[b, h], vn[b, h])
        u.flush()
        u.decode(w.q[b, h * g:(h + 1) * g, :], w.softmax_scale)

    t0 = time.perf_counter()
    done = 0
    with ThreadPoolExecutor(max_workers=threads) as ex:
        while done < len(order):
            wave = order[done:done + threads]
            list(ex.map(unit, wave))
            done += len(wave)
            if time.perf_counter() - t0 >= budget_s:
                break
    el = time.perf_counter() - t0
    return el / done * len(order), done


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from bit_kv_cache_16_b200 import synth
    import oracle
    oracle.build()
    w = synth.make_config(1)
    cores = host_cores()
    per_step = []
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
                             "sample": "%d of %d (sequence, kv head) units per step on %d threads, extrapolated"
                                       % (units, B * HKV, cores)},
            "e2e": {"value": us, "unit": "us/step", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# Cross-rank pieces (weak scaling: every rank runs its own batch)
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


# ---------------------------------------------------------------------------
# GPU leg
# ---------------------------------------------------------------------------

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

    w = rank_workload(rank)
    kn, vn = synth.streaming_token(w, 0)
    to_pinned = lambda a: torch.from_numpy(np.ascontiguousarray(a.view(np.int16))).pin_memory()
    hk, hv, hq = to_pinned(w.k), to_pinned(w.v), to_pinned(w.q)
    hkn, hvn = to_pinned(kn), to_pinned(vn)
    hcu = torch.from_numpy(w.cu_seqlens.astype(np.int32)).pin_memory()
    dk, dv, dq = hk.to(dev), hv.to(dev), hq.to(dev)
    dkn, dvn, dcu = hkn.to(dev), hvn.to(dev), hcu.to(dev)

    cache = kvq.Cache(kvq.KVQ_FORMAT_INT4, B, HQ, HKV, N_CTX, group=G, residual=R, device=dev)
    splits = args.splits or kvq.kvq_decode_default_splits(cache.desc, N_CTX)
    ws = torch.empty(cache.workspace_bytes(splits, N_CTX), dtype=torch.uint8, device=dev)
    out = torch.empty(B, HQ, D, dtype=torch.float32, device=dev)
    hout = torch.empty(B, HQ, D, dtype=torch.float32).pin_memory()
    l2 = torch.empty(512 * 2 ** 20, dtype=torch.uint8, device=dev)
    l2_words = l2.view(torch.int64)

    def flush_l2():
        # Write 512 MB (evicts everything), then read it back: the read makes
        # the L2 write back its dirty lines here, so the next timed kernel
        # starts on a cold, clean L2 instead of paying for this buffer's
        # write-back.
        l2.zero_()
        l2_words.sum()

    stream = torch.cuda.current_stream()
    scale = 1.0 / np.sqrt(D)

    def ev():
        return torch.cuda.Event(enable_timing=True)

    def step(timed):
        flush_l2()
        e = [ev() for _ in range(5)]
        e[0].record(stream)
        cache.quantize_prefill(dk, dv, dcu, N_PREFILL, stream)
        e[1].record(stream)
        flush_l2()
        e[2].record(stream)
        cache.append_flush(dkn, dvn, stream)
        e[3].record(stream)
        cache.decode_attention(dq, out, scale, ws, splits, N_CTX, stream)
        e[4].record(stream)
        return e

    # correctness guard for this exact launch configuration (state, not timing)
    step(False)
    torch.cuda.synchronize()
    assert cache.error() == 0
    assert torch.isfinite(out).all()

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    evs = [step(True) for _ in range(args.steps)]
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    ph = {"prefill": [], "append_flush": [], "decode": []}
    for e in evs:
        ph["prefill"].append(e[0].elapsed_time(e[1]) * 1e3)
        ph["append_flush"].append(e[2].elapsed_time(e[3]) * 1e3)
        ph["decode"].append(e[3].elapsed_time(e[4]) * 1e3)
    step_us = max_over_ranks(sum(sum(v) for v in ph.values()) / args.steps, dev, world)

    # end to end through the public API with host buffers (pinned): per step
    # copy the prefill K/V, lengths, query and the new token in, read `out` back
    h2d = sum(t.numel() * t.element_size() for t in (hk, hv, hcu, hq, hkn, hvn))
    d2h = hout.numel() * hout.element_size()

    def e2e_step():
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        dcu.copy_(hcu, non_blocking=True)
        dq.copy_(hq, non_blocking=True)
        dkn.copy_(hkn, non_blocking=True)
        dvn.copy_(hvn, non_blocking=True)
        cache.quantize_prefill(dk, dv, dcu, N_PREFILL, stream)
        cache.append_flush(dkn, dvn, stream)
        cache.decode_attention(dq, out, scale, ws, splits, N_CTX, stream)
        hout.copy_(out, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = ev(), ev()
    flush_l2()
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_us = max_over_ranks(e0.elapsed_time(e1) * 1e3 / args.steps, dev, world)

    if rank == 0:
        peak, peak_kind = measured_peak_gbs()
        ab = algorithmic_bytes()
        kern = {}
        for k, v in ph.items():
            us = statistics.mean(v)
            gbs = ab[k] / (us * 1e-6) / 1e9
            kern[k] = {"us": round(us, 3), "bytes": ab[k], "GB/s": round(gbs, 1), "frac": round(gbs / peak, 4)}
        dom = max(kern, key=lambda k: kern[k]["us"])
        traffic = load_traffic(dom)
        line = {"metric": METRIC, "value": round(step_us, 3), "unit": "us/step", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_us / 1e3, 6),
                "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "int4-codes/f16-mma/f32",
                "data": "synthetic (seeded; K outlier channels x20, V heavy tokens x5, q outliers x5)",
                "config": {"workload": WORKLOAD, "batch": B, "seq_len": N_CTX, "q_heads": HQ, "kv_heads": HKV,
                           "bits": 4, "group": G, "residual": R, "decode_splits": splits,
                           "l2": "512 MB write then read before prefill and before append (cold, clean L2), outside the timed windows",
                           "parallelism": "dp%d (independent batch per GPU)" % world},
                "phases": kern,
                "decode_tokens_per_s": round(world * B / (kern["decode"]["us"] * 1e-6), 1),
                "roofline": {"bound": "hbm", "kernel": dom, "achieved": kern[dom]["GB/s"],
                             "peak": peak, "peak_kind": peak_kind + " hbm_gbs (copy)", "unit": "GB/s",
                             "frac": kern[dom]["frac"], "traffic": traffic},
                "decode_roofline": {"bound": "hbm", "achieved": kern["decode"]["GB/s"], "peak": peak,
                                    "unit": "GB/s", "frac": kern["decode"]["frac"],
                                    "traffic": load_traffic("decode")},
                "e2e": {"value": round(e2e_us, 3), "unit": "us/step", "h2d_bytes_per_step": h2d,
                        "d2h_bytes_per_step": d2h},
                "gpu_launches": args.steps * LAUNCHES_PER_STEP,
                "clocks": clocks}
        if not args.no_cpu_baseline:
            t, units = oracle_step_sample(w, budget_s=args.cpu_budget)
            line["cpu_baseline"] = {"value": round(t * 1e6, 1), "unit": "us/step", "cores": 1, "kind": "oracle",
                                    "sample": "%d of %d (sequence, kv head) units of one step, extrapolated"
                                              % (units, B * HKV)}
            cores = host_cores()
            t, units = oracle_step_sample(w, budget_s=args.cpu_budget, threads=cores)
            line["cpu_baseline"]["all_cores"] = {
                "value": round(t * 1e6, 1), "unit": "us/step", "cores": cores,
                "sample": "%d of %d units of one step on %d threads, extrapolated" % (units, B * HKV, cores)}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# --sweep: prefill and decode of every named workload, and the streaming runs
# step by step (flush steps apart from the others).  One JSON line each.
# ---------------------------------------------------------------------------

SWEEP = [  # (workload, config id, bits)
    ("tiny_b1_n512_int2_g32_r32", 0, 2),
    ("llama3_8b_layer_b8_n8192_int4_g32_r128", 1, 4),
    ("llama3_70b_layer_b1_n131072_int4_g32_r128", 2, 4),
    ("llama3_70b_layer_b1_n131072_int2_g32_r128", 2, 2),
    ("paged_ragged_b64_n1k_32k_int4_g16_r16", 3, 4),
]
STREAMING = [
    ("streaming_b16_n4096_512steps_int2_g32_r128", 4, 2),
    ("streaming_b16_n4096_512steps_fp8_e4m3", 4, 8),
]
STREAM_STEPS = 512


def quantized_split(n: int, group: int, residual: int):
    """(n_q, r): quantized tokens and window tokens of a sequence of n tokens."""
    nq = group * (max(n - residual, 0) // group)
    return nq, n - nq


def _cache_bytes(w, n: int) -> int:
    """Bytes of one (sequence, kv head) cache of n tokens: codes, fp16
    scale/zero and the bf16 window (e4m3 codes only for FP8)."""
    D = w.head_dim
    if w.bits == 8:
        return n * D * 2
    nq, r = quantized_split(n, w.group, w.residual)
    return nq * D * w.bits // 8 * 2 + (nq // w.group) * 2 * D * 2 + nq * 4 + r * D * 2 * 2


def sweep_decode_bytes(w, lengths) -> int:
    """Algorithmic bytes of one decode call at these sequence lengths."""
    return w.batch * w.num_q_heads * w.head_dim * 2 + sum(w.num_kv_heads * _cache_bytes(w, int(n)) for n in lengths)


def sweep_prefill_bytes(w) -> int:
    """Algorithmic bytes of the prefill: read K and V once, write the cache."""
    return sum(w.num_kv_heads * (int(n) * w.head_dim * 2 * 2 + _cache_bytes(w, int(n))) for n in w.lengths)


def run_sweep(args):
    import torch
    from bit_kv_cache_16_b200 import kvq, synth
    from bit_kv_cache_16_b200.build import build_libkvq

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    build_libkvq()
    kvq.load()
    peak, peak_kind = measured_peak_gbs()
    stream = torch.cuda.current_stream()
    l2 = torch.empty(512 * 2 ** 20, dtype=torch.uint8, device=dev)
    l2_words = l2.view(torch.int64)
    iters = args.sweep_iters

    def flush_l2():
        l2.zero_()
        l2_words.sum()

    def dev_bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a.view(np.int16))).to(dev)

    def make_cache(w, extra):
        if w.page_size:
            table, P = synth.page_table(w, extra)
            c = kvq.Cache(w.bits, w.batch, w.num_q_heads, w.num_kv_heads, table.shape[1] * w.page_size,
                          group=w.group, residual=w.residual, page_size=w.page_size,
                          max_pages_per_seq=table.shape[1], num_pages=P, device=dev)
            c.set_page_table(torch.from_numpy(table).to(dev))
            return c
        step = max(w.group, 16)
        cap = (int(w.lengths.max()) + extra + step - 1) // step * step
        if w.bits == 8:
            return kvq.Cache(8, w.batch, w.num_q_heads, w.num_kv_heads, cap, group=32, residual=0, device=dev)
        return kvq.Cache(w.bits, w.batch, w.num_q_heads, w.num_kv_heads, cap, group=w.group, residual=w.residual,
                         device=dev)

    def timed(fn, n):
        """Device time of fn (us) n times, each after an L2 flush outside the window."""
        evs = []
        for _ in range(n):
            flush_l2()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            evs.append((e0, e1))
        torch.cuda.synchronize()
        return [a.elapsed_time(b) * 1e3 for a, b in evs]

    def rate(us, nbytes):
        gbs = nbytes / (us * 1e-6) / 1e9
        return {"us": round(us, 3), "bytes": nbytes, "GB/s": round(gbs, 1), "frac": round(gbs / peak, 4)}

    common = {"peak_gbs": peak, "peak_kind": peak_kind, "iters": iters,
              "l2": "512 MB write then read before every timed call, outside the timed window"}
    for name, cid, bits in SWEEP:
        w = synth.make_config(cid, bits=bits)
        k, v, q = dev_bf16(w.k), dev_bf16(w.v), dev_bf16(w.q)
        cu = torch.from_numpy(w.cu_seqlens.astype(np.int32)).to(dev)
        max_len = int(w.lengths.max())
        c = make_cache(w, 0)
        splits = kvq.kvq_decode_default_splits(c.desc, max_len)
        ws = torch.empty(max(c.workspace_bytes(splits, max_len), 16), dtype=torch.uint8, device=dev)
        out = torch.empty(w.batch, w.num_q_heads, w.head_dim, dtype=torch.float32, device=dev)
        pre = lambda: c.quantize_prefill(k, v, cu, max_len, stream)
        dec = lambda: c.decode_attention(q, out, w.softmax_scale, ws, splits, max_len, stream)
        for _ in range(3):
            pre()
            dec()
        torch.cuda.synchronize()
        assert c.error() == 0 and bool(torch.isfinite(out).all())
        tp = statistics.median(timed(pre, iters))
        td = statistics.median(timed(dec, iters))
        line = {"sweep": name, "batch": w.batch, "max_len": max_len, "decode_splits": splits,
                "prefill": rate(tp, sweep_prefill_bytes(w)), "decode": rate(td, sweep_decode_bytes(w, w.lengths)),
                "decode_tokens_per_s": round(w.batch / (td * 1e-6), 1), **common}
        print(json.dumps(line), flush=True)
        del c, k, v, ws
        torch.cuda.empty_cache()

    for name, cid, bits in STREAMING:
        w = synth.make_config(cid, bits=bits)
        k, v, q = dev_bf16(w.k), dev_bf16(w.v), dev_bf16(w.q)
        cu = torch.from_numpy(w.cu_seqlens.astype(np.int32)).to(dev)
        n0 = int(w.lengths.max())
        toks = [synth.streaming_token(w, s) for s in range(STREAM_STEPS)]
        kn = dev_bf16(np.stack([t[0] for t in toks]))
        vn = dev_bf16(np.stack([t[1] for t in toks]))
        c = make_cache(w, STREAM_STEPS)
        splits = [kvq.kvq_decode_default_splits(c.desc, n0 + s + 1) for s in range(STREAM_STEPS)]
        ws = torch.empty(max(max(c.workspace_bytes(sp, n0 + STREAM_STEPS) for sp in set(splits)), 16),
                         dtype=torch.uint8, device=dev)
        out = torch.empty(w.batch, w.num_q_heads, w.head_dim, dtype=torch.float32, device=dev)

        def stream_pass(timed_pass):
            c.quantize_prefill(k, v, cu, n0, stream)
            evs = []
            for s in range(STREAM_STEPS):
                if timed_pass:
                    flush_l2()
                e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
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
        if bits == 8:
            flush_steps = set()
        else:
            flush_steps = {s for s in range(STREAM_STEPS)
                           if quantized_split(n0 + s + 1, w.group, w.residual)[0]
                           != quantized_split(n0 + s, w.group, w.residual)[0]}
        plain = [s for s in range(STREAM_STEPS) if s not in flush_steps]
        mean = lambda xs: statistics.mean(xs) if xs else None
        r2 = lambda x: None if x is None else round(x, 3)
        ends = {"first_32": range(32), "last_32": range(STREAM_STEPS - 32, STREAM_STEPS)}
        decode = {}
        for key, rg in ends.items():
            us = mean([t[s][1] for s in rg])
            nbytes = round(mean([sweep_decode_bytes(w, [n0 + s + 1] * w.batch) for s in rg]))
            decode[key] = rate(us, nbytes)
        line = {"sweep": name, "batch": w.batch, "start_len": n0, "steps": STREAM_STEPS,
                "flush_steps": len(flush_steps),
                "append_flush_us": {"flush_steps": r2(mean([t[s][0] for s in flush_steps])),
                                    "other_steps": r2(mean([t[s][0] for s in plain]))},
                "decode_us_mean": r2(mean([x[1] for x in t])),
                "step_us": {"flush_steps": r2(mean([sum(t[s]) for s in flush_steps])),
                            "other_steps": r2(mean([sum(t[s]) for s in plain]))},
                "decode": decode, **common}
        line["iters"] = 1
        line["l2"] = "512 MB write then read before every step, outside the timed windows"
        print(json.dumps(line), flush=True)
        del c, k, v, ws
        torch.cuda.empty_cache()


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
    ap.add_argument("--sweep", action="store_true",
                    help="time prefill and decode on every named workload and the streaming runs (one GPU)")
    ap.add_argument("--sweep-iters", type=int, default=50)
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    elif args.sweep:
        run_sweep(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
