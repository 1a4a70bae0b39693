"""GPU parity of the pieces of sequence sharding: the decode's ln-sum-exp
output, the merge kernel, and a long sequence split over emulated ranks
(every rank's shard decoded on this one GPU, then merged), against the
oracle's unsharded cache."""
import numpy as np
import pytest
import torch

import oracle
from bit_kv_cache_16_b200 import kvq, seqshard, synth

from gpu_harness import assert_close, gpu_decode, gpu_prefill, oracle_cache, to_dev

pytestmark = pytest.mark.gpu

LSE_ATOL = 1e-3    # ln-sum-exp: its error is at most the largest score error


def _lse_decode(c, w, max_len):
    rows = w.batch * w.num_q_heads
    q = to_dev(w.q)
    out = torch.full((w.batch, w.num_q_heads, 128), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((rows,), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(max(c.workspace_bytes(0, max_len), 16), dtype=torch.uint8, device="cuda")
    c.decode_attention_lse(q, out, lse, w.softmax_scale, ws, 0, max_len)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def _logsumexp(lg):
    if lg.shape[1] == 0:
        return np.full(lg.shape[0], -np.inf)
    m = lg.max(axis=1)
    return m + np.log(np.exp(lg - m[:, None]).sum(axis=1))


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_decode_lse_is_the_softmax_denominator(bits):
    lengths = [0, 37, 300, 1029]
    R = 0 if bits == 8 else 64
    w = synth.make_workload("lse", 7400 + bits, lengths, 8, 2, bits, 32, R)
    c = gpu_prefill(w)
    oc = oracle_cache(w, c.shape.capacity)
    out, lse = _lse_decode(c, w, max(lengths))
    assert_close(out, oc.decode(w.q, w.softmax_scale))
    g = 4
    lse = lse.reshape(w.batch, w.num_q_heads)
    for b, n in enumerate(lengths):
        for h in range(w.num_kv_heads):
            if bits == 8:
                kh = oracle.e4m3_decode(oc.k_codes[b, h, :n]).astype(np.float64) * float(oc.Sk[h])
                vh = oracle.e4m3_decode(oc.v_codes[b, h, :n]).astype(np.float64) * float(oc.Sv[h])
            else:
                kh, vh = oc.units[b][h].materialize()
            _, lg = oracle.attend(kh, vh, w.q[b, h * g:(h + 1) * g], w.softmax_scale, return_logits=True)
            ref = _logsumexp(lg)
            got = lse[b, h * g:(h + 1) * g]
            if n == 0:
                assert np.all(np.isneginf(got))
            else:
                assert np.max(np.abs(got - ref)) <= LSE_ATOL, (b, h, np.max(np.abs(got - ref)))


def test_merge_kernel_formula():
    rng = np.random.default_rng(7500)
    P, rows = 3, 37
    outs = rng.standard_normal((P, rows, 128)).astype(np.float32)
    lses = (rng.standard_normal((P, rows)) * 20).astype(np.float32)
    lses[1, 5] = -np.inf                     # a part with no tokens in row 5
    lses[:, 9] = -np.inf                     # a row with no tokens anywhere
    lses[0, 11], lses[2, 11] = 80.0, -80.0   # very different weights
    d_out = torch.empty(rows, 128, dtype=torch.float32, device="cuda")
    d_lse = torch.empty(rows, dtype=torch.float32, device="cuda")
    kvq.kvq_merge_partials(torch.from_numpy(outs).cuda(), torch.from_numpy(lses).cuda(), P, rows, d_out, d_lse)
    torch.cuda.synchronize()
    o64, l64 = outs.astype(np.float64), lses.astype(np.float64)
    M = l64.max(axis=0)
    safe = np.where(np.isfinite(M), M, 0.0)
    wts = np.where(np.isfinite(l64), np.exp(l64 - safe), 0.0)
    tot = wts.sum(axis=0)
    ref = np.einsum("pr,prd->rd", wts, o64) / np.where(tot > 0, tot, 1.0)[:, None]
    ref[tot == 0] = 0.0
    ref_lse = np.where(tot > 0, safe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    got, got_lse = d_out.cpu().numpy(), d_lse.cpu().numpy()
    assert np.max(np.abs(got - ref)) <= 1e-5 * max(1.0, np.abs(ref).max())
    assert np.all(got[9] == 0.0) and np.isneginf(got_lse[9])
    fin = np.isfinite(ref_lse)
    assert np.max(np.abs(got_lse[fin] - ref_lse[fin])) <= 1e-5 * np.abs(ref_lse[fin]).max()


def _shard_workload(w, bounds_per_seq, p):
    """Rank p's part of every sequence of w as a workload of its own."""
    ks, vs, lens = [], [], []
    for b in range(w.batch):
        lo, hi = bounds_per_seq[b][p]
        ks.append(w.seq_k(b)[lo:hi])
        vs.append(w.seq_v(b)[lo:hi])
        lens.append(hi - lo)
    cu = np.zeros(w.batch + 1, np.int32)
    cu[1:] = np.cumsum(lens)
    return np.concatenate(ks), np.concatenate(vs), cu, max(lens)


@pytest.mark.parametrize("bits,G,R,parts", [(4, 32, 128, 2), (2, 32, 128, 3), (4, 16, 16, 4)])
def test_sharded_sequences_merge_to_the_unsharded_decode(bits, G, R, parts):
    """Each emulated rank holds whole key groups of every sequence (the last
    one also the window) in a cache of its own; their lse decodes merged by
    the merge kernel equal the oracle's attention over the whole sequences."""
    lengths = [4099, 1500, 200]
    w = synth.make_workload("shard", 7600 + parts, lengths, 8, 2, bits, G, R)
    bounds = [seqshard.shard_bounds(n, G, R, parts) for n in lengths]
    q = to_dev(w.q)
    rows = w.batch * w.num_q_heads
    outs = torch.empty(parts, rows, 128, dtype=torch.float32, device="cuda")
    lses = torch.empty(parts, rows, dtype=torch.float32, device="cuda")
    for p in range(parts):
        k, v, cu, mx = _shard_workload(w, bounds, p)
        cap = max(G, (mx + G - 1) // G * G)
        c = kvq.Cache(bits, w.batch, w.num_q_heads, w.num_kv_heads, cap, group=G,
                      residual=seqshard.shard_residual(p, parts, R))
        c.quantize_prefill(to_dev(k), to_dev(v), torch.from_numpy(cu).cuda(), mx)
        ws = torch.empty(max(c.workspace_bytes(0, max(mx, 1)), 16), dtype=torch.uint8, device="cuda")
        c.decode_attention_lse(q, outs[p], lses[p], w.softmax_scale, ws, 0, max(mx, 1))
        torch.cuda.synchronize()
        assert c.error() == 0
    out = torch.empty(w.batch, w.num_q_heads, 128, dtype=torch.float32, device="cuda")
    kvq.kvq_merge_partials(outs, lses, parts, rows, out)
    torch.cuda.synchronize()
    oc = oracle_cache(w, (max(lengths) + G - 1) // G * G)
    assert_close(out.cpu().numpy().astype(np.float64), oc.decode(w.q, w.softmax_scale))
    # and the unsharded GPU decode agrees with both
    c = gpu_prefill(w)
    assert_close(gpu_decode(c, w, max(lengths)), oc.decode(w.q, w.softmax_scale))


def test_decode_sharded_on_a_side_stream():
    """decode_sharded given a stream that is not torch's current one: the
    decode, the all-gather and the merge are ordered on that stream (one NCCL
    rank on this GPU), and the result equals the oracle's attention."""
    import socket

    import torch.distributed as dist
    lengths = [3000, 640]
    bits, G, R = 4, 32, 128
    w = synth.make_workload("shard_stream", 7800, lengths, 8, 2, bits, G, R)
    c = gpu_prefill(w)
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % port, rank=0, world_size=1,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        side = torch.cuda.Stream()
        q = to_dev(w.q)
        out = torch.full((w.batch, w.num_q_heads, 128), float("nan"), dtype=torch.float32, device="cuda")
        ws = torch.empty(max(c.workspace_bytes(0, max(lengths)), 16), dtype=torch.uint8, device="cuda")
        side.wait_stream(torch.cuda.current_stream())      # inputs are ready before the side stream reads them
        for _ in range(3):
            seqshard.decode_sharded(c, q, out, w.softmax_scale, ws, 0, max(lengths), stream=side)
        side.synchronize()
    finally:
        dist.destroy_process_group()
    oc = oracle_cache(w, c.shape.capacity)
    assert_close(out.cpu().numpy().astype(np.float64), oc.decode(w.q, w.softmax_scale))
