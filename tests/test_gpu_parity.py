"""CUDA path vs the CPU oracle, through the C ABI, on seeded inputs.

Codes, scales, zero points, window slots and counters must match bit for
bit; decode outputs within max-abs 2e-3 and cosine 0.9999 per row.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_kv_cache_16_b200 import kvq, synth

from gpu_harness import (assert_close, assert_fp8_state, assert_unit_state, gpu_decode, gpu_prefill, heads_of,
                         make_gpu_cache, oracle_cache, round_up, to_dev)
from layout import GpuState

pytestmark = pytest.mark.gpu


def _all_units(w):
    return [(b, h) for b in range(w.batch) for h in range(w.num_kv_heads)]


def _run_prefill_decode(w, units=None, num_splits=0, check_state=True):
    c = gpu_prefill(w)
    st = GpuState(c)
    oc = oracle_cache(w, c.shape.capacity, units=units)
    units = units or _all_units(w)
    if check_state:
        for b, h in units:
            assert_unit_state(st, oc, b, h)
    out = gpu_decode(c, w, int(w.lengths.max(initial=0)), num_splits)
    ref = oc.decode(w.q, w.softmax_scale, units=units)
    assert_close(out, ref, rows=heads_of(w, units))
    assert c.error() == 0
    return out, ref


# ---------------------------------------------------------------------------
# Small cases: several tiles, ragged tails, every GQA ratio, group and window
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("G,R", [(32, 128), (32, 32), (16, 16), (64, 0), (128, 64), (16, 0)])
def test_ragged_prefill_and_decode(bits, G, R):
    lengths = [0, 1, 15, 16, 17, R + G - 1, R + G, R + G + 1, 3 * G + R + 5, 700]
    w = synth.make_workload("ragged", 1000 + G + R, lengths, 8, 2, bits, G, R)
    _run_prefill_decode(w)


@pytest.mark.parametrize("gq", [1, 2, 4, 8])
@pytest.mark.parametrize("bits", [2, 4])
def test_gqa_ratios(gq, bits):
    w = synth.make_workload("gqa", 2000 + gq, [517, 1024, 260], 2 * gq, 2, bits, 32, 32)
    _run_prefill_decode(w)


def test_tiny_config_int2():
    """The tiny KIVI check: B=1, one head, n=512, INT2, G=32, R=32."""
    w = synth.make_config(0)
    out, ref = _run_prefill_decode(w)
    assert out.shape == (1, 1, 128)


@pytest.mark.parametrize("num_splits", [2, 3, 7, 33, 1000])
def test_split_count_does_not_change_result(num_splits):
    w = synth.make_workload("splits", 3000, [4000, 1500], 8, 1, 4, 32, 128)
    _run_prefill_decode(w, num_splits=num_splits)


def test_workspace_reuse_across_calls():
    """Two decodes with different queries on one workspace: the second call
    merges only its own partials, never ones left by the first."""
    w = synth.make_workload("reuse", 3050, [4000, 1500, 900], 8, 2, 4, 32, 128)
    c = gpu_prefill(w)
    oc = oracle_cache(w, c.shape.capacity)
    max_len = int(w.lengths.max())
    ws = torch.empty(c.workspace_bytes(0, max_len), dtype=torch.uint8, device="cuda")
    rng = np.random.default_rng(7)
    for trial in range(3):
        q = w.q if trial == 0 else torch.from_numpy(rng.standard_normal(w.q.shape).astype(np.float32)) \
            .to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        out = torch.full((w.batch, w.num_q_heads, 128), float("nan"), dtype=torch.float32, device="cuda")
        c.decode_attention(to_dev(q), out, w.softmax_scale, ws, 0, max_len)
        torch.cuda.synchronize()
        assert_close(out.cpu().numpy().astype(np.float64), oc.decode(q, w.softmax_scale))
    assert c.error() == 0


def test_extreme_values_and_constant_groups():
    """Constant key groups (scale 0), huge and tiny magnitudes, -0."""
    w = synth.make_workload("extreme", 3100, [320, 96], 4, 1, 4, 32, 32)
    k = synth.bf16_bits_to_f32(w.k).copy()
    v = synth.bf16_bits_to_f32(w.v).copy()
    k[:32] = 0.75                      # first group of sequence 0 constant
    k[32:64, :, :8] = -0.0
    k[64:96] *= 1e3
    v[100:110] *= 1e-4
    v[110:120] = 0.0
    to_bits = lambda a: torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy() \
        .view(np.uint16)
    w.k, w.v = to_bits(k), to_bits(v)
    _run_prefill_decode(w)


# ---------------------------------------------------------------------------
# Streaming: append + flush equals the oracle's state machine
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("bits,G,R", [(2, 32, 128), (4, 16, 16), (4, 32, 0)])
def test_streaming_append_flush(bits, G, R, fused):
    B, steps = 3, 2 * (R + G) + 7
    w = synth.make_workload("stream", 4000 + bits + G, [R + 3, 2 * G + R, 5 * G + R + 9], 8, 2, bits, G, R)
    c = gpu_prefill(w, extra_tokens=steps)
    oc = oracle_cache(w, c.shape.capacity)
    for step in range(steps):
        kn, vn = synth.streaming_token(w, step)
        if fused:
            c.append_flush(to_dev(kn), to_dev(vn))
        else:
            c.append_token(to_dev(kn), to_dev(vn))
            c.flush_group()
        oc.append(kn, vn)
        oc.flush()
        if step % 11 == 0 or step == steps - 1:
            torch.cuda.synchronize()
            st = GpuState(c)
            for b in range(B):
                for h in range(2):
                    assert_unit_state(st, oc, b, h)
            max_len = int(w.lengths.max()) + step + 1
            out = gpu_decode(c, w, max_len)
            assert_close(out, oc.decode(w.q, w.softmax_scale))
    assert c.error() == 0


def test_append_without_flush_reports_full_window():
    w = synth.make_workload("full", 4100, [32 + 31], 2, 1, 2, 32, 32)   # window holds R+G-1
    c = gpu_prefill(w, extra_tokens=4)
    kn, vn = synth.streaming_token(w, 0)
    c.append_token(to_dev(kn), to_dev(vn))       # fills the window (R+G)
    assert c.error() == 0
    c.append_token(to_dev(kn), to_dev(vn))       # no flush: must be refused
    assert c.error() & kvq.KVQ_DEVERR_APPEND_FULL
    torch.cuda.synchronize()
    assert GpuState(c).seq_len[0] == 64
    c.clear_error()
    c.flush_group()
    c.append_token(to_dev(kn), to_dev(vn))
    assert c.error() == 0 and GpuState(c).seq_len[0] == 65


@pytest.mark.parametrize("bits,G,R", [(4, 16, 16), (2, 32, 32)])
def test_prefill_batch_of_1100_ragged_sequences(bits, G, R):
    """1100 ragged sequences of 0 to 96 tokens: every state counter is
    checked, and codes, scales, window and decode on sampled units."""
    u = synth.draw_uniform(4100 + G, 6, 0, 1100)
    lengths = np.floor(u * 97).astype(np.int64)
    lengths[[0, 1023, 1024]] = [96, 0, 95]
    w = synth.make_workload("many", 4100 + G, lengths, 2, 1, bits, G, R)
    units = [(b, 0) for b in (0, 1, 2, 511, 1022, 1023, 1024, 1025, 1050, 1099)]
    c = gpu_prefill(w)
    st = GpuState(c)
    oc = oracle_cache(w, c.shape.capacity, units=units)
    for b in range(w.batch):
        n = int(lengths[b])
        assert st.seq_len[b] == n and st.n_quant[b] == G * (max(n - R, 0) // G), b
    for b, h in units:
        assert_unit_state(st, oc, b, h)
    out = gpu_decode(c, w, int(lengths.max()))
    assert_close(out, oc.decode(w.q, w.softmax_scale, units=units), rows=heads_of(w, units))
    assert c.error() == 0


@pytest.mark.parametrize("bits", [4, 8])
def test_prefill_rejects_sequences_longer_than_max_len(bits):
    """max_len bounds the lengths: a longer sequence is flagged and stored
    empty, like one above the capacity, and the others are quantized as if it
    were not there (for FP8 it takes no part in the amax either)."""
    w = synth.make_workload("under", 4150, [700, 300, 517], 4, 2, bits, 32, 0 if bits == 8 else 64)
    c = make_gpu_cache(w)
    cu = torch.from_numpy(w.cu_seqlens.astype(np.int32)).cuda()
    c.quantize_prefill(to_dev(w.k), to_dev(w.v), cu, 517)
    torch.cuda.synchronize()
    assert c.error() & kvq.KVQ_DEVERR_PREFILL_LEN
    st = GpuState(c)
    # the oracle sees sequence 0 as empty and the other two unchanged
    k_o, v_o = w.k[700:], w.v[700:]
    cu_o = np.array([0, 0, 300, 817], dtype=np.int32)
    if bits == 8:
        oc = oracle.FP8Cache(3, 4, 2, 128, c.shape.capacity)
        oc.prefill(k_o, v_o, cu_o)
        assert_fp8_state(st, oc, _all_units(w))
    else:
        oc = oracle.Cache(bits, 3, 4, 2, 128, 32, 64, c.shape.capacity)
        oc.prefill(k_o, v_o, cu_o)
        for b, h in _all_units(w):
            assert_unit_state(st, oc, b, h)
    out = gpu_decode(c, w, 517)
    assert_close(out, oc.decode(w.q, w.softmax_scale))


def test_prefill_longer_than_capacity_is_rejected():
    w = synth.make_workload("long", 4200, [100, 40], 2, 1, 4, 32, 32)
    c = make_gpu_cache(w, capacity=64)
    cu = torch.from_numpy(w.cu_seqlens.astype(np.int32)).cuda()
    c.quantize_prefill(to_dev(w.k), to_dev(w.v), cu, 100)
    assert c.error() & kvq.KVQ_DEVERR_PREFILL_LEN
    st = GpuState(c)
    assert st.seq_len[0] == 0 and st.seq_len[1] == 40


def test_capacity_reached_on_append():
    w = synth.make_workload("cap", 4300, [60], 2, 1, 4, 32, 0)
    c = make_gpu_cache(w, capacity=64)
    cu = torch.from_numpy(w.cu_seqlens.astype(np.int32)).cuda()
    c.quantize_prefill(to_dev(w.k), to_dev(w.v), cu, 60)
    kn, vn = synth.streaming_token(w, 0)
    for _ in range(4):
        c.append_token(to_dev(kn), to_dev(vn))
        c.flush_group()
    assert c.error() == 0
    c.append_token(to_dev(kn), to_dev(vn))
    assert c.error() & kvq.KVQ_DEVERR_APPEND_FULL


# ---------------------------------------------------------------------------
# Paged cache
# ---------------------------------------------------------------------------

def test_paged_matches_oracle():
    w = synth.make_workload("paged", 5000, [0, 5, 31, 32, 33, 250, 1037], 8, 2, 4, 16, 16, page_size=16)
    _run_prefill_decode(w)


@pytest.mark.parametrize("fused", [False, True])
def test_paged_streaming(fused):
    w = synth.make_workload("paged_stream", 5100, [40, 300], 4, 1, 4, 16, 16, page_size=16)
    steps = 50
    c = gpu_prefill(w, extra_tokens=steps)
    oc = oracle_cache(w, c.shape.capacity)
    for step in range(steps):
        kn, vn = synth.streaming_token(w, step)
        if fused:
            c.append_flush(to_dev(kn), to_dev(vn))
        else:
            c.append_token(to_dev(kn), to_dev(vn))
            c.flush_group()
        oc.append(kn, vn)
        oc.flush()
    torch.cuda.synchronize()
    st = GpuState(c)
    for b in range(2):
        assert_unit_state(st, oc, b, 0)
    out = gpu_decode(c, w, 300 + steps)
    assert_close(out, oc.decode(w.q, w.softmax_scale))
    assert c.error() == 0


@pytest.mark.parametrize("hkv,bits,G,R", [(8, 4, 32, 128), (8, 2, 16, 0), (16, 4, 32, 32), (3, 2, 64, 64)])
def test_append_flush_equals_two_calls(hkv, bits, G, R):
    """The one-launch append+flush leaves every cache region byte-identical
    to append_token followed by flush_group (one cluster of H_kv CTAs per
    sequence for H_kv <= 8, the two calls beyond)."""
    lens = [R + G - 2, 3 * G + R, 5 * G + R + 3]
    w = synth.make_workload("fused", 5300 + hkv + G, lens, 4 * hkv if hkv <= 4 else hkv, hkv, bits, G, R)
    steps = 2 * (R + G) + 5
    a = gpu_prefill(w, extra_tokens=steps)
    f = gpu_prefill(w, extra_tokens=steps)
    for step in range(steps):
        kn, vn = synth.streaming_token(w, step)
        kd, vd = to_dev(kn), to_dev(vn)
        a.append_token(kd, vd)
        a.flush_group()
        f.append_flush(kd, vd)
    torch.cuda.synchronize()
    for name in ("k_codes", "k_meta", "v_codes", "v_meta", "k_res", "v_res", "seq_len", "n_quant"):
        assert torch.equal(a.region(name), f.region(name)), name
    assert a.error() == 0 and f.error() == 0


def test_append_flush_errors_match_two_calls():
    """Capacity reached: the same error bit and the same state."""
    w = synth.make_workload("fused_cap", 5400, [60], 2, 1, 4, 32, 0)
    caches = []
    for fused in (False, True):
        c = make_gpu_cache(w, capacity=64)
        cu = torch.from_numpy(w.cu_seqlens.astype(np.int32)).cuda()
        c.quantize_prefill(to_dev(w.k), to_dev(w.v), cu, 60)
        kn, vn = synth.streaming_token(w, 0)
        for _ in range(5):
            if fused:
                c.append_flush(to_dev(kn), to_dev(vn))
            else:
                c.append_token(to_dev(kn), to_dev(vn))
                c.flush_group()
        caches.append(c)
    a, f = caches
    assert a.error() & kvq.KVQ_DEVERR_APPEND_FULL and f.error() == a.error()
    for name in ("seq_len", "n_quant", "k_codes", "k_res"):
        assert torch.equal(a.region(name), f.region(name)), name


def test_paged_bad_page_is_flagged_not_read():
    w = synth.make_workload("paged_bad", 5200, [200], 4, 1, 4, 16, 16, page_size=16)
    c = gpu_prefill(w)
    assert c.error() == 0
    pt = c.region("page_table").view(torch.int32)
    pt[3] = c.shape.num_pages + 7           # out of range
    out = gpu_decode(c, w, 200)
    assert c.error() & kvq.KVQ_DEVERR_PAGE_RANGE
    assert np.all(np.isfinite(out))


# ---------------------------------------------------------------------------
# FP8-E4M3 comparison cache
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("lengths", [[4096, 1000, 17], [1, 16, 33, 250]])
def test_fp8_prefill_decode(lengths):
    w = synth.make_workload("fp8", 6000 + len(lengths), lengths, 8, 2, 8, 16, 0)
    c = gpu_prefill(w, extra_tokens=20)
    oc = oracle_cache(w, c.shape.capacity)
    st = GpuState(c)
    assert_fp8_state(st, oc, _all_units(w))
    out = gpu_decode(c, w, max(lengths))
    assert_close(out, oc.decode(w.q, w.softmax_scale))
    for step in range(20):
        kn, vn = synth.streaming_token(w, step)
        c.append_token(to_dev(kn), to_dev(vn))
        c.flush_group()
        oc.append(kn, vn)
    torch.cuda.synchronize()
    assert_fp8_state(GpuState(c), oc, _all_units(w))
    out = gpu_decode(c, w, max(lengths) + 20)
    assert_close(out, oc.decode(w.q, w.softmax_scale))
    assert c.error() == 0


# ---------------------------------------------------------------------------
# Empty batch member and zero query
# ---------------------------------------------------------------------------

def test_empty_sequences_decode_to_zero():
    """All sequences empty.  The K/V inputs must still be valid pointers (a
    zero-element torch tensor has none), so one dummy row is passed."""
    w = synth.make_workload("empty", 7000, [0, 0], 4, 1, 4, 32, 32)
    c = make_gpu_cache(w, capacity=64)
    dummy = torch.zeros(1, 1, 128, dtype=torch.int16, device="cuda")
    cu = torch.zeros(3, dtype=torch.int32, device="cuda")
    c.quantize_prefill(dummy, dummy, cu, 0)
    out = gpu_decode(c, w, 0)
    assert np.all(out == 0.0)
    assert c.error() == 0


@pytest.mark.parametrize("bits", [4, 2, 8])
def test_inconsistent_state_is_flagged_and_skipped(bits):
    """seq_len / n_quant that no prefill, append or flush can produce
    (seq_len beyond the capacity, n_quant beyond seq_len, n_quant off a group
    boundary): the decode sets KVQ_DEVERR_STATE, gives those sequences zero
    rows, and leaves every other sequence's output as the oracle computes it;
    a flush on such a state sets the bit and changes nothing."""
    lengths = [300, 500, 200, 700]
    R = 0 if bits == 8 else 32
    w = synth.make_workload("badstate", 4700 + bits, lengths, 8, 2, bits, 32, R)
    c = gpu_prefill(w)
    cap = c.shape.capacity
    ok = [0, 3]
    if bits == 8:
        bad = {1: (cap + 5, cap + 5), 2: (-3, -3)}
    else:
        bad = {1: (cap + 5, 480),               # seq_len beyond the capacity
               2: (200, 232)}                   # n_quant beyond seq_len
    seq_len, n_quant = c.seq_len(), c.n_quant()
    for b, (n, nq) in bad.items():
        seq_len[b] = n
        n_quant[b] = nq
    torch.cuda.synchronize()
    out = gpu_decode(c, w, cap)
    assert c.error() & kvq.KVQ_DEVERR_STATE
    oc = oracle_cache(w, cap)
    units = [(b, h) for b in ok for h in range(w.num_kv_heads)]
    assert_close(out, oc.decode(w.q, w.softmax_scale, units=units), rows=heads_of(w, units))
    for b in bad:
        assert np.all(out[b] == 0.0)
    if bits != 8:
        # a window that looks full (seq_len - n_quant = R + G) over an n_quant
        # off a group boundary: the flush refuses it
        c.clear_error()
        before = GpuState(c)
        seq_len[0] = 17 + R + 32
        n_quant[0] = 17
        torch.cuda.synchronize()
        c.flush_group()
        torch.cuda.synchronize()
        assert c.error() & kvq.KVQ_DEVERR_STATE
        after = GpuState(c)
        assert after.n_quant[0] == 17 and after.seq_len[0] == 17 + R + 32
        assert np.array_equal(before.kc, after.kc) and np.array_equal(before.km, after.km)
