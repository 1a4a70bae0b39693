"""INT8 per-token dynamic cache on the GPU against the oracle: codes and
per-token key/value scale and zero bit-exact, decode within the decode
tolerance.  Lengths that end inside a 16-token tile, empty sequences, every
GQA ratio, split counts, appends one token at a time, and the 8B-layer and
streaming shapes at full size."""
import numpy as np
import pytest
import torch

import oracle
from bit_kv_cache_16_b200 import kvq, synth

from gpu_harness import (assert_close, assert_int8_state, each_unit, gpu_decode, gpu_prefill, oracle_cache,
                         to_dev)
from layout import GpuState

pytestmark = pytest.mark.gpu

I8 = kvq.KVQ_FORMAT_INT8


def _units(w):
    return [(b, h) for b in range(w.batch) for h in range(w.num_kv_heads)]


@pytest.mark.parametrize("gq", [1, 4, 8])
def test_int8_prefill_and_decode_ragged(gq):
    lengths = [0, 1, 15, 16, 17, 300, 1029, 2048]
    w = synth.make_workload("i8", 9000 + gq, lengths, 2 * gq, 2, I8, 16, 0)
    c = gpu_prefill(w)
    oc = oracle_cache(w, c.shape.capacity)
    assert_int8_state(GpuState(c), oc, _units(w))
    assert_close(gpu_decode(c, w, max(lengths)), oc.decode(w.q, w.softmax_scale))
    assert c.error() == 0


@pytest.mark.parametrize("num_splits", [1, 3, 57, 444, 1000])
def test_int8_split_count_does_not_change_result(num_splits):
    w = synth.make_workload("i8s", 9100, [700, 33, 4099], 16, 4, I8, 16, 0)
    c = gpu_prefill(w)
    oc = oracle_cache(w, c.shape.capacity)
    assert_close(gpu_decode(c, w, 4099, num_splits=num_splits), oc.decode(w.q, w.softmax_scale))


@pytest.mark.parametrize("fused", [False, True])
def test_int8_append_one_token_at_a_time(fused):
    """Appends land in token seq_len with their own scale and zero (also
    across tile boundaries); decode after every few steps."""
    w = synth.make_workload("i8a", 9200, [5, 31, 250], 8, 2, I8, 16, 0)
    steps = 40
    c = gpu_prefill(w, extra_tokens=steps)
    oc = oracle_cache(w, c.shape.capacity)
    for step in range(steps):
        kn, vn = synth.streaming_token(w, step)
        if fused:
            c.append_flush(to_dev(kn), to_dev(vn))
        else:
            c.append_token(to_dev(kn), to_dev(vn))
            c.flush_group()                       # a no-op for this format
        assert oc.append(kn, vn).all()
        if step % 7 == 0 or step == steps - 1:
            torch.cuda.synchronize()
            assert_int8_state(GpuState(c), oc, _units(w))
            assert_close(gpu_decode(c, w, 250 + step + 1), oc.decode(w.q, w.softmax_scale))
    assert c.error() == 0


def test_int8_capacity_reached_on_append():
    w = synth.make_workload("i8c", 9300, [32, 20], 4, 1, I8, 16, 0)
    c = gpu_prefill(w, capacity=32)
    kn, vn = synth.streaming_token(w, 0)
    c.append_token(to_dev(kn), to_dev(vn))        # sequence 0 is full: dropped, flagged
    assert c.error() & kvq.KVQ_DEVERR_APPEND_FULL
    st = GpuState(c)
    assert st.seq_len[0] == 32 and st.seq_len[1] == 21 and st.n_quant[1] == 21


def test_int8_extreme_rows():
    """Constant rows, -0, tiny and huge magnitudes and NaN: the state equals
    the oracle's bit for bit (NaN is ignored by min/max and encodes as 0)."""
    rng = np.random.default_rng(9400)
    n, D = 48, 128
    K = rng.normal(size=(n, D)).astype(np.float32)
    V = rng.normal(size=(n, D)).astype(np.float32)
    K[3, :] = 1.25                      # constant row
    K[4, :] = -0.0
    K[5, :] *= 1e-30                    # tiny
    K[6, :] *= 1e4                      # large
    K[7, 9] = np.nan
    V[8, :] = 0.0
    V[9, 100] = np.nan
    V[10, :] *= 3e3
    to_bf16 = lambda x: torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    w = synth.make_workload("i8x", 9400, [n], 4, 1, I8, 16, 0)
    w.k = to_bf16(K)[:, None, :].copy()
    w.v = to_bf16(V)[:, None, :].copy()
    c = gpu_prefill(w)
    oc = oracle_cache(w, c.shape.capacity)
    assert_int8_state(GpuState(c), oc, _units(w))


def test_int8_llama3_8b_layer_full():
    """B = 8, 32 / 8 heads, 8192 tokens each, every unit."""
    w = synth.make_config(1, bits=I8)
    c = gpu_prefill(w)
    units = _units(w)
    oc = oracle.Int8Cache(w.batch, w.num_q_heads, w.num_kv_heads, 128, c.shape.capacity)
    each_unit(lambda bh: oc.prefill(w.k, w.v, w.cu_seqlens, units=[bh]), units)
    assert_int8_state(GpuState(c), oc, units)
    out = gpu_decode(c, w, 8192)
    ref = each_unit(lambda bh: oc.decode_unit(w.q, bh[0], bh[1], w.softmax_scale), units)
    assert_close(out, np.stack(ref).reshape(w.batch, w.num_q_heads, 128))
    assert c.error() == 0


def test_int8_streaming_full():
    """The streaming shapes (B = 16, 4096 tokens, then 512 appended), every
    unit's state and decode at four steps."""
    w = synth.make_config(4, bits=I8)
    steps = 512
    c = gpu_prefill(w, extra_tokens=steps)
    units = _units(w)
    oc = oracle.Int8Cache(w.batch, w.num_q_heads, w.num_kv_heads, 128, c.shape.capacity)
    each_unit(lambda bh: oc.prefill(w.k, w.v, w.cu_seqlens, units=[bh]), units)
    for step in range(steps):
        kn, vn = synth.streaming_token(w, step)
        c.append_flush(to_dev(kn), to_dev(vn))
        oc.append(kn, vn)
        if step in (0, 37, 255, 511):
            torch.cuda.synchronize()
            assert_int8_state(GpuState(c), oc, units)
            out = gpu_decode(c, w, 4096 + step + 1)
            ref = each_unit(lambda bh: oc.decode_unit(w.q, bh[0], bh[1], w.softmax_scale), units)
            assert_close(out, np.stack(ref).reshape(w.batch, w.num_q_heads, 128))
    assert c.error() == 0
