"""The five named workloads at full size, in the launch configuration the
bench times (default split count), checked against the oracle on every
unit it finishes quickly and on samples where it does not.

  tiny       B=1, 1/1 heads, n=512, INT2, G=32, R=32            (all units)
  8B layer   B=8, 32/8 heads, n=8192, INT4, G=32, R=128         (all 64 units;
             prefill 8191 + one-launch append + flush + decode, as timed)
  70B 128K   B=1, 64/8 heads, n=131072, INT4 and INT2, RoPE K   (all 8 units)
  paged      B=64, n ~ U{1024..32768}, 32/8 heads, INT4, G=16=page, R=16
             (6 sampled units: shortest, longest, two more)
  streaming  B=16, 32/8 heads, 4096 -> 4608 over 512 steps, INT2, G=32, R=128
             (state of sampled units after every flush; decode sampled), and
             the FP8-E4M3 cache of the same shapes
"""
import numpy as np
import pytest
import torch

import oracle
from bit_kv_cache_16_b200 import synth

from gpu_harness import (assert_close, assert_fp8_state, assert_unit_state, gpu_decode, gpu_prefill, heads_of,
                         make_gpu_cache, oracle_cache, to_dev)
from layout import GpuState

pytestmark = pytest.mark.gpu


def test_tiny_full():
    w = synth.make_config(0)
    c = gpu_prefill(w)
    oc = oracle_cache(w, c.shape.capacity)
    st = GpuState(c)
    assert_unit_state(st, oc, 0, 0)
    assert_close(gpu_decode(c, w, 512), oc.decode(w.q, w.softmax_scale))


def test_llama3_8b_layer_full_as_benched():
    w = synth.make_config(1, lengths=[8191] * 8)
    c = gpu_prefill(w, extra_tokens=1, capacity=8192)
    oc = oracle_cache(w, 8192)
    kn, vn = synth.streaming_token(w, 0)
    c.append_flush(to_dev(kn), to_dev(vn))        # the bench's one-launch append + flush
    oc.append(kn, vn)
    assert oc.flush().all()                       # the window filled: one group quantized
    torch.cuda.synchronize()
    st = GpuState(c)
    for b in range(8):
        for h in range(8):
            assert_unit_state(st, oc, b, h)
    assert st.n_quant[0] == 8064 and st.seq_len[0] == 8192
    out = gpu_decode(c, w, 8192)
    assert_close(out, oc.decode(w.q, w.softmax_scale))
    assert c.error() == 0


@pytest.mark.parametrize("bits", [4, 2])
def test_llama3_70b_128k_full(bits):
    w = synth.make_config(2, bits=bits)
    c = gpu_prefill(w)
    oc = oracle_cache(w, c.shape.capacity)
    st = GpuState(c)
    for h in range(8):
        assert_unit_state(st, oc, 0, h)
    assert st.n_quant[0] == 130944
    assert_close(gpu_decode(c, w, 131072), oc.decode(w.q, w.softmax_scale))
    assert c.error() == 0


def test_paged_ragged_full_sampled():
    w = synth.make_config(3)
    c = gpu_prefill(w)
    L = w.lengths
    b_short, b_long = int(np.argmin(L)), int(np.argmax(L))
    units = [(b_short, 0), (b_long, 7), (b_long, 3), (5, 2), (33, 5), (b_short, 6)]
    oc = oracle_cache(w, c.shape.capacity, units=units)
    st = GpuState(c)
    for b, h in units:
        assert_unit_state(st, oc, b, h)
    out = gpu_decode(c, w, int(L.max()))
    assert_close(out, oc.decode(w.q, w.softmax_scale, units=units), rows=heads_of(w, units))
    # every other output row: finite and of the right scale
    assert np.all(np.isfinite(out))
    assert c.error() == 0


@pytest.mark.parametrize("fused", [False, True])
def test_streaming_int2_full_sampled(fused):
    w = synth.make_config(4)
    steps = 512
    c = gpu_prefill(w, extra_tokens=steps)
    units = [(0, 0), (7, 3), (15, 7)]
    oc = oracle.Cache(2, 16, 32, 8, 128, 32, 128, c.shape.capacity)
    oc.prefill(w.k, w.v, w.cu_seqlens, units=units)
    for step in range(steps):
        kn, vn = synth.streaming_token(w, step)
        if fused:
            c.append_flush(to_dev(kn), to_dev(vn))
        else:
            c.append_token(to_dev(kn), to_dev(vn))
            c.flush_group()
        for b, h in units:
            oc.units[b][h].append(kn[b, h], vn[b, h])
            oc.units[b][h].flush()
        if step % 32 == 31 or step in (0, 255, 511):
            torch.cuda.synchronize()
            st = GpuState(c)
            for b, h in units:
                assert_unit_state(st, oc, b, h)
            if step in (0, 31, 255, 511):
                out = gpu_decode(c, w, 4096 + step + 1)
                assert_close(out, oc.decode(w.q, w.softmax_scale, units=units), rows=heads_of(w, units))
    assert c.error() == 0


def test_streaming_fp8_full_sampled():
    w = synth.make_config(4, bits=8)
    steps = 512
    c = gpu_prefill(w, extra_tokens=steps)
    oc = oracle.FP8Cache(16, 32, 8, 128, c.shape.capacity)
    oc.prefill(w.k, w.v, w.cu_seqlens)
    units = [(0, 0), (9, 4), (15, 7)]
    for step in range(steps):
        kn, vn = synth.streaming_token(w, step)
        c.append_token(to_dev(kn), to_dev(vn))
        oc.append(kn, vn)
        if step in (0, 100, 511):
            torch.cuda.synchronize()
            assert_fp8_state(GpuState(c), oc, units)
            out = gpu_decode(c, w, 4096 + step + 1)
            assert_close(out, oc.decode(w.q, w.softmax_scale, units=units), rows=heads_of(w, units))
    assert c.error() == 0
