"""The five named workloads at full size, in the launch configuration the
bench times (default split count), checked against the oracle on every
unit it finishes quickly and on samples where it does not.

  tiny       B=1, 1/1 heads, n=512, INT2, G=32, R=32            (all units)
  8B layer   B=8, 32/8 heads, n=8192, INT4, G=32, R=128         (all 64 units;
             prefill 8191 + one-launch append + flush + decode, as timed)
  70B 128K   B=1, 64/8 heads, n=131072, INT4 and INT2, RoPE K   (all 8 units)
  paged      B=64, n ~ U{1024..32768}, 32/8 heads, INT4, G=16=page, R=16
             (all 512 units: state and decode)
  streaming  B=16, 32/8 heads, 4096 -> 4608 over 512 steps, INT2, G=32, R=128
             (state of all 128 units after every flush, decode of all units
             at four steps), and the FP8-E4M3 cache of the same shapes
The oracle runs unit by unit on a pool of host threads.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_kv_cache_16_b200 import synth

from gpu_harness import (assert_close, assert_fp8_state, assert_unit_state, assert_unit_state_of, each_unit,
                         gpu_decode, gpu_prefill, heads_of, make_gpu_cache, oracle_cache, to_dev)
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


def test_paged_ragged_full_all_units():
    """All 64 x 8 units of the paged ragged batch: codes, scales, zeros and
    window slots bit-exact after the page-table gather, every output row
    within the decode tolerance."""
    w = synth.make_config(3)
    c = gpu_prefill(w)
    L = w.lengths
    out = gpu_decode(c, w, int(L.max()))
    st = GpuState(c)
    g = w.num_q_heads // w.num_kv_heads
    units = [(b, h) for b in range(w.batch) for h in range(w.num_kv_heads)]

    def one(bh):
        b, h = bh
        u = oracle.Unit(4, 128, w.group, w.residual, (int(L[b]) + 15) // 16 * 16)
        lo, hi = int(w.cu_seqlens[b]), int(w.cu_seqlens[b + 1])
        u.prefill(w.k[lo:hi, h, :], w.v[lo:hi, h, :])
        assert_unit_state_of(st, u, b, h)
        return u.decode(w.q[b, h * g:(h + 1) * g], w.softmax_scale)

    ref = np.stack(each_unit(one, units)).reshape(w.batch, w.num_q_heads, 128)
    assert_close(out, ref)
    assert c.error() == 0


@pytest.mark.parametrize("fused", [False, True])
def test_streaming_int2_full_all_units(fused):
    """512 streaming steps on all 16 x 8 units: state after every flush step
    (and steps 0, 255), decode of every row at steps 0, 31, 255 and 511."""
    w = synth.make_config(4)
    steps = 512
    c = gpu_prefill(w, extra_tokens=steps)
    oc = oracle.Cache(2, 16, 32, 8, 128, 32, 128, c.shape.capacity)
    units = [(b, h) for b in range(w.batch) for h in range(w.num_kv_heads)]
    each_unit(lambda bh: oc.units[bh[0]][bh[1]].prefill(w.seq_k(bh[0])[:, bh[1], :], w.seq_v(bh[0])[:, bh[1], :]),
              units)
    for step in range(steps):
        kn, vn = synth.streaming_token(w, step)
        if fused:
            c.append_flush(to_dev(kn), to_dev(vn))
        else:
            c.append_token(to_dev(kn), to_dev(vn))
            c.flush_group()
        assert oc.append(kn, vn).all()
        oc.flush()
        if step % 32 == 31 or step in (0, 255, 511):
            torch.cuda.synchronize()
            st = GpuState(c)
            each_unit(lambda bh: assert_unit_state(st, oc, bh[0], bh[1]), units)
            if step in (0, 31, 255, 511):
                out = gpu_decode(c, w, 4096 + step + 1)
                g = w.num_q_heads // w.num_kv_heads
                ref = each_unit(lambda bh: oc.decode_unit(w.q, bh[0], bh[1], w.softmax_scale), units)
                assert_close(out, np.stack(ref).reshape(w.batch, w.num_q_heads, 128))
    assert c.error() == 0


def test_streaming_fp8_full_all_units():
    w = synth.make_config(4, bits=8)
    steps = 512
    c = gpu_prefill(w, extra_tokens=steps)
    oc = oracle.FP8Cache(16, 32, 8, 128, c.shape.capacity)
    oc.prefill(w.k, w.v, w.cu_seqlens)
    units = [(b, h) for b in range(w.batch) for h in range(w.num_kv_heads)]
    for step in range(steps):
        kn, vn = synth.streaming_token(w, step)
        c.append_token(to_dev(kn), to_dev(vn))
        oc.append(kn, vn)
        if step in (0, 100, 511):
            torch.cuda.synchronize()
            assert_fp8_state(GpuState(c), oc, units)
            out = gpu_decode(c, w, 4096 + step + 1)
            ref = each_unit(lambda bh: oc.decode_unit(w.q, bh[0], bh[1], w.softmax_scale), units)
            assert_close(out, np.stack(ref).reshape(w.batch, w.num_q_heads, 128))
    assert c.error() == 0
