"""Dense-and-sparse caches (each key set and value set keeps its largest
value aside, exactly) on the GPU against the oracle: codes, scales, zeros,
kept values and their positions bit-exact; decode (which uses the kept
values in place of the dense ones) within the decode tolerance.  G of 16 and
32, INT2 and INT4, GQA 1 to 8, split counts, streaming appends and flushes,
and the 8B-layer shape at full size."""
import numpy as np
import pytest
import torch

from bit_kv_cache_16_b200 import kvq, synth

from gpu_harness import (assert_close, assert_unit_state, each_unit, gpu_decode, gpu_prefill, oracle_cache,
                         to_dev)
from layout import GpuState

pytestmark = pytest.mark.gpu


def _units(w):
    return [(b, h) for b in range(w.batch) for h in range(w.num_kv_heads)]


@pytest.mark.parametrize("bits,G,R,gq", [(4, 32, 128, 4), (2, 32, 32, 8), (4, 16, 16, 1), (2, 16, 0, 4)])
def test_sparse_prefill_and_decode(bits, G, R, gq):
    lengths = [0, 9, 140, 1029, 3000]
    w = synth.make_workload("sp", 9700 + bits + G + gq, lengths, 2 * gq, 2, bits, G, R)
    c = gpu_prefill(w, sparse=True)
    oc = oracle_cache(w, c.shape.capacity, sparse=True)
    st = GpuState(c)
    for b, h in _units(w):
        assert_unit_state(st, oc, b, h)
    assert_close(gpu_decode(c, w, max(lengths)), oc.decode(w.q, w.softmax_scale))
    assert c.error() == 0


def test_sparse_kept_outliers_matter():
    """Keys with one huge value per channel set and values with one per
    token: the dense-and-sparse decode follows the oracle, and differs from
    the plain cache's."""
    rng = np.random.default_rng(9750)
    lengths = [700, 300]
    w = synth.make_workload("spo", 9751, lengths, 8, 2, 4, 32, 32)
    K = synth.bf16_bits_to_f32(w.k).copy()
    V = synth.bf16_bits_to_f32(w.v).copy()
    T = K.shape[0]
    for t in rng.choice(T, T // 40, replace=False):
        K[t, :, rng.integers(0, 128)] *= 30.0
        V[t, :, rng.integers(0, 128)] *= 30.0
    to_bf16 = lambda x: torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    w.k, w.v = to_bf16(K), to_bf16(V)
    c = gpu_prefill(w, sparse=True)
    oc = oracle_cache(w, c.shape.capacity, sparse=True)
    st = GpuState(c)
    for b, h in _units(w):
        assert_unit_state(st, oc, b, h)
    out = gpu_decode(c, w, 700)
    assert_close(out, oc.decode(w.q, w.softmax_scale))
    plain = oracle_cache(w, c.shape.capacity).decode(w.q, w.softmax_scale)
    assert np.max(np.abs(out - plain)) > 1e-2


@pytest.mark.parametrize("num_splits", [1, 7, 1000])
def test_sparse_split_count_does_not_change_result(num_splits):
    lengths = [2500, 33]
    w = synth.make_workload("sps", 9760, lengths, 16, 4, 4, 32, 64)
    c = gpu_prefill(w, sparse=True)
    oc = oracle_cache(w, c.shape.capacity, sparse=True)
    assert_close(gpu_decode(c, w, 2500, num_splits=num_splits), oc.decode(w.q, w.softmax_scale))


@pytest.mark.parametrize("fused", [False, True])
def test_sparse_streaming(fused):
    lengths = [150, 61]
    w = synth.make_workload("spa", 9770, lengths, 8, 2, 2, 32, 64)
    steps = 100
    c = gpu_prefill(w, extra_tokens=steps, sparse=True)
    oc = oracle_cache(w, c.shape.capacity, sparse=True)
    for step in range(steps):
        kn, vn = synth.streaming_token(w, step)
        if fused:
            c.append_flush(to_dev(kn), to_dev(vn))
        else:
            c.append_token(to_dev(kn), to_dev(vn))
            c.flush_group()
        assert oc.append(kn, vn).all()
        flushed = oc.flush()
        if flushed.any() or step == steps - 1:
            torch.cuda.synchronize()
            st = GpuState(c)
            for b, h in _units(w):
                assert_unit_state(st, oc, b, h)
        if step % 30 == 0 or step == steps - 1:
            assert_close(gpu_decode(c, w, 150 + step + 1), oc.decode(w.q, w.softmax_scale))
    assert c.error() == 0


def test_sparse_llama3_8b_layer_full():
    w = synth.make_config(1)
    c = gpu_prefill(w, sparse=True)
    oc = oracle_cache(w, c.shape.capacity, units=[], sparse=True)
    units = _units(w)
    each_unit(lambda bh: oc.units[bh[0]][bh[1]].prefill(w.seq_k(bh[0])[:, bh[1], :], w.seq_v(bh[0])[:, bh[1], :]),
              units)
    st = GpuState(c)
    each_unit(lambda bh: assert_unit_state(st, oc, bh[0], bh[1]), units)
    out = gpu_decode(c, w, 8192)
    ref = each_unit(lambda bh: oc.decode_unit(w.q, bh[0], bh[1], w.softmax_scale), units)
    assert_close(out, np.stack(ref).reshape(w.batch, w.num_q_heads, 128))
    assert c.error() == 0
