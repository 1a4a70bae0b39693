"""MIXED 2/4-bit cache (a group at the widest class of its tokens) on the GPU
against the oracle: codes, scales, zeros, group widths and window classes
bit-exact, decode within the decode tolerance.  Ragged lengths, G of 32, 64
and 128, GQA 4 and 8, split counts, one class everywhere, streaming appends
with their classes, and the 8B-layer shape at full size."""
import numpy as np
import pytest
import torch

import oracle
from bit_kv_cache_16_b200 import kvq, synth

from gpu_harness import (assert_close, assert_unit_state, assert_unit_state_of, each_unit, gpu_decode,
                         gpu_prefill, oracle_cache, to_dev)
from layout import GpuState

pytestmark = pytest.mark.gpu

MX = kvq.KVQ_FORMAT_MIXED


def _units(w):
    return [(b, h) for b in range(w.batch) for h in range(w.num_kv_heads)]


@pytest.mark.parametrize("G,R,gq,frac,span", [(32, 32, 4, 0.3, (64, 512)), (64, 64, 8, 0.5, (16, 100)),
                                               (128, 16, 4, 0.3, (1, 40)), (32, 128, 2, 0.05, (1, 1))])
def test_mixed_prefill_and_decode(G, R, gq, frac, span):
    lengths = [0, 5, 31, 200, 1029, 3000]
    w = synth.make_workload("mx", 9500 + G + gq, lengths, 2 * gq, 2, MX, G, R)
    cls = synth.token_classes(w.seed, lengths, high_fraction=frac, span=span)
    c = gpu_prefill(w, classes=cls)
    oc = oracle_cache(w, c.shape.capacity, classes=cls)
    st = GpuState(c)
    seen = set()
    for b, h in _units(w):
        assert_unit_state(st, oc, b, h)
        u = oc.units[b][h]
        seen |= set(u.group_bits[:u.n_q // G].tolist())
    assert seen == {2, 4}
    assert_close(gpu_decode(c, w, max(lengths)), oc.decode(w.q, w.softmax_scale))
    assert c.error() == 0


@pytest.mark.parametrize("cls_value,bits", [(4, 4), (2, 2)])
def test_mixed_with_one_class_decodes_like_the_uniform_cache(cls_value, bits):
    lengths = [700, 4099, 77]
    w = synth.make_workload("mx1", 9600 + bits, lengths, 16, 4, MX, 32, 128)
    cls = np.full(sum(lengths), cls_value, np.uint8)
    c = gpu_prefill(w, classes=cls)
    wu = synth.make_workload("mx1", 9600 + bits, lengths, 16, 4, bits, 32, 128)
    cu = gpu_prefill(wu)
    assert np.array_equal(gpu_decode(c, w, 4099), gpu_decode(cu, wu, 4099))


@pytest.mark.parametrize("num_splits", [1, 7, 444, 1000])
def test_mixed_split_count_does_not_change_result(num_splits):
    lengths = [2500, 33, 1200]
    w = synth.make_workload("mxs", 9700, lengths, 16, 4, MX, 32, 64)
    cls = synth.token_classes(w.seed, lengths, high_fraction=0.4, span=(8, 100))
    c = gpu_prefill(w, classes=cls)
    oc = oracle_cache(w, c.shape.capacity, classes=cls)
    assert_close(gpu_decode(c, w, 2500, num_splits=num_splits), oc.decode(w.q, w.softmax_scale))


@pytest.mark.parametrize("fused", [False, True])
def test_mixed_streaming(fused):
    """Appends carry their classes; every flush stores the group at the
    widest class of its tokens; state after every step that flushes."""
    lengths = [150, 290, 31]
    G, R = 32, 64
    w = synth.make_workload("mxa", 9800, lengths, 8, 2, MX, G, R)
    cls = synth.token_classes(w.seed, lengths, high_fraction=0.3, span=(4, 60))
    steps = 130
    c = gpu_prefill(w, extra_tokens=steps, classes=cls)
    oc = oracle_cache(w, c.shape.capacity, classes=cls)
    rng = np.random.default_rng(9800)
    for step in range(steps):
        kn, vn = synth.streaming_token(w, step)
        sc = np.where(rng.random(w.batch) < 0.1, 4, 2).astype(np.uint8)
        d = torch.from_numpy(sc).cuda()
        if fused:
            c.append_flush_mixed(to_dev(kn), to_dev(vn), d)
        else:
            c.append_token_mixed(to_dev(kn), to_dev(vn), d)
            c.flush_group()
        assert oc.append(kn, vn, sc).all()
        flushed = oc.flush()
        if flushed.any() or step in (0, steps - 1):
            torch.cuda.synchronize()
            st = GpuState(c)
            for b, h in _units(w):
                assert_unit_state(st, oc, b, h)
        if step % 25 == 0 or step == steps - 1:
            assert_close(gpu_decode(c, w, 290 + step + 1), oc.decode(w.q, w.softmax_scale))
    assert c.error() == 0


def test_mixed_llama3_8b_layer_full():
    """B = 8, 32 / 8 heads, 8192 tokens each, G = 32, R = 128, the seeded
    span classes (about 68% of the tokens at 2 bits): every unit."""
    w = synth.make_config(1, bits=MX)
    cls = synth.token_classes(w.seed, w.lengths)
    c = gpu_prefill(w, classes=cls)
    st = GpuState(c)
    g = w.num_q_heads // w.num_kv_heads

    def one(bh):
        b, h = bh
        u = oracle.Unit(0, 128, w.group, w.residual, c.shape.capacity, mixed=True)
        lo, hi = int(w.cu_seqlens[b]), int(w.cu_seqlens[b + 1])
        u.prefill(w.k[lo:hi, h, :], w.v[lo:hi, h, :], cls[lo:hi])
        assert_unit_state_of(st, u, b, h)
        return u.decode(w.q[b, h * g:(h + 1) * g], w.softmax_scale)

    ref = np.stack(each_unit(one, _units(w))).reshape(w.batch, w.num_q_heads, 128)
    assert_close(gpu_decode(c, w, 8192), ref)
    assert c.error() == 0
