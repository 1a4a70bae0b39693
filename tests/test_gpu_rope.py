"""Keys stored before RoPE and rotated at read (KVQuant's pre-RoPE key
quantization) on the GPU against the oracle: the cache holds un-rotated
keys (codes and scales bit-exact, as any INT cache), and the decode, which
turns key t by its position before the scores (window keys too), matches the
oracle's rotated attention within the decode tolerance."""
import numpy as np
import pytest
import torch

from bit_kv_cache_16_b200 import kvq, synth

from gpu_harness import (assert_close, assert_unit_state, each_unit, gpu_decode, gpu_prefill, oracle_cache,
                         to_dev)
from layout import GpuState

pytestmark = pytest.mark.gpu

THETA = 500000.0


def _units(w):
    return [(b, h) for b in range(w.batch) for h in range(w.num_kv_heads)]


@pytest.mark.parametrize("bits,G,R,gq", [(4, 32, 128, 4), (2, 32, 32, 8), (4, 64, 0, 2), (2, 128, 64, 4)])
def test_rope_at_read_ragged(bits, G, R, gq):
    lengths = [0, 7, 130, 1029, 5000]
    w = synth.make_workload("rope", 9900 + bits + G, lengths, 2 * gq, 2, bits, G, R)
    c = gpu_prefill(w, rope_theta=THETA)
    oc = oracle_cache(w, c.shape.capacity)
    st = GpuState(c)
    for b, h in _units(w):
        assert_unit_state(st, oc, b, h)
    assert_close(gpu_decode(c, w, max(lengths)), oc.decode(w.q, w.softmax_scale, rope_theta=THETA))
    assert c.error() == 0


@pytest.mark.parametrize("theta", [10000.0, 500000.0])
def test_rope_split_counts_and_bases(theta):
    lengths = [3000, 333]
    w = synth.make_workload("ropes", 9950, lengths, 16, 4, 4, 32, 128)
    c = gpu_prefill(w, rope_theta=theta)
    oc = oracle_cache(w, c.shape.capacity)
    ref = oc.decode(w.q, w.softmax_scale, rope_theta=theta)
    for ns in (1, 5, 444):
        assert_close(gpu_decode(c, w, 3000, num_splits=ns), ref)
    # a different base gives a different answer (the rotation is applied)
    other = oc.decode(w.q, w.softmax_scale, rope_theta=theta * 3)
    assert np.max(np.abs(other - ref)) > 1e-2


def test_rope_streaming():
    """Appends and flushes of un-rotated keys; decode at growing positions."""
    lengths = [200, 61]
    w = synth.make_workload("ropea", 9960, lengths, 8, 2, 2, 32, 64)
    steps = 100
    c = gpu_prefill(w, extra_tokens=steps, rope_theta=THETA)
    oc = oracle_cache(w, c.shape.capacity)
    for step in range(steps):
        kn, vn = synth.streaming_token(w, step)
        c.append_flush(to_dev(kn), to_dev(vn))
        oc.append(kn, vn)
        oc.flush()
        if step % 33 == 0 or step == steps - 1:
            torch.cuda.synchronize()
            assert_close(gpu_decode(c, w, 200 + step + 1), oc.decode(w.q, w.softmax_scale, rope_theta=THETA))
    assert c.error() == 0


@pytest.mark.parametrize("bits", [4, 2])
def test_rope_llama3_70b_128k_full(bits):
    """The Llama-3-70B 131072-token layer with its keys kept before RoPE
    (the same seeded keys as the post-RoPE workload, not rotated): every
    unit, every output row."""
    w = synth.make_config(2, bits=bits, rope=False)
    c = gpu_prefill(w, rope_theta=synth.ROPE_THETA_70B)
    oc = oracle_cache(w, c.shape.capacity, units=[])
    g = w.num_q_heads // w.num_kv_heads

    def one(h):
        u = oc.units[0][h]
        u.prefill(w.k[:, h, :], w.v[:, h, :])
        return u.decode(w.q[0, h * g:(h + 1) * g], w.softmax_scale, synth.ROPE_THETA_70B)

    ref = np.stack(each_unit(one, list(range(w.num_kv_heads)))).reshape(1, w.num_q_heads, 128)
    st = GpuState(c)
    for h in range(w.num_kv_heads):
        assert_unit_state(st, oc, 0, h)
    assert_close(gpu_decode(c, w, 131072), ref)
    assert c.error() == 0
