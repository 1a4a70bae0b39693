"""Algorithmic byte counts and streaming flush steps used by bench.py --sweep
(host logic only)."""
import types

import numpy as np

import bench
from bit_kv_cache_16_b200 import synth


def shape(batch, hq, hkv, bits, group, residual, lengths):
    return types.SimpleNamespace(batch=batch, num_q_heads=hq, num_kv_heads=hkv, head_dim=128, bits=bits,
                                 group=group, residual=residual, lengths=np.asarray(lengths))


def test_decode_bytes_by_hand():
    # Llama-3-8B layer: 8 sequences x 8 kv heads of n_q = 8064 INT4 tokens
    # (codes 64 B per token for K and for V), 252 key groups of 512 B, 4 B of
    # value scale/zero per token, 128 window tokens of 512 B, and the query.
    w = shape(8, 32, 8, 4, 32, 128, [8192] * 8)
    per_unit = 8064 * 64 * 2 + 252 * 512 + 8064 * 4 + 128 * 512
    assert bench.sweep_decode_bytes(w, w.lengths) == 64 * per_unit + 8 * 32 * 256
    assert bench.sweep_decode_bytes(w, w.lengths) == bench.algorithmic_bytes()["decode"]


def test_fp8_bytes_are_one_byte_per_element():
    w = shape(16, 32, 8, 8, 32, 0, [4608] * 16)
    assert bench.sweep_decode_bytes(w, w.lengths) == 16 * 8 * 4608 * 256 + 16 * 32 * 256
    assert bench.sweep_prefill_bytes(w) == 16 * 8 * 4608 * (512 + 256)


def test_int2_halves_the_code_bytes():
    w4 = shape(1, 64, 8, 4, 32, 128, [131072])
    w2 = shape(1, 64, 8, 2, 32, 128, [131072])
    nq = 130944
    assert bench.sweep_decode_bytes(w4, w4.lengths) - bench.sweep_decode_bytes(w2, w2.lengths) == 8 * nq * 32 * 2


def test_streaming_flushes_once_per_group():
    w = synth.make_config(4, lengths=[8] * 2)      # only the shape fields are read
    n0 = 4096
    flushes = [s for s in range(bench.STREAM_STEPS)
               if bench.quantized_split(n0 + s + 1, w.group, w.residual)[0]
               != bench.quantized_split(n0 + s, w.group, w.residual)[0]]
    assert len(flushes) == bench.STREAM_STEPS // w.group
    # the window holds R..R+G-1 tokens after every step
    for s in range(bench.STREAM_STEPS):
        _, r = bench.quantized_split(n0 + s + 1, w.group, w.residual)
        assert w.residual <= r < w.residual + w.group
