"""Algorithmic byte counts and streaming flush steps used by bench.py
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
    assert bench.wl_decode_bytes(w, w.lengths) == 64 * per_unit + 8 * 32 * 256
    assert bench.decode_bytes(4, 32, 128, 32, 8, [8192] * 8) == 64 * per_unit + 8 * 32 * 256


def test_prefill_bytes_by_hand():
    # 8191 tokens: n_q = 8032 (251 groups), 159 window tokens; K and V read once
    per_unit = 8191 * 512 + 8032 * 64 * 2 + 251 * 512 + 8032 * 4 + 159 * 512
    assert bench.prefill_bytes(4, 32, 128, 8, [8191] * 8) == 64 * per_unit


def test_append_flush_bytes_flush_steps():
    # 8191 -> 8192 fills the window (8192 - 8032 = 160 = R + G): a flush
    per_append = 128 * 2 * 2 * 2
    per_flush = 32 * 512 + 32 * 64 * 2 + 512 + 32 * 4
    assert bench.append_flush_bytes(4, 32, 128, 8, 8, 8191) == 64 * (per_append + per_flush)
    assert bench.append_flush_bytes(4, 32, 128, 8, 8, 8192) == 64 * per_append
    flushing = [n for n in range(8191, 8191 + 96) if bench.append_flush_bytes(4, 32, 128, 1, 1, n) > per_append]
    assert flushing == [8191, 8223, 8255]
    # FP8 and INT8: the token is encoded straight into the cache (read bf16, write codes [+ scale/zero])
    assert bench.append_flush_bytes(8, 32, 0, 1, 1, 5000) == 512 + 256
    assert bench.append_flush_bytes(16, 16, 0, 1, 1, 5000) == 512 + 256 + 8


def test_int8_bytes_per_token():
    w = shape(8, 32, 8, 16, 16, 0, [8192] * 8)
    assert bench.wl_decode_bytes(w, w.lengths) == 64 * 8192 * (256 + 8) + 8 * 32 * 256


def test_fp8_bytes_are_one_byte_per_element():
    w = shape(16, 32, 8, 8, 32, 0, [4608] * 16)
    assert bench.wl_decode_bytes(w, w.lengths) == 16 * 8 * 4608 * 256 + 16 * 32 * 256
    assert bench.wl_prefill_bytes(w) == 16 * 8 * 4608 * (512 + 256)


def test_int2_halves_the_code_bytes():
    w4 = shape(1, 64, 8, 4, 32, 128, [131072])
    w2 = shape(1, 64, 8, 2, 32, 128, [131072])
    nq = 130944
    assert bench.wl_decode_bytes(w4, w4.lengths) - bench.wl_decode_bytes(w2, w2.lengths) == 8 * nq * 32 * 2


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


def test_seqshard_parts_tile_the_sequence():
    w = synth.make_workload("ss", 5, [1000, 333], 8, 2, 4, 32, 128)
    for world in (1, 2, 3):
        ks, lens_all = [], []
        for rank in range(world):
            k, v, cu, lens, res = bench.seqshard_part(w, rank, world)
            assert k.shape[0] == cu[-1] == lens.sum()
            assert res == (128 if rank == world - 1 else 0)
            ks.append((k, cu))
            lens_all.append(lens)
        assert np.array_equal(np.sum(lens_all, axis=0), w.lengths)
        for b in range(w.batch):
            parts = [k[cu[b]:cu[b + 1]] for k, cu in ks]
            assert np.array_equal(np.concatenate(parts), w.seq_k(b))
            for p in parts[:-1]:
                assert p.shape[0] % w.group == 0         # whole key groups before the last rank


def test_mixed_bytes_follow_the_group_widths():
    """A mixed cache's bytes are those of INT4 for groups with a class-4
    token and of INT2 for the others; one class everywhere gives the uniform
    cache's bytes."""
    n, G, R = 8192, 32, 128
    assert bench.mixed_unit_bytes([4] * n, G, R) == bench.unit_cache_bytes(4, G, R, n)
    assert bench.mixed_unit_bytes([2] * n, G, R) == bench.unit_cache_bytes(2, G, R, n)
    cls = [2] * n
    cls[5] = 4                      # one token of class 4: its group at 4 bits
    cls[8100] = 4                   # a window token: no effect on the quantized part
    assert bench.mixed_unit_bytes(cls, G, R) == bench.unit_cache_bytes(2, G, R, n) + G * 128 * (4 - 2) // 8 * 2


def test_sparse_bytes():
    # 8191 tokens -> 251 groups of 32 (128 kept keys each) and 8032 kept values, 4 bytes each
    w = shape(8, 32, 8, 4, 32, 128, [8191] * 8)
    assert bench.sparse_bytes(w) == 64 * (251 * 128 * 4 + 8032 * 4)
