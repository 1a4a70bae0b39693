"""The C ABI library, on any machine: it builds for sm_100a, loads, exports
every entry point include/kvq.h declares, and rejects bad arguments on the
host before launching anything (no call here reaches a kernel)."""
import ctypes
import os
import re

import pytest

from bit_kv_cache_16_b200 import build, kvq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build_libkvq()
    return kvq.load()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "kvq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 10
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(kvq.EXPORTED)
    assert kvq.kvq_version().count(".") == 2


def test_struct_layouts_match_header():
    # 11 int32 shape fields, the RoPE base (float) and the sparse flag, then 16 pointers
    assert ctypes.sizeof(kvq.KvqShape) == 52
    assert kvq.KvqCache.k_codes.offset == 56
    assert ctypes.sizeof(kvq.KvqCache) == 56 + 16 * 8
    assert kvq.KvqCache.v_sparse.offset == 56 + 15 * 8


def _shape(**kw):
    base = dict(format=4, batch=8, num_q_heads=32, num_kv_heads=8, head_dim=128, group=32, residual=128,
                capacity=8192, page_size=0, max_pages_per_seq=0, num_pages=0, rope_theta=0.0, sparse=0)
    base.update(kw)
    return kvq.KvqShape(*[base[f] for f, _ in kvq.KvqShape._fields_])


def _bytes(shape, region):
    n = ctypes.c_size_t(0)
    st = kvq.load().kvq_buffer_bytes(ctypes.byref(shape), region, ctypes.byref(n))
    return st, n.value


def test_buffer_bytes_contiguous(lib):
    s = _shape()
    B, H, cap = 8, 8, 8192
    assert _bytes(s, 0) == (0, B * H * cap * 64)               # K codes, 4-bit rows of 64 bytes
    assert _bytes(s, 1) == (0, B * H * (cap // 32) * 2 * 128 * 2)
    assert _bytes(s, 2) == (0, B * H * cap * 64)               # V tiles
    assert _bytes(s, 3) == (0, B * H * cap * 4)
    assert _bytes(s, 4) == (0, B * H * 160 * 128 * 2)          # window ring of R + G slots
    assert _bytes(s, 6) == (0, B * 4)
    assert _bytes(s, 8) == (0, 0)                              # no page table
    assert _bytes(s, 9) == (0, 0)                              # no fp8 scales
    s2 = _shape(format=2)
    assert _bytes(s2, 0) == (0, B * H * cap * 32)
    s8 = _shape(format=8)
    assert _bytes(s8, 0) == (0, B * H * cap * 128)
    assert _bytes(s8, 1) == (0, 0) and _bytes(s8, 4) == (0, 0)
    assert _bytes(s8, 9) == (0, 2 * H * 4)
    # INT8 per token: byte codes, a (scale, zero) per token for K and for V, no window
    s16 = _shape(format=16, group=0, residual=0)
    assert _bytes(s16, 0) == (0, B * H * cap * 128) and _bytes(s16, 2) == (0, B * H * cap * 128)
    assert _bytes(s16, 1) == (0, B * H * cap * 4) and _bytes(s16, 3) == (0, B * H * cap * 4)
    assert _bytes(s16, 4) == (0, 0) and _bytes(s16, 5) == (0, 0) and _bytes(s16, 9) == (0, 0)
    # MIXED: regions sized as INT4, plus the group widths and the window classes
    s6 = _shape(format=6)
    assert _bytes(s6, 0) == (0, B * H * cap * 64) and _bytes(s6, 2) == (0, B * H * cap * 64)
    assert _bytes(s6, 1) == (0, B * H * (cap // 32) * 2 * 128 * 2)
    assert _bytes(s6, 12) == (0, B * (cap // 32)) and _bytes(s6, 13) == (0, B * 160)
    assert _bytes(s, 12) == (0, 0) and _bytes(s, 13) == (0, 0)
    # dense-and-sparse: a kept key per (group, channel) and a kept value per token, 4 bytes each
    ssp = _shape(sparse=1)
    assert _bytes(ssp, 14) == (0, B * H * (cap // 32) * 128 * 4) and _bytes(ssp, 15) == (0, B * H * cap * 4)
    assert _bytes(s, 14) == (0, 0) and _bytes(s, 15) == (0, 0)


def test_buffer_bytes_paged(lib):
    s = _shape(group=16, residual=16, page_size=16, max_pages_per_seq=2048, capacity=2048 * 16, num_pages=1000,
               batch=64)
    assert _bytes(s, 0) == (0, 1000 * 8 * 16 * 64)
    assert _bytes(s, 1) == (0, 1000 * 8 * 2 * 128 * 2)
    assert _bytes(s, 3) == (0, 1000 * 8 * 16 * 4)
    assert _bytes(s, 8) == (0, 64 * 2048 * 4)


@pytest.mark.parametrize("kw,status", [
    (dict(head_dim=64), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(num_q_heads=30), kvq.KVQ_ERR_SHAPE),
    (dict(num_q_heads=128), kvq.KVQ_ERR_UNSUPPORTED),          # 16 query heads per kv head
    (dict(format=3), kvq.KVQ_ERR_INVALID_ARG),
    (dict(group=24), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(group=48), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(group=256), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(capacity=8200), kvq.KVQ_ERR_SHAPE),
    (dict(batch=0), kvq.KVQ_ERR_INVALID_ARG),
    (dict(residual=-1), kvq.KVQ_ERR_INVALID_ARG),
    (dict(page_size=16, group=32, max_pages_per_seq=4, num_pages=4, capacity=64), kvq.KVQ_ERR_SHAPE),
    (dict(page_size=32, group=32, max_pages_per_seq=4, num_pages=4, capacity=128), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(page_size=16, group=16, max_pages_per_seq=4, num_pages=4, capacity=80), kvq.KVQ_ERR_SHAPE),
    (dict(format=16, page_size=16, group=16, max_pages_per_seq=4, num_pages=4, capacity=64),
     kvq.KVQ_ERR_UNSUPPORTED),                                 # INT8 is contiguous only
    (dict(format=16, capacity=8200), kvq.KVQ_ERR_SHAPE),       # whole 16-token tiles
    (dict(format=6, group=16, residual=16), kvq.KVQ_ERR_UNSUPPORTED),   # mixed: groups of 32 or more
    (dict(rope_theta=-1.0), kvq.KVQ_ERR_INVALID_ARG),
    (dict(rope_theta=float("nan")), kvq.KVQ_ERR_INVALID_ARG),
    (dict(rope_theta=5e5, format=8), kvq.KVQ_ERR_UNSUPPORTED),          # RoPE at read: INT2 / INT4 only
    (dict(rope_theta=5e5, format=6), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(rope_theta=5e5, group=16, residual=16, page_size=16, max_pages_per_seq=4, num_pages=4, capacity=64),
     kvq.KVQ_ERR_UNSUPPORTED),
    (dict(sparse=2), kvq.KVQ_ERR_INVALID_ARG),
    (dict(sparse=1, group=64), kvq.KVQ_ERR_UNSUPPORTED),                 # dense-and-sparse: G of 16 or 32
    (dict(sparse=1, format=16), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(sparse=1, rope_theta=5e5), kvq.KVQ_ERR_UNSUPPORTED),
    (dict(format=6, group=16, residual=16, page_size=16, max_pages_per_seq=4, num_pages=4, capacity=64),
     kvq.KVQ_ERR_UNSUPPORTED),
])
def test_shape_validation(lib, kw, status):
    assert _bytes(_shape(**kw), 0)[0] == status


def _fake_cache(shape, **override):
    """A descriptor with aligned dummy pointers: only ever handed to calls
    that must fail validation before any launch."""
    vals = {n: 0x1000 * (i + 1) for i, n in enumerate(kvq.REGIONS)}
    vals.update(override)
    return kvq.KvqCache(shape, *[vals[f] for f, _ in kvq.KvqCache._fields_[1:]])


def test_host_validation_before_launch(lib):
    s = _shape()
    c = _fake_cache(s)
    L = kvq.load()
    # null cache / query / out
    assert L.kvq_decode_attention(None, 16, 16, 1.0, 16, 1 << 30, 0, 8192, None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_decode_attention(ctypes.byref(c), None, 16, 1.0, 16, 1 << 30, 0, 8192, None) == kvq.KVQ_ERR_INVALID_ARG
    # misaligned query
    assert L.kvq_decode_attention(ctypes.byref(c), 17, 16, 1.0, 16, 1 << 30, 0, 8192, None) == kvq.KVQ_ERR_ALIGNMENT
    # workspace too small
    need = L.kvq_decode_workspace_bytes(ctypes.byref(c), 0, 8192)
    assert need > 0
    assert L.kvq_decode_attention(ctypes.byref(c), 16, 16, 1.0, 16, need - 1, 0, 8192, None) == kvq.KVQ_ERR_WORKSPACE
    # a negative split count
    assert L.kvq_decode_attention(ctypes.byref(c), 16, 16, 1.0, 16, 1 << 30, -1, 8192, None) == kvq.KVQ_ERR_INVALID_ARG
    # NaN softmax scale
    assert L.kvq_decode_attention(ctypes.byref(c), 16, 16, float("nan"), 16, 1 << 30, 0, 8192, None) == \
        kvq.KVQ_ERR_INVALID_ARG
    # a missing or misaligned cache region
    assert L.kvq_flush_group(ctypes.byref(_fake_cache(s, k_meta=0)), None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_flush_group(ctypes.byref(_fake_cache(s, v_res=0x1008)), None) == kvq.KVQ_ERR_ALIGNMENT
    assert L.kvq_append_token(ctypes.byref(c), 16, None, None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_append_flush(ctypes.byref(c), 16, None, None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_append_flush(ctypes.byref(c), 16, 24, None) == kvq.KVQ_ERR_ALIGNMENT
    assert L.kvq_append_flush(ctypes.byref(_fake_cache(s, k_res=0)), 16, 16, None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_quantize_prefill(ctypes.byref(c), 16, 16, None, 8192, None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_quantize_prefill(ctypes.byref(c), 16, 16, 16, -1, None) == kvq.KVQ_ERR_INVALID_ARG
    # paged cache without a page table
    sp = _shape(group=16, residual=16, page_size=16, max_pages_per_seq=4, num_pages=4, capacity=64)
    assert L.kvq_flush_group(ctypes.byref(_fake_cache(sp, page_table=0)), None) == kvq.KVQ_ERR_INVALID_ARG
    # decode with the ln-sum-exp output: it must be given and aligned
    assert L.kvq_decode_attention_lse(ctypes.byref(c), 16, 16, None, 1.0, 16, 1 << 30, 0, 8192, None) == \
        kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_decode_attention_lse(ctypes.byref(c), 16, 16, 20, 1.0, 16, 1 << 30, 0, 8192, None) == \
        kvq.KVQ_ERR_ALIGNMENT
    assert L.kvq_decode_attention_lse(ctypes.byref(c), 16, 16, 32, 1.0, 16, need - 1, 0, 8192, None) == \
        kvq.KVQ_ERR_WORKSPACE
    # merge of partial attentions
    assert L.kvq_merge_partials(None, 16, 2, 8, 16, None, None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_merge_partials(16, 16, 0, 8, 16, None, None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_merge_partials(16, 16, 2, -1, 16, None, None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_merge_partials(16, 16, 2, 1 << 31, 16, None, None) == kvq.KVQ_ERR_UNSUPPORTED
    assert L.kvq_merge_partials(16, 20, 2, 8, 16, None, None) == kvq.KVQ_ERR_ALIGNMENT
    assert L.kvq_merge_partials(16, 16, 2, 8, 16, 24, None) == kvq.KVQ_ERR_ALIGNMENT
    # nothing to merge: no launch, so no device is needed
    assert L.kvq_merge_partials(16, 16, 2, 0, 16, None, None) == kvq.KVQ_OK


def test_default_splits_and_workspace(lib):
    c = _fake_cache(_shape())
    L = kvq.load()
    n = L.kvq_decode_default_splits(ctypes.byref(c), 8192)
    assert n >= 1
    # INT formats: one partial slot per (streaming warp, unit segment): 4 warps
    # per CTA of the grid plus one per (sequence, kv head), gq heads x 130 floats
    sh = c.shape
    gq = sh.num_q_heads // sh.num_kv_heads
    slots = 4 * n + sh.batch * sh.num_kv_heads
    ml_floats = (slots * gq * 2 + 63) // 64 * 64     # (m, l) area, padded to 256 bytes
    assert L.kvq_decode_workspace_bytes(ctypes.byref(c), n, 8192) == (ml_floats + slots * gq * 128) * 4
    c8 = _fake_cache(_shape(format=8))
    n8 = L.kvq_decode_default_splits(ctypes.byref(c8), 4096)
    assert n8 >= 1
    # FP8: one partial per (sequence, query head, split)
    assert L.kvq_decode_workspace_bytes(ctypes.byref(c8), n8, 4096) == \
        c8.shape.batch * c8.shape.num_q_heads * n8 * 130 * 4


def test_status_strings(lib):
    for st in range(7):
        assert kvq.kvq_status_string(st) not in ("", "unknown status")
    assert kvq.kvq_status_string(99) == "unknown status"


@pytest.mark.parametrize("kw,args,status", [
    (dict(head_dim=64), {}, kvq.KVQ_ERR_UNSUPPORTED),
    (dict(num_q_heads=30), {}, kvq.KVQ_ERR_SHAPE),
    (dict(format=3), {}, kvq.KVQ_ERR_INVALID_ARG),
    (dict(), dict(num_splits=70000), kvq.KVQ_ERR_INVALID_ARG),
    (dict(), dict(num_splits=-1), kvq.KVQ_ERR_INVALID_ARG),
    (dict(), dict(q=17), kvq.KVQ_ERR_ALIGNMENT),
    (dict(), dict(out=None), kvq.KVQ_ERR_INVALID_ARG),
    (dict(), dict(scale=float("nan")), kvq.KVQ_ERR_INVALID_ARG),
    (dict(), dict(cache=dict(v_meta=0)), kvq.KVQ_ERR_INVALID_ARG),
])
def test_noalloc_rejects_like_the_workspace_entry(lib, kw, args, status):
    """A bad argument gives the same status from the allocation-free decode
    as from the entry point with a caller workspace (checked on the host,
    before the scratch-size test and before any launch)."""
    c = _fake_cache(_shape(**kw), **args.get("cache", {}))
    L = kvq.load()
    q, out = args.get("q", 16), args.get("out", 16)
    scale, splits = args.get("scale", 1.0), args.get("num_splits", 0)
    ws = L.kvq_decode_attention(ctypes.byref(c), q, out, scale, 16, 1 << 40, splits, 8192, None)
    na = L.kvq_decode_attention_noalloc(ctypes.byref(c), q, out, scale, splits, 8192, None)
    assert ws == status and na == status


def test_mixed_write_calls_need_the_classes(lib):
    """A MIXED cache is written only through the calls that take the token
    classes; the others refuse it (and the mixed calls refuse other formats)."""
    L = kvq.load()
    m = _fake_cache(_shape(format=6))
    i4 = _fake_cache(_shape())
    assert L.kvq_quantize_prefill(ctypes.byref(m), 16, 16, 16, 8192, None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_append_token(ctypes.byref(m), 16, 16, None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_append_flush(ctypes.byref(m), 16, 16, None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_quantize_prefill_mixed(ctypes.byref(i4), 16, 16, 16, 16, 8192, None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_append_token_mixed(ctypes.byref(i4), 16, 16, 16, None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_quantize_prefill_mixed(ctypes.byref(m), 16, 16, None, 16, 8192, None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_append_flush_mixed(ctypes.byref(m), 16, 16, None, None) == kvq.KVQ_ERR_INVALID_ARG
    assert L.kvq_flush_group(ctypes.byref(_fake_cache(_shape(format=6), group_bits=0)), None) == \
        kvq.KVQ_ERR_INVALID_ARG
