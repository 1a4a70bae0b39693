"""kvq_decode_attention_noalloc: the decode entry point for callers that
cannot allocate device memory (no workspace argument; the split partials live
in the library's fixed device array).  Collected last on purpose, so that a
run stopping at the first failure has run everything else first; it also
passes alone in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

from bit_kv_cache_16_b200 import kvq, synth

from gpu_harness import assert_close, gpu_decode, gpu_prefill, oracle_cache, to_dev

pytestmark = pytest.mark.gpu


def _noalloc(c, w, max_len, num_splits=0):
    out = torch.full((w.batch, w.num_q_heads, 128), float("nan"), dtype=torch.float32, device="cuda")
    st = kvq.load().kvq_decode_attention_noalloc(ctypes.byref(c.desc), ctypes.c_void_p(to_dev(w.q).data_ptr()),
                                                 ctypes.c_void_p(out.data_ptr()), w.softmax_scale, num_splits,
                                                 max_len, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == kvq.KVQ_OK, kvq.status_string(st)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("bits", [4, 2])
def test_noalloc_matches_workspace_entry_twice(bits):
    w = synth.make_workload("noalloc", 9100 + bits, [8192, 5000, 777, 130], 32, 8, bits, 32, 128)
    c = gpu_prefill(w)
    ref = gpu_decode(c, w, 8192)                   # the entry point with a caller workspace
    oref = oracle_cache(w, c.shape.capacity).decode(w.q, w.softmax_scale)
    for _ in range(2):                             # two calls in a row share the fixed array
        got = _noalloc(c, w, 8192)
        assert_close(got, ref)
        assert_close(got, oref)                    # and the oracle's attention
    assert c.error() == 0


def test_noalloc_rejects_partials_beyond_the_array():
    # 1024 parts x 4 warps (+ 512 units) x 8 heads x 130 floats = 19 MB of partials > 8 MiB
    c = kvq.Cache(kvq.KVQ_FORMAT_INT4, 64, 64, 8, 64, group=32, residual=32)
    need = c.workspace_bytes(1024, 64)
    assert need > (8 << 20)
    q = torch.zeros(64, 64, 128, dtype=torch.int16, device="cuda")
    out = torch.zeros(64, 64, 128, dtype=torch.float32, device="cuda")
    st = kvq.load().kvq_decode_attention_noalloc(ctypes.byref(c.desc), ctypes.c_void_p(q.data_ptr()),
                                                 ctypes.c_void_p(out.data_ptr()), 0.1, 1024, 64, None)
    assert st == kvq.KVQ_ERR_WORKSPACE
