"""Python binding of libkvq (argument marshalling only).

Every function here forwards to the C entry point of the same name declared
in include/kvq.h; all work runs in the library's CUDA kernels.  PyTorch is
used for device memory and streams only.  If libkvq.so is missing the import
of the library fails loudly: there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from .build import LIB_PATH

KVQ_OK = 0
KVQ_ERR_INVALID_ARG = 1
KVQ_ERR_SHAPE = 2
KVQ_ERR_UNSUPPORTED = 3
KVQ_ERR_ALIGNMENT = 4
KVQ_ERR_WORKSPACE = 5
KVQ_ERR_CUDA = 6

KVQ_FORMAT_INT2 = 2
KVQ_FORMAT_INT4 = 4
KVQ_FORMAT_FP8_E4M3 = 8
KVQ_FORMAT_INT8 = 16
KVQ_FORMAT_MIXED = 6

KVQ_DEVERR_APPEND_FULL = 0x1
KVQ_DEVERR_PAGE_RANGE = 0x2
KVQ_DEVERR_PREFILL_LEN = 0x4
KVQ_DEVERR_WAIT_TIMEOUT = 0x8
KVQ_DEVERR_STATE = 0x10

REGIONS = ["k_codes", "k_meta", "v_codes", "v_meta", "k_res", "v_res", "seq_len", "n_quant",
           "page_table", "fp8_scale", "fp8_amax", "err_word", "group_bits", "window_class", "k_sparse", "v_sparse"]

EXPORTED = ["kvq_buffer_bytes", "kvq_quantize_prefill", "kvq_append_token", "kvq_flush_group", "kvq_append_flush",
            "kvq_quantize_prefill_mixed", "kvq_append_token_mixed", "kvq_append_flush_mixed",
            "kvq_decode_attention", "kvq_decode_attention_lse", "kvq_merge_partials",
            "kvq_decode_attention_noalloc", "kvq_decode_workspace_bytes", "kvq_decode_default_splits",
            "kvq_read_error", "kvq_status_string", "kvq_version"]


class KvqShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("format", "batch", "num_q_heads", "num_kv_heads", "head_dim", "group", "residual",
                 "capacity", "page_size", "max_pages_per_seq", "num_pages")] + [("rope_theta", ctypes.c_float),
                                                                                ("sparse", ctypes.c_int32)]


class KvqCache(ctypes.Structure):
    _fields_ = [("shape", KvqShape)] + [(n, ctypes.c_void_p) for n in REGIONS]


class KvqError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__("%s failed: %s (status %d)" % (fn, status_string(status), status))
        self.status = status


_lib = None


def load(path: Optional[str] = None):
    """Load libkvq.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise ImportError("libkvq.so not found at %s; build it with bit_kv_cache_16_b200.build.build_libkvq()"
                          % path)
    lib = ctypes.CDLL(path)
    vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    pc = ctypes.POINTER(KvqCache)
    sig = {
        "kvq_buffer_bytes": (i32, [ctypes.POINTER(KvqShape), i32, ctypes.POINTER(sz)]),
        "kvq_quantize_prefill": (i32, [pc, vp, vp, vp, i32, vp]),
        "kvq_append_token": (i32, [pc, vp, vp, vp]),
        "kvq_flush_group": (i32, [pc, vp]),
        "kvq_append_flush": (i32, [pc, vp, vp, vp]),
        "kvq_quantize_prefill_mixed": (i32, [pc, vp, vp, vp, vp, i32, vp]),
        "kvq_append_token_mixed": (i32, [pc, vp, vp, vp, vp]),
        "kvq_append_flush_mixed": (i32, [pc, vp, vp, vp, vp]),
        "kvq_decode_attention": (i32, [pc, vp, vp, f32, vp, sz, i32, i32, vp]),
        "kvq_decode_attention_lse": (i32, [pc, vp, vp, vp, f32, vp, sz, i32, i32, vp]),
        "kvq_merge_partials": (i32, [vp, vp, i32, ctypes.c_int64, vp, vp, vp]),
        "kvq_decode_attention_noalloc": (i32, [pc, vp, vp, f32, i32, i32, vp]),
        "kvq_decode_workspace_bytes": (sz, [pc, i32, i32]),
        "kvq_decode_default_splits": (i32, [pc, i32]),
        "kvq_read_error": (i32, [pc, ctypes.POINTER(ctypes.c_uint32), vp]),
        "kvq_status_string": (ctypes.c_char_p, [i32]),
        "kvq_version": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t) -> ctypes.c_void_p:
    if t is None:
        return ctypes.c_void_p(0)
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    return ctypes.c_void_p(t.data_ptr())


def _check(fn: str, status: int):
    if status != KVQ_OK:
        raise KvqError(fn, status)


# --------------------------------------------------------------------------
# Entry points (same names as the C ABI)
# --------------------------------------------------------------------------

def status_string(status: int) -> str:
    return load().kvq_status_string(status).decode()


def kvq_status_string(status: int) -> str:
    return status_string(status)


def kvq_version() -> str:
    return load().kvq_version().decode()


def kvq_buffer_bytes(shape: KvqShape, region: int) -> int:
    n = ctypes.c_size_t(0)
    _check("kvq_buffer_bytes", load().kvq_buffer_bytes(ctypes.byref(shape), region, ctypes.byref(n)))
    return n.value


def kvq_quantize_prefill(cache: KvqCache, k, v, cu_seqlens, max_len: int, stream=None):
    _check("kvq_quantize_prefill", load().kvq_quantize_prefill(ctypes.byref(cache), _ptr(k), _ptr(v),
                                                               _ptr(cu_seqlens), int(max_len), _stream(stream)))


def kvq_append_token(cache: KvqCache, k_new, v_new, stream=None):
    _check("kvq_append_token", load().kvq_append_token(ctypes.byref(cache), _ptr(k_new), _ptr(v_new),
                                                       _stream(stream)))


def kvq_flush_group(cache: KvqCache, stream=None):
    _check("kvq_flush_group", load().kvq_flush_group(ctypes.byref(cache), _stream(stream)))


def kvq_append_flush(cache: KvqCache, k_new, v_new, stream=None):
    _check("kvq_append_flush", load().kvq_append_flush(ctypes.byref(cache), _ptr(k_new), _ptr(v_new),
                                                       _stream(stream)))


def kvq_quantize_prefill_mixed(cache: KvqCache, k, v, token_class, cu_seqlens, max_len: int, stream=None):
    """Prefill of a MIXED cache: token_class uint8 [T_total] (2 or 4) on the device."""
    _check("kvq_quantize_prefill_mixed",
           load().kvq_quantize_prefill_mixed(ctypes.byref(cache), _ptr(k), _ptr(v), _ptr(token_class),
                                             _ptr(cu_seqlens), int(max_len), _stream(stream)))


def kvq_append_token_mixed(cache: KvqCache, k_new, v_new, token_class, stream=None):
    """Append to a MIXED cache: token_class uint8 [B] (2 or 4) on the device."""
    _check("kvq_append_token_mixed", load().kvq_append_token_mixed(ctypes.byref(cache), _ptr(k_new), _ptr(v_new),
                                                                   _ptr(token_class), _stream(stream)))


def kvq_append_flush_mixed(cache: KvqCache, k_new, v_new, token_class, stream=None):
    _check("kvq_append_flush_mixed", load().kvq_append_flush_mixed(ctypes.byref(cache), _ptr(k_new), _ptr(v_new),
                                                                   _ptr(token_class), _stream(stream)))


def kvq_decode_workspace_bytes(cache: KvqCache, num_splits: int, max_len: int) -> int:
    return int(load().kvq_decode_workspace_bytes(ctypes.byref(cache), int(num_splits), int(max_len)))


def kvq_decode_default_splits(cache: KvqCache, max_len: int) -> int:
    return int(load().kvq_decode_default_splits(ctypes.byref(cache), int(max_len)))


def kvq_decode_attention(cache: KvqCache, q, out, softmax_scale: float, workspace, ws_bytes: int,
                         num_splits: int, max_len: int, stream=None):
    _check("kvq_decode_attention",
           load().kvq_decode_attention(ctypes.byref(cache), _ptr(q), _ptr(out), float(softmax_scale),
                                       _ptr(workspace), int(ws_bytes), int(num_splits), int(max_len),
                                       _stream(stream)))


def kvq_decode_attention_lse(cache: KvqCache, q, out, lse, softmax_scale: float, workspace, ws_bytes: int,
                             num_splits: int, max_len: int, stream=None):
    """kvq_decode_attention that also writes each row's ln-sum-exp into
    `lse` (float [B][H_q])."""
    _check("kvq_decode_attention_lse",
           load().kvq_decode_attention_lse(ctypes.byref(cache), _ptr(q), _ptr(out), _ptr(lse), float(softmax_scale),
                                           _ptr(workspace), int(ws_bytes), int(num_splits), int(max_len),
                                           _stream(stream)))


def kvq_merge_partials(outs, lses, parts: int, rows: int, out, lse_out=None, stream=None):
    """Merge `parts` attentions of the same rows over disjoint token sets:
    outs float [parts][rows][128], lses float [parts][rows] -> out [rows][128]
    (and the merged ln-sum-exp into lse_out [rows] when given)."""
    _check("kvq_merge_partials",
           load().kvq_merge_partials(_ptr(outs), _ptr(lses), int(parts), int(rows), _ptr(out), _ptr(lse_out),
                                     _stream(stream)))


def kvq_decode_attention_noalloc(cache: KvqCache, q, out, softmax_scale: float, num_splits: int, max_len: int,
                                 stream=None):
    """Decode without a workspace: the split partials use the library's fixed
    device array (see include/kvq.h for its size and sharing rules)."""
    _check("kvq_decode_attention_noalloc",
           load().kvq_decode_attention_noalloc(ctypes.byref(cache), _ptr(q), _ptr(out), float(softmax_scale),
                                               int(num_splits), int(max_len), _stream(stream)))


def kvq_read_error(cache: KvqCache, stream=None) -> int:
    v = ctypes.c_uint32(0)
    _check("kvq_read_error", load().kvq_read_error(ctypes.byref(cache), ctypes.byref(v), _stream(stream)))
    return v.value


# --------------------------------------------------------------------------
# A cache whose buffers are torch device tensors
# --------------------------------------------------------------------------

class Cache:
    """Allocates every region of a cache (torch uint8 tensors on `device`)
    and keeps the C descriptor pointing at them."""

    def __init__(self, fmt: int, batch: int, num_q_heads: int, num_kv_heads: int, capacity: int,
                 group: int = 32, residual: int = 128, page_size: int = 0, max_pages_per_seq: int = 0,
                 num_pages: int = 0, head_dim: int = 128, device="cuda", rope_theta: float = 0.0,
                 sparse: bool = False):
        load()
        self.shape = KvqShape(fmt, batch, num_q_heads, num_kv_heads, head_dim, group, residual, capacity,
                              page_size, max_pages_per_seq, num_pages, float(rope_theta), int(sparse))
        self.device = torch.device(device)
        self.buffers = {}
        for i, name in enumerate(REGIONS):
            n = kvq_buffer_bytes(self.shape, i)
            # torch's caching allocator hands out 256-byte aligned blocks
            t = torch.zeros(max(n, 16), dtype=torch.uint8, device=self.device) if n else None
            self.buffers[name] = t
        self.desc = KvqCache(self.shape, *[self.buffers[n].data_ptr() if self.buffers[n] is not None else None
                                           for n in REGIONS])

    @property
    def fmt(self) -> int:
        return self.shape.format

    def region(self, name: str) -> torch.Tensor:
        return self.buffers[name]

    def seq_len(self) -> torch.Tensor:
        return self.buffers["seq_len"].view(torch.int32)

    def n_quant(self) -> torch.Tensor:
        return self.buffers["n_quant"].view(torch.int32)

    def set_page_table(self, table: torch.Tensor):
        t = self.buffers["page_table"].view(torch.int32).view(self.shape.batch, self.shape.max_pages_per_seq)
        t.copy_(table.to(torch.int32))

    def clear_error(self):
        self.buffers["err_word"].zero_()

    def error(self, stream=None) -> int:
        return kvq_read_error(self.desc, stream)

    def quantize_prefill(self, k, v, cu_seqlens, max_len: int, stream=None):
        kvq_quantize_prefill(self.desc, k, v, cu_seqlens, max_len, stream)

    def append_token(self, k_new, v_new, stream=None):
        kvq_append_token(self.desc, k_new, v_new, stream)

    def flush_group(self, stream=None):
        kvq_flush_group(self.desc, stream)

    def append_flush(self, k_new, v_new, stream=None):
        kvq_append_flush(self.desc, k_new, v_new, stream)

    def quantize_prefill_mixed(self, k, v, token_class, cu_seqlens, max_len: int, stream=None):
        kvq_quantize_prefill_mixed(self.desc, k, v, token_class, cu_seqlens, max_len, stream)

    def append_token_mixed(self, k_new, v_new, token_class, stream=None):
        kvq_append_token_mixed(self.desc, k_new, v_new, token_class, stream)

    def append_flush_mixed(self, k_new, v_new, token_class, stream=None):
        kvq_append_flush_mixed(self.desc, k_new, v_new, token_class, stream)

    def workspace_bytes(self, num_splits: int, max_len: int) -> int:
        return kvq_decode_workspace_bytes(self.desc, num_splits, max_len)

    def decode_attention(self, q, out, softmax_scale: float, workspace, num_splits: int, max_len: int,
                         stream=None):
        kvq_decode_attention(self.desc, q, out, softmax_scale, workspace, workspace.numel() * workspace.element_size(),
                             num_splits, max_len, stream)

    def decode_attention_lse(self, q, out, lse, softmax_scale: float, workspace, num_splits: int, max_len: int,
                             stream=None):
        kvq_decode_attention_lse(self.desc, q, out, lse, softmax_scale, workspace,
                                 workspace.numel() * workspace.element_size(), num_splits, max_len, stream)
