"""CPU oracle of the asymmetric low-bit KV cache (TEST INFRASTRUCTURE ONLY).

Only `tests/`, the package's `smoke()` check and the bench's CPU-baseline leg
may import this module.  The product path (the CUDA library and its Python
binding) never does, and this module never imports the product path: the two
share only the seeded inputs from the synthetic-workload module.

The arithmetic lives in kvq_oracle.c (plain single-threaded C, built with
-O2 -ffp-contract=off and no fast-math); this file builds it and marshals
numpy arrays.  Each C routine's header comment names the page passage it
follows.  Parity status of every function is pinned by tests/test_oracle_*.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkvq_oracle.so")
_lib = None

C_FLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", *C_FLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Unit(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int32), ("D", ctypes.c_int32), ("G", ctypes.c_int32),
                ("R", ctypes.c_int32), ("cap", ctypes.c_int32), ("n", ctypes.c_int32),
                ("n_q", ctypes.c_int32),
                ("k_codes", ctypes.c_void_p), ("k_scale", ctypes.c_void_p), ("k_zero", ctypes.c_void_p),
                ("v_codes", ctypes.c_void_p), ("v_scale", ctypes.c_void_p), ("v_zero", ctypes.c_void_p),
                ("k_ring", ctypes.c_void_p), ("v_ring", ctypes.c_void_p),
                ("group_bits", ctypes.c_void_p), ("ring_class", ctypes.c_void_p),
                ("k_out", ctypes.c_void_p), ("k_out_idx", ctypes.c_void_p),
                ("v_out", ctypes.c_void_p), ("v_out_idx", ctypes.c_void_p)]


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i32, i64, f32, f64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_double
    u8, u16 = ctypes.c_uint8, ctypes.c_uint16
    sig = {
        "oracle_bf16_to_f32": (f32, [u16]),
        "oracle_f16_to_f32": (f32, [u16]),
        "oracle_f32_to_f16": (u16, [f32]),
        "oracle_e4m3_decode": (f32, [u8]),
        "oracle_e4m3_encode": (u8, [f32]),
        "oracle_e4m3_encode_bruteforce": (u8, [f32]),
        "oracle_quant_params": (None, [f32, f32, i32, vp, vp]),
        "oracle_encode": (u8, [f32, u16, u16, i32]),
        "oracle_encode_truediv": (u8, [f32, u16, u16, i32]),
        "oracle_quantize_set": (None, [vp, i64, i64, i32, vp, i64, vp, vp]),
        "oracle_quantize_set_sparse": (i32, [vp, vp, i64, i64, i32, vp, i64, vp, vp, vp]),
        "oracle_dequant": (f64, [u8, u16, u16]),
        "oracle_pack": (None, [vp, i64, i32, vp]),
        "oracle_unpack": (None, [vp, i64, i32, vp]),
        "oracle_kv_bytes": (i64, [i64, i64, i64, i64, i64]),
        "oracle_unit_prefill": (i32, [ctypes.POINTER(_Unit), vp, vp, i64, i32]),
        "oracle_unit_append": (i32, [ctypes.POINTER(_Unit), vp, vp]),
        "oracle_unit_flush": (i32, [ctypes.POINTER(_Unit)]),
        "oracle_unit_prefill_mixed": (i32, [ctypes.POINTER(_Unit), vp, vp, i64, i32, vp]),
        "oracle_unit_append_mixed": (i32, [ctypes.POINTER(_Unit), vp, vp, i32]),
        "oracle_unit_materialize": (None, [ctypes.POINTER(_Unit), vp, vp]),
        "oracle_attend": (None, [vp, vp, i32, i32, vp, i64, i32, f64, vp, vp, vp]),
        "oracle_unit_decode": (None, [ctypes.POINTER(_Unit), vp, i64, i32, f64, vp, vp]),
        "oracle_rope_rows": (None, [vp, i64, i32, f64, i64]),
        "oracle_unit_decode_rope": (None, [ctypes.POINTER(_Unit), vp, i64, i32, f64, f64, vp, vp]),
        "oracle_fp8_scale": (f32, [f32]),
        "oracle_amax_rows": (None, [vp, i64, i64, i32, vp]),
        "oracle_fp8_encode_rows": (None, [vp, i64, i64, i32, f32, vp]),
        "oracle_fp8_decode": (None, [vp, vp, i32, i32, f32, f32, vp, i64, i32, f64, vp, vp]),
        "oracle_int8_encode_rows": (None, [vp, i64, i64, i32, vp, vp, vp]),
        "oracle_int8_materialize": (None, [vp, vp, vp, vp, vp, vp, i32, i32, vp, vp]),
        "oracle_int8_decode": (None, [vp, vp, vp, vp, vp, vp, i32, i32, vp, i64, i32, f64, vp, vp]),
        "oracle_f32_to_f16_array": (None, [vp, i64, vp]),
        "oracle_f16_to_f32_array": (None, [vp, i64, vp]),
        "oracle_e4m3_encode_array": (None, [vp, i64, vp]),
        "oracle_e4m3_encode_bruteforce_array": (None, [vp, i64, vp]),
        "oracle_e4m3_decode_array": (None, [vp, i64, vp]),
        "oracle_encode_array": (None, [vp, i64, u16, u16, i32, i32, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


# --------------------------------------------------------------------------
# Scalar and array routines
# --------------------------------------------------------------------------

def f32_to_f16(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().oracle_f32_to_f16_array(_p(x), x.size, _p(out))
    return out


def f16_to_f32(h) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(h.shape, dtype=np.float32)
    _load().oracle_f16_to_f32_array(_p(h), h.size, _p(out))
    return out


def e4m3_encode(x, bruteforce: bool = False) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    f = _load().oracle_e4m3_encode_bruteforce_array if bruteforce else _load().oracle_e4m3_encode_array
    f(_p(x), x.size, _p(out))
    return out


def e4m3_decode(c) -> np.ndarray:
    c = np.ascontiguousarray(c, dtype=np.uint8)
    out = np.empty(c.shape, dtype=np.float32)
    _load().oracle_e4m3_decode_array(_p(c), c.size, _p(out))
    return out


def quant_params(mn: float, mx: float, bits: int):
    s, z = ctypes.c_uint16(), ctypes.c_uint16()
    _load().oracle_quant_params(float(mn), float(mx), bits, ctypes.byref(s), ctypes.byref(z))
    return s.value, z.value


def encode(x, s16: int, z16: int, bits: int, truediv: bool = False) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    _load().oracle_encode_array(_p(x), x.size, s16, z16, bits, int(truediv), _p(out))
    return out


def quantize_set_sparse(x_bits, bits: int):
    """Dense-and-sparse quantization of one set given as bf16 bits: returns
    codes, s16, z16, the kept value's bf16 bits and its index."""
    xb = np.ascontiguousarray(x_bits, dtype=np.uint16).reshape(-1)
    xf = np.ascontiguousarray((xb.astype(np.uint32) << 16).view(np.float32))
    codes = np.empty(xb.size, dtype=np.uint8)
    s, z, o = ctypes.c_uint16(), ctypes.c_uint16(), ctypes.c_uint16()
    idx = _load().oracle_quantize_set_sparse(_p(xf), _p(xb), xb.size, 1, bits, _p(codes), 1, ctypes.byref(s),
                                             ctypes.byref(z), ctypes.byref(o))
    return codes, s.value, z.value, o.value, int(idx)


def quantize_set(x, bits: int):
    """One (scale, zero) over all of x (float32): returns codes, s16, z16."""
    x = np.ascontiguousarray(x, dtype=np.float32).reshape(-1)
    codes = np.empty(x.size, dtype=np.uint8)
    s, z = ctypes.c_uint16(), ctypes.c_uint16()
    _load().oracle_quantize_set(_p(x), x.size, 1, bits, _p(codes), 1, ctypes.byref(s), ctypes.byref(z))
    return codes, s.value, z.value


def dequant(codes, s16, z16) -> np.ndarray:
    """code * s + z in double (vectorised over broadcastable arrays)."""
    s = f16_to_f32(np.asarray(s16, dtype=np.uint16)).astype(np.float64)
    z = f16_to_f32(np.asarray(z16, dtype=np.uint16)).astype(np.float64)
    return np.asarray(codes, dtype=np.float64) * s + z


def quantize_matrix(x, bits: int, axis: int):
    """Quantize a 2-D float32 matrix with one (scale, zero) per slice along
    `axis` (axis=0: per column, i.e. the range over rows; axis=1: per row).
    Returns the dequantized matrix (double)."""
    x = np.asarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.float64)
    if axis == 0:
        for c in range(x.shape[1]):
            codes, s, z = quantize_set(x[:, c], bits)
            out[:, c] = dequant(codes, s, z)
    else:
        for r in range(x.shape[0]):
            codes, s, z = quantize_set(x[r, :], bits)
            out[r, :] = dequant(codes, s, z)
    return out


def pack(codes, bits: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8).reshape(-1)
    out = np.empty(codes.size * bits // 8, dtype=np.uint8)
    _load().oracle_pack(_p(codes), codes.size, bits, _p(out))
    return out


def unpack(packed, count: int, bits: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8).reshape(-1)
    out = np.empty(count, dtype=np.uint8)
    _load().oracle_unpack(_p(packed), count, bits, _p(out))
    return out


def rope_rows(x, theta: float, pos0: int = 0) -> np.ndarray:
    """RoPE of rows x [n, D] (double) at positions pos0, pos0 + 1, ..."""
    y = np.ascontiguousarray(x, dtype=np.float64).copy()
    n, D = y.shape
    _load().oracle_rope_rows(_p(y), n, D, float(theta), int(pos0))
    return y


def kv_bytes(layers: int, kv_heads: int, tokens: int, head_dim: int, bits_per_elem: int) -> int:
    return int(_load().oracle_kv_bytes(layers, kv_heads, tokens, head_dim, bits_per_elem))


def attend(khat, vhat, q_bits, scale: float, return_logits: bool = False):
    """Softmax attention in double of bf16 query rows over given K^, V^ rows."""
    khat = np.ascontiguousarray(khat, dtype=np.float64)
    vhat = np.ascontiguousarray(vhat, dtype=np.float64)
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    n, D = khat.shape
    nh = q_bits.shape[0]
    out = np.empty((nh, D), dtype=np.float64)
    lg = np.empty((nh, n), dtype=np.float64) if return_logits else None
    work = np.empty(max(n, 1), dtype=np.float64)
    _load().oracle_attend(_p(khat), _p(vhat), n, D, _p(q_bits), D, nh, scale, _p(out),
                          None if lg is None else _p(lg), _p(work))
    return (out, lg) if return_logits else out


# --------------------------------------------------------------------------
# The cache
# --------------------------------------------------------------------------

class Unit:
    """One (sequence, kv head) unit of the low-bit cache.  mixed=True: every
    group is stored at 2 or 4 bits by its tokens' classes (prefill and
    append then take the classes; `bits` is unused).  sparse=True: every key
    and value set keeps its largest-magnitude value aside (dense-and-sparse)."""

    def __init__(self, bits: int, head_dim: int, group: int, residual: int, capacity: int, mixed: bool = False,
                 sparse: bool = False):
        if capacity % group:
            raise ValueError("capacity must be a multiple of the group")
        D, G, R = head_dim, group, residual
        self.mixed = mixed
        self.group_bits = np.zeros(capacity // G, np.uint8) if mixed else None
        self.ring_class = np.zeros(R + G, np.uint8) if mixed else None
        self.sparse = sparse
        self.k_out = np.zeros((capacity // G, D), np.uint16) if sparse else None
        self.k_out_idx = np.zeros((capacity // G, D), np.uint8) if sparse else None
        self.v_out = np.zeros(capacity, np.uint16) if sparse else None
        self.v_out_idx = np.zeros(capacity, np.uint8) if sparse else None
        ptr = lambda a: None if a is None else a.ctypes.data
        self.k_codes = np.zeros((capacity, D), np.uint8)
        self.k_scale = np.zeros((capacity // G, D), np.uint16)
        self.k_zero = np.zeros((capacity // G, D), np.uint16)
        self.v_codes = np.zeros((capacity, D), np.uint8)
        self.v_scale = np.zeros(capacity, np.uint16)
        self.v_zero = np.zeros(capacity, np.uint16)
        self.k_ring = np.zeros((R + G, D), np.uint16)
        self.v_ring = np.zeros((R + G, D), np.uint16)
        self.s = _Unit(bits, D, G, R, capacity, 0, 0,
                       self.k_codes.ctypes.data, self.k_scale.ctypes.data, self.k_zero.ctypes.data,
                       self.v_codes.ctypes.data, self.v_scale.ctypes.data, self.v_zero.ctypes.data,
                       self.k_ring.ctypes.data, self.v_ring.ctypes.data,
                       ptr(self.group_bits), ptr(self.ring_class),
                       ptr(self.k_out), ptr(self.k_out_idx), ptr(self.v_out), ptr(self.v_out_idx))

    @property
    def n(self) -> int:
        return self.s.n

    @property
    def n_q(self) -> int:
        return self.s.n_q

    def prefill(self, k_rows, v_rows, classes=None):
        """k_rows, v_rows: bf16 bits [n, D] (any row stride); classes: the
        tokens' classes (2 or 4) for a mixed unit."""
        k_rows = np.asarray(k_rows, dtype=np.uint16)
        v_rows = np.asarray(v_rows, dtype=np.uint16)
        n, D = k_rows.shape
        assert k_rows.strides == v_rows.strides and k_rows.strides[1] == 2
        ld = k_rows.strides[0] // 2
        if self.mixed:
            cls = np.ascontiguousarray(classes, dtype=np.uint8).reshape(-1)
            assert cls.size == n
            rc = _load().oracle_unit_prefill_mixed(ctypes.byref(self.s), ctypes.c_void_p(k_rows.ctypes.data),
                                                   ctypes.c_void_p(v_rows.ctypes.data), ld, n, _p(cls))
        else:
            rc = _load().oracle_unit_prefill(ctypes.byref(self.s), ctypes.c_void_p(k_rows.ctypes.data),
                                             ctypes.c_void_p(v_rows.ctypes.data), ld, n)
        if rc != 0:
            raise ValueError("prefill rejected (capacity)")

    def append(self, k_tok, v_tok, cls=None) -> bool:
        k_tok = np.ascontiguousarray(k_tok, dtype=np.uint16)
        v_tok = np.ascontiguousarray(v_tok, dtype=np.uint16)
        if self.mixed:
            return _load().oracle_unit_append_mixed(ctypes.byref(self.s), _p(k_tok), _p(v_tok), int(cls)) == 0
        return _load().oracle_unit_append(ctypes.byref(self.s), _p(k_tok), _p(v_tok)) == 0

    def flush(self) -> bool:
        return _load().oracle_unit_flush(ctypes.byref(self.s)) == 1

    def materialize(self):
        n, D = self.s.n, self.s.D
        kh = np.empty((n, D), np.float64)
        vh = np.empty((n, D), np.float64)
        _load().oracle_unit_materialize(ctypes.byref(self.s), _p(kh), _p(vh))
        return kh, vh

    def decode(self, q_rows, scale: float, rope_theta: float = 0.0) -> np.ndarray:
        """rope_theta > 0: the unit's keys are pre-RoPE; key t is rotated by
        its position t before the scores."""
        q_rows = np.ascontiguousarray(q_rows, dtype=np.uint16)
        nh, D = q_rows.shape
        out = np.empty((nh, D), np.float64)
        work = np.empty(2 * self.s.n * D + self.s.n + 1, np.float64)
        if rope_theta > 0.0:
            _load().oracle_unit_decode_rope(ctypes.byref(self.s), _p(q_rows), D, nh, scale, rope_theta, _p(out),
                                            _p(work))
        else:
            _load().oracle_unit_decode(ctypes.byref(self.s), _p(q_rows), D, nh, scale, _p(out), _p(work))
        return out

    def ring_slot(self, t: int) -> int:
        return t % (self.s.R + self.s.G)


class Cache:
    """The whole batch: units[b][kv].  mixed=True: 2/4-bit groups by token
    class; sparse=True: dense-and-sparse sets."""

    def __init__(self, bits: int, batch: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                 group: int, residual: int, capacity: int, mixed: bool = False, sparse: bool = False):
        self.bits, self.B, self.H_q, self.H_kv, self.D = bits, batch, num_q_heads, num_kv_heads, head_dim
        self.G, self.R, self.cap, self.mixed, self.sparse = group, residual, capacity, mixed, sparse
        self.units = [[Unit(bits, head_dim, group, residual, capacity, mixed, sparse) for _ in range(num_kv_heads)]
                      for _ in range(batch)]

    def prefill(self, k, v, cu_seqlens, units=None, classes=None):
        """k, v: bf16 bits [T_total, H_kv, D]; units: optional list of (b, kv)
        to fill; classes: [T_total] token classes (2 or 4) for a mixed cache."""
        todo = units if units is not None else [(b, h) for b in range(self.B) for h in range(self.H_kv)]
        for b, h in todo:
            lo, hi = int(cu_seqlens[b]), int(cu_seqlens[b + 1])
            self.units[b][h].prefill(k[lo:hi, h, :], v[lo:hi, h, :],
                                     None if classes is None else classes[lo:hi])

    def append(self, k_new, v_new, classes=None) -> np.ndarray:
        """k_new, v_new: [B, H_kv, D]; classes: [B] for a mixed cache.
        Returns per-(b, kv) acceptance."""
        return np.array([[self.units[b][h].append(k_new[b, h], v_new[b, h],
                                                  None if classes is None else classes[b])
                          for h in range(self.H_kv)] for b in range(self.B)])

    def flush(self) -> np.ndarray:
        return np.array([[self.units[b][h].flush() for h in range(self.H_kv)] for b in range(self.B)])

    def decode_unit(self, q, b: int, kv: int, scale: float, rope_theta: float = 0.0) -> np.ndarray:
        g = self.H_q // self.H_kv
        return self.units[b][kv].decode(q[b, kv * g:(kv + 1) * g, :], scale, rope_theta)

    def decode(self, q, scale: float, units=None, rope_theta: float = 0.0) -> np.ndarray:
        """q: bf16 bits [B, H_q, D] -> out [B, H_q, D] (double); NaN where not
        computed.  rope_theta > 0: keys are pre-RoPE, rotated at read."""
        g = self.H_q // self.H_kv
        out = np.full((self.B, self.H_q, self.D), np.nan)
        todo = units if units is not None else [(b, h) for b in range(self.B) for h in range(self.H_kv)]
        for b, h in todo:
            out[b, h * g:(h + 1) * g, :] = self.decode_unit(q, b, h, scale, rope_theta)
        return out


class FP8Cache:
    """FP8-E4M3 cache with one static scale per (kv head, K|V), set by the prefill."""

    def __init__(self, batch: int, num_q_heads: int, num_kv_heads: int, head_dim: int, capacity: int):
        self.B, self.H_q, self.H_kv, self.D, self.cap = batch, num_q_heads, num_kv_heads, head_dim, capacity
        self.k_codes = np.zeros((batch, num_kv_heads, capacity, head_dim), np.uint8)
        self.v_codes = np.zeros((batch, num_kv_heads, capacity, head_dim), np.uint8)
        self.Sk = np.ones(num_kv_heads, np.float32)
        self.Sv = np.ones(num_kv_heads, np.float32)
        self.n = np.zeros(batch, np.int64)

    def prefill(self, k, v, cu_seqlens):
        lib = _load()
        for h in range(self.H_kv):
            ak, av = ctypes.c_float(0.0), ctypes.c_float(0.0)
            for b in range(self.B):
                lo, hi = int(cu_seqlens[b]), int(cu_seqlens[b + 1])
                kr, vr = k[lo:hi, h, :], v[lo:hi, h, :]
                if hi > lo:
                    lib.oracle_amax_rows(ctypes.c_void_p(kr.ctypes.data), kr.strides[0] // 2, hi - lo, self.D,
                                         ctypes.byref(ak))
                    lib.oracle_amax_rows(ctypes.c_void_p(vr.ctypes.data), vr.strides[0] // 2, hi - lo, self.D,
                                         ctypes.byref(av))
            self.Sk[h] = lib.oracle_fp8_scale(ak.value)
            self.Sv[h] = lib.oracle_fp8_scale(av.value)
        for b in range(self.B):
            lo, hi = int(cu_seqlens[b]), int(cu_seqlens[b + 1])
            if hi - lo > self.cap:
                raise ValueError("prefill rejected (capacity)")
            for h in range(self.H_kv):
                self._encode(k[lo:hi, h, :], self.Sk[h], self.k_codes[b, h, :hi - lo])
                self._encode(v[lo:hi, h, :], self.Sv[h], self.v_codes[b, h, :hi - lo])
            self.n[b] = hi - lo

    def _encode(self, rows, S, out):
        if rows.shape[0] == 0:
            return
        tmp = np.empty(rows.shape, np.uint8)
        _load().oracle_fp8_encode_rows(ctypes.c_void_p(rows.ctypes.data), rows.strides[0] // 2, rows.shape[0],
                                       self.D, float(S), _p(tmp))
        out[...] = tmp

    def append(self, k_new, v_new) -> np.ndarray:
        ok = np.zeros((self.B, self.H_kv), bool)
        for b in range(self.B):
            if self.n[b] >= self.cap:
                continue
            for h in range(self.H_kv):
                self._encode(np.ascontiguousarray(k_new[b, h][None, :]), self.Sk[h],
                             self.k_codes[b, h, self.n[b]:self.n[b] + 1])
                self._encode(np.ascontiguousarray(v_new[b, h][None, :]), self.Sv[h],
                             self.v_codes[b, h, self.n[b]:self.n[b] + 1])
                ok[b, h] = True
            self.n[b] += 1
        return ok

    def decode_unit(self, q, b: int, kv: int, scale: float) -> np.ndarray:
        g = self.H_q // self.H_kv
        n = int(self.n[b])
        kc = np.ascontiguousarray(self.k_codes[b, kv, :n])
        vc = np.ascontiguousarray(self.v_codes[b, kv, :n])
        qr = np.ascontiguousarray(q[b, kv * g:(kv + 1) * g, :])
        out = np.empty((g, self.D), np.float64)
        work = np.empty(2 * n * self.D + n + 1, np.float64)
        _load().oracle_fp8_decode(_p(kc), _p(vc), n, self.D, float(self.Sk[kv]), float(self.Sv[kv]),
                                  _p(qr), self.D, g, scale, _p(out), _p(work))
        return out

    def decode(self, q, scale: float, units=None) -> np.ndarray:
        g = self.H_q // self.H_kv
        out = np.full((self.B, self.H_q, self.D), np.nan)
        todo = units if units is not None else [(b, h) for b in range(self.B) for h in range(self.H_kv)]
        for b, h in todo:
            out[b, h * g:(h + 1) * g, :] = self.decode_unit(q, b, h, scale)
        return out


class Int8Cache:
    """INT8 per-token dynamic cache: every key and value row quantized over
    its channels at 8 bits when it is written (one fp16 scale and zero per
    token for K and for V); no window."""

    def __init__(self, batch: int, num_q_heads: int, num_kv_heads: int, head_dim: int, capacity: int):
        self.B, self.H_q, self.H_kv, self.D, self.cap = batch, num_q_heads, num_kv_heads, head_dim, capacity
        shp = (batch, num_kv_heads, capacity)
        self.k_codes = np.zeros(shp + (head_dim,), np.uint8)
        self.v_codes = np.zeros(shp + (head_dim,), np.uint8)
        self.k_scale = np.zeros(shp, np.uint16)
        self.k_zero = np.zeros(shp, np.uint16)
        self.v_scale = np.zeros(shp, np.uint16)
        self.v_zero = np.zeros(shp, np.uint16)
        self.n = np.zeros(batch, np.int64)

    def _encode(self, rows, codes, s, z):
        """rows: bf16 bits [m, D] (any row stride) into codes [m, D], s, z [m]."""
        m = rows.shape[0]
        if m == 0:
            return
        rows = np.asarray(rows, dtype=np.uint16)
        assert rows.strides[1] == 2
        c = np.empty((m, self.D), np.uint8)
        ss = np.empty(m, np.uint16)
        zz = np.empty(m, np.uint16)
        _load().oracle_int8_encode_rows(ctypes.c_void_p(rows.ctypes.data), rows.strides[0] // 2, m, self.D,
                                        _p(c), _p(ss), _p(zz))
        codes[...] = c
        s[...] = ss
        z[...] = zz

    def prefill(self, k, v, cu_seqlens, units=None):
        todo = units if units is not None else [(b, h) for b in range(self.B) for h in range(self.H_kv)]
        for b in range(self.B):
            lo, hi = int(cu_seqlens[b]), int(cu_seqlens[b + 1])
            if hi - lo > self.cap:
                raise ValueError("prefill rejected (capacity)")
            self.n[b] = hi - lo
        for b, h in todo:
            lo, hi = int(cu_seqlens[b]), int(cu_seqlens[b + 1])
            n = hi - lo
            self._encode(k[lo:hi, h, :], self.k_codes[b, h, :n], self.k_scale[b, h, :n], self.k_zero[b, h, :n])
            self._encode(v[lo:hi, h, :], self.v_codes[b, h, :n], self.v_scale[b, h, :n], self.v_zero[b, h, :n])

    def append(self, k_new, v_new) -> np.ndarray:
        ok = np.zeros((self.B, self.H_kv), bool)
        for b in range(self.B):
            t = int(self.n[b])
            if t >= self.cap:
                continue
            for h in range(self.H_kv):
                self._encode(np.ascontiguousarray(k_new[b, h][None, :]), self.k_codes[b, h, t:t + 1],
                             self.k_scale[b, h, t:t + 1], self.k_zero[b, h, t:t + 1])
                self._encode(np.ascontiguousarray(v_new[b, h][None, :]), self.v_codes[b, h, t:t + 1],
                             self.v_scale[b, h, t:t + 1], self.v_zero[b, h, t:t + 1])
                ok[b, h] = True
            self.n[b] += 1
        return ok

    def _unit_arrays(self, b: int, kv: int):
        n = int(self.n[b])
        c = lambda a: np.ascontiguousarray(a[b, kv, :n])
        return (n, c(self.k_codes), c(self.k_scale), c(self.k_zero), c(self.v_codes), c(self.v_scale),
                c(self.v_zero))

    def materialize(self, b: int, kv: int):
        n, kc, ks, kz, vc, vs, vz = self._unit_arrays(b, kv)
        kh = np.empty((n, self.D), np.float64)
        vh = np.empty((n, self.D), np.float64)
        _load().oracle_int8_materialize(_p(kc), _p(ks), _p(kz), _p(vc), _p(vs), _p(vz), n, self.D, _p(kh), _p(vh))
        return kh, vh

    def decode_unit(self, q, b: int, kv: int, scale: float) -> np.ndarray:
        g = self.H_q // self.H_kv
        n, kc, ks, kz, vc, vs, vz = self._unit_arrays(b, kv)
        qr = np.ascontiguousarray(q[b, kv * g:(kv + 1) * g, :])
        out = np.empty((g, self.D), np.float64)
        work = np.empty(2 * n * self.D + n + 1, np.float64)
        _load().oracle_int8_decode(_p(kc), _p(ks), _p(kz), _p(vc), _p(vs), _p(vz), n, self.D, _p(qr), self.D, g,
                                   scale, _p(out), _p(work))
        return out

    def decode(self, q, scale: float, units=None) -> np.ndarray:
        g = self.H_q // self.H_kv
        out = np.full((self.B, self.H_q, self.D), np.nan)
        todo = units if units is not None else [(b, h) for b in range(self.B) for h in range(self.H_kv)]
        for b, h in todo:
            out[b, h * g:(h + 1) * g, :] = self.decode_unit(q, b, h, scale)
        return out
