"""Seeded synthetic workloads for the KV-cache quantization path.

This module only draws numbers and lays them out; it contains no
quantization, packing or attention arithmetic.  Both the CUDA path (through
the bench and the GPU tests) and the CPU oracle (through the tests) receive
their inputs from here, so that the two sides see identical bf16 tensors.

Value structure follows the KV statistics described on the source pages
(arganzheng.life "KV cache compression", section 2.1; door4ai-lab "KV Cache
lab", experiment 03): keys carry a few fixed outlier channels, values carry a
few heavy tokens, and long-context keys are rotated by RoPE.

Streams (sub-stream ids of the counter-based generator in synth.c):
  1 K, 2 V, 3 q, 4 outlier-channel choice, 5 heavy-token choice,
  6 sequence lengths, 7 page permutation, 100+step streaming K,
  200+step streaming V, 300+step streaming heavy-token draw.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_PATH = os.path.join(_HERE, "libkvq_synth.so")
_lib = None

SEED_BASE = 0xB17C0000
K_OUTLIER_FACTOR = 20.0
Q_OUTLIER_FACTOR = 5.0
V_HEAVY_FACTOR = 5.0
N_OUTLIER_CHANNELS = 4
HEAVY_FRACTION = 0.01
ROPE_THETA_70B = 500000.0


def build(force: bool = False) -> str:
    """Compile synth.c into libkvq_synth.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        u64, i64, i32, dbl = ctypes.c_uint64, ctypes.c_int64, ctypes.c_int32, ctypes.c_double
        vp = ctypes.c_void_p
        lib.synth_u64.argtypes = [u64, u64, u64, i64, vp]
        lib.synth_uniform.argtypes = [u64, u64, u64, i64, vp]
        lib.synth_normal.argtypes = [u64, u64, u64, i64, vp]
        lib.synth_fill_rows_bf16.argtypes = [u64, u64, u64, i64, i32, i32, vp, vp, dbl, vp, vp]
        for f in (lib.synth_u64, lib.synth_uniform, lib.synth_normal, lib.synth_fill_rows_bf16):
            f.restype = None
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def draw_u64(seed: int, stream: int, first: int, count: int) -> np.ndarray:
    out = np.empty(count, dtype=np.uint64)
    _load().synth_u64(seed, stream, first, count, _ptr(out))
    return out


def draw_uniform(seed: int, stream: int, first: int, count: int) -> np.ndarray:
    out = np.empty(count, dtype=np.float64)
    _load().synth_uniform(seed, stream, first, count, _ptr(out))
    return out


def draw_normal(seed: int, stream: int, first: int, count: int) -> np.ndarray:
    out = np.empty(count, dtype=np.float64)
    _load().synth_normal(seed, stream, first, count, _ptr(out))
    return out


def fill_rows_bf16(seed: int, stream: int, index0: int, n_tok: int, H: int, D: int,
                   chan_factor: Optional[np.ndarray] = None,
                   tok_factor: Optional[np.ndarray] = None,
                   rope_theta: float = 0.0,
                   positions: Optional[np.ndarray] = None) -> np.ndarray:
    """bf16 bits, shape [n_tok, H, D]; see synth_fill_rows_bf16 in synth.c."""
    if D > 1024 or D % 2:
        raise ValueError("head_dim must be even and at most 1024")
    out = np.empty((n_tok, H, D), dtype=np.uint16)
    cf = None if chan_factor is None else np.ascontiguousarray(chan_factor, dtype=np.float64).reshape(H, D)
    tf = None if tok_factor is None else np.ascontiguousarray(tok_factor, dtype=np.float64).reshape(n_tok)
    pos = None
    if rope_theta > 0.0:
        pos = np.ascontiguousarray(positions, dtype=np.int64).reshape(n_tok)
    _load().synth_fill_rows_bf16(seed, stream, index0, n_tok, H, D, _ptr(cf), _ptr(tf),
                                 float(rope_theta), _ptr(pos), _ptr(out))
    return out


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32 (a 16-bit shift)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def smallest_keys(seed: int, stream: int, first: int, n: int, m: int) -> np.ndarray:
    """Indices of the m smallest of n seeded 64-bit keys (a seeded m-subset), sorted."""
    keys = draw_u64(seed, stream, first, n)
    return np.sort(np.argsort(keys, kind="stable")[:m])


# --------------------------------------------------------------------------
# Workloads
# --------------------------------------------------------------------------

@dataclasses.dataclass
class Workload:
    """One batch of synthetic decode-attention inputs.

    k, v: bf16 bits [T_total, H_kv, D], sequences packed back to back
          (token-major, ragged, offsets in cu_seqlens)
    q:    bf16 bits [B, H_q, D]
    """
    name: str
    seed: int
    bits: int                 # cache format: 2, 4 (INT), 6 (mixed 2/4), 8 (FP8-E4M3), 16 (INT8 per token)
    group: int                # G
    residual: int             # R
    page_size: int            # 0 = contiguous cache, else tokens per page
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    lengths: np.ndarray       # int64 [B]
    cu_seqlens: np.ndarray    # int32 [B+1]
    k: np.ndarray
    v: np.ndarray
    q: np.ndarray
    outlier_channels: np.ndarray   # int64 [H_kv, 4]
    heavy_tokens: list             # per sequence, sorted token positions
    rope_theta: float = 0.0

    @property
    def batch(self) -> int:
        return int(self.lengths.shape[0])

    @property
    def softmax_scale(self) -> float:
        return 1.0 / float(np.sqrt(self.head_dim))

    def seq_k(self, b: int) -> np.ndarray:
        return self.k[self.cu_seqlens[b]:self.cu_seqlens[b + 1]]

    def seq_v(self, b: int) -> np.ndarray:
        return self.v[self.cu_seqlens[b]:self.cu_seqlens[b + 1]]


def outlier_channels(seed: int, H_kv: int, D: int) -> np.ndarray:
    return np.stack([smallest_keys(seed, 4, h * D, D, N_OUTLIER_CHANNELS) for h in range(H_kv)])


def make_workload(name: str, seed: int, lengths, num_q_heads: int, num_kv_heads: int,
                  bits: int, group: int, residual: int, page_size: int = 0,
                  head_dim: int = 128, rope_theta: float = 0.0,
                  k_outlier: float = K_OUTLIER_FACTOR, q_outlier: float = Q_OUTLIER_FACTOR,
                  v_heavy: float = V_HEAVY_FACTOR) -> Workload:
    lengths = np.asarray(lengths, dtype=np.int64).reshape(-1)
    B = lengths.shape[0]
    H_kv, H_q, D = num_kv_heads, num_q_heads, head_dim
    cu = np.zeros(B + 1, dtype=np.int64)
    cu[1:] = np.cumsum(lengths)
    T = int(cu[-1])
    oc = outlier_channels(seed, H_kv, D)
    kf = np.ones((H_kv, D))
    for h in range(H_kv):
        kf[h, oc[h]] = k_outlier
    heavy = []
    vf = np.ones(T)
    for b in range(B):
        n = int(lengths[b])
        m = int(round(HEAVY_FRACTION * n))
        ht = smallest_keys(seed, 5, b << 40, n, m) if m > 0 else np.zeros(0, dtype=np.int64)
        heavy.append(ht)
        vf[cu[b] + ht] = v_heavy
    pos = None
    if rope_theta > 0.0:
        pos = np.concatenate([np.arange(int(n), dtype=np.int64) for n in lengths]) if T else np.zeros(0, np.int64)
    k = fill_rows_bf16(seed, 1, 0, T, H_kv, D, chan_factor=kf, rope_theta=rope_theta, positions=pos)
    v = fill_rows_bf16(seed, 2, 0, T, H_kv, D, tok_factor=vf)
    g = H_q // H_kv
    qf = np.ones((H_q, D))
    for h in range(H_q):
        qf[h, oc[h // g]] = q_outlier
    q = fill_rows_bf16(seed, 3, 0, B, H_q, D, chan_factor=qf)
    return Workload(name=name, seed=seed, bits=bits, group=group, residual=residual,
                    page_size=page_size, num_q_heads=H_q, num_kv_heads=H_kv, head_dim=D,
                    lengths=lengths, cu_seqlens=cu.astype(np.int32), k=k, v=v, q=q,
                    outlier_channels=oc, heavy_tokens=heavy, rope_theta=rope_theta)


MIXED_HIGH_FRACTION = 0.30      # share of tokens in classes kept at 4 bits (the rest at 2)
MIXED_SPAN = (64, 512)          # token classes come in spans of these lengths (uniform)


def token_classes(seed: int, lengths, high_fraction: float = MIXED_HIGH_FRACTION, span=MIXED_SPAN,
                  stream: int = 8) -> np.ndarray:
    """Seeded per-token classes for a mixed 2/4-bit cache: uint8 [sum(lengths)],
    2 or 4.  Agent contexts come as stretches of one kind (a system prompt, a
    tool schema, a chain of thought, a tool call, an observation), so the
    classes are drawn per stretch: each sequence is cut into spans of
    uniform length in [span[0], span[1]], and a span is class 4 with
    probability high_fraction, else class 2."""
    lengths = np.asarray(lengths, dtype=np.int64).reshape(-1)
    out = np.empty(int(lengths.sum()), np.uint8)
    off = 0
    for b, n in enumerate(lengths):
        n = int(n)
        u = draw_uniform(seed, stream, b << 40, 2 * (n // span[0] + 2))
        t = i = 0
        while t < n:
            L = span[0] + int(u[2 * i] * (span[1] - span[0] + 1))
            out[off + t:off + min(n, t + L)] = 4 if u[2 * i + 1] < high_fraction else 2
            t += L
            i += 1
        off += n
    return out


def streaming_class(w: "Workload", step: int) -> np.ndarray:
    """Class (2 or 4) of the token appended at streaming step `step`, per
    sequence: the class of the span the sequence is in continues."""
    return token_classes(w.seed, w.lengths + step + 1)[np.cumsum(w.lengths + step + 1) - 1]


def config_lengths(config_id: int, batch: int) -> np.ndarray:
    """Sequence lengths of the ragged paged batch: uniform on {1024..32768}."""
    u = draw_uniform(SEED_BASE + config_id, 6, 0, batch)
    return (1024 + np.floor(u * (32768 - 1024 + 1))).astype(np.int64)


def make_config(config_id: int, bits: Optional[int] = None, lengths=None, rope: bool = True) -> Workload:
    """The five named workloads (sizes as stated with each):

    0  tiny KIVI check: B=1, 1 q head, 1 kv head, n=512, INT2, G=32, R=32
    1  Llama-3-8B layer: B=8, 32/8 heads, n=8192, INT4, G=32, R=128
    2  Llama-3-70B long context: B=1, 64/8 heads, n=131072, INT4 or INT2,
       G=32, R=128, K rotated by RoPE (theta 500000)
    3  paged ragged batch: B=64, n ~ U{1024..32768}, 32/8 heads, INT4,
       G=16 = page size, R=16
    4  streaming start state: B=16, 32/8 heads, n=4096, INT2 (or 8 = FP8),
       G=32, R=128
    `lengths` overrides the sequence lengths (smaller parity cases with the
    same distributions).  rope=False gives config 2's keys before RoPE (the
    same seeded values, not rotated), for a cache that rotates keys at read.
    """
    seed = SEED_BASE + config_id
    if config_id == 0:
        L = [512] if lengths is None else lengths
        return make_workload("c0_tiny_int2", seed, L, 1, 1, bits or 2, 32, 32)
    if config_id == 1:
        L = [8192] * 8 if lengths is None else lengths
        b = bits or 4
        name = {16: "c1_llama3_8b_int8_per_token", 6: "c1_llama3_8b_mixed24"}.get(b, "c1_llama3_8b_int%d" % b)
        return make_workload(name, seed, L, 32, 8, b, 32 if b != 16 else 16, 128 if b != 16 else 0)
    if config_id == 2:
        b = bits or 4
        L = [131072] if lengths is None else lengths
        return make_workload("c2_llama3_70b_128k_int%d%s" % (b, "" if rope else "_pre_rope"), seed, L, 64, 8, b,
                             32, 128, rope_theta=ROPE_THETA_70B if rope else 0.0)
    if config_id == 3:
        L = config_lengths(3, 64) if lengths is None else lengths
        return make_workload("c3_paged_ragged_int4", seed, L, 32, 8, bits or 4, 16, 16, page_size=16)
    if config_id == 4:
        b = bits or 2
        L = [4096] * 16 if lengths is None else lengths
        name = {8: "fp8", 16: "int8_per_token"}.get(b, "int%d" % b)
        tok = b in (8, 16)                  # every token quantized on write: no window
        return make_workload("c4_streaming_%s" % name, seed, L, 32, 8, b, 16 if tok else 32, 0 if tok else 128)
    raise ValueError("unknown config %r" % (config_id,))


def streaming_token(w: Workload, step: int):
    """K and V of the token appended at streaming step `step`: bf16 bits [B, H_kv, D].

    Same distributions as the prefill: K outlier channels x20, and the token
    is heavy (V x5 over all kv heads) with probability 1%.
    """
    B, H_kv, D = w.batch, w.num_kv_heads, w.head_dim
    kf = np.ones((H_kv, D))
    for h in range(H_kv):
        kf[h, w.outlier_channels[h]] = K_OUTLIER_FACTOR
    heavy = draw_uniform(w.seed, 300 + step, 0, B) < HEAVY_FRACTION
    vf = np.where(heavy, V_HEAVY_FACTOR, 1.0)
    pos = None
    if w.rope_theta > 0.0:
        pos = w.lengths + step
    k = fill_rows_bf16(w.seed, 100 + step, 0, B, H_kv, D, chan_factor=kf,
                       rope_theta=w.rope_theta, positions=pos)
    v = fill_rows_bf16(w.seed, 200 + step, 0, B, H_kv, D, tok_factor=vf)
    return k, v


def page_table(w: Workload, extra_tokens: int = 0, max_pages_per_seq: Optional[int] = None):
    """Seeded page placement for a paged cache: sequence b owns
    ceil((n_b + extra_tokens) / page) logical pages; the pool holds exactly
    their sum, and physical ids are a seeded permutation of the pool.
    Returns (table int32 [B, max_pages_per_seq] with -1 past each sequence's
    pages, num_pages)."""
    P = w.page_size
    need = [int((int(n) + extra_tokens + P - 1) // P) for n in w.lengths]
    total = int(sum(need))
    mp = max_pages_per_seq or max(1, max(need))
    keys = draw_u64(w.seed, 7, 0, max(total, 1))
    perm = np.argsort(keys, kind="stable")[:total].astype(np.int32)
    table = np.full((w.batch, mp), -1, dtype=np.int32)
    off = 0
    for b, k in enumerate(need):
        table[b, :k] = perm[off:off + k]
        off += k
    return table, max(total, 1)
