"""Shared harness of the GPU parity tests: run the CUDA path through the C ABI
and the CPU oracle on the same seeded inputs, and compare."""
import os

import numpy as np
import torch

import oracle
from bit_kv_cache_16_b200 import kvq, synth

from layout import GpuState

ATOL = 2e-3          # max-abs error of the decode output
COS_MIN = 0.9999     # cosine similarity per output row


def to_dev(a: np.ndarray) -> torch.Tensor:
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def round_up(x: int, m: int) -> int:
    return (x + m - 1) // m * m


def make_gpu_cache(w: synth.Workload, extra_tokens: int = 0, capacity: int = 0, rope_theta: float = 0.0,
                   sparse: bool = False):
    """A libkvq cache sized for w plus extra_tokens appended tokens
    (rope_theta > 0: keys stored before RoPE, rotated at read)."""
    B, Hq, Hkv = w.batch, w.num_q_heads, w.num_kv_heads
    fmt = w.bits
    if w.page_size:
        table, P = synth.page_table(w, extra_tokens)
        mp = table.shape[1]
        c = kvq.Cache(fmt, B, Hq, Hkv, mp * 16, group=16, residual=w.residual, page_size=16,
                      max_pages_per_seq=mp, num_pages=P)
        c.set_page_table(torch.from_numpy(table).cuda())
        return c
    tok = fmt in (8, 16)        # every token quantized on write: group and residual unused
    G = 16 if tok else w.group
    cap = capacity or max(round_up(int(w.lengths.max(initial=0)) + extra_tokens, max(G, 16)), max(G, 16))
    return kvq.Cache(fmt, B, Hq, Hkv, cap, group=G if not tok else 32, residual=w.residual if not tok else 0,
                     rope_theta=rope_theta, sparse=sparse)


def gpu_prefill(w: synth.Workload, extra_tokens: int = 0, capacity: int = 0, classes=None, rope_theta: float = 0.0,
                sparse: bool = False):
    c = make_gpu_cache(w, extra_tokens, capacity, rope_theta, sparse)
    k, v = to_dev(w.k), to_dev(w.v)
    cu = torch.from_numpy(w.cu_seqlens.astype(np.int32)).cuda()
    if w.bits == 6:
        c.quantize_prefill_mixed(k, v, torch.from_numpy(np.ascontiguousarray(classes)).cuda(), cu,
                                 int(w.lengths.max(initial=0)))
    else:
        c.quantize_prefill(k, v, cu, int(w.lengths.max(initial=0)))
    torch.cuda.synchronize()
    return c


def gpu_decode(c, w: synth.Workload, max_len: int, num_splits: int = 0, q=None):
    qd = to_dev(w.q if q is None else q)
    out = torch.full((w.batch, w.num_q_heads, 128), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(max(c.workspace_bytes(num_splits, max_len), 16), dtype=torch.uint8, device="cuda")
    c.decode_attention(qd, out, w.softmax_scale, ws, num_splits, max_len)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def oracle_cache(w: synth.Workload, capacity: int, units=None, classes=None, sparse: bool = False):
    if w.bits == 6:
        oc = oracle.Cache(0, w.batch, w.num_q_heads, w.num_kv_heads, 128, w.group, w.residual, capacity, mixed=True)
        oc.prefill(w.k, w.v, w.cu_seqlens, units=units, classes=classes)
        return oc
    if w.bits == 16:
        oc = oracle.Int8Cache(w.batch, w.num_q_heads, w.num_kv_heads, 128, capacity)
        oc.prefill(w.k, w.v, w.cu_seqlens, units=units)
        return oc
    if w.bits == 8:
        oc = oracle.FP8Cache(w.batch, w.num_q_heads, w.num_kv_heads, 128, capacity)
        oc.prefill(w.k, w.v, w.cu_seqlens)
        return oc
    oc = oracle.Cache(w.bits, w.batch, w.num_q_heads, w.num_kv_heads, 128, w.group, w.residual, capacity,
                      sparse=sparse)
    oc.prefill(w.k, w.v, w.cu_seqlens, units=units)
    return oc


def assert_unit_state(st: GpuState, oc, b: int, h: int):
    """Codes, scales, zeros, window slots and counters of one unit, bit-exact."""
    assert_unit_state_of(st, oc.units[b][h], b, h)


def assert_unit_state_of(st: GpuState, o, b: int, h: int):
    """assert_unit_state against one oracle Unit `o` (the GPU's unit (b, h));
    for a mixed unit also the group widths and the window slots' classes."""
    if getattr(o, "sparse", False):
        ng = o.n_q // o.s.G
        ks = st.k_sparse[b, h, :ng]
        assert np.array_equal((ks & 0xFFFF).astype(np.uint16), o.k_out[:ng]), "kept keys differ (b=%d h=%d)" % (b, h)
        assert np.array_equal((ks >> 16).astype(np.uint8), o.k_out_idx[:ng]), "kept key positions differ"
        vs = st.v_sparse[b, h, :o.n_q]
        assert np.array_equal((vs & 0xFFFF).astype(np.uint16), o.v_out[:o.n_q]), "kept values differ"
        assert np.array_equal((vs >> 16).astype(np.uint8), o.v_out_idx[:o.n_q]), "kept value channels differ"
    if getattr(o, "mixed", False):
        ng = o.n_q // o.s.G
        assert np.array_equal(st.group_bits[b, :ng], o.group_bits[:ng]), "group widths differ (b=%d)" % b
        W = o.s.R + o.s.G
        for t in range(o.n_q, o.n):
            assert st.window_class[b, t % W] == o.ring_class[t % W], "window class differs"
    assert st.seq_len[b] == o.n and st.n_quant[b] == o.n_q, (b, st.seq_len[b], o.n, st.n_quant[b], o.n_q)
    nq = o.n_q
    if nq:
        u = st.unit(b, h, nq)
        G = o.s.G
        assert np.array_equal(u["k_codes"], o.k_codes[:nq]), "K codes differ (b=%d h=%d)" % (b, h)
        assert np.array_equal(u["k_scale"], o.k_scale[:nq // G]), "K scales differ"
        assert np.array_equal(u["k_zero"], o.k_zero[:nq // G]), "K zeros differ"
        assert np.array_equal(u["v_codes"], o.v_codes[:nq]), "V codes differ (b=%d h=%d)" % (b, h)
        assert np.array_equal(u["v_scale"], o.v_scale[:nq]), "V scales differ"
        assert np.array_equal(u["v_zero"], o.v_zero[:nq]), "V zeros differ"
    W = o.s.R + o.s.G
    for t in range(nq, o.n):
        assert np.array_equal(st.k_ring[b, h, t % W], o.k_ring[t % W]), "K window slot differs"
        assert np.array_equal(st.v_ring[b, h, t % W], o.v_ring[t % W]), "V window slot differs"


def assert_fp8_state(st: GpuState, oc, units):
    assert np.array_equal(st.fp8_scale[0].view(np.uint32), oc.Sk.view(np.uint32))
    assert np.array_equal(st.fp8_scale[1].view(np.uint32), oc.Sv.view(np.uint32))
    for b, h in units:
        n = int(oc.n[b])
        assert st.seq_len[b] == n and st.n_quant[b] == n
        n16 = n // 16 * 16
        if n16:
            u = st.unit(b, h, n16)
            assert np.array_equal(u["k_codes"], oc.k_codes[b, h, :n16])
            assert np.array_equal(u["v_codes"], oc.v_codes[b, h, :n16])
        if n > n16:   # partial last tile
            u = st.unit(b, h, n16 + 16)
            assert np.array_equal(u["k_codes"][n16:n], oc.k_codes[b, h, n16:n])
            assert np.array_equal(u["v_codes"][n16:n], oc.v_codes[b, h, n16:n])


def assert_int8_state(st: GpuState, oc, units):
    """INT8 per-token cache: codes and per-token key/value scale and zero of
    every held token, bit-exact (tokens of the last tile past the length are
    unspecified and not compared)."""
    for b, h in units:
        n = int(oc.n[b])
        assert st.seq_len[b] == n and st.n_quant[b] == n, (b, st.seq_len[b], n)
        if n == 0:
            continue
        u = st.unit(b, h, (n + 15) // 16 * 16)
        for name, ref in (("k_codes", oc.k_codes), ("v_codes", oc.v_codes), ("k_scale", oc.k_scale),
                          ("k_zero", oc.k_zero), ("v_scale", oc.v_scale), ("v_zero", oc.v_zero)):
            assert np.array_equal(u[name][:n], ref[b, h, :n]), "%s differs (b=%d h=%d)" % (name, b, h)


def _report(out, ref, err):
    """With KVQ_TEST_REPORT=<path>, append the test id and its error figures."""
    path = os.environ.get("KVQ_TEST_REPORT")
    if not path:
        return
    num = np.sum(out * ref, axis=1)
    den = np.linalg.norm(out, axis=1) * np.linalg.norm(ref, axis=1)
    cos = float(np.min(num[den > 0] / den[den > 0])) if np.any(den > 0) else 1.0
    with open(path, "a") as f:
        f.write("%s max_abs=%.3e min_cos=%.8f\n" % (os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0], err, cos))


def assert_close(out: np.ndarray, ref: np.ndarray, rows=None):
    """Decode outputs [B, H_q, D]: max-abs <= ATOL and cosine >= COS_MIN per row."""
    if rows is not None:
        out = np.stack([out[b, h] for b, h in rows])
        ref = np.stack([ref[b, h] for b, h in rows])
    out = out.reshape(-1, 128)
    ref = ref.reshape(-1, 128)
    assert np.all(np.isfinite(out)), "non-finite output"
    err = np.max(np.abs(out - ref))
    _report(out, ref, err)
    assert err <= ATOL, "max abs error %.3g" % err
    num = np.sum(out * ref, axis=1)
    den = np.linalg.norm(out, axis=1) * np.linalg.norm(ref, axis=1)
    nz = den > 0
    cos = num[nz] / den[nz]
    assert cos.size == 0 or cos.min() >= COS_MIN, "min cosine %.6f" % cos.min()
    # rows of exactly zero (empty sequences) must be zero on both sides
    assert np.all(np.abs(out[~nz]) <= ATOL)
    return err


def heads_of(w: synth.Workload, units):
    g = w.num_q_heads // w.num_kv_heads
    return [(b, h * g + i) for b, h in units for i in range(g)]


def host_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return os.cpu_count() or 1


def each_unit(fn, units, threads: int = 0):
    """fn(unit) over the units on a pool of host threads (the C oracle
    releases the interpreter lock); returns the results in order and
    re-raises the first failure."""
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=threads or host_threads()) as ex:
        return list(ex.map(fn, units))
