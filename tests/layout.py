"""Decoding of libkvq's documented device layouts (include/kvq.h) into the
canonical per-element form the oracle keeps: index shuffling only, no
quantization arithmetic."""
import numpy as np

D = 128
TILE = 16


def _vtile_index(bits: int):
    """(byte index, bit shift) of every (token i, channel c) of one value tile."""
    i = np.arange(TILE)[:, None]
    c = np.arange(D)[None, :]
    n, j = c // 16, c % 16
    l, s, o = (i % 8) // 2, i // 8, i % 2
    lane = 4 * n + l
    if bits == 4:
        w = j // 2
        p = (j % 2) + 2 * o + 4 * s
        addr = 16 * lane + 4 * (w % 4) + 512 * (w // 4)
        return addr + p // 2, 4 * (p % 2)
    if bits == 2:
        w = j // 4
        p = (j % 4) + 4 * o + 8 * s
        addr = 16 * lane + 4 * w
        return addr + p // 4, 2 * (p % 4)
    # fp8: one byte per code
    addr = 16 * lane + 512 * (j // 4) + 4 * (j % 4) + 2 * s + o
    return addr, np.zeros_like(addr)


def kmeta_natural(rows: np.ndarray, bits: int) -> np.ndarray:
    """Key scale/zero rows [..., D] from pair order back to channel order."""
    c = np.arange(D)
    l, u = c // 32, c % 32
    if bits == 4:
        J, v = u // 8, u % 8
        h, r = (v // 2) % 2, v % 2 + 2 * (v // 4)
        pos = 32 * l + 8 * J + 2 * r + h
    else:
        J, r, h = u // 16, u % 8, (u % 16) // 8
        pos = 32 * l + 16 * J + 2 * r + h
    return rows[..., pos]


def unpack_rows(packed: np.ndarray, bits: int) -> np.ndarray:
    """Canonical packed rows [..., D*bits/8] -> codes [..., D] (fp8 and
    INT8, format 16: one byte per code, identity)."""
    if bits in (8, 16):
        return packed.copy()
    per = 8 // bits
    sh = (bits * np.arange(per)).astype(np.uint8)
    codes = (packed[..., :, None] >> sh) & ((1 << bits) - 1)
    return codes.reshape(*packed.shape[:-1], D).astype(np.uint8)


def unpack_vtiles(tiles: np.ndarray, bits: int) -> np.ndarray:
    """Value tiles [..., TB] -> codes [..., 16, D] (INT8, format 16, uses the
    fp8 byte layout)."""
    idx, sh = _vtile_index(8 if bits == 16 else bits)
    b = tiles[..., idx]
    if bits in (8, 16):
        return b.astype(np.uint8)
    return ((b >> sh.astype(np.uint8)) & ((1 << bits) - 1)).astype(np.uint8)


def row_bytes(bits: int) -> int:
    """Bytes per key row (MIXED, format 6, is laid out as INT4)."""
    return D if bits in (8, 16) else (64 if bits == 6 else D * bits // 8)


class GpuState:
    """Host copy of a libkvq cache; unit(b, h) decodes one (sequence, kv
    head) into the canonical per-element arrays the oracle keeps."""

    def __init__(self, cache):
        s = cache.shape
        self.bits = s.format
        self.B, self.H, self.cap, self.G, self.R = s.batch, s.num_kv_heads, s.capacity, s.group, s.residual
        self.paged = s.page_size != 0
        g = lambda n: cache.region(n).cpu().numpy() if cache.region(n) is not None else None
        self.seq_len = g("seq_len").view(np.int32).copy()
        self.n_quant = g("n_quant").view(np.int32).copy()
        rb = row_bytes(self.bits)
        tb = TILE * rb
        if self.paged:
            P = s.num_pages
            self.kc = g("k_codes").reshape(P, self.H, TILE, rb)
            self.vc = g("v_codes").reshape(P, self.H, tb)
            self.km = g("k_meta").view(np.uint16).reshape(P, self.H, 2, D)
            self.vm = g("v_meta").view(np.uint16).reshape(P, self.H, TILE, 2)
            self.page_table = g("page_table").view(np.int32).reshape(self.B, s.max_pages_per_seq)
        else:
            self.kc = g("k_codes").reshape(self.B, self.H, self.cap, rb)
            self.vc = g("v_codes").reshape(self.B, self.H, self.cap // TILE, tb)
            if self.bits == 16:
                self.km = g("k_meta").view(np.uint16).reshape(self.B, self.H, self.cap, 2)
                self.vm = g("v_meta").view(np.uint16).reshape(self.B, self.H, self.cap, 2)
            elif self.bits != 8:
                self.km = g("k_meta").view(np.uint16).reshape(self.B, self.H, self.cap // self.G, 2, D)
                self.vm = g("v_meta").view(np.uint16).reshape(self.B, self.H, self.cap, 2)
        self.sparse = bool(getattr(s, "sparse", 0))
        if self.sparse:
            # dense-and-sparse: kept key per (group, channel), kept value per token
            self.k_sparse = g("k_sparse").view(np.uint32).reshape(self.B, self.H, self.cap // self.G, D)
            self.v_sparse = g("v_sparse").view(np.uint32).reshape(self.B, self.H, self.cap)
        if self.bits == 6:
            # MIXED: regions laid out as INT4, plus the widths and window classes
            self.group_bits = g("group_bits").reshape(self.B, self.cap // self.G)
            self.window_class = g("window_class").reshape(self.B, self.R + self.G)
        if self.bits == 16:
            pass
        elif self.bits != 8:
            W = self.R + self.G
            self.k_ring = g("k_res").view(np.uint16).reshape(self.B, self.H, W, D)
            self.v_ring = g("v_res").view(np.uint16).reshape(self.B, self.H, W, D)
        else:
            self.fp8_scale = g("fp8_scale").view(np.float32).reshape(2, self.H)

    def unit(self, b: int, h: int, ntok: int):
        """Canonical arrays of the first ntok tokens of unit (b, h)
        (ntok a multiple of 16, and of G for the key metadata)."""
        nt = ntok // TILE
        out = {}
        if self.paged:
            ids = self.page_table[b, :nt]
            out["k_codes"] = unpack_rows(self.kc[ids, h], self.bits).reshape(ntok, D)
            out["v_codes"] = unpack_vtiles(self.vc[ids, h], self.bits).reshape(ntok, D)
            km = kmeta_natural(self.km[ids, h], self.bits)           # [nt, 2, D]
            out["k_scale"], out["k_zero"] = km[:, 0, :], km[:, 1, :]
            vm = self.vm[ids, h].reshape(ntok, 2)
            out["v_scale"], out["v_zero"] = vm[:, 0], vm[:, 1]
        elif self.bits == 6:
            # per group: INT4 slot as is, or a 2-bit group packed in the first
            # half of its slot (key rows of 32 bytes, each value tile's first
            # 512 bytes), key scale/zero rows in that width's pair order
            G = self.G
            kc, vc = [], []
            ks, kz = [], []
            kslots = self.kc[b, h].reshape(self.cap // G, G * 64)
            for gi in range(ntok // G):
                bits = int(self.group_bits[b, gi])
                slot = kslots[gi]
                tiles = self.vc[b, h, gi * (G // TILE):(gi + 1) * (G // TILE)]
                if bits == 4:
                    kc.append(unpack_rows(slot.reshape(G, 64), 4))
                    vc.append(unpack_vtiles(tiles, 4).reshape(G, D))
                else:
                    kc.append(unpack_rows(slot[:G * 32].reshape(G, 32), 2))
                    vc.append(unpack_vtiles(tiles[:, :512], 2).reshape(G, D))
                km = kmeta_natural(self.km[b, h, gi], bits)
                ks.append(km[0])
                kz.append(km[1])
            out["k_codes"] = np.concatenate(kc) if kc else np.zeros((0, D), np.uint8)
            out["v_codes"] = np.concatenate(vc) if vc else np.zeros((0, D), np.uint8)
            out["k_scale"] = np.stack(ks) if ks else np.zeros((0, D), np.uint16)
            out["k_zero"] = np.stack(kz) if kz else np.zeros((0, D), np.uint16)
            vm = self.vm[b, h, :ntok]
            out["v_scale"], out["v_zero"] = vm[:, 0], vm[:, 1]
        elif self.bits == 16:
            out["k_codes"] = unpack_rows(self.kc[b, h, :ntok], self.bits)
            out["v_codes"] = unpack_vtiles(self.vc[b, h, :nt], self.bits).reshape(ntok, D)
            out["k_scale"], out["k_zero"] = self.km[b, h, :ntok, 0], self.km[b, h, :ntok, 1]
            out["v_scale"], out["v_zero"] = self.vm[b, h, :ntok, 0], self.vm[b, h, :ntok, 1]
        else:
            out["k_codes"] = unpack_rows(self.kc[b, h, :ntok], self.bits)
            out["v_codes"] = unpack_vtiles(self.vc[b, h, :nt], self.bits).reshape(ntok, D)
            if self.bits != 8:
                km = kmeta_natural(self.km[b, h, :ntok // self.G], self.bits)
                out["k_scale"], out["k_zero"] = km[:, 0, :], km[:, 1, :]
                vm = self.vm[b, h, :ntok]
                out["v_scale"], out["v_zero"] = vm[:, 0], vm[:, 1]
        return out
