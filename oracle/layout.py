"""Byte layout of the compressed KV cache, written from its prose spec.

Test infrastructure only (see oracle/__init__.py).  This is an independent
implementation of the layout the C header documents; it shares no code with
the CUDA path.

The pages do not fix a layout (reading).  The spec:

* The cache of one layer is one byte buffer holding, for every sequence b
  and KV head h (b-major), ``capacity / 128`` tiles of 128 tokens.  Tile
  ``(b, h, t)`` starts at byte ``((b * H_kv + h) * n_tiles + t) * tile_bytes``.
* A tile holds, in this order, 128 tokens of each section:
    1. key code bit-planes: mb planes (mb = key_bits - 1); plane p is
       [128 tokens][d/8 bytes] and holds bit p of every Lloyd-Max index;
    2. the QJL sign plane: [128][d/8], bit = 1 for sign +1;
    3. value codes: for 2-bit values, packed codes [128 tokens][d/4 bytes],
       byte i holding channels 4i .. 4i+3, channel 4i + m in bits 2m, 2m+1;
       for 3- and 4-bit values, vb bit-planes [128][d/8] each (bit p of the
       code);
    4. norms: [128] x (nk, rn) as two little-endian fp16 (4 bytes a token);
    5. value scale/zero: [128][d/group] x (scale, zero) as two fp16.
* Inside a plane row, byte i, bit k (LSB = 0) holds coordinate 8 i + k.
* Record bytes per (token, KV head): R = (mb + 1 + vb) d/8 + 4 + 4 d/group,
  tile_bytes = 128 R.
* TurboQuant-MSE values (value_mode "mse"): section 3 holds vb bit-planes of
  the values' Lloyd-Max cell indices at every vb, and section 5 holds the
  value norms [128] x fp16 (2 bytes a token) instead of scale/zero pairs:
  R = (mb + 1 + vb) d/8 + 4 + 2 (102 bytes at 3-bit keys and values).
"""

from __future__ import annotations

import numpy as np

TILE = 128


def record_bytes(d: int, key_bits: int, value_bits: int, group: int,
                 value_mode: str = "group") -> int:
    mb = key_bits - 1
    tail = 2 if value_mode == "mse" else 4 * (d // group)
    return (mb + 1 + value_bits) * d // 8 + 4 + tail


def tile_bytes(d, key_bits, value_bits, group, value_mode="group") -> int:
    return TILE * record_bytes(d, key_bits, value_bits, group, value_mode)


def section_offsets(d, key_bits, value_bits, group, value_mode="group") -> dict:
    mb = key_bits - 1
    plane = TILE * d // 8
    off = {}
    o = 0
    off["kplanes"] = o
    o += mb * plane
    off["signs"] = o
    o += plane
    off["vplanes"] = o
    o += value_bits * plane
    off["norms"] = o
    o += TILE * 4
    off["vsz"] = o
    o += TILE * 2 if value_mode == "mse" else TILE * 4 * (d // group)
    off["end"] = o
    return off


def cache_bytes(batch, h_kv, capacity, d, key_bits, value_bits, group, value_mode="group") -> int:
    assert capacity % TILE == 0
    return batch * h_kv * (capacity // TILE) * tile_bytes(d, key_bits, value_bits, group, value_mode)


def _bits_to_plane_row(bits: np.ndarray) -> np.ndarray:
    """[..., d] of 0/1 -> [..., d/8] bytes, byte i bit k = coordinate 8i+k."""
    b = np.asarray(bits, np.uint8).reshape(*bits.shape[:-1], -1, 8)
    weights = (1 << np.arange(8)).astype(np.uint16)
    return (b.astype(np.uint16) * weights).sum(axis=-1).astype(np.uint8)


def _codes_to_packed2_row(codes: np.ndarray) -> np.ndarray:
    """[..., d] codes in 0..3 -> [..., d/4] bytes, channel 4i+m at bits 2m, 2m+1."""
    c = np.asarray(codes, np.uint16).reshape(*codes.shape[:-1], -1, 4)
    weights = (1 << (2 * np.arange(4))).astype(np.uint16)
    return (c * weights).sum(axis=-1).astype(np.uint8)


def _packed2_row_to_codes(rows: np.ndarray, d: int) -> np.ndarray:
    r = np.asarray(rows, np.uint8)
    m = (2 * np.arange(4)).astype(np.uint8)
    c = (r[..., :, None] >> m) & 3
    return c.reshape(*r.shape[:-1], d)


def _plane_row_to_bits(rows: np.ndarray, d: int) -> np.ndarray:
    r = np.asarray(rows, np.uint8)
    k = np.arange(8, dtype=np.uint8)
    bits = (r[..., :, None] >> k) & 1
    return bits.reshape(*r.shape[:-1], d)


class CacheSpec:
    def __init__(self, batch, h_kv, capacity, d, key_bits, value_bits, group, value_mode="group"):
        self.batch, self.h_kv, self.capacity = batch, h_kv, capacity
        self.d, self.key_bits, self.value_bits, self.group = d, key_bits, value_bits, group
        self.value_mode = value_mode
        self.mse = value_mode == "mse"
        self.mb = key_bits - 1
        self.ntiles = capacity // TILE
        self.tile_bytes = tile_bytes(d, key_bits, value_bits, group, value_mode)
        self.off = section_offsets(d, key_bits, value_bits, group, value_mode)
        self.nbytes = cache_bytes(batch, h_kv, capacity, d, key_bits, value_bits, group, value_mode)

    def tile_base(self, b, h, t) -> int:
        return ((b * self.h_kv + h) * self.ntiles + t) * self.tile_bytes

    def empty(self) -> np.ndarray:
        return np.zeros(self.nbytes, np.uint8)

    # -- writing -----------------------------------------------------------
    def write(self, buf: np.ndarray, b: int, h: int, pos: int, keyrec: dict,
              valrec: dict, i: int) -> None:
        """Write record i of the logical (keyrec, valrec) fields for one
        (token, head) at token position ``pos`` of sequence b, head h."""
        d = self.d
        t, slot = divmod(pos, TILE)
        base = self.tile_base(b, h, t)
        rowb = d // 8
        plane = TILE * rowb
        idx = keyrec["idx"][i]
        for p in range(self.mb):
            o = base + self.off["kplanes"] + p * plane + slot * rowb
            buf[o:o + rowb] = _bits_to_plane_row((idx >> p) & 1)
        o = base + self.off["signs"] + slot * rowb
        buf[o:o + rowb] = _bits_to_plane_row(keyrec["sign"][i])
        codes = valrec["vidx"][i] if self.mse else valrec["codes"][i]
        if self.value_bits == 2 and not self.mse:
            o = base + self.off["vplanes"] + slot * (d // 4)
            buf[o:o + d // 4] = _codes_to_packed2_row(codes)
        else:
            for p in range(self.value_bits):
                o = base + self.off["vplanes"] + p * plane + slot * rowb
                buf[o:o + rowb] = _bits_to_plane_row((codes >> p) & 1)
        o = base + self.off["norms"] + slot * 4
        buf[o:o + 4] = np.array([keyrec["nk16"][i], keyrec["rn16"][i]],
                                np.float16).view(np.uint8)
        if self.mse:
            o = base + self.off["vsz"] + slot * 2
            buf[o:o + 2] = np.array([valrec["nv16"][i]], np.float16).view(np.uint8)
            return
        ng = d // self.group
        o = base + self.off["vsz"] + slot * 4 * ng
        sz = np.stack([valrec["scale16"][i], valrec["zero16"][i]], axis=1)
        buf[o:o + 4 * ng] = sz.astype(np.float16).reshape(-1).view(np.uint8)

    def write_sequence(self, buf, b, h, pos0, keyrec, valrec) -> None:
        """Write n consecutive records at positions pos0 .. pos0+n-1 of (b, h);
        the same bytes as n calls of ``write``, gathered per section."""
        n = len(keyrec["nk16"])
        d = self.d
        rowb = d // 8
        plane = TILE * rowb
        ng = d // self.group
        pos = pos0 + np.arange(n)
        t, slot = pos // TILE, pos % TILE
        base = np.array([self.tile_base(b, h, int(tt)) for tt in t])

        def put(offsets, rows):          # rows [n, width] bytes at offsets [n]
            buf[offsets[:, None] + np.arange(rows.shape[1])[None, :]] = rows

        idx = np.asarray(keyrec["idx"])
        for p in range(self.mb):
            put(base + self.off["kplanes"] + p * plane + slot * rowb,
                _bits_to_plane_row((idx >> p) & 1))
        put(base + self.off["signs"] + slot * rowb, _bits_to_plane_row(keyrec["sign"]))
        codes = np.asarray(valrec["vidx"] if self.mse else valrec["codes"])
        if self.value_bits == 2 and not self.mse:
            put(base + self.off["vplanes"] + slot * (d // 4), _codes_to_packed2_row(codes))
        else:
            for p in range(self.value_bits):
                put(base + self.off["vplanes"] + p * plane + slot * rowb,
                    _bits_to_plane_row((codes >> p) & 1))
        nr = np.stack([keyrec["nk16"], keyrec["rn16"]], axis=1).astype(np.float16)
        put(base + self.off["norms"] + slot * 4, nr.view(np.uint8).reshape(n, 4))
        if self.mse:
            nv = np.asarray(valrec["nv16"]).astype(np.float16)
            put(base + self.off["vsz"] + slot * 2, nv.view(np.uint8).reshape(n, 2))
            return
        sz = np.stack([valrec["scale16"], valrec["zero16"]], axis=2).astype(np.float16)
        put(base + self.off["vsz"] + slot * 4 * ng, sz.reshape(n, 2 * ng).view(np.uint8))

    # -- reading -----------------------------------------------------------
    def read(self, buf: np.ndarray, b: int, h: int, start: int, count: int) -> dict:
        """Logical fields of tokens [start, start+count) of (b, h), gathered
        per section (vectorised form of ``read_one``)."""
        d = self.d
        rowb = d // 8
        plane = TILE * rowb
        ng = d // self.group
        buf = np.asarray(buf, np.uint8)
        pos = start + np.arange(count)
        t, slot = pos // TILE, pos % TILE
        base = ((b * self.h_kv + h) * self.ntiles + t) * self.tile_bytes

        def get(offsets, width):
            return buf[offsets[:, None] + np.arange(width)[None, :]]

        idx = np.zeros((count, d), np.int64)
        for p in range(self.mb):
            rows = get(base + self.off["kplanes"] + p * plane + slot * rowb, rowb)
            idx |= _plane_row_to_bits(rows, d).astype(np.int64) << p
        sign = _plane_row_to_bits(get(base + self.off["signs"] + slot * rowb, rowb), d)
        codes = np.zeros((count, d), np.int64)
        if self.value_bits == 2 and not self.mse:
            rows = get(base + self.off["vplanes"] + slot * (d // 4), d // 4)
            codes = _packed2_row_to_codes(rows, d).astype(np.int64)
        else:
            for p in range(self.value_bits):
                rows = get(base + self.off["vplanes"] + p * plane + slot * rowb, rowb)
                codes |= _plane_row_to_bits(rows, d).astype(np.int64) << p
        nr = get(base + self.off["norms"] + slot * 4, 4).copy().view(np.float16)
        nr = nr.astype(np.float64).reshape(count, 2)
        if self.mse:
            nv = get(base + self.off["vsz"] + slot * 2, 2).copy().view(np.float16)
            return {"idx": idx, "sign": sign.astype(np.uint8), "nk16": nr[:, 0],
                    "rn16": nr[:, 1], "vidx": codes, "nv16": nv.astype(np.float64).reshape(count)}
        sz = get(base + self.off["vsz"] + slot * 4 * ng, 4 * ng).copy().view(np.float16)
        sz = sz.astype(np.float64).reshape(count, ng, 2)
        return {"idx": idx, "sign": sign.astype(np.uint8), "nk16": nr[:, 0],
                "rn16": nr[:, 1], "codes": codes, "scale16": sz[:, :, 0],
                "zero16": sz[:, :, 1]}

    def read_one(self, buf: np.ndarray, b: int, h: int, start: int, count: int) -> dict:
        """Logical fields of tokens [start, start+count) of (b, h), one record
        at a time straight from the spec."""
        d = self.d
        rowb = d // 8
        plane = TILE * rowb
        ng = d // self.group
        idx = np.zeros((count, d), np.int64)
        sign = np.zeros((count, d), np.uint8)
        codes = np.zeros((count, d), np.int64)
        nk = np.zeros(count)
        rn = np.zeros(count)
        sc = np.zeros((count, ng))
        ze = np.zeros((count, ng))
        for i in range(count):
            pos = start + i
            t, slot = divmod(pos, TILE)
            base = self.tile_base(b, h, t)
            for p in range(self.mb):
                o = base + self.off["kplanes"] + p * plane + slot * rowb
                idx[i] |= _plane_row_to_bits(buf[o:o + rowb], d).astype(np.int64) << p
            o = base + self.off["signs"] + slot * rowb
            sign[i] = _plane_row_to_bits(buf[o:o + rowb], d)
            if self.value_bits == 2 and not self.mse:
                o = base + self.off["vplanes"] + slot * (d // 4)
                codes[i] = _packed2_row_to_codes(buf[o:o + d // 4], d)
            else:
                for p in range(self.value_bits):
                    o = base + self.off["vplanes"] + p * plane + slot * rowb
                    codes[i] |= _plane_row_to_bits(buf[o:o + rowb], d).astype(np.int64) << p
            o = base + self.off["norms"] + slot * 4
            nr = buf[o:o + 4].copy().view(np.float16).astype(np.float64)
            nk[i], rn[i] = nr[0], nr[1]
            if self.mse:
                o = base + self.off["vsz"] + slot * 2
                sc[i, 0] = buf[o:o + 2].copy().view(np.float16).astype(np.float64)[0]
                continue
            o = base + self.off["vsz"] + slot * 4 * ng
            sz = buf[o:o + 4 * ng].copy().view(np.float16).astype(np.float64).reshape(ng, 2)
            sc[i], ze[i] = sz[:, 0], sz[:, 1]
        if self.mse:
            return {"idx": idx, "sign": sign, "nk16": nk, "rn16": rn, "vidx": codes,
                    "nv16": sc[:, 0].copy()}
        return {"idx": idx, "sign": sign, "nk16": nk, "rn16": rn,
                "codes": codes, "scale16": sc, "zero16": ze}
