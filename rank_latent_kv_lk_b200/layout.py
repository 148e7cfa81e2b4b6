"""Host-side view of the latent cache layout declared in include/lk.h.

Pure index arithmetic (byte permutations and plane offsets), used to load a
cache from logical per-(batch, head) code rows or to read one back for
inspection.  It performs no quantisation or packing of values.

Layout: for batch row b and head h the code plane holds capacity * rb_h bytes
(rb_h = r_h for int8, r_h / 2 for int4) at byte offset
(b * sum_h rb_h + sum_{h'<h} rb_h') * capacity; tokens are stored in blocks of
16.  Inside a block, K caches are chunk-major over each token's code row
(chunk size cs = 16, 8 or 4 bytes, the largest dividing rb); V caches are
dimension-major (int8: dim d of token t at d * 16 + t % 16; int4: dim d of
tokens 2i, 2i + 1 share byte d * 8 + i, low nibble = even token).  Scales:
fp32 [capacity] per (b, h) (int8) or fp16 [capacity][ng_h] per (b, h)
(int4), planes in the same (b, h) order.
"""
from __future__ import annotations

import numpy as np


def row_bytes(r, kind):
    return r if kind == "i8" else r // 2


def n_groups(r, kind, group):
    if kind == "i8":
        return 1
    g = min(group, r)
    return -(-r // g)


def chunk_bytes(rb):
    if rb % 16 == 0:
        return 16
    if rb % 8 == 0:
        return 8
    return 4


def tile_index(T, rb):
    """Flat plane index of byte k of token t, as an int64 array [T, rb]."""
    cs = chunk_bytes(rb)
    t = np.arange(T, dtype=np.int64)[:, None]
    k = np.arange(rb, dtype=np.int64)[None, :]
    return (t // 16) * 16 * rb + (k // cs) * 16 * cs + (t % 16) * cs + (k % cs)


def _nibbles(rows):
    """uint8 [T, nb] -> the 4-bit fields [T, 2 nb], low nibble first."""
    out = np.empty(rows.shape[:-1] + (2 * rows.shape[-1],), np.uint8)
    out[..., 0::2] = rows & 0xF
    out[..., 1::2] = rows >> 4
    return out


def v_plane_from_rows(rows, rb, kind, capacity):
    """Token rows of code bytes [T, rb] -> a dimension-major V plane [capacity * rb]."""
    T = rows.shape[0]
    Tp = (T + 15) // 16 * 16
    plane = np.zeros(capacity * rb, np.uint8)
    if kind == "i8":
        full = np.zeros((Tp, rb), np.uint8)
        full[:T] = rows
        blocks = full.reshape(Tp // 16, 16, rb).transpose(0, 2, 1)   # [blk][dim][16 tokens]
        plane[:Tp * rb] = blocks.reshape(-1)
        return plane
    nib = np.zeros((Tp, 2 * rb), np.uint8)
    nib[:T] = _nibbles(rows)
    blocks = nib.reshape(Tp // 16, 16, 2 * rb).transpose(0, 2, 1)     # [blk][dim][16 tokens]
    packed = blocks[..., 0::2] | (blocks[..., 1::2] << 4)                # [blk][dim][8 bytes]
    plane[:Tp * rb] = packed.reshape(-1)
    return plane


def rows_from_v_plane(plane, T, rb, kind):
    """Inverse of v_plane_from_rows for the first T tokens."""
    Tp = (T + 15) // 16 * 16
    flat = np.asarray(plane[:Tp * rb], np.uint8)
    if kind == "i8":
        blocks = flat.reshape(Tp // 16, rb, 16).transpose(0, 2, 1)
        return blocks.reshape(Tp, rb)[:T].copy()
    blocks = flat.reshape(Tp // 16, 2 * rb, 8)                           # [blk][dim][8 bytes]
    nib = np.empty((Tp // 16, 2 * rb, 16), np.uint8)
    nib[..., 0::2] = blocks & 0xF
    nib[..., 1::2] = blocks >> 4
    tok = nib.transpose(0, 2, 1).reshape(Tp, 2 * rb)[:T]               # [token][dim]
    return (tok[:, 0::2] | (tok[:, 1::2] << 4)).astype(np.uint8)


class CacheGeometry:
    """Plane offsets of one cache (one layer, K or V)."""

    def __init__(self, batch, ranks, capacity, kind, group=32, role="k"):
        assert capacity % 16 == 0
        assert role in ("k", "v")
        self.role = role
        self.batch = batch
        self.ranks = [int(r) for r in ranks]
        self.capacity = capacity
        self.kind = kind
        self.group = group
        self.rb = [row_bytes(r, kind) for r in self.ranks]
        self.ng = [n_groups(r, kind, group) for r in self.ranks]
        self.sum_rb = sum(self.rb)
        self.sum_ng = sum(self.ng)
        self.pref_rb = np.concatenate([[0], np.cumsum(self.rb)[:-1]]).astype(np.int64)
        self.pref_ng = np.concatenate([[0], np.cumsum(self.ng)[:-1]]).astype(np.int64)
        self.scale_dtype = np.float32 if kind == "i8" else np.float16

    @property
    def codes_bytes(self):
        return self.batch * self.sum_rb * self.capacity

    @property
    def scales_elems(self):
        return self.batch * self.sum_ng * self.capacity

    def code_plane(self, b, h):
        off = (b * self.sum_rb + int(self.pref_rb[h])) * self.capacity
        return off, self.rb[h] * self.capacity

    def scale_plane(self, b, h):
        off = (b * self.sum_ng + int(self.pref_ng[h])) * self.capacity
        return off, self.ng[h] * self.capacity

    def pack(self, rows, scales):
        """rows[b][h]: uint8 [T_bh, rb_h] code bytes; scales[b][h]: [T_bh] or [T_bh, ng_h].

        Returns host arrays (codes uint8 [codes_bytes], scales [scales_elems]);
        unused positions are zero.
        """
        codes = np.zeros(self.codes_bytes, np.uint8)
        sc = np.zeros(self.scales_elems, self.scale_dtype)
        for b in range(self.batch):
            for h in range(len(self.ranks)):
                r = np.asarray(rows[b][h], np.uint8)
                T = r.shape[0]
                assert T <= self.capacity and r.shape[1] == self.rb[h]
                off, n = self.code_plane(b, h)
                if self.role == "k":
                    codes[off + tile_index(T, self.rb[h])] = r
                else:
                    codes[off:off + n] = v_plane_from_rows(r, self.rb[h], self.kind, self.capacity)
                soff, _ = self.scale_plane(b, h)
                s = np.asarray(scales[b][h], self.scale_dtype).reshape(T, self.ng[h])
                sc[soff:soff + T * self.ng[h]] = s.reshape(-1)
        return codes, sc

    def unpack(self, codes, scales, lens):
        """Inverse of pack for the first lens[b] tokens of every (b, h)."""
        codes = np.asarray(codes, np.uint8)
        scales = np.asarray(scales).view(self.scale_dtype)
        rows, sc = [], []
        for b in range(self.batch):
            rr, ss = [], []
            for h in range(len(self.ranks)):
                T = int(lens[b])
                off, n = self.code_plane(b, h)
                if self.role == "k":
                    rr.append(codes[off + tile_index(T, self.rb[h])])
                else:
                    rr.append(rows_from_v_plane(codes[off:off + n], T, self.rb[h], self.kind))
                soff, _ = self.scale_plane(b, h)
                s = scales[soff:soff + T * self.ng[h]].reshape(T, self.ng[h])
                ss.append(s[:, 0].copy() if self.kind == "i8" else s.copy())
            rows.append(rr)
            sc.append(ss)
        return rows, sc

    def unpack_unit(self, plane, scale_plane, h, T):
        """Code rows [T, rb_h] and scales of one (b, h) from that plane's bytes
        (``plane``: the capacity * rb_h code bytes; ``scale_plane``: its
        capacity * ng_h scales)."""
        plane = np.asarray(plane, np.uint8)
        if self.role == "k":
            rows = plane[tile_index(T, self.rb[h])]
        else:
            rows = rows_from_v_plane(plane, T, self.rb[h], self.kind)
        s = np.asarray(scale_plane).view(self.scale_dtype)[:T * self.ng[h]].reshape(T, self.ng[h])
        return rows, (s[:, 0].copy() if self.kind == "i8" else s.copy())
