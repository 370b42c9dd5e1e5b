"""Test-side packing of logical states into the pool byte layout and back.

The layout is the one documented in include/ssq.h (offsets from
ssq_pool_layout; element order, nibble order and two's complement codes as
the header states).  This module is written from that documentation alone; it
shares no code with the library or with the oracle.  It lets the tests upload
an oracle state into a GPU pool and read a GPU pool back as a logical state,
so that no oracle input ever comes from the CUDA path.
"""
from __future__ import annotations

import numpy as np

F32, BF16, I8S, I8A, I4S, I4A = range(6)


def bits(fmt):
    return {I8S: 8, I8A: 8, I4S: 4, I4A: 4, BF16: 16}.get(fmt, 32)


def is_quant(fmt):
    return fmt in (I8S, I8A, I4S, I4A)


def is_sym(fmt):
    return fmt in (I8S, I4S)


class Codec:
    def __init__(self, fmt, nheads, headdim, d_state, layout, perm):
        self.fmt, self.H, self.P, self.N = fmt, nheads, headdim, d_state
        self.L = layout
        self.perm = list(perm)
        self.pos = {h: i for i, h in enumerate(self.perm)}   # head -> region pos
        self.Hq = layout["n_quant_heads"]

    def _slot_base(self, slot):
        return self.L["header_bytes"] + slot * self.L["slot_bytes"] - self.buf_offset

    buf_offset = 0   # byte offset in the pool of buf[0] (partial copies)

    def slot_range(self, slot):
        """(first byte, byte count) of one slot in the pool."""
        return self.L["header_bytes"] + slot * self.L["slot_bytes"], self.L["slot_bytes"]

    def _region(self, h):
        i = self.pos[h]
        return (True, i) if i < self.Hq else (False, i - self.Hq)

    def write(self, buf, slot, layer, q, delta, zero, val):
        """Write one (slot, layer) logical state (natural row order
        r = h*P + p) into the uint8 pool image buf."""
        L, P, N = self.L, self.P, self.N
        base = self._slot_base(slot)
        for h in range(self.H):
            quant, i = self._region(h)
            for p in range(P):
                r = h * P + p
                rr = i * P + p
                if quant:
                    rb = L["row_code_bytes"]
                    off = base + L["codes_off"] + layer * L["codes_layer_bytes"] + rr * rb
                    buf[off:off + rb] = self.encode_codes(q[r])
                    moff = base + L["meta_off"] + layer * L["meta_layer_bytes"] \
                        + rr * L["row_meta_bytes"]
                    if is_sym(self.fmt):
                        meta = np.array([delta[r]], np.float32)
                    else:
                        meta = np.array([delta[r], zero[r]], np.float32)
                    buf[moff:moff + meta.nbytes] = meta.view(np.uint8)
                else:
                    eb = L["fp_elem_bytes"]
                    off = base + L["fp_off"] + layer * L["fp_layer_bytes"] + rr * N * eb
                    v = np.asarray(val[r], np.float32)
                    if eb == 2:
                        raw = (v.view(np.uint32) >> 16).astype(np.uint16)
                        buf[off:off + N * 2] = raw.view(np.uint8)
                    else:
                        buf[off:off + N * 4] = v.view(np.uint8)

    def read(self, buf, slot, layer):
        """Read one (slot, layer) state back: (q, delta, zero, val) in natural
        row order."""
        L, P, N, H = self.L, self.P, self.N, self.H
        q = np.zeros((H * P, N), np.int32)
        delta = np.zeros(H * P, np.float32)
        zero = np.zeros(H * P, np.float32)
        val = np.zeros((H * P, N), np.float32)
        base = self._slot_base(slot)
        for h in range(H):
            quant, i = self._region(h)
            for p in range(P):
                r = h * P + p
                rr = i * P + p
                if quant:
                    rb = L["row_code_bytes"]
                    off = base + L["codes_off"] + layer * L["codes_layer_bytes"] + rr * rb
                    q[r] = self.decode_codes(buf[off:off + rb])
                    moff = base + L["meta_off"] + layer * L["meta_layer_bytes"] \
                        + rr * L["row_meta_bytes"]
                    m = buf[moff:moff + L["row_meta_bytes"]].copy().view(np.float32)
                    delta[r] = m[0]
                    zero[r] = 0.0 if is_sym(self.fmt) else m[1]
                else:
                    eb = L["fp_elem_bytes"]
                    off = base + L["fp_off"] + layer * L["fp_layer_bytes"] + rr * N * eb
                    raw = buf[off:off + N * eb].copy()
                    if eb == 2:
                        val[r] = (raw.view(np.uint16).astype(np.uint32) << 16).view(np.float32)
                    else:
                        val[r] = raw.view(np.float32)
        return q, delta, zero, val

    def encode_codes(self, q):
        q = np.asarray(q, np.int64)
        if bits(self.fmt) == 8:
            return (q & 0xFF).astype(np.uint8)
        nib = (q & 0xF).astype(np.uint8)
        return (nib[0::2] | (nib[1::2] << 4)).astype(np.uint8)

    def decode_codes(self, raw):
        raw = np.asarray(raw, np.uint8)
        if bits(self.fmt) == 8:
            return raw.view(np.int8).astype(np.int32) if is_sym(self.fmt) \
                else raw.astype(np.int32)
        lo = (raw & 0xF).astype(np.int32)
        hi = (raw >> 4).astype(np.int32)
        out = np.empty(raw.size * 2, np.int32)
        out[0::2], out[1::2] = lo, hi
        if is_sym(self.fmt):
            out = np.where(out >= 8, out - 16, out)
        return out


class DampCodec:
    """Packing of one (layer, request)'s DAMP state (oracle.DampState arrays
    hi[H][K][P], q[H][N-K][P], delta/zero[H][N-K]) into the DAMP pool layout
    of include/ssq.h: per (slot, layer, head) a block of head_bytes with the
    FP16 tier at hi_off (position-major halves), uint8 codes at codes_off and
    {float Delta, float z} per INT8 position at meta_off."""

    buf_offset = 0   # byte offset in the pool of buf[0] (partial copies)

    def __init__(self, nheads, headdim, d_state, n_protected, layout):
        self.H, self.P, self.N, self.K = nheads, headdim, d_state, n_protected
        self.L = layout

    def layer_range(self, slot, layer):
        """(offset, size) of one (slot, layer)'s heads in the pool."""
        L = self.L
        return (L["header_bytes"] + slot * L["slot_bytes"] + layer * L["layer_bytes"],
                L["layer_bytes"])

    def _head(self, slot, layer, h):
        L = self.L
        return (L["header_bytes"] + slot * L["slot_bytes"] + layer * L["layer_bytes"]
                + h * L["head_bytes"] - self.buf_offset)

    def write(self, buf, slot, layer, hi, q, delta, zero):
        H, P, N, K = self.H, self.P, self.N, self.K
        L = self.L
        for h in range(H):
            o = self._head(slot, layer, h)
            half = np.asarray(hi[h], np.float32).astype(np.float16).reshape(-1)
            # hi holds values already on the fp16 grid: the cast is exact
            assert np.array_equal(half.astype(np.float32), np.asarray(hi[h], np.float32).reshape(-1))
            hb = half.view(np.uint8)
            buf[o + L["hi_off"]: o + L["hi_off"] + hb.size] = hb
            cb = np.asarray(q[h], np.int32).reshape(-1)
            assert cb.size == 0 or (cb.min() >= 0 and cb.max() <= 255)
            buf[o + L["codes_off"]: o + L["codes_off"] + cb.size] = cb.astype(np.uint8)
            meta = np.stack([np.asarray(delta[h], np.float32), np.asarray(zero[h], np.float32)],
                            axis=1).reshape(-1).view(np.uint8)
            buf[o + L["meta_off"]: o + L["meta_off"] + meta.size] = meta

    def read(self, buf, slot, layer):
        H, P, N, K = self.H, self.P, self.N, self.K
        L = self.L
        hi = np.zeros((H, K, P), np.float32)
        q = np.zeros((H, N - K, P), np.int32)
        delta = np.zeros((H, N - K), np.float32)
        zero = np.zeros((H, N - K), np.float32)
        for h in range(H):
            o = self._head(slot, layer, h)
            hb = buf[o + L["hi_off"]: o + L["hi_off"] + 2 * K * P].copy()
            hi[h] = hb.view(np.float16).astype(np.float32).reshape(K, P)
            q[h] = buf[o + L["codes_off"]: o + L["codes_off"] + (N - K) * P].astype(
                np.int32).reshape(N - K, P)
            m = buf[o + L["meta_off"]: o + L["meta_off"] + 8 * (N - K)].copy().view(
                np.float32).reshape(N - K, 2)
            delta[h], zero[h] = m[:, 0], m[:, 1]
        return hi, q, delta, zero

    def read_hi_bits(self, buf, slot, layer):
        """The FP16 tier as raw uint16 patterns [H][K][P]."""
        H, P, K = self.H, self.P, self.K
        L = self.L
        out = np.zeros((H, K, P), np.uint16)
        for h in range(H):
            o = self._head(slot, layer, h)
            out[h] = buf[o + L["hi_off"]: o + L["hi_off"] + 2 * K * P].copy().view(
                np.uint16).reshape(K, P)
        return out
