"""Serialized JoLT stream: writer and reader (oracle side, independent of the C library).

Test infrastructure only; see oracle/__init__.py. The pages publish no format (the news
summary says the code is not public), so this layout is this project's own; the C
library implements the same layout from its header description, with no shared code.

Layout, all little-endian:
    0   4  magic b"JOLT"
    4   4  u32 version (1)
    8   4  u32 header_bytes = 64 + 24 * num_groups rounded up to a multiple of 16
    12  4  u32 flags: bit0 has V, bit1 float32 output, bit2 separate K/V budgets,
                      bit3 randomized Hadamard rotation (else Haar), bits 8..15 encoder
                      (1 exact, 2 sketch)
    16  4  i32 layers        20  4  i32 heads      24  4  i32 tokens
    28  4  i32 head_dim      32  4  i32 num_groups 36  4  i32 rank_step
    40  4  i32 rt_max        44  4  i32 reserved (0)
    48  8  u64 seed          56  8  u64 body_bytes
    64     alloc table: for g, for kind in (K, V): i32 r_t, r_d, b (zeros for an absent V)
    header_bytes: body
    end: u32 CRC-32 (IEEE 802.3 polynomial, as zlib) of header and body

Body: for lt = 2 * layer + kind (kind 1 skipped without V), for the parts U_T [T][r_t] bf16,
U_D [D][r_d] bf16, G [H][r_t][r_d] bf16, scales [H][T] fp16, codes [H][T][D b / 8] u8 (the
last two absent when b = 0): each part starts at the next multiple of 256 bytes from the
body start; body_bytes ends at the last part's last byte.
"""
from __future__ import annotations

import struct
import zlib

import numpy as np

from .jolt import KINDS, LTCode, OracleStream, group_ranges, pack_codes, unpack_codes
from .numerics import bf16_bits, bf16_from_bits, fp16_bits, fp16_from_bits

MAGIC = b"JOLT"
VERSION = 1
ALIGN = 256


class CorruptStream(ValueError):
    pass


def header_bytes(num_groups: int) -> int:
    n = 64 + 24 * num_groups
    return (n + 15) // 16 * 16


def part_sizes(H, T, D, rt, rd, b):
    return [T * rt * 2, D * rd * 2, H * rt * rd * 2,
            H * T * 2 if b > 0 else 0, H * T * (D * b // 8) if b > 0 else 0]


def body_layout(L, H, T, D, has_v, num_groups, alloc):
    """{lt: [(offset, size)] * 5} and the body size, from the allocation table."""
    group_of = {}
    for g, lay in enumerate(group_ranges(L, num_groups)):
        for l in lay:
            group_of[l] = g
    cur = 0
    out = {}
    for l in range(L):
        for k in ((0, 1) if has_v else (0,)):
            rt, rd, b = (int(v) for v in alloc[group_of[l]][k])
            parts = []
            for sz in part_sizes(H, T, D, rt, rd, b):
                off = (cur + ALIGN - 1) // ALIGN * ALIGN
                parts.append((off, sz))
                cur = off + sz
            out[l * KINDS + k] = parts
    return out, cur


def _flags(st: OracleStream) -> int:
    enc = 1 if st.encoder == "exact" else 2
    return (int(st.has_v) | (int(st.out_f32) << 1) | (int(st.split_kv) << 2) |
            (int(st.rotation == "hadamard") << 3) | (enc << 8))


def serialize(st: OracleStream) -> bytes:
    hb = header_bytes(st.num_groups)
    layout, body_n = body_layout(st.L, st.H, st.T, st.D, st.has_v, st.num_groups, st.alloc)
    head = bytearray(hb)
    struct.pack_into("<4sIII", head, 0, MAGIC, VERSION, hb, _flags(st))
    struct.pack_into("<8i", head, 16, st.L, st.H, st.T, st.D, st.num_groups, st.rank_step,
                     st.rt_max, 0)
    struct.pack_into("<QQ", head, 48, st.seed, body_n)
    for g in range(st.num_groups):
        for k in range(2):
            struct.pack_into("<3i", head, 64 + 24 * g + 12 * k, *(int(v) for v in st.alloc[g][k]))
    body = bytearray(body_n)
    for lt, parts in layout.items():
        c = st.lts[lt]
        blobs = [bf16_bits(c.U_T).tobytes(), bf16_bits(c.U_D).tobytes(), bf16_bits(c.G).tobytes()]
        if c.b > 0:
            blobs += [fp16_bits(c.scales).tobytes(), pack_codes(c.codes, c.b).tobytes()]
        else:
            blobs += [b"", b""]
        for (off, sz), blob in zip(parts, blobs):
            assert len(blob) == sz, (lt, sz, len(blob))
            body[off:off + sz] = blob
    data = bytes(head) + bytes(body)
    return data + struct.pack("<I", zlib.crc32(data) & 0xFFFFFFFF)


def parse(buf: bytes, lts=None) -> OracleStream:
    """Inverse of `serialize`; raises CorruptStream on a bad magic, version, size or CRC.
    `lts`: unpack only these layer-tensors (all when None); the whole buffer is still checked."""
    if len(buf) < 68 or buf[:4] != MAGIC:
        raise CorruptStream("bad magic or short buffer")
    _, ver, hb, flags = struct.unpack_from("<4sIII", buf, 0)
    if ver != VERSION:
        raise CorruptStream(f"version {ver}")
    L, H, T, D, G, step, rtm, _ = struct.unpack_from("<8i", buf, 16)
    seed, body_n = struct.unpack_from("<QQ", buf, 48)
    if hb != header_bytes(G) or len(buf) != hb + body_n + 4:
        raise CorruptStream("size mismatch")
    (crc,) = struct.unpack_from("<I", buf, hb + body_n)
    if crc != (zlib.crc32(buf[:hb + body_n]) & 0xFFFFFFFF):
        raise CorruptStream("CRC mismatch")
    has_v = bool(flags & 1)
    alloc = np.zeros((G, 2, 3), dtype=np.int64)
    for g in range(G):
        for k in range(2):
            alloc[g, k] = struct.unpack_from("<3i", buf, 64 + 24 * g + 12 * k)
    enc = "exact" if ((flags >> 8) & 0xFF) == 1 else "sketch"
    st = OracleStream(L, H, T, D, has_v, G, seed, enc, step, rtm, bool(flags & 4),
                      bool(flags & 2), alloc, rotation="hadamard" if flags & 8 else "haar")
    layout, n = body_layout(L, H, T, D, has_v, G, alloc)
    if n != body_n:
        raise CorruptStream("body size does not match the allocation table")
    body = memoryview(buf)[hb:hb + body_n]
    group_of = {l: g for g, lay in enumerate(group_ranges(L, G)) for l in lay}
    for lt, parts in layout.items():
        if lts is not None and lt not in lts:
            continue
        rt, rd, b = (int(v) for v in alloc[group_of[lt // KINDS]][lt % KINDS])
        raw = [np.frombuffer(body[o:o + s], dtype=np.uint8) for o, s in parts]
        U_T = bf16_from_bits(raw[0].view(np.uint16)).reshape(T, rt)
        U_D = bf16_from_bits(raw[1].view(np.uint16)).reshape(D, rd)
        Gc = bf16_from_bits(raw[2].view(np.uint16)).reshape(H, rt, rd)
        if b > 0:
            sc = fp16_from_bits(raw[3].view(np.uint16)).reshape(H, T)
            codes = unpack_codes(raw[4].reshape(H, T, D * b // 8), b, D)
        else:
            sc = np.zeros((H, 0))
            codes = np.zeros((H, T, 0), dtype=np.int64)
        st.lts[lt] = LTCode(rt, rd, b, U_T, U_D, Gc, sc, codes)
    return st
