"""Packed 3-bit code layout (oracle).  The pages fix only "packed 3-bit tensors"
([RQ-abs]; [RQ-news] section "妙处不只是压缩，而是不再展开") and that codes should be
read a word at a time and unpacked in registers ([TQ-RQ] section "真正的瓶颈").  The
bit layout below is this project's own; this module implements it from its written
specification, independently of the CUDA packer.

Chunk: 32 codes y_0..y_31 (3 bits each) in 12 bytes = three little-endian uint32
words W_0, W_1, W_2:
    for w in 0..2, j in 0..7:
        bits [4j, 4j+3) of W_w  = y_{8w+j}
        bit  4j+3       of W_w  = bit w of y_{24+j}

K record, one per token, 48 bytes = chunks c = 0..3 at bytes [12c, 12c+12);
    slot s of chunk c holds rotated coordinate 32c + s.

V block, one per 16 consecutive positions 16b .. 16b+15 of a (sequence, kv head), 768 bytes
= 64 chunks; chunk (g, tq, h) with g in 0..7, tq in 0..3, h in 0..1 sits at bytes
[12 q, 12 q + 12) with q = 2 (4 g + tq) + h.  Slot s = 8 floor(m/2) + 4 (m mod 2) + j of
chunk (g, tq, h), for m in 0..7 and j in 0..3, holds
    token  u = 8 floor(j/2) + 2 tq + (j mod 2)       (position 16b + u)
    coord  x = 16 m + g + 8 h
so token u owns nibbles j and j+4 (all four bits, spare bit included) of the three words of
the sixteen chunks (g, tq(u), h): no other token has a bit there.
"""

import numpy as np

K_BYTES = 48
V_BLOCK_TOKENS = 16
V_BLOCK_BYTES = 768


def pack_chunk(y):
    """32 codes -> 12 bytes (see module docstring)."""
    y = [int(v) & 7 for v in y]
    assert len(y) == 32
    out = bytearray()
    for w in range(3):
        word = 0
        for j in range(8):
            word |= y[8 * w + j] << (4 * j)
            word |= ((y[24 + j] >> w) & 1) << (4 * j + 3)
        out += word.to_bytes(4, "little")
    return bytes(out)


def unpack_chunk(b):
    """12 bytes -> 32 codes."""
    b = bytes(b)
    assert len(b) == 12
    words = [int.from_bytes(b[4 * w : 4 * w + 4], "little") for w in range(3)]
    y = [0] * 32
    for w in range(3):
        for j in range(8):
            y[8 * w + j] = (words[w] >> (4 * j)) & 7
            y[24 + j] |= ((words[w] >> (4 * j + 3)) & 1) << w
    return y


def k_slot_coord(c, s):
    return 32 * c + s


def v_chunk_index(g, tq, h):
    return 2 * (4 * g + tq) + h


def v_slot_token_coord(g, tq, h, s):
    """(token within the block, coordinate) held by slot s of V chunk (g, tq, h)."""
    m = 2 * (s // 8) + (s % 8) // 4
    j = s % 4
    return 8 * (j // 2) + 2 * tq + (j % 2), 16 * m + g + 8 * h


def pack_k(codes):
    """codes (T, 128) -> (T, 48) uint8 K records."""
    codes = np.asarray(codes)
    T = codes.shape[0]
    out = np.zeros((T, K_BYTES), dtype=np.uint8)
    for t in range(T):
        rec = bytearray()
        for c in range(4):
            rec += pack_chunk([codes[t, k_slot_coord(c, s)] for s in range(32)])
        out[t] = np.frombuffer(bytes(rec), dtype=np.uint8)
    return out


def unpack_k(records):
    records = np.asarray(records, dtype=np.uint8)
    T = records.shape[0]
    codes = np.zeros((T, 128), dtype=np.uint8)
    for t in range(T):
        for c in range(4):
            y = unpack_chunk(records[t, 12 * c : 12 * c + 12].tobytes())
            for s in range(32):
                codes[t, k_slot_coord(c, s)] = y[s]
    return codes


def pack_v(codes):
    """codes (T, 128) -> (ceil(T/16), 768) uint8 V blocks; slots of positions >= T are zero."""
    codes = np.asarray(codes)
    T = codes.shape[0]
    NB = (T + 15) // 16
    out = np.zeros((NB, V_BLOCK_BYTES), dtype=np.uint8)
    for blk in range(NB):
        rec = bytearray(V_BLOCK_BYTES)
        for g in range(8):
            for tq in range(4):
                for h in range(2):
                    y = []
                    for s in range(32):
                        u, x = v_slot_token_coord(g, tq, h, s)
                        t = 16 * blk + u
                        y.append(codes[t, x] if t < T else 0)
                    q = v_chunk_index(g, tq, h)
                    rec[12 * q : 12 * q + 12] = pack_chunk(y)
        out[blk] = np.frombuffer(bytes(rec), dtype=np.uint8)
    return out


def unpack_v(records, T=None):
    records = np.asarray(records, dtype=np.uint8)
    NB = records.shape[0]
    if T is None:
        T = 16 * NB
    codes = np.zeros((T, 128), dtype=np.uint8)
    for blk in range(NB):
        for g in range(8):
            for tq in range(4):
                for h in range(2):
                    q = v_chunk_index(g, tq, h)
                    y = unpack_chunk(records[blk, 12 * q : 12 * q + 12].tobytes())
                    for s in range(32):
                        u, x = v_slot_token_coord(g, tq, h, s)
                        t = 16 * blk + u
                        if t < T:
                            codes[t, x] = y[s]
    return codes


def v_bit_owner():
    """For each of the 6144 bits of a V block (byte-major, bit 0 first), the token (0..15)
    whose code it stores, from the slot map and the chunk bit layout."""
    owner = np.full(V_BLOCK_BYTES * 8, -1)
    for g in range(8):
        for tq in range(4):
            for h in range(2):
                base = 96 * v_chunk_index(g, tq, h)
                for w in range(3):
                    for nib in range(8):
                        u_direct, _ = v_slot_token_coord(g, tq, h, 8 * w + nib)
                        u_spare, _ = v_slot_token_coord(g, tq, h, 24 + nib)
                        for bit in range(3):
                            owner[base + 32 * w + 4 * nib + bit] = u_direct
                        owner[base + 32 * w + 4 * nib + 3] = u_spare
    return owner


# --------------------------------------------------------------------- vectorised forms
# The same layout written with numpy array operations for large inputs; tests check them
# against the per-slot loops above.
def _chunk_words(y):
    """y: (..., 32) codes -> (..., 3) uint32 words."""
    y = np.asarray(y, dtype=np.uint32) & 7
    j = np.arange(8, dtype=np.uint32)
    words = []
    for w in range(3):
        word = np.bitwise_or.reduce(y[..., 8 * w : 8 * w + 8] << (4 * j), axis=-1)
        word |= np.bitwise_or.reduce(((y[..., 24:32] >> w) & 1) << (4 * j + 3), axis=-1)
        words.append(word)
    return np.stack(words, axis=-1).astype(np.uint32)


def _words_chunk(words):
    """(..., 3) uint32 words -> (..., 32) codes."""
    words = np.asarray(words, dtype=np.uint32)
    j = np.arange(8, dtype=np.uint32)
    y = np.zeros(words.shape[:-1] + (32,), dtype=np.uint32)
    for w in range(3):
        y[..., 8 * w : 8 * w + 8] = (words[..., w : w + 1] >> (4 * j)) & 7
        y[..., 24:32] |= ((words[..., w : w + 1] >> (4 * j + 3)) & 1) << w
    return y.astype(np.uint8)


_VB_TOK = np.zeros((64, 32), dtype=np.int64)
_VB_COORD = np.zeros((64, 32), dtype=np.int64)
for _g in range(8):
    for _tq in range(4):
        for _h in range(2):
            for _s in range(32):
                _VB_TOK[v_chunk_index(_g, _tq, _h), _s], _VB_COORD[v_chunk_index(_g, _tq, _h), _s] = \
                    v_slot_token_coord(_g, _tq, _h, _s)


def pack_k_fast(codes):
    codes = np.asarray(codes)
    T = codes.shape[0]
    y = codes.reshape(T, 4, 32)  # chunk c holds coordinates 32c .. 32c+31 in slot order
    return _chunk_words(y).reshape(T, 12).view("<u4").view(np.uint8).reshape(T, K_BYTES)


def unpack_k_fast(records):
    records = np.ascontiguousarray(np.asarray(records, dtype=np.uint8))
    T = records.shape[0]
    words = records.view("<u4").reshape(T, 4, 3)
    return _words_chunk(words).reshape(T, 128)


def pack_v_fast(codes):
    codes = np.asarray(codes)
    T = codes.shape[0]
    NB = (T + 15) // 16
    pad = np.zeros((16 * NB, 128), dtype=codes.dtype)
    pad[:T] = codes
    blocks = pad.reshape(NB, 16, 128)
    y = blocks[:, _VB_TOK, _VB_COORD]  # (NB, 64, 32)
    return _chunk_words(y).reshape(NB, 192).view("<u4").view(np.uint8).reshape(NB, V_BLOCK_BYTES)


def unpack_v_fast(records, T=None):
    records = np.ascontiguousarray(np.asarray(records, dtype=np.uint8))
    NB = records.shape[0]
    if T is None:
        T = 16 * NB
    y = _words_chunk(records.view("<u4").reshape(NB, 64, 3))  # (NB, 64, 32)
    blocks = np.zeros((NB, 16, 128), dtype=np.uint8)
    blocks[:, _VB_TOK, _VB_COORD] = y
    return blocks.reshape(16 * NB, 128)[:T]
