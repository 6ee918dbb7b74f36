"""Packed code layout (oracle).  The pages fix only "packed 3-bit tensors"
([RQ-abs]; [RQ-news] section "妙处不只是压缩，而是不再展开") and that codes should be
read a word at a time and unpacked in registers ([TQ-RQ] section "真正的瓶颈"); 2- and
4-bit codes follow [TQ-RQ] section "K 和 V 的非对称需求" (more bits for K than for V).  The
bit layout below is this project's own; this module implements it from its written
specification, independently of the CUDA packer.

Chunk: 32 codes y_0..y_31 of b bits each in 4b bytes = b little-endian uint32 words:
  b = 3 (12 bytes, W_0..W_2): for w in 0..2, j in 0..7:
        bits [4j, 4j+3) of W_w  = y_{8w+j}
        bit  4j+3       of W_w  = bit w of y_{24+j}
  b = 4 (16 bytes, W_0..W_3): bits [4j, 4j+4) of W_w = y_{8w+j}
  b = 2 (8 bytes, W_0, W_1):  for w in 0..1, j in 0..7:
        bits [4j, 4j+2) of W_w = y_{16w+j},  bits [4j+2, 4j+4) of W_w = y_{16w+8+j}
In every width, "nibble j of selector word w" (w = 0..3) names slot 8w + j.

K record, one per token, 16b bytes = chunks c = 0..3 at bytes [4bc, 4bc + 4b);
    slot s of chunk c holds rotated coordinate 32c + s.

V block, one per 16 consecutive positions 16b .. 16b+15 of a (sequence, kv head), 256 b
bytes = 64 chunks; chunk (g, tq, h) with g in 0..7, tq in 0..3, h in 0..1 sits at bytes
[4b q, 4b q + 4b) with q = 2 (4 g + tq) + h.  Slot s = 8 floor(m/2) + 4 (m mod 2) + j of
chunk (g, tq, h), for m in 0..7 and j in 0..3, holds
    token  u = 8 floor(j/2) + 2 tq + (j mod 2)       (position 16b + u)
    coord  x = 16 m + g + 8 h
so token u owns nibbles j and j+4 of the selector words of the sixteen chunks
(g, tq(u), h): in every width no other token has a bit in the storage of those slots.
"""

import numpy as np

K_BYTES = 48
V_BLOCK_TOKENS = 16
V_BLOCK_BYTES = 768
BITS = (2, 3, 4)


def chunk_bytes(bits=3):
    return 4 * bits


def k_record_bytes(bits=3):
    return 16 * bits


def v_block_bytes(bits=3):
    return 256 * bits


def pack_chunk(y, bits=3):
    """32 codes -> 4*bits bytes (see module docstring)."""
    y = [int(v) for v in y]
    assert len(y) == 32 and all(0 <= v < (1 << bits) for v in y)
    out = bytearray()
    for w in range(bits):
        word = 0
        for j in range(8):
            if bits == 3:
                word |= y[8 * w + j] << (4 * j)
                word |= ((y[24 + j] >> w) & 1) << (4 * j + 3)
            elif bits == 4:
                word |= y[8 * w + j] << (4 * j)
            else:
                word |= y[16 * w + j] << (4 * j)
                word |= y[16 * w + 8 + j] << (4 * j + 2)
        out += word.to_bytes(4, "little")
    return bytes(out)


def unpack_chunk(b, bits=3):
    """4*bits bytes -> 32 codes."""
    b = bytes(b)
    assert len(b) == 4 * bits
    words = [int.from_bytes(b[4 * w : 4 * w + 4], "little") for w in range(bits)]
    y = [0] * 32
    for w in range(bits):
        for j in range(8):
            if bits == 3:
                y[8 * w + j] = (words[w] >> (4 * j)) & 7
                y[24 + j] |= ((words[w] >> (4 * j + 3)) & 1) << w
            elif bits == 4:
                y[8 * w + j] = (words[w] >> (4 * j)) & 15
            else:
                y[16 * w + j] = (words[w] >> (4 * j)) & 3
                y[16 * w + 8 + j] = (words[w] >> (4 * j + 2)) & 3
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


def pack_k(codes, bits=3):
    """codes (T, 128) -> (T, 16*bits) uint8 K records."""
    codes = np.asarray(codes)
    T = codes.shape[0]
    out = np.zeros((T, k_record_bytes(bits)), dtype=np.uint8)
    for t in range(T):
        rec = bytearray()
        for c in range(4):
            rec += pack_chunk([codes[t, k_slot_coord(c, s)] for s in range(32)], bits)
        out[t] = np.frombuffer(bytes(rec), dtype=np.uint8)
    return out


def unpack_k(records, bits=3):
    records = np.asarray(records, dtype=np.uint8)
    T = records.shape[0]
    cb = chunk_bytes(bits)
    codes = np.zeros((T, 128), dtype=np.uint8)
    for t in range(T):
        for c in range(4):
            y = unpack_chunk(records[t, cb * c : cb * c + cb].tobytes(), bits)
            for s in range(32):
                codes[t, k_slot_coord(c, s)] = y[s]
    return codes


def pack_v(codes, bits=3):
    """codes (T, 128) -> (ceil(T/16), 256*bits) uint8 V blocks; slots of positions >= T are zero."""
    codes = np.asarray(codes)
    T = codes.shape[0]
    NB = (T + 15) // 16
    cb = chunk_bytes(bits)
    out = np.zeros((NB, v_block_bytes(bits)), dtype=np.uint8)
    for blk in range(NB):
        rec = bytearray(v_block_bytes(bits))
        for g in range(8):
            for tq in range(4):
                for h in range(2):
                    y = []
                    for s in range(32):
                        u, x = v_slot_token_coord(g, tq, h, s)
                        t = 16 * blk + u
                        y.append(codes[t, x] if t < T else 0)
                    q = v_chunk_index(g, tq, h)
                    rec[cb * q : cb * q + cb] = pack_chunk(y, bits)
        out[blk] = np.frombuffer(bytes(rec), dtype=np.uint8)
    return out


def unpack_v(records, T=None, bits=3):
    records = np.asarray(records, dtype=np.uint8)
    NB = records.shape[0]
    if T is None:
        T = 16 * NB
    cb = chunk_bytes(bits)
    codes = np.zeros((T, 128), dtype=np.uint8)
    for blk in range(NB):
        for g in range(8):
            for tq in range(4):
                for h in range(2):
                    q = v_chunk_index(g, tq, h)
                    y = unpack_chunk(records[blk, cb * q : cb * q + cb].tobytes(), bits)
                    for s in range(32):
                        u, x = v_slot_token_coord(g, tq, h, s)
                        t = 16 * blk + u
                        if t < T:
                            codes[t, x] = y[s]
    return codes


def v_bit_owner(bits=3):
    """For each bit of a V block (byte-major, bit 0 first), the token (0..15) whose code it
    stores, found by packing one-hot code patterns (each bit of each slot alone) through
    pack_chunk and reading where they land."""
    cb = chunk_bytes(bits)
    owner = np.full(v_block_bytes(bits) * 8, -1)
    for g in range(8):
        for tq in range(4):
            for h in range(2):
                base = 8 * cb * v_chunk_index(g, tq, h)
                for s in range(32):
                    u, _ = v_slot_token_coord(g, tq, h, s)
                    for bit in range(bits):
                        y = [0] * 32
                        y[s] = 1 << bit
                        words = int.from_bytes(pack_chunk(y, bits), "little")
                        pos = words.bit_length() - 1
                        owner[base + pos] = u
    return owner


# --------------------------------------------------------------------- vectorised forms
# The same layout written with numpy array operations for large inputs; tests check them
# against the per-slot loops above.
def _chunk_words(y, bits=3):
    """y: (..., 32) codes -> (..., bits) uint32 words."""
    y = np.asarray(y, dtype=np.uint32)
    j = np.arange(8, dtype=np.uint32)
    words = []
    for w in range(bits):
        if bits == 3:
            word = np.bitwise_or.reduce((y[..., 8 * w : 8 * w + 8] & 7) << (4 * j), axis=-1)
            word |= np.bitwise_or.reduce(((y[..., 24:32] >> w) & 1) << (4 * j + 3), axis=-1)
        elif bits == 4:
            word = np.bitwise_or.reduce((y[..., 8 * w : 8 * w + 8] & 15) << (4 * j), axis=-1)
        else:
            word = np.bitwise_or.reduce((y[..., 16 * w : 16 * w + 8] & 3) << (4 * j), axis=-1)
            word |= np.bitwise_or.reduce((y[..., 16 * w + 8 : 16 * w + 16] & 3) << (4 * j + 2), axis=-1)
        words.append(word)
    return np.stack(words, axis=-1).astype(np.uint32)


def _words_chunk(words, bits=3):
    """(..., bits) uint32 words -> (..., 32) codes."""
    words = np.asarray(words, dtype=np.uint32)
    j = np.arange(8, dtype=np.uint32)
    y = np.zeros(words.shape[:-1] + (32,), dtype=np.uint32)
    for w in range(bits):
        ww = words[..., w : w + 1]
        if bits == 3:
            y[..., 8 * w : 8 * w + 8] = (ww >> (4 * j)) & 7
            y[..., 24:32] |= ((ww >> (4 * j + 3)) & 1) << w
        elif bits == 4:
            y[..., 8 * w : 8 * w + 8] = (ww >> (4 * j)) & 15
        else:
            y[..., 16 * w : 16 * w + 8] = (ww >> (4 * j)) & 3
            y[..., 16 * w + 8 : 16 * w + 16] = (ww >> (4 * j + 2)) & 3
    return y.astype(np.uint8)


_VB_TOK = np.zeros((64, 32), dtype=np.int64)
_VB_COORD = np.zeros((64, 32), dtype=np.int64)
for _g in range(8):
    for _tq in range(4):
        for _h in range(2):
            for _s in range(32):
                _VB_TOK[v_chunk_index(_g, _tq, _h), _s], _VB_COORD[v_chunk_index(_g, _tq, _h), _s] = \
                    v_slot_token_coord(_g, _tq, _h, _s)


def pack_k_fast(codes, bits=3):
    codes = np.asarray(codes)
    T = codes.shape[0]
    y = codes.reshape(T, 4, 32)  # chunk c holds coordinates 32c .. 32c+31 in slot order
    return _chunk_words(y, bits).reshape(T, 4 * bits).view("<u4").view(np.uint8).reshape(T, k_record_bytes(bits))


def unpack_k_fast(records, bits=3):
    records = np.ascontiguousarray(np.asarray(records, dtype=np.uint8))
    T = records.shape[0]
    words = records.view("<u4").reshape(T, 4, bits)
    return _words_chunk(words, bits).reshape(T, 128)


def pack_v_fast(codes, bits=3):
    codes = np.asarray(codes)
    T = codes.shape[0]
    NB = (T + 15) // 16
    pad = np.zeros((16 * NB, 128), dtype=codes.dtype)
    pad[:T] = codes
    blocks = pad.reshape(NB, 16, 128)
    y = blocks[:, _VB_TOK, _VB_COORD]  # (NB, 64, 32)
    return _chunk_words(y, bits).reshape(NB, 64 * bits).view("<u4").view(np.uint8).reshape(NB, v_block_bytes(bits))


def unpack_v_fast(records, T=None, bits=3):
    records = np.ascontiguousarray(np.asarray(records, dtype=np.uint8))
    NB = records.shape[0]
    if T is None:
        T = 16 * NB
    y = _words_chunk(records.view("<u4").reshape(NB, 64, bits), bits)  # (NB, 64, 32)
    blocks = np.zeros((NB, 16, 128), dtype=np.uint8)
    blocks[:, _VB_TOK, _VB_COORD] = y
    return blocks.reshape(16 * NB, 128)[:T]
