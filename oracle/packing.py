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

V record, one per token pair (2p, 2p+1), 96 bytes = chunks g = 0..7 at bytes
[12g, 12g+12); slot s of chunk g holds
    token  2p + (1 if s mod 4 >= 2 else 0)
    coord  16g + 2*floor(s/4) + (s mod 2)
so every byte belongs to one token of the pair: even bytes to token 2p, odd bytes
to token 2p+1.
"""

import numpy as np

K_BYTES = 48
V_PAIR_BYTES = 96


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


def v_slot_token_coord(g, s):
    return (1 if (s % 4) >= 2 else 0), 16 * g + 2 * (s // 4) + (s % 2)


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
    """codes (T, 128) -> (ceil(T/2), 96) uint8 V records.  For odd T the last record's
    odd bytes (the missing partner's) are left zero."""
    codes = np.asarray(codes)
    T = codes.shape[0]
    P = (T + 1) // 2
    out = np.zeros((P, V_PAIR_BYTES), dtype=np.uint8)
    for p in range(P):
        rec = bytearray()
        for g in range(8):
            y = []
            for s in range(32):
                tok, coord = v_slot_token_coord(g, s)
                t = 2 * p + tok
                y.append(codes[t, coord] if t < T else 0)
            rec += pack_chunk(y)
        out[p] = np.frombuffer(bytes(rec), dtype=np.uint8)
    return out


def unpack_v(records, T=None):
    records = np.asarray(records, dtype=np.uint8)
    P = records.shape[0]
    if T is None:
        T = 2 * P
    codes = np.zeros((T, 128), dtype=np.uint8)
    for p in range(P):
        for g in range(8):
            y = unpack_chunk(records[p, 12 * g : 12 * g + 12].tobytes())
            for s in range(32):
                tok, coord = v_slot_token_coord(g, s)
                t = 2 * p + tok
                if t < T:
                    codes[t, coord] = y[s]
    return codes


def v_byte_owner():
    """For each of the 96 bytes of a V record, which token of the pair (0 or 1) owns it."""
    return np.arange(V_PAIR_BYTES) % 2


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


_V_TOK = np.array([1 if (s % 4) >= 2 else 0 for s in range(32)])
_V_COORD = np.array([[16 * g + 2 * (s // 4) + (s % 2) for s in range(32)] for g in range(8)])


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
    P = (T + 1) // 2
    pad = np.zeros((2 * P, 128), dtype=codes.dtype)
    pad[:T] = codes
    pairs = pad.reshape(P, 2, 128)
    y = pairs[:, _V_TOK[None, :], _V_COORD]  # (P, 8, 32)
    return _chunk_words(y).reshape(P, 24).view("<u4").view(np.uint8).reshape(P, V_PAIR_BYTES)


def unpack_v_fast(records, T=None):
    records = np.ascontiguousarray(np.asarray(records, dtype=np.uint8))
    P = records.shape[0]
    if T is None:
        T = 2 * P
    y = _words_chunk(records.view("<u4").reshape(P, 8, 3))  # (P, 8, 32)
    pairs = np.zeros((P, 2, 128), dtype=np.uint8)
    pairs[:, _V_TOK[None, :], _V_COORD] = y
    return pairs.reshape(2 * P, 128)[:T]
