"""ctypes binding of libiq (include/iq.h): argument marshalling only.

Every entry point keeps its C name.  Device buffers are torch CUDA tensors (PyTorch is used
for device memory and streams only); every step of the computation runs in libiq's kernels.
Loading fails loudly when libiq.so is missing: there is no CPU fallback.
"""

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libiq.so")

IQ_OK = 0
IQ_ERR_INVALID_ARG = 1
IQ_ERR_UNSUPPORTED = 2
IQ_ERR_CAPACITY = 3
IQ_ERR_WORKSPACE = 4
IQ_ERR_ALIGNMENT = 5
IQ_ERR_CUDA = 6
IQ_F16 = 0
IQ_F32 = 1
IQ_DEVERR_POSITION = 1
IQ_DEVERR_PAGE = 2
IQ_DEVERR_CTX = 4
IQ_DEVERR_TIMEOUT = 8
IQ_DEVERR_WORKSPACE = 16
IQ_ROT_ISO = 0
IQ_ROT_QUAT = 1
IQ_ROT_PLANAR = 2
ROTATIONS = {"iso": IQ_ROT_ISO, "quat": IQ_ROT_QUAT, "planar": IQ_ROT_PLANAR}
WIDTHS = ((2, 2), (3, 2), (3, 3), (4, 2), (4, 3), (4, 4))  # supported (K bits, V bits)

HEAD_DIM = 128
V_BLOCK_TOKENS = 16
TILE_TOKENS = 32


def k_record_bytes(bits=3):
    return 16 * bits


def v_block_bytes(bits=3):
    return 256 * bits


def tile_bytes(k_bits=3, v_bits=3):
    """32 K records | 2 V blocks | 32 K norms | 32 V norms (3200 bytes for 3/3)."""
    return 32 * k_record_bytes(k_bits) + 2 * v_block_bytes(v_bits) + 128


K_RECORD_BYTES = k_record_bytes(3)
V_BLOCK_BYTES = v_block_bytes(3)
TILE_BYTES = tile_bytes(3, 3)


class IqError(RuntimeError):
    def __init__(self, fn, status):
        super().__init__(f"{fn}: {iq_status_string(status)} (status {status})")
        self.status = status


class iq_cache(ctypes.Structure):
    _fields_ = [
        ("pool", ctypes.c_void_p),
        ("n_layers", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("n_pages", ctypes.c_int32),
        ("block_table_dev", ctypes.c_void_p),
        ("max_pages_per_seq", ctypes.c_int32),
        ("status_dev", ctypes.c_void_p),
        ("k_bits", ctypes.c_int32),
        ("v_bits", ctypes.c_int32),
        ("rotation", ctypes.c_int32),
    ]


class iq_fp16_prefix(ctypes.Structure):
    _fields_ = [
        ("k_dev", ctypes.c_void_p),
        ("v_dev", ctypes.c_void_p),
        ("len_dev", ctypes.c_void_p),
        ("max_len", ctypes.c_int32),
    ]


_lib = None


def lib():
    """Load libiq.so once; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libiq.so not built at {LIB_PATH}; run `python -m rotated_bit_kv_iq_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        P = ctypes.POINTER(iq_cache)
        L.iq_version.restype = ctypes.c_char_p
        L.iq_version.argtypes = []
        L.iq_status_string.restype = ctypes.c_char_p
        L.iq_status_string.argtypes = [ctypes.c_int]
        L.iq_cache_bytes.restype = ctypes.c_int
        L.iq_cache_bytes.argtypes = [i32, i32, i32, i32, i32, i32, ctypes.POINTER(sz)]
        L.iq_init_rotation.restype = ctypes.c_int
        L.iq_init_rotation.argtypes = [ctypes.c_uint64, i32, i32, vp]
        L.iq_init_rotation_variant.restype = ctypes.c_int
        L.iq_init_rotation_variant.argtypes = [ctypes.c_uint64, i32, i32, i32, vp]
        L.iq_rotation_params_per_head.restype = i32
        L.iq_rotation_params_per_head.argtypes = [i32]
        L.iq_encode_append.restype = ctypes.c_int
        L.iq_encode_append.argtypes = [P, i32, vp, vp, i32, i32, vp, vp, vp]
        L.iq_decode_workspace_size.restype = sz
        L.iq_decode_workspace_size.argtypes = [i32, i32, i32, i32]
        L.iq_decode_attention.restype = ctypes.c_int
        L.iq_decode_attention.argtypes = [P, i32, vp, ctypes.c_int, i32, i32, vp, i32, vp, vp, vp, sz, vp]
        L.iq_decode_step.restype = ctypes.c_int
        L.iq_decode_step.argtypes = [P, i32, vp, ctypes.c_int, vp, vp, i32, i32, vp, i32, vp, vp, vp, sz, vp]
        L.iq_decode_attention_noalloc.restype = ctypes.c_int
        L.iq_decode_attention_noalloc.argtypes = [P, i32, vp, ctypes.c_int, i32, i32, vp, i32, vp, vp, vp]
        L.iq_decode_deferred_workspace_size.restype = sz
        L.iq_decode_deferred_workspace_size.argtypes = [i32, i32, i32, i32, i32]
        L.iq_decode_step_deferred.restype = ctypes.c_int
        L.iq_decode_step_deferred.argtypes = [P, i32, ctypes.POINTER(iq_fp16_prefix), vp, ctypes.c_int, vp, vp, i32,
                                              i32, vp, i32, vp, vp, vp, sz, vp]
        L.iq_prefill_workspace_size.restype = sz
        L.iq_prefill_workspace_size.argtypes = [i32, i32, i32, i32]
        L.iq_prefill_attention.restype = ctypes.c_int
        L.iq_prefill_attention.argtypes = [P, i32, vp, ctypes.c_int, i32, i32, i32, vp, i32, vp, vp, vp, sz, vp]
        L.iq_export_codes.restype = ctypes.c_int
        L.iq_export_codes.argtypes = [P, i32, i32, i32, i32, i32, vp, vp, vp]
        _lib = L
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch

        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn, st):
    if st != IQ_OK:
        raise IqError(fn, st)


# ----------------------------------------------------------------------- entry points
def iq_version():
    return lib().iq_version().decode()


def iq_status_string(status):
    return lib().iq_status_string(int(status)).decode()


def iq_cache_bytes(n_layers, n_kv_heads, page_size, n_pages, k_bits=3, v_bits=3):
    a = ctypes.c_size_t(0)
    _check("iq_cache_bytes", lib().iq_cache_bytes(n_layers, n_kv_heads, page_size, n_pages, k_bits, v_bits,
                                                  ctypes.byref(a)))
    return a.value


def iq_init_rotation(seed, n_layers, n_kv_heads):
    """Seeded rotation parameters as a host float32 array [L][Hkv][32][2][4]."""
    out = np.zeros((n_layers, n_kv_heads, 32, 2, 4), dtype=np.float32)
    _check("iq_init_rotation", lib().iq_init_rotation(ctypes.c_uint64(seed), n_layers, n_kv_heads,
                                                      out.ctypes.data_as(ctypes.c_void_p)))
    return out


def iq_rotation_params_per_head(rotation):
    return int(lib().iq_rotation_params_per_head(int(rotation)))


PARAM_SHAPE = {IQ_ROT_ISO: (32, 2, 4), IQ_ROT_QUAT: (32, 4), IQ_ROT_PLANAR: (64, 2)}


def iq_init_rotation_variant(seed, rotation, n_layers, n_kv_heads):
    """Seeded parameters of any rotation variant: host float32 [L][Hkv][...] (see include/iq.h)."""
    rot = ROTATIONS.get(rotation, rotation)
    out = np.zeros((n_layers, n_kv_heads) + PARAM_SHAPE[rot], dtype=np.float32)
    _check("iq_init_rotation_variant", lib().iq_init_rotation_variant(ctypes.c_uint64(seed), rot, n_layers,
                                                                      n_kv_heads, out.ctypes.data_as(ctypes.c_void_p)))
    return out


def iq_encode_append(cache, layer, k, v, start_pos, params, stream=None):
    """k, v: fp16 [batch][n_new][Hkv][128] CUDA tensors (either may be None)."""
    ref = k if k is not None else v
    batch, n_new = int(ref.shape[0]), int(ref.shape[1])
    _check("iq_encode_append", lib().iq_encode_append(ctypes.byref(cache.c), layer, _ptr(k), _ptr(v), batch, n_new,
                                                      _ptr(start_pos), _ptr(params), _stream(stream)))


def iq_decode_workspace_size(batch, n_q_heads, n_kv_heads, max_ctx):
    return int(lib().iq_decode_workspace_size(batch, n_q_heads, n_kv_heads, max_ctx))


def iq_decode_attention(cache, layer, q, ctx_len, max_ctx, params, out, workspace, stream=None):
    """q: [batch][Hq][128] fp16|fp32; out: fp32 [batch][Hq][128]; workspace: uint8 CUDA tensor,
    zero-filled before its first use (torch.zeros); calls leave it ready for the next one."""
    import torch

    dtype = IQ_F32 if q.dtype == torch.float32 else IQ_F16
    _check("iq_decode_attention", lib().iq_decode_attention(
        ctypes.byref(cache.c), layer, _ptr(q), dtype, int(q.shape[0]), int(q.shape[1]), _ptr(ctx_len), int(max_ctx),
        _ptr(params), _ptr(out), _ptr(workspace), int(workspace.numel() * workspace.element_size()), _stream(stream)))


def iq_decode_step(cache, layer, q, k_new, v_new, ctx_len, max_ctx, params, out, workspace, stream=None):
    """Append one token per sequence (k_new, v_new: fp16 [batch][Hkv][128]) at position ctx_len-1 and
    attend over [0, ctx_len)."""
    import torch

    dtype = IQ_F32 if q.dtype == torch.float32 else IQ_F16
    _check("iq_decode_step", lib().iq_decode_step(
        ctypes.byref(cache.c), layer, _ptr(q), dtype, _ptr(k_new), _ptr(v_new), int(q.shape[0]), int(q.shape[1]),
        _ptr(ctx_len), int(max_ctx), _ptr(params), _ptr(out), _ptr(workspace),
        int(workspace.numel() * workspace.element_size()), _stream(stream)))


def iq_decode_deferred_workspace_size(batch, n_q_heads, n_kv_heads, max_ctx, max_len):
    return int(lib().iq_decode_deferred_workspace_size(batch, n_q_heads, n_kv_heads, max_ctx, max_len))


def iq_decode_step_deferred(cache, layer, k16, v16, prefix_len, q, k_new, v_new, ctx_len, max_ctx, params, out,
                            workspace, stream=None):
    """Decode step over an fp16 prefix (k16, v16: fp16 [batch][Hkv][max_len][128], prefix_len: int32
    [batch]) followed by the packed cache; the new token is appended (quantised) as by iq_decode_step."""
    import torch

    dtype = IQ_F32 if q.dtype == torch.float32 else IQ_F16
    pre = iq_fp16_prefix(k16.data_ptr(), v16.data_ptr(), prefix_len.data_ptr(), int(k16.shape[2]))
    _check("iq_decode_step_deferred", lib().iq_decode_step_deferred(
        ctypes.byref(cache.c), layer, ctypes.byref(pre), _ptr(q), dtype, _ptr(k_new), _ptr(v_new), int(q.shape[0]),
        int(q.shape[1]), _ptr(ctx_len), int(max_ctx), _ptr(params), _ptr(out), _ptr(workspace),
        int(workspace.numel() * workspace.element_size()), _stream(stream)))


def iq_prefill_workspace_size(batch, n_tokens, n_kv_heads, max_ctx):
    return int(lib().iq_prefill_workspace_size(batch, n_tokens, n_kv_heads, max_ctx))


def iq_prefill_attention(cache, layer, q, start_pos, max_ctx, params, out, workspace, stream=None):
    """q: [batch][n_tokens][Hq][128] fp16|fp32; out: fp32 of the same shape; query token i of sequence b
    at position start_pos[b] + i attends causally to the cache's positions 0 .. start_pos[b] + i."""
    import torch

    dtype = IQ_F32 if q.dtype == torch.float32 else IQ_F16
    ws_bytes = 0 if workspace is None else int(workspace.numel() * workspace.element_size())
    _check("iq_prefill_attention", lib().iq_prefill_attention(
        ctypes.byref(cache.c), layer, _ptr(q), dtype, int(q.shape[0]), int(q.shape[1]), int(q.shape[2]),
        _ptr(start_pos), int(max_ctx), _ptr(params), _ptr(out), _ptr(workspace), ws_bytes, _stream(stream)))


IQ_NOALLOC_SCRATCH_BYTES = 4 << 20


def iq_decode_attention_noalloc(cache, layer, q, ctx_len, max_ctx, params, out, stream=None):
    """iq_decode_attention with the library's fixed device scratch instead of a caller workspace."""
    import torch

    dtype = IQ_F32 if q.dtype == torch.float32 else IQ_F16
    _check("iq_decode_attention_noalloc", lib().iq_decode_attention_noalloc(
        ctypes.byref(cache.c), layer, _ptr(q), dtype, int(q.shape[0]), int(q.shape[1]), _ptr(ctx_len), int(max_ctx),
        _ptr(params), _ptr(out), _stream(stream)))


def iq_export_codes(cache, layer, kv, seq, t0, n, codes, norms=None, stream=None):
    """codes: uint8 [Hkv][n][128] CUDA tensor; norms: int16/uint16 [Hkv][n] or None."""
    _check("iq_export_codes", lib().iq_export_codes(ctypes.byref(cache.c), layer, kv, seq, t0, n, _ptr(codes),
                                                    _ptr(norms), _stream(stream)))


# ----------------------------------------------------------------------- cache holder
class PagedCache:
    """Device pool of a packed K/V cache (one torch tensor of tile records) and the iq_cache
    struct over it.

    page_size tokens per page (a multiple of 32); with block_table None, sequence b owns page b
    (a contiguous cache of capacity page_size tokens per sequence).  k_bits / v_bits are the
    code widths, rotation the variant ("iso", "quat", "planar" or its IQ_ROT_* value).  The
    k_codes, v_codes, k_norms and v_norms attributes are strided views of the pool's tile records."""

    def __init__(self, n_layers, n_kv_heads, page_size, n_pages, block_table=None, device="cuda", k_bits=3, v_bits=3,
                 rotation=IQ_ROT_ISO):
        import torch

        self.k_bits, self.v_bits = k_bits, v_bits
        self.rotation = ROTATIONS.get(rotation, rotation)
        self.tile_bytes = tile_bytes(k_bits, v_bits)
        self.pool = torch.empty(iq_cache_bytes(n_layers, n_kv_heads, page_size, n_pages, k_bits, v_bits),
                                dtype=torch.uint8, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.block_table = block_table
        self.n_layers, self.n_kv_heads, self.page_size, self.n_pages = n_layers, n_kv_heads, page_size, n_pages
        self.max_pages_per_seq = int(block_table.shape[1]) if block_table is not None else 1
        t = self.tiles()
        kv0 = 32 * k_record_bytes(k_bits)
        kn0 = kv0 + 2 * v_block_bytes(v_bits)
        self.k_codes = t[..., 0:kv0]
        self.v_codes = t[..., kv0:kn0]
        self.k_norms = t[..., kn0:kn0 + 64].view(torch.int16)
        self.v_norms = t[..., kn0 + 64:kn0 + 128].view(torch.int16)
        self.c = iq_cache(
            self.pool.data_ptr(), n_layers, n_kv_heads, HEAD_DIM, page_size, n_pages,
            block_table.data_ptr() if block_table is not None else None,
            self.max_pages_per_seq, self.status.data_ptr(), k_bits, v_bits, self.rotation,
        )

    def tiles(self):
        """[L][n_pages][Hkv][page_size/32][tile_bytes] tile records."""
        return self.pool.view(self.n_layers, self.n_pages, self.n_kv_heads, self.page_size // TILE_TOKENS,
                              self.tile_bytes)

    # Views with the records' logical shapes (for writing oracle-made records in tests).
    def k_code_view(self):
        """[L][n_pages][Hkv][page_size/32][32][16 k_bits]"""
        return self.k_codes.view(*self.k_codes.shape[:-1], TILE_TOKENS, k_record_bytes(self.k_bits))

    def v_code_view(self):
        """[L][n_pages][Hkv][page_size/32][2][256 v_bits]"""
        return self.v_codes.view(*self.v_codes.shape[:-1], 2, v_block_bytes(self.v_bits))

    def k_norm_view(self):
        """[L][n_pages][Hkv][page_size/32][32] int16"""
        return self.k_norms

    def v_norm_view(self):
        return self.v_norms
