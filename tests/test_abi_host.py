"""Host-side checks of the C ABI (no GPU needed): exported symbols, host-only entry points,
and argument validation that must reject a call before any kernel launch."""

import ctypes
import os
import re

import numpy as np
import pytest
import torch

from oracle import rotation
from rotated_bit_kv_iq_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from rotated_bit_kv_iq_b200 import build

    build.build()
    return B.lib()


def test_library_exports_every_declared_symbol(lib):
    hdr = open(os.path.join(ROOT, "include", "iq.h")).read()
    names = set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b(iq_\w+)\s*\(", hdr, flags=re.M))
    assert {"iq_init_rotation", "iq_encode_append", "iq_decode_attention", "iq_decode_workspace_size",
            "iq_export_codes", "iq_status_string", "iq_cache_bytes", "iq_version", "iq_decode_step",
            "iq_init_rotation_variant", "iq_rotation_params_per_head", "iq_prefill_attention",
            "iq_prefill_workspace_size", "iq_decode_step_deferred", "iq_decode_deferred_workspace_size"} <= names
    for n in names:
        assert hasattr(lib, n), n
        assert ctypes.cast(getattr(lib, n), ctypes.c_void_p).value


def test_status_strings_and_version(lib):
    assert "libiq" in B.iq_version()
    for s in range(7):
        assert B.iq_status_string(s)
    assert B.iq_status_string(99) == "unknown status"


def test_init_rotation_is_bit_identical_to_oracle(lib):
    got = B.iq_init_rotation(1, 3, 4)
    want = rotation.init_rotation(1, 3, 4)
    assert got.dtype == np.float32 and got.shape == (3, 4, 32, 2, 4)
    np.testing.assert_array_equal(got.view(np.uint32), want.view(np.uint32))
    got = B.iq_init_rotation(0xDEADBEEFCAFEF00D, 2, 3)
    np.testing.assert_array_equal(got.view(np.uint32), rotation.init_rotation(0xDEADBEEFCAFEF00D, 2, 3).view(np.uint32))


@pytest.mark.parametrize("variant", ["quat", "planar"])
def test_variant_params_are_bit_identical_to_oracle(lib, variant):
    got = B.iq_init_rotation_variant(3, variant, 2, 3)
    want = rotation.init_rotation(3, 2, 3, variant)
    assert got.shape == want.shape and got.dtype == np.float32
    np.testing.assert_array_equal(got.view(np.uint32), want.view(np.uint32))
    assert B.iq_rotation_params_per_head(B.ROTATIONS[variant]) == 128
    assert B.iq_rotation_params_per_head(0) == 256 and B.iq_rotation_params_per_head(3) == 0
    iso = B.iq_init_rotation_variant(1, "iso", 1, 2)
    np.testing.assert_array_equal(iso.view(np.uint32), B.iq_init_rotation(1, 1, 2).view(np.uint32))
    assert B.lib().iq_init_rotation_variant(1, 7, 1, 1, got.ctypes.data_as(ctypes.c_void_p)) == B.IQ_ERR_UNSUPPORTED


def test_cache_bytes_and_workspace(lib):
    pb = B.iq_cache_bytes(2, 4, 64, 10)
    assert pb == 2 * 4 * 64 * 10 * 100  # 48 + 48 code bytes and 2 + 2 norm bytes per slot and kv head
    for kb, vb in B.WIDTHS:  # 16 (kb + vb) code bytes and 4 norm bytes per slot and kv head
        assert B.iq_cache_bytes(1, 2, 64, 3, kb, vb) == 2 * 64 * 3 * (16 * (kb + vb) + 4)
    with pytest.raises(B.IqError):
        B.iq_cache_bytes(1, 1, 48, 1)  # page size not a multiple of 32
    with pytest.raises(B.IqError):
        B.iq_cache_bytes(1, 1, 64, 1, 2, 3)  # V wider than K: not built
    w1 = B.iq_decode_workspace_size(1, 32, 4, 32768)
    w2 = B.iq_decode_workspace_size(2, 32, 4, 32768)
    assert 0 < w1 <= w2
    assert B.iq_decode_workspace_size(1, 32, 0, 10) == 0


# --- validation: fake but aligned device addresses; every call below must be rejected
# on the host.  Skipped on a GPU machine so that a validation bug can never launch a
# kernel on these addresses.
cpu_only = pytest.mark.skipif(torch.cuda.is_available(), reason="fake-pointer checks run only without a GPU")


def _fake_cache(**kw):
    c = B.iq_cache(0x10000, 2, 2, 128, 64, 4, None, 1, None)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def _enc(c, layer=0, k=0x50000, v=0x60000, batch=1, n_new=4, start=0x70000, params=0x80000):
    return B.lib().iq_encode_append(ctypes.byref(c) if c is not None else None, layer, k, v, batch, n_new, start,
                                    params, None)


def _dec(c, layer=0, q=0x50000, dtype=0, batch=1, hq=8, ctx=0x70000, max_ctx=32, params=0x80000, out=0x90000,
         ws=0xA0000, ws_bytes=1 << 30):
    return B.lib().iq_decode_attention(ctypes.byref(c) if c is not None else None, layer, q, dtype, batch, hq, ctx,
                                       max_ctx, params, out, ws, ws_bytes, None)


@cpu_only
def test_encode_rejects_bad_arguments(lib):
    assert _enc(None) == B.IQ_ERR_INVALID_ARG
    assert _enc(_fake_cache(head_dim=64)) == B.IQ_ERR_UNSUPPORTED
    assert _enc(_fake_cache(page_size=24)) == B.IQ_ERR_INVALID_ARG
    assert _enc(_fake_cache(), layer=2) == B.IQ_ERR_INVALID_ARG
    assert _enc(_fake_cache(), layer=-1) == B.IQ_ERR_INVALID_ARG
    assert _enc(_fake_cache(pool=None)) == B.IQ_ERR_INVALID_ARG
    assert _enc(_fake_cache(pool=0x10004)) == B.IQ_ERR_ALIGNMENT
    assert _enc(_fake_cache(), k=None, v=None) == B.IQ_ERR_INVALID_ARG
    assert _enc(_fake_cache(), start=None) == B.IQ_ERR_INVALID_ARG
    assert _enc(_fake_cache(), params=None) == B.IQ_ERR_INVALID_ARG
    assert _enc(_fake_cache(), k=0x50008) == B.IQ_ERR_ALIGNMENT
    assert _enc(_fake_cache(), n_new=65) == B.IQ_ERR_CAPACITY          # > page_size without a block table
    assert _enc(_fake_cache(), batch=5) == B.IQ_ERR_CAPACITY           # more sequences than pages
    assert _enc(_fake_cache(), n_new=-1) == B.IQ_ERR_INVALID_ARG
    assert _enc(_fake_cache(block_table_dev=0xB0000, max_pages_per_seq=0)) == B.IQ_ERR_INVALID_ARG


@cpu_only
def test_calls_reject_unsupported_formats(lib):
    for kw in (dict(k_bits=5), dict(k_bits=2, v_bits=3), dict(v_bits=1), dict(rotation=3), dict(rotation=-1)):
        assert _enc(_fake_cache(**kw)) == B.IQ_ERR_UNSUPPORTED, kw
        assert _dec(_fake_cache(**kw)) == B.IQ_ERR_UNSUPPORTED, kw


@cpu_only
def test_decode_rejects_bad_arguments(lib):
    assert _dec(None) == B.IQ_ERR_INVALID_ARG
    assert _dec(_fake_cache(head_dim=96)) == B.IQ_ERR_UNSUPPORTED
    assert _dec(_fake_cache(), hq=18) == B.IQ_ERR_UNSUPPORTED         # group size 9
    assert _dec(_fake_cache(), hq=5) == B.IQ_ERR_INVALID_ARG          # not a multiple of Hkv
    assert _dec(_fake_cache(), dtype=7) == B.IQ_ERR_UNSUPPORTED
    assert _dec(_fake_cache(), max_ctx=65) == B.IQ_ERR_CAPACITY
    assert _dec(_fake_cache(), ws_bytes=16) == B.IQ_ERR_WORKSPACE
    assert _dec(_fake_cache(), ws=None) == B.IQ_ERR_WORKSPACE
    assert _dec(_fake_cache(), ws=0xA0010) == B.IQ_ERR_ALIGNMENT
    assert _dec(_fake_cache(), q=0x50004) == B.IQ_ERR_ALIGNMENT
    assert _dec(_fake_cache(), out=None) == B.IQ_ERR_INVALID_ARG
    assert _dec(_fake_cache(), ctx=None) == B.IQ_ERR_INVALID_ARG
    assert _dec(_fake_cache(), batch=-1) == B.IQ_ERR_INVALID_ARG
    assert _dec(_fake_cache(), max_ctx=-1) == B.IQ_ERR_INVALID_ARG


@cpu_only
def test_decode_step_rejects_bad_arguments(lib):
    f = B.lib().iq_decode_step

    def step(c, k=0x58000, v=0x5C000, max_ctx=32, hq=8, ws_bytes=1 << 30):
        return f(ctypes.byref(c), 0, 0x50000, 0, k, v, 1, hq, 0x70000, max_ctx, 0x80000, 0x90000, 0xA0000, ws_bytes,
                 None)

    assert step(_fake_cache(), k=None) == B.IQ_ERR_INVALID_ARG
    assert step(_fake_cache(), v=None) == B.IQ_ERR_INVALID_ARG
    assert step(_fake_cache(), k=0x58008) == B.IQ_ERR_ALIGNMENT
    assert step(_fake_cache(), max_ctx=0) == B.IQ_ERR_INVALID_ARG   # the new token needs a slot
    assert step(_fake_cache(), max_ctx=65) == B.IQ_ERR_CAPACITY
    assert step(_fake_cache(), hq=18) == B.IQ_ERR_UNSUPPORTED
    assert step(_fake_cache(), ws_bytes=8) == B.IQ_ERR_WORKSPACE
    assert step(_fake_cache(head_dim=64)) == B.IQ_ERR_UNSUPPORTED


@cpu_only
def test_prefill_rejects_bad_arguments(lib):
    f = B.lib().iq_prefill_attention

    def pre(c, q=0x50000, dtype=0, batch=1, n_tok=8, hq=8, start=0x70000, max_ctx=32, ws=0xA0000, ws_bytes=1 << 30):
        return f(ctypes.byref(c), 0, q, dtype, batch, n_tok, hq, start, max_ctx, 0x80000, 0x90000, ws, ws_bytes, None)

    assert pre(_fake_cache(), n_tok=40) == B.IQ_ERR_INVALID_ARG      # max_ctx below the chunk
    assert pre(_fake_cache(), max_ctx=65) == B.IQ_ERR_CAPACITY
    assert pre(_fake_cache(), hq=18) == B.IQ_ERR_UNSUPPORTED
    assert pre(_fake_cache(), hq=5) == B.IQ_ERR_INVALID_ARG
    assert pre(_fake_cache(), dtype=3) == B.IQ_ERR_UNSUPPORTED
    assert pre(_fake_cache(), start=None) == B.IQ_ERR_INVALID_ARG
    assert pre(_fake_cache(), q=0x50004) == B.IQ_ERR_ALIGNMENT
    assert pre(_fake_cache(), ws=None) == B.IQ_ERR_WORKSPACE
    assert pre(_fake_cache(), ws_bytes=64) == B.IQ_ERR_WORKSPACE
    assert pre(_fake_cache(), ws=0xA0040) == B.IQ_ERR_ALIGNMENT
    assert pre(_fake_cache(k_bits=5)) == B.IQ_ERR_UNSUPPORTED
    assert pre(_fake_cache(), batch=5) == B.IQ_ERR_CAPACITY
    assert B.iq_prefill_workspace_size(1, 512, 8, 8192) > 0


@cpu_only
def test_deferred_step_rejects_bad_arguments(lib):
    f = B.lib().iq_decode_step_deferred

    def step(c, pre, max_ctx=32, hq=8, ws=0xA0000, ws_bytes=1 << 30):
        return f(ctypes.byref(c), 0, ctypes.byref(pre) if pre is not None else None, 0x50000, 0, 0x58000, 0x5C000, 1,
                 hq, 0x70000, max_ctx, 0x80000, 0x90000, ws, ws_bytes, None)

    good = B.iq_fp16_prefix(0x100000, 0x200000, 0x300000, 16)
    assert step(_fake_cache(), None) == B.IQ_ERR_INVALID_ARG
    assert step(_fake_cache(), B.iq_fp16_prefix(None, 0x200000, 0x300000, 16)) == B.IQ_ERR_INVALID_ARG
    assert step(_fake_cache(), B.iq_fp16_prefix(0x100000, 0x200000, None, 16)) == B.IQ_ERR_INVALID_ARG
    assert step(_fake_cache(), B.iq_fp16_prefix(0x100008, 0x200000, 0x300000, 16)) == B.IQ_ERR_ALIGNMENT
    assert step(_fake_cache(), B.iq_fp16_prefix(0x100000, 0x200000, 0x300000, -1)) == B.IQ_ERR_INVALID_ARG
    assert step(_fake_cache(), good, max_ctx=65) == B.IQ_ERR_CAPACITY
    assert step(_fake_cache(), good, hq=18) == B.IQ_ERR_UNSUPPORTED
    assert step(_fake_cache(), good, ws_bytes=64) == B.IQ_ERR_WORKSPACE
    assert step(_fake_cache(k_bits=1), good) == B.IQ_ERR_UNSUPPORTED
    assert B.iq_decode_deferred_workspace_size(1, 32, 8, 8704, 8192) > B.iq_decode_workspace_size(1, 32, 8, 8704)


@cpu_only
def test_export_rejects_bad_arguments(lib):
    c = _fake_cache()
    f = B.lib().iq_export_codes
    assert f(ctypes.byref(c), 0, 2, 0, 0, 4, 0x50000, None, None) == B.IQ_ERR_INVALID_ARG
    assert f(ctypes.byref(c), 0, 0, 4, 0, 4, 0x50000, None, None) == B.IQ_ERR_CAPACITY
    assert f(ctypes.byref(c), 0, 0, 0, 60, 8, 0x50000, None, None) == B.IQ_ERR_CAPACITY
    assert f(ctypes.byref(c), 0, 0, 0, 0, 4, None, None, None) == B.IQ_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(B, "_lib", None)
    monkeypatch.setattr(B, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="not built"):
        B.lib()
