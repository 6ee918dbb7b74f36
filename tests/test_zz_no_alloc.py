"""iq_decode_attention_noalloc: the same decode attention as iq_decode_attention, with the
split-K scratch in the library's fixed device array, for callers that may not allocate
device memory (plugins whose host owns every allocation, services that must not allocate
after start-up).  Collected last on purpose; it must pass alone and after the other tests."""

import ctypes

import numpy as np
import pytest
import torch

from rotated_bit_kv_iq_b200 import binding as B
from rotated_bit_kv_iq_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 2e-3  # the attention tolerance used by the parity tests


def _max_rel(a, b):
    a = a.reshape(-1, 128).astype(np.float64)
    b = b.reshape(-1, 128).astype(np.float64)
    return float((np.abs(a - b).max(1) / np.maximum(np.abs(b).max(1), 1e-30)).max())


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    """Ragged paged batch (contexts 2500, 1, 777 over shuffled 64-token pages), group size 8:
    two calls in a row with different queries, each against iq_decode_attention with a
    workspace from torch."""
    from rotated_bit_kv_iq_b200 import build

    build.build()
    Bn, Hq, Hkv, ps, maxp = 3, 16, 2, 64, 40
    max_ctx = ps * maxp
    ctx = torch.tensor([2500, 1, 777], dtype=torch.int32, device=DEV)
    P = torch.from_numpy(B.iq_init_rotation(inputs.ROTATION_SEED, 1, Hkv)).to(DEV)
    table = torch.from_numpy(inputs.page_permutation(2, Bn * maxp).reshape(Bn, maxp)).to(DEV)
    cache = B.PagedCache(1, Hkv, ps, Bn * maxp, block_table=table)
    g = torch.Generator(device=DEV).manual_seed(5)
    cache.k_codes.copy_(torch.randint(0, 256, cache.k_codes.shape, generator=g, device=DEV, dtype=torch.uint8))
    cache.v_codes.copy_(torch.randint(0, 256, cache.v_codes.shape, generator=g, device=DEV, dtype=torch.uint8))
    cache.k_norms.copy_((torch.rand(cache.k_norms.shape, generator=g, device=DEV) * 40 + 1).half().view(torch.int16))
    cache.v_norms.copy_((torch.rand(cache.v_norms.shape, generator=g, device=DEV) * 40 + 1).half().view(torch.int16))
    need = B.iq_decode_workspace_size(Bn, Hq, Hkv, max_ctx)
    assert need <= B.IQ_NOALLOC_SCRATCH_BYTES
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
    for call in range(2):  # the second call reuses the scratch the first one left behind
        q = torch.randn((Bn, Hq, 128), generator=g, device=DEV).half()
        ref = torch.empty((Bn, Hq, 128), dtype=torch.float32, device=DEV)
        got = torch.full((Bn, Hq, 128), float("nan"), dtype=torch.float32, device=DEV)
        B.iq_decode_attention(cache, 0, q, ctx, max_ctx, P, ref, ws)
        B.iq_decode_attention_noalloc(cache, 0, q, ctx, max_ctx, P, got)
        torch.cuda.synchronize()
        gn, rn = got.cpu().numpy(), ref.cpu().numpy()
        assert np.isfinite(gn).all(), call
        assert _max_rel(gn, rn) <= TOL, (call, _max_rel(gn, rn))
    assert cache.status.item() == 0


def test_noalloc_rejects_problems_larger_than_its_scratch():
    # sizes whose split-K scratch exceeds the fixed array are refused on the host, before any launch
    from rotated_bit_kv_iq_b200 import build

    build.build()
    assert B.iq_decode_workspace_size(256, 64, 8, 1 << 20) > B.IQ_NOALLOC_SCRATCH_BYTES
    c = B.iq_cache(0x10000, 1, 8, 128, 1 << 20, 256, None, 1, None)
    st = B.lib().iq_decode_attention_noalloc(ctypes.byref(c), 0, 0x50000, 0, 256, 64, 0x70000, 1 << 20, 0x80000,
                                             0x90000, None)
    assert st == B.IQ_ERR_WORKSPACE
