"""GPU parity of the other code widths (2, 3 and 4 bits, K and V separately) and the rotation
variants (one quaternion per block, Givens pairs; no WHT) against the fp64 oracle, through the
C ABI: codes bit-exact outside the boundary band, norms within 1 ulp, attention within 2e-3."""

import numpy as np
import pytest
import torch

from oracle import attention, encode, packing
from rotated_bit_kv_iq_b200 import binding as B
from rotated_bit_kv_iq_b200 import inputs
from tests._helpers import Guarded, max_rel_err, oracle_params, record_parity, upload_sequence

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 2e-3

# (K bits, V bits, rotation): every width pair with the WHT + quaternion-pair rotation, and the
# two variants without the WHT at symmetric and asymmetric widths
FORMS = [(2, 2, "iso"), (3, 2, "iso"), (4, 2, "iso"), (4, 3, "iso"), (4, 4, "iso"), (3, 3, "quat"),
         (3, 3, "planar"), (4, 2, "planar"), (4, 3, "quat")]


@pytest.fixture(scope="module", autouse=True)
def _built():
    from rotated_bit_kv_iq_b200 import build

    build.build()
    B.lib()


def _pd(P):
    return torch.from_numpy(np.ascontiguousarray(P)).to(DEV)


def _export(cache, layer, kv, seq, t0, n):
    codes = torch.empty((cache.n_kv_heads, n, 128), dtype=torch.uint8, device=DEV)
    norms = torch.empty((cache.n_kv_heads, n), dtype=torch.int16, device=DEV)
    B.iq_export_codes(cache, layer, kv, seq, t0, n, codes, norms)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), norms.cpu().numpy().view(np.uint16)


def _check(gpu_codes, gpu_n16, ref, label, rec):
    near = ref["near"]
    diff = gpu_codes != ref["codes"]
    bad = diff & ~near
    assert not bad.any(), f"{label}: {int(bad.sum())} code mismatches outside the boundary band"
    assert np.all(np.abs(gpu_codes.astype(int) - ref["codes"].astype(int))[diff] == 1)
    ulp = np.abs(gpu_n16.astype(np.int64) - ref["norm16"].astype(np.int64))
    assert ulp.max() <= 1, f"{label}: norm off by {ulp.max()} ulp"
    rec["excluded"] = rec.get("excluded", 0) + int(near.sum())
    rec["codes"] = rec.get("codes", 0) + int(near.size)
    rec["norm_ulp"] = max(rec.get("norm_ulp", 0), int(ulp.max()))


@pytest.mark.parametrize("kb,vb,rot", FORMS)
def test_encode_formats_match_oracle(kb, vb, rot):
    """Bulk encode (ragged paged sequences, odd starts, 5% Student-t tokens) and single-token
    appends; codes, norms and the K records' bytes checked."""
    Hkv, ps, n_pages, L, layer = 2, 64, 16, 2, 1
    P = oracle_params(7, L, Hkv, rot)
    table = torch.from_numpy(inputs.page_permutation(3, n_pages).reshape(2, 8)).to(DEV)
    cache = B.PagedCache(L, Hkv, ps, n_pages, block_table=table, k_bits=kb, v_bits=vb, rotation=rot)
    starts = np.array([0, 37], dtype=np.int32)
    n_new = 150
    X = {}
    for which in (0, 1):
        arr = np.zeros((2, n_new, Hkv, 128), dtype=np.float16)
        for b in range(2):
            for h in range(Hkv):
                arr[b, :, h] = inputs.kv_tokens(11 + b, layer, h, which, 0, n_new, heavy_frac=0.05)
        X[which] = arr
    B.iq_encode_append(cache, layer, torch.from_numpy(X[0]).to(DEV), torch.from_numpy(X[1]).to(DEV),
                       torch.from_numpy(starts).to(DEV), _pd(P))
    # then two single-token appends per sequence (the one-warp path) right after the bulk run
    extra = {w: np.stack([np.stack([inputs.kv_tokens(40 + b, layer, h, w, 0, 2) for h in range(Hkv)], axis=1)
                          for b in range(2)]) for w in (0, 1)}
    for i in range(2):
        pos = torch.from_numpy(starts + n_new + i).to(DEV)
        B.iq_encode_append(cache, layer, torch.from_numpy(extra[0][:, i:i + 1].copy()).to(DEV),
                           torch.from_numpy(extra[1][:, i:i + 1].copy()).to(DEV), pos, _pd(P))
    torch.cuda.synchronize()
    assert cache.status.item() == 0
    rec = {}
    for b in range(2):
        for which, bits in ((0, kb), (1, vb)):
            codes, n16 = _export(cache, layer, which, b, int(starts[b]), n_new + 2)
            for h in range(Hkv):
                x = np.concatenate([X[which][b, :, h], extra[which][b, :, h]])
                ref = encode.encode(x, P[layer, h], bits, rot)
                _check(codes[h], n16[h], ref, f"b={b} h={h} kv={which}", rec)
    # byte-level: sequence 0's first page as the oracle packer writes it (GPU codes where excluded)
    codes, _ = _export(cache, layer, 0, 0, 0, 64)
    ref = encode.encode(X[0][0, :64, 0], P[layer, 0], kb, rot)
    expect = np.where(ref["near"], codes[0], ref["codes"])
    page0 = int(table[0, 0])
    got = cache.k_code_view()[layer, page0, 0].reshape(-1, B.k_record_bytes(kb))[:64].cpu().numpy()
    np.testing.assert_array_equal(got, packing.pack_k_fast(expect, kb))
    codes, _ = _export(cache, layer, 1, 0, 0, 64)
    ref = encode.encode(X[1][0, :64, 0], P[layer, 0], vb, rot)
    expect = np.where(ref["near"], codes[0], ref["codes"])
    got = cache.v_code_view()[layer, page0, 0].reshape(-1, B.v_block_bytes(vb))[:4].cpu().numpy()
    np.testing.assert_array_equal(got, packing.pack_v_fast(expect, vb))
    record_parity(f"encode K{kb}/V{vb} {rot}, ragged paged + appends", **rec)


def _oracle_seq(P_layer, layer, Hkv, T, seed, kb, vb, rot):
    kc, kn, vc, vn = [], [], [], []
    for h in range(Hkv):
        ek = encode.encode(inputs.kv_tokens(seed, layer, h, 0, 0, T), P_layer[h], kb, rot)
        ev = encode.encode(inputs.kv_tokens(seed, layer, h, 1, 0, T), P_layer[h], vb, rot)
        kc.append(ek["codes"]); kn.append(ek["norm16"]); vc.append(ev["codes"]); vn.append(ev["norm16"])
    return np.stack(kc), np.stack(kn), np.stack(vc), np.stack(vn)


@pytest.mark.parametrize("kb,vb,rot", FORMS)
@pytest.mark.parametrize("G", [4, 8])
def test_decode_formats_match_oracle(kb, vb, rot, G):
    """Decode attention and the fused step over ragged paged sequences (both mma layouts)."""
    Hkv = 2
    Hq = G * Hkv
    ctx = [1, 40, 300, 777]
    ps, maxp = 64, 13
    P = oracle_params(5, 1, Hkv, rot)
    table_np = inputs.page_permutation(8, len(ctx) * maxp).reshape(len(ctx), maxp)
    cache = B.PagedCache(1, Hkv, ps, len(ctx) * maxp, block_table=torch.from_numpy(table_np).to(DEV), k_bits=kb,
                         v_bits=vb, rotation=rot)
    q = inputs.queries(6, 0, len(ctx), Hq)
    refs, knew, vnew = [], np.zeros((len(ctx), Hkv, 128), np.float16), np.zeros((len(ctx), Hkv, 128), np.float16)
    for b, T in enumerate(ctx):
        kc, kn, vc, vn = _oracle_seq(P[0], 0, Hkv, T, 300 + b, kb, vb, rot)
        for h in range(Hkv):
            # tokens 0..T-2 from the oracle; token T-1 is appended by the fused step below
            upload_sequence(cache, 0, table_np[b], h, kc[h, :T - 1], kn[h, :T - 1], vc[h, :T - 1], vn[h, :T - 1])
            knew[b, h] = inputs.kv_tokens(300 + b, 0, h, 0, T - 1, 1)[0]
            vnew[b, h] = inputs.kv_tokens(300 + b, 0, h, 1, T - 1, 1)[0]
        refs.append(attention.attention_rotated(q[b].astype(np.float64), kc, kn, vc, vn, P[0], kb, vb, rot))
    max_ctx = maxp * ps
    out = Guarded((len(ctx), Hq, 128), torch.float32, fill=float("nan"))
    ws = Guarded((B.iq_decode_workspace_size(len(ctx), Hq, Hkv, max_ctx),), torch.uint8, fill=0)
    B.iq_decode_step(cache, 0, torch.from_numpy(q).to(DEV), torch.from_numpy(knew).to(DEV),
                     torch.from_numpy(vnew).to(DEV), torch.tensor(ctx, dtype=torch.int32, device=DEV), max_ctx, _pd(P),
                     out.t, ws.t)
    torch.cuda.synchronize()
    out.check("out")
    ws.check("workspace")
    o = out.t.cpu().numpy()
    err_step = max(max_rel_err(o[b], refs[b]) for b in range(len(ctx)))
    # plain decode attention over the now complete cache gives the same result
    out2 = torch.empty((len(ctx), Hq, 128), dtype=torch.float32, device=DEV)
    B.iq_decode_attention(cache, 0, torch.from_numpy(q).to(DEV), torch.tensor(ctx, dtype=torch.int32, device=DEV),
                          max_ctx, _pd(P), out2, ws.t)
    torch.cuda.synchronize()
    o2 = out2.cpu().numpy()
    err_plain = max(max_rel_err(o2[b], refs[b]) for b in range(len(ctx)))
    rec = {"max_rel_err": max(err_step, err_plain)}
    for b, T in enumerate(ctx):  # the appended records
        for which, bits, x in ((0, kb, knew), (1, vb, vnew)):
            codes, n16 = _export(cache, 0, which, b, T - 1, 1)
            for h in range(Hkv):
                _check(codes[h], n16[h], encode.encode(x[b, h:h + 1], P[0, h], bits, rot), f"b={b}", rec)
    record_parity(f"decode + step K{kb}/V{vb} {rot} (G={G})", **rec)
    assert err_step < TOL and err_plain < TOL, (err_step, err_plain)
    assert cache.status.item() == 0


@pytest.mark.parametrize("kb,vb", [(4, 3), (3, 2)])
@pytest.mark.parametrize("shape", ["llama8b_8k", "qwen30b_32k"])
def test_decode_asymmetric_full_layers(kb, vb, shape):
    """Asymmetric K/V widths on a whole layer of the 8K (32 q / 8 kv heads) and 32K (32 q / 4 kv
    heads) workloads through the fused step; every output row compared."""
    cfg = inputs.CONFIGS[shape]
    Hq, Hkv, T = cfg["n_q_heads"], cfg["n_kv_heads"], cfg["ctx"]
    P = oracle_params(inputs.ROTATION_SEED, 1, Hkv)
    cache = B.PagedCache(1, Hkv, T, 1, k_bits=kb, v_bits=vb)
    kc, kn, vc, vn = _oracle_seq(P[0], 0, Hkv, T, 0, kb, vb, "iso")
    for h in range(Hkv):
        upload_sequence(cache, 0, [0], h, kc[h, :T - 1], kn[h, :T - 1], vc[h, :T - 1], vn[h, :T - 1])
    knew = np.stack([inputs.kv_tokens(0, 0, h, 0, T - 1, 1)[0] for h in range(Hkv)])[None]
    vnew = np.stack([inputs.kv_tokens(0, 0, h, 1, T - 1, 1)[0] for h in range(Hkv)])[None]
    q = inputs.queries(0, 0, 1, Hq)
    out = Guarded((1, Hq, 128), torch.float32, fill=float("nan"))
    ws = Guarded((B.iq_decode_workspace_size(1, Hq, Hkv, T),), torch.uint8, fill=0)
    B.iq_decode_step(cache, 0, torch.from_numpy(q).to(DEV), torch.from_numpy(knew).to(DEV),
                     torch.from_numpy(vnew).to(DEV), torch.tensor([T], dtype=torch.int32, device=DEV), T, _pd(P),
                     out.t, ws.t)
    torch.cuda.synchronize()
    out.check("out")
    ws.check("workspace")
    ref = attention.attention_rotated(q[0].astype(np.float64), kc, kn, vc, vn, P[0], kb, vb)
    err = max_rel_err(out.t.cpu().numpy()[0], ref)
    record_parity(f"decode step K{kb}/V{vb} {shape} full layer", max_rel_err=err)
    assert err < TOL, err
    assert cache.status.item() == 0
