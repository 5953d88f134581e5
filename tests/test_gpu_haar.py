"""The Haar-QR rotation (turboquant-plus-rs README, Modules: rotation: a
Haar-random rotation from a QR factorization), GPU against the oracle.

Same bars as the Walsh-Hadamard path: codes and QJL signs bit-exact outside
the 1e-5 boundary band, norms / dequantized vectors / scores within 1e-4
relative, attention within 2e-3 absolute.  Scores, dequantization and decode
read codes the oracle produced (uploaded), so they see identical codes.
"""
import numpy as np
import pytest
import torch

import oracle
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("kv_cache_vector_10_b200")

DEV = "cuda"


def _pair(d, bits, m, seed):
    return tq.Codec(d, bits, m, seed, rotation="haar"), oracle.Codec(d, bits, m, seed, rotation="haar")


def _cap(T):
    return max(16, (T + 15) // 16 * 16)


@pytest.mark.parametrize("bits", [2, 3, 4, 5])
@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
def test_haar_encode_matches_oracle(bits, dtype):
    g = torch.Generator().manual_seed(bits * 7 + dtype.itemsize)
    B, H, T, d = 2, 3, 301, 128
    k = (torch.randn(B, H, T, d, generator=g) * 2).to(dtype)
    v = torch.randn(B, H, T, d, generator=g).to(dtype)
    gc, oc = _pair(d, bits, 128, 17 + bits)
    cache = gc.alloc(B, H, _cap(T))
    gc.encode_kv(k.to(DEV), v.to(DEV), cache)
    torch.cuda.synchronize()
    assert gc.status() == (0, 0)
    ek, ev = pu.oracle_encode(oc, k, True), pu.oracle_encode(oc, v, False)
    kg, vg = cache.k.cpu().numpy(), cache.v.cpu().numpy()
    rep = {}
    for b in range(B):
        for h in range(H):
            pu.compare_k(kg[b, h, :T], ek[b][h], oc, rep)
            pu.compare_v(vg[b, h, :T], ev[b][h], oc, rep)
    assert rep["k_rows_flipped"] <= 3 and rep["v_index_flips"] <= 3, rep


@pytest.mark.parametrize("d,m", [(64, 64), (128, 256)])
def test_haar_encode_dims_and_projections(d, m):
    g = torch.Generator().manual_seed(d + m)
    k = torch.randn(1, 2, 200, d, generator=g).to(torch.bfloat16)
    v = torch.randn(1, 2, 200, d, generator=g).to(torch.bfloat16)
    gc, oc = _pair(d, 3, m, 5)
    cache = gc.alloc(1, 2, 208)
    gc.encode_kv(k.to(DEV), v.to(DEV), cache)
    ek, ev = pu.oracle_encode(oc, k, True), pu.oracle_encode(oc, v, False)
    rep = {}
    for h in range(2):
        pu.compare_k(cache.k[0, h, :200].cpu().numpy(), ek[0][h], oc, rep)
        pu.compare_v(cache.v[0, h, :200].cpu().numpy(), ev[0][h], oc, rep)


def test_haar_power_of_two_scaling_tiny_and_nonfinite_rows():
    """The row is scaled by a power of two before the tensor-core rotation, so
    scaling the input by 2^-75 or 2^40 gives the same codes and norms scaled
    by the same power; rows with max |x_j| below 2^-100 and zero rows encode
    as zero rows; non-finite rows are counted."""
    g = torch.Generator().manual_seed(3)
    k = torch.randn(1, 2, 40, 128, generator=g)
    v = torch.randn(1, 2, 40, 128, generator=g)
    gc = tq.Codec(128, 4, 128, 9, rotation="haar")
    outs = []
    for s in (1.0, 2.0 ** -75, 2.0 ** 40, 2.0 ** -110, 0.0):
        c = gc.alloc(1, 2, 48)
        gc.encode_kv((k * s).to(DEV), (v * s).to(DEV), c)
        outs.append((c.k[:, :, :40].cpu().numpy(), c.v[:, :, :40].cpu().numpy()))
    torch.cuda.synchronize()
    assert gc.status() == (0, 0)
    bk, bv = outs[0]
    for (kk, vv), s in zip(outs[1:3], (2.0 ** -75, 2.0 ** 40)):
        assert np.array_equal(kk[..., :-8], bk[..., :-8]) and np.array_equal(vv[..., :-4], bv[..., :-4])
        assert np.array_equal(kk[..., -8:].copy().view(np.float32), bk[..., -8:].copy().view(np.float32) * np.float32(s))
        assert np.array_equal(vv[..., -4:].copy().view(np.float32), bv[..., -4:].copy().view(np.float32) * np.float32(s))
    assert np.array_equal(outs[3][0], outs[4][0]) and np.array_equal(outs[3][1], outs[4][1])
    k2 = k.clone()
    k2[0, 1, 5, 7] = float("inf")
    c = gc.alloc(1, 2, 48)
    gc.encode_kv(k2.to(DEV), v.to(DEV), c)
    assert gc.status() == (1, 0)
    z = gc.alloc(1, 2, 48)
    gc.encode_kv(torch.zeros(1, 2, 40, 128, device=DEV), torch.zeros(1, 2, 40, 128, device=DEV), z)
    assert np.array_equal(c.k[0, 1, 5].cpu().numpy(), z.k[0, 1, 5].cpu().numpy())


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_haar_encode_many_tiles_per_cta_strided_offset(d, dtype):
    """Enough 128-row tiles (16 heads x 33 tiles) that the persistent encoder's
    CTAs each take several, crossing heads, so the rotation pieces of sqrt(d) Q
    are reloaded mid-CTA; the input is a [B, T, H, d] tensor viewed as
    [B, H, T, d] (token stride H d), written at token offset 37 with a ragged
    last tile.  Sampled heads are compared with the oracle in full, and the
    rows outside the written range stay zero."""
    g = torch.Generator().manual_seed(d + 3 * dtype.itemsize)
    B, H, T, off = 1, 16, 33 * 128 - 51, 37
    base = torch.randn(B, T, H, d, generator=g).to(dtype)
    k, v = base.permute(0, 2, 1, 3), (base * 0.5).permute(0, 2, 1, 3)
    gc, oc = _pair(d, 4, 128, 31)
    cache = gc.alloc(B, H, _cap(T + off))
    gc.encode_kv(base.to(DEV).permute(0, 2, 1, 3), (base * 0.5).to(DEV).permute(0, 2, 1, 3), cache, off)
    torch.cuda.synchronize()
    assert gc.status() == (0, 0)
    rep = {}
    for h in (0, 5, 10, 15):
        ek = oc.encode(k[0, h].double().numpy(), h, True)
        ev = oc.encode(v[0, h].double().numpy(), h, False)
        pu.compare_k(cache.k[0, h, off:off + T].cpu().numpy(), ek, oc, rep)
        pu.compare_v(cache.v[0, h, off:off + T].cpu().numpy(), ev, oc, rep)
    assert rep["k_rows_flipped"] <= 12 and rep["v_index_flips"] <= 12, rep
    assert int(cache.k[:, :, :off].abs().sum()) == 0 and int(cache.v[:, :, off + T:].abs().sum()) == 0


@pytest.mark.parametrize("dtype,scale", [(torch.float16, 2.0 ** -18), (torch.float16, 2.0 ** -10),
                                         (torch.float16, 2.0 ** 13), (torch.bfloat16, 2.0 ** -40),
                                         (torch.bfloat16, 2.0 ** 40)])
def test_haar_encode_16bit_extreme_magnitudes(dtype, scale):
    """16-bit rows are rotated in their own type against sqrt(d) Q split into
    16-bit pieces, without a row scale: binary16 subnormals (2^-18), rows
    mixing subnormal and normal entries (2^-10), rows near the binary16
    maximum (2^13) and bfloat16 rows far from 1 (2^-40, 2^40) encode like the
    oracle at d = 128 and d = 64."""
    g = torch.Generator().manual_seed(int(abs(np.log2(scale))) + 7 * dtype.itemsize)
    k = (torch.randn(1, 2, 260, 128, generator=g) * scale).to(dtype)
    v = (torch.randn(1, 2, 260, 128, generator=g) * scale).to(dtype)
    for d in (128, 64):
        gc, oc = _pair(d, 4, 64, 21)
        kd, vd = k[..., :d].contiguous(), v[..., :d].contiguous()
        cache = gc.alloc(1, 2, 272)
        gc.encode_kv(kd.to(DEV), vd.to(DEV), cache)
        torch.cuda.synchronize()
        assert gc.status() == (0, 0)
        ek, ev = pu.oracle_encode(oc, kd, True), pu.oracle_encode(oc, vd, False)
        rep = {}
        for h in range(2):
            pu.compare_k(cache.k[0, h, :260].cpu().numpy(), ek[0][h], oc, rep)
            pu.compare_v(cache.v[0, h, :260].cpu().numpy(), ev[0][h], oc, rep)
        assert rep["k_rows_flipped"] <= 3 and rep["v_index_flips"] <= 3, rep


@pytest.mark.parametrize("bits", [2, 4])
def test_haar_scores_and_dequant_match_oracle(bits):
    g = torch.Generator().manual_seed(40 + bits)
    B, H, Hq, T, d = 2, 2, 4, 150, 128
    k = torch.randn(B, H, T, d, generator=g)
    v = torch.randn(B, H, T, d, generator=g)
    q = torch.randn(B, Hq, d, generator=g)
    gc, oc = _pair(d, bits, 128, 77)
    ek, ev = pu.oracle_encode(oc, k, True), pu.oracle_encode(oc, v, False)
    cache = gc.alloc(B, H, _cap(T))
    pu.upload_rows(cache.k, ek, T)
    pu.upload_rows(cache.v, ev, T)
    s = gc.attention_scores(cache, q.to(DEV), T).cpu().numpy()
    kh, vh = gc.dequantize(cache, T)
    kh, vh = kh.cpu().numpy(), vh.cpu().numpy()
    for b in range(B):
        for h in range(H):
            okh = oc.dequant(ek[b][h]["rows"], h, True)
            ovh = oc.dequant(ev[b][h]["rows"], h, False)
            assert np.all(np.abs(kh[b, h] - okh) <= pu.vec_tolerance(okh))
            assert np.all(np.abs(vh[b, h] - ovh) <= pu.vec_tolerance(ovh))
            for j in range(h * 2, h * 2 + 2):
                qq = q[b, j].double().numpy()
                ref = oc.scores(qq, ek[b][h]["rows"], h)
                assert np.all(np.abs(s[b, j] - ref) <= pu.scores_tolerance(ref, qq, okh))


@pytest.mark.parametrize("Hq,Hkv,bits,T", [(4, 4, 4, 700), (8, 2, 2, 513)])
def test_haar_decode_matches_oracle(Hq, Hkv, bits, T):
    g = torch.Generator().manual_seed(Hq * 31 + T)
    B, d = 2, 128
    k = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, T, d, generator=g).to(torch.bfloat16)
    q = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16)
    gc, oc = _pair(d, bits, 128, 1)
    ek, ev = pu.oracle_encode(oc, k, True), pu.oracle_encode(oc, v, False)
    cache = gc.alloc(B, Hkv, _cap(T))
    pu.upload_rows(cache.k, ek, T)
    pu.upload_rows(cache.v, ev, T)
    segs = [tq.Segment(cache, T, b, 1, codes_batch=b) for b in range(B)]
    out = tq.decode_attention(segs, q.to(DEV), Hkv, out_dtype=torch.float32).cpu().numpy()
    G = Hq // Hkv
    for b in range(B):
        for j in range(Hq):
            h = j // G
            ref = oracle.attention(q[b, j].double().numpy(), [(oc, h, ek[b][h]["rows"], ev[b][h]["rows"])])
            assert np.max(np.abs(out[b, j] - ref)) <= pu.ATTN_ABS


def test_haar_end_to_end_and_append():
    """GPU encode -> GPU decode with an appended token, against oracle encode
    -> oracle attention; the appended rows against the oracle's encode."""
    g = torch.Generator().manual_seed(12)
    B, H, Hq, T, d = 2, 4, 8, 600, 128
    k = torch.randn(B, H, T + 1, d, generator=g).to(torch.float16)
    v = torch.randn(B, H, T + 1, d, generator=g).to(torch.float16)
    q = torch.randn(B, Hq, d, generator=g).to(torch.float16)
    gc, oc = _pair(d, 3, 128, 4)
    cache = gc.alloc(B, H, 608)
    gc.encode_kv(k[:, :, :T].to(DEV), v[:, :, :T].to(DEV), cache)
    segs = [tq.Segment(cache, T, b, 1, codes_batch=b) for b in range(B)]
    out = tq.decode_append(segs, k[:, :, T].to(DEV), v[:, :, T].to(DEV), q.to(DEV), H,
                           out_dtype=torch.float32).cpu().numpy()
    rep = {}
    for b in range(B):
        for h in range(H):
            pu.compare_k(cache.k[b, h, T:T + 1].cpu().numpy(), oc.encode(k[b, h, T:T + 1].double().numpy(), h, True),
                         oc, rep)
            pu.compare_v(cache.v[b, h, T:T + 1].cpu().numpy(), oc.encode(v[b, h, T:T + 1].double().numpy(), h, False),
                         oc, rep)
            ek = oc.encode(k[b, h].double().numpy(), h, True)
            ev = oc.encode(v[b, h].double().numpy(), h, False)
            for j in range(h * 2, h * 2 + 2):
                ref = oracle.attention(q[b, j].double().numpy(), [(oc, h, ek["rows"], ev["rows"])])
                assert np.max(np.abs(out[b, j] - ref)) <= pu.ATTN_ABS


def test_haar_rejects_unknown_rotation():
    with pytest.raises(tq.TQError, match="TQ_ERR_DIM"):
        tq.tq_create_ex(128, 3, 128, 1, 7)
