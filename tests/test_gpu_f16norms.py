"""Binary16 key norms (tq_create_format, TQ_NORMS_F16): key rows end in n_s
and gamma rounded to binary16 (turboquant-plus-rs README, "Compression
formats": turbo4 at 4.25 bits per value), GPU against the oracle's same
format.

Codes and QJL signs bit-exact outside the 1e-5 boundary band; the stored
norms within 1e-4 relative plus one binary16 step (the kernel rounds its fp32
norm, the oracle its fp64 norm); scores, dequantized vectors and attention on
uploaded oracle rows as in the fp32 format; rows whose norms overflow
binary16 are zero rows and counted, as in the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("kv_cache_vector_10_b200")

DEV = "cuda"


def _pair(d, bits, m, seed, rotation="hadamard"):
    return (tq.Codec(d, bits, m, seed, rotation=rotation, norms="f16"),
            oracle.Codec(d, bits, m, seed, rotation=rotation, norms="f16"))


def _cap(T):
    return max(16, (T + 15) // 16 * 16)


def test_f16_row_bytes():
    gc = tq.Codec(128, 4, 128, 1, norms="f16")
    assert gc.k_row_bytes == 68 and gc.v_row_bytes == 68
    assert tq.Codec(128, 4, 128, 1).k_row_bytes == 72
    with pytest.raises(tq.TQError, match="TQ_ERR_DIM"):
        tq.tq_create_format(128, 4, 128, 1, 0, 5)


@pytest.mark.parametrize("bits", [2, 3, 4, 5])
@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
def test_f16_encode_matches_oracle(bits, dtype):
    g = torch.Generator().manual_seed(bits * 17 + dtype.itemsize)
    B, H, T, d = 2, 3, 301, 128
    k = (torch.randn(B, H, T, d, generator=g) * torch.rand(B, H, T, 1, generator=g) * 40).to(dtype)
    v = torch.randn(B, H, T, d, generator=g).to(dtype)
    gc, oc = _pair(d, bits, 128, 3 + bits)
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


@pytest.mark.parametrize("d,m,rotation", [(64, 64, "hadamard"), (128, 256, "hadamard"), (128, 128, "haar"),
                                          (64, 96, "haar")])
def test_f16_encode_dims_and_rotations(d, m, rotation):
    g = torch.Generator().manual_seed(d + m)
    k = torch.randn(1, 2, 200, d, generator=g).to(torch.bfloat16)
    v = torch.randn(1, 2, 200, d, generator=g).to(torch.bfloat16)
    gc, oc = _pair(d, 3, m, 5, rotation)
    cache = gc.alloc(1, 2, 208)
    gc.encode_kv(k.to(DEV), v.to(DEV), cache)
    ek, ev = pu.oracle_encode(oc, k, True), pu.oracle_encode(oc, v, False)
    rep = {}
    for h in range(2):
        pu.compare_k(cache.k[0, h, :200].cpu().numpy(), ek[0][h], oc, rep)
        pu.compare_v(cache.v[0, h, :200].cpu().numpy(), ev[0][h], oc, rep)


def test_f16_overflow_rows_are_zero_rows_and_counted():
    """Rows whose n_s rounds to binary16 infinity are the oracle's zero row
    and counted; neighbouring rows are unaffected."""
    g = torch.Generator().manual_seed(9)
    k = torch.randn(1, 2, 40, 128, generator=g)
    v = torch.randn(1, 2, 40, 128, generator=g)
    k[0, 0, 5] *= 1e5
    k[0, 1, 17] *= 2e3
    gc, oc = _pair(128, 4, 128, 2)
    cache = gc.alloc(1, 2, 48)
    gc.encode_kv(k.to(DEV), v.to(DEV), cache)
    torch.cuda.synchronize()
    ek, ev = pu.oracle_encode(oc, k, True), pu.oracle_encode(oc, v, False)
    assert ek[0][0]["nonfinite"] == 1 and ek[0][1]["nonfinite"] == 0
    assert gc.status() == (1, 0)
    zero = oc.encode(np.zeros((1, 128)), 0, True)["rows"][0]
    assert np.array_equal(cache.k[0, 0, 5].cpu().numpy(), zero)
    rep = {}
    for h in range(2):
        pu.compare_k(cache.k[0, h, :40].cpu().numpy(), ek[0][h], oc, rep)


@pytest.mark.parametrize("bits", [2, 4])
def test_f16_scores_dequant_decode_on_oracle_rows(bits):
    g = torch.Generator().manual_seed(60 + bits)
    B, H, Hq, T, d = 2, 2, 4, 517, 128
    k = torch.randn(B, H, T, d, generator=g) * 3
    v = torch.randn(B, H, T, d, generator=g)
    q = torch.randn(B, Hq, d, generator=g)
    gc, oc = _pair(d, bits, 128, 77)
    ek, ev = pu.oracle_encode(oc, k, True), pu.oracle_encode(oc, v, False)
    cache = gc.alloc(B, H, _cap(T))
    pu.upload_rows(cache.k, ek, T)
    pu.upload_rows(cache.v, ev, T)
    s = gc.attention_scores(cache, q.to(DEV), T).cpu().numpy()
    kh, vh = gc.dequantize(cache, T)
    kh = kh.cpu().numpy()
    segs = [tq.Segment(cache, T, b, 1, codes_batch=b) for b in range(B)]
    out = tq.decode_attention(segs, q.to(DEV), H, out_dtype=torch.float32).cpu().numpy()
    for b in range(B):
        for h in range(H):
            okh = oc.dequant(ek[b][h]["rows"], h, True)
            assert np.all(np.abs(kh[b, h] - okh) <= pu.vec_tolerance(okh))
            for j in range(h * 2, h * 2 + 2):
                qq = q[b, j].double().numpy()
                ref = oc.scores(qq, ek[b][h]["rows"], h)
                assert np.all(np.abs(s[b, j] - ref) <= pu.scores_tolerance(ref, qq, okh))
                att = oracle.attention(qq, [(oc, h, ek[b][h]["rows"], ev[b][h]["rows"])])
                assert np.max(np.abs(out[b, j] - att)) <= pu.ATTN_ABS


def test_f16_append_and_mixed_format_segments():
    """The append step writes binary16-norm rows like the oracle; a decode
    over a binary16-norm prefix and an fp32-norm tail (two contexts) matches
    the oracle over both."""
    g = torch.Generator().manual_seed(21)
    B, H, Hq, T, d = 2, 2, 4, 300, 128
    k = torch.randn(B, H, T + 1, d, generator=g).to(torch.float16)
    v = torch.randn(B, H, T + 1, d, generator=g).to(torch.float16)
    q = torch.randn(B, Hq, d, generator=g).to(torch.float16)
    gc, oc = _pair(d, 4, 128, 8)
    cache = gc.alloc(B, H, 304)
    gc.encode_kv(k[:, :, :T].to(DEV), v[:, :, :T].to(DEV), cache)
    segs = [tq.Segment(cache, T, b, 1, codes_batch=b) for b in range(B)]
    out = tq.decode_append(segs, k[:, :, T].to(DEV), v[:, :, T].to(DEV), q.to(DEV), H,
                           out_dtype=torch.float32).cpu().numpy()
    rep = {}
    for b in range(B):
        for h in range(H):
            pu.compare_k(cache.k[b, h, T:T + 1].cpu().numpy(), oc.encode(k[b, h, T:T + 1].double().numpy(), h, True),
                         oc, rep)
            ek = oc.encode(k[b, h].double().numpy(), h, True)
            ev = oc.encode(v[b, h].double().numpy(), h, False)
            for j in range(h * 2, h * 2 + 2):
                ref = oracle.attention(q[b, j].double().numpy(), [(oc, h, ek["rows"], ev["rows"])])
                assert np.max(np.abs(out[b, j] - ref)) <= pu.ATTN_ABS
    # prefix in binary16 norms (context gc), tail in fp32 norms at the same
    # bit width (context g2): rows of different lengths in one decode step
    g2, o2 = tq.Codec(d, 4, 128, 8), oracle.Codec(d, 4, 128, 8)
    Tt = 90
    kt = torch.randn(B, H, Tt, d, generator=g)
    vt = torch.randn(B, H, Tt, d, generator=g)
    tail = g2.alloc(B, H, 96)
    ekt, evt = pu.oracle_encode(o2, kt, True), pu.oracle_encode(o2, vt, False)
    pu.upload_rows(tail.k, ekt, Tt)
    pu.upload_rows(tail.v, evt, Tt)
    segs = []
    for b in range(B):
        segs += [tq.Segment(cache, T + 1, b, 1, codes_batch=b), tq.Segment(tail, Tt, b, 1, codes_batch=b)]
    out = tq.decode_attention(segs, q.to(DEV), H, out_dtype=torch.float32).cpu().numpy()
    for b in range(B):
        for h in range(H):
            ek = oc.encode(k[b, h].double().numpy(), h, True)
            ev = oc.encode(v[b, h].double().numpy(), h, False)
            for j in range(h * 2, h * 2 + 2):
                ref = oracle.attention(q[b, j].double().numpy(), [(oc, h, ek["rows"], ev["rows"]),
                                                                  (o2, h, ekt[b][h]["rows"], evt[b][h]["rows"])])
                assert np.max(np.abs(out[b, j] - ref)) <= pu.ATTN_ABS


def test_f16_split_decode():
    """Channel-split decode with binary16-norm codecs on both groups."""
    g = torch.Generator().manual_seed(31)
    B, Hkv, Hq, T = 2, 2, 4, 260
    k = torch.randn(B, Hkv, T, 128, generator=g) * torch.cat([torch.full((64,), 5.0), torch.ones(64)])
    v = torch.randn(B, Hkv, T, 128, generator=g)
    q = torch.randn(B, Hq, 128, generator=g)
    go, oo = _pair(64, 4, 64, 3)
    gn, on = _pair(64, 3, 64, 4)
    co, cn = go.alloc(B, Hkv, 272), gn.alloc(B, Hkv, 272)
    eko, evo = pu.oracle_encode(oo, k[..., :64], True), pu.oracle_encode(oo, v[..., :64], False)
    ekn, evn = pu.oracle_encode(on, k[..., 64:], True), pu.oracle_encode(on, v[..., 64:], False)
    for cache, ek, ev in ((co, eko, evo), (cn, ekn, evn)):
        pu.upload_rows(cache.k, ek, T)
        pu.upload_rows(cache.v, ev, T)
    out = tq.decode_split(go, co, gn, cn, T, q.to(DEV), out_dtype=torch.float32).cpu().numpy()
    for b in range(B):
        for j in range(Hq):
            h = j // 2
            ref = oracle.attention_split(q[b, j].double().numpy(), (oo, h, eko[b][h]["rows"], evo[b][h]["rows"]),
                                         (on, h, ekn[b][h]["rows"], evn[b][h]["rows"]))
            assert np.max(np.abs(out[b, j] - ref)) <= pu.ATTN_ABS
