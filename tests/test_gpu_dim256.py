"""head_dim 256 (bitpolar src/kv_cache.rs, KvCacheConfig { head_dim }): the
whole path at d = 256 against the oracle -- encode for every input type and
bit width, scores, dequantization, decode (multi-head, grouped-query, split,
shared prefix, 16-bit output) and the append step.  Same bars as d = 128:
codes and QJL signs bit-exact outside the 1e-5 boundary band, vectors and
scores within 1e-4 relative, attention within 2e-3 (plus the rounding to a
16-bit output type)."""
import numpy as np
import pytest
import torch

import oracle
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("kv_cache_vector_10_b200")

DEV = "cuda"
D = 256


def _cap(T):
    return max(16, (T + 15) // 16 * 16)


@pytest.mark.parametrize("bits", [2, 3, 4, 5])
@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
def test_encode_d256(bits, dtype):
    g = torch.Generator().manual_seed(bits * 7 + 1)
    B, H, T, m = 2, 2, 300, 128
    k = (torch.randn(B, H, T, D, generator=g) * 1.5).to(dtype)
    v = torch.randn(B, H, T, D, generator=g).to(dtype)
    gc, oc = tq.Codec(D, bits, m, 17), oracle.Codec(D, bits, m, 17)
    cache = gc.alloc(B, H, _cap(T))
    gc.encode_kv(k.to(DEV), v.to(DEV), cache)
    torch.cuda.synchronize()
    ek, ev = pu.oracle_encode(oc, k, True), pu.oracle_encode(oc, v, False)
    kg, vg = cache.k.cpu().numpy(), cache.v.cpu().numpy()
    rep = {}
    for b in range(B):
        for h in range(H):
            pu.compare_k(kg[b, h, :T], ek[b][h], oc, rep)
            pu.compare_v(vg[b, h, :T], ev[b][h], oc, rep)
    assert gc.status() == (0, 0)


@pytest.mark.parametrize("m", [64, 192])
def test_encode_d256_projections(m):
    g = torch.Generator().manual_seed(m)
    k = torch.randn(1, 3, 257, D, generator=g).to(torch.bfloat16)
    gc, oc = tq.Codec(D, 4, m, 5), oracle.Codec(D, 4, m, 5)
    cache = gc.alloc(1, 3, _cap(257))
    gc.encode_kv(k.to(DEV), None, cache)
    torch.cuda.synchronize()
    ek = pu.oracle_encode(oc, k, True)
    kg = cache.k.cpu().numpy()
    for h in range(3):
        pu.compare_k(kg[0, h, :257], ek[0][h], oc, {})


@pytest.mark.parametrize("bits", [2, 4])
def test_scores_and_dequantize_d256(bits):
    g = torch.Generator().manual_seed(40 + bits)
    B, Hkv, Hq, T = 1, 2, 4, 200
    k = torch.randn(B, Hkv, T, D, generator=g) * 2
    v = torch.randn(B, Hkv, T, D, generator=g)
    q = torch.randn(B, Hq, D, generator=g)
    gc, oc = tq.Codec(D, bits, 128, 9), oracle.Codec(D, bits, 128, 9)
    ek, ev = pu.oracle_encode(oc, k, True), pu.oracle_encode(oc, v, False)
    cache = gc.alloc(B, Hkv, _cap(T))
    pu.upload_rows(cache.k, ek, T)
    pu.upload_rows(cache.v, ev, T)
    s = gc.attention_scores(cache, q.to(DEV), T).cpu().numpy()
    kh, vh = gc.dequantize(cache, T)
    for j in range(Hq):
        h = j // 2
        ref = oc.scores(q[0, j].double().numpy(), ek[0][h]["rows"], h)
        khat = oc.dequant(ek[0][h]["rows"], h, True)
        assert np.all(np.abs(s[0, j] - ref) <= pu.scores_tolerance(ref, q[0, j].double().numpy(), khat))
    for h in range(Hkv):
        rk = oc.dequant(ek[0][h]["rows"], h, True)
        rv = oc.dequant(ev[0][h]["rows"], h, False)
        assert np.all(np.abs(kh[0, h].cpu().numpy() - rk) <= pu.vec_tolerance(rk))
        assert np.all(np.abs(vh[0, h].cpu().numpy() - rv) <= pu.vec_tolerance(rv))


def _decode_case(specs, q, Hkv, out_dtype=torch.float32):
    """specs: dict(bits, k [Bc,H,T,d], v, first_seq, n_seqs, stride) -> worst error / tolerance."""
    B, Hq, _ = q.shape
    G = Hq // Hkv
    gsegs, osegs, keep = [], [], []
    for sp in specs:
        gc, oc = tq.Codec(D, sp["bits"], 128, 42), oracle.Codec(D, sp["bits"], 128, 42)
        Bc, H, T, _ = sp["k"].shape
        ek, ev = pu.oracle_encode(oc, sp["k"], True), pu.oracle_encode(oc, sp["v"], False)
        cache = gc.alloc(Bc, H, _cap(T))
        pu.upload_rows(cache.k, ek, T)
        pu.upload_rows(cache.v, ev, T)
        keep += [gc, cache]
        for cb in range(Bc):
            fs = sp["first_seq"] + cb * sp.get("stride", 0)
            gsegs.append(tq.Segment(cache, T, fs, sp["n_seqs"], codes_batch=cb))
            osegs.append((oc, ek, ev, cb, fs, sp["n_seqs"], T))
    out = tq.decode_attention(gsegs, q.to(DEV), Hkv, out_dtype=out_dtype).float().cpu().numpy()
    worst = 0.0
    for b in range(B):
        for j in range(Hq):
            h = j // G
            segs = [(oc, h, ek[cb][h]["rows"][:T], ev[cb][h]["rows"][:T])
                    for oc, ek, ev, cb, fs, ns, T in osegs if fs <= b < fs + ns]
            ref = oracle.attention(q[b, j].double().numpy(), segs)
            worst = max(worst, float(np.max(np.abs(out[b, j] - ref) / pu.attn_tolerance(ref, out_dtype))))
    return worst


@pytest.mark.parametrize("Hq,Hkv,bits,T", [(2, 2, 4, 1000), (8, 2, 3, 700), (4, 1, 2, 3000), (2, 1, 5, 400)])
def test_decode_d256(Hq, Hkv, bits, T):
    g = torch.Generator().manual_seed(Hq + T)
    B = 2
    k = torch.randn(B, Hkv, T, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, T, D, generator=g).to(torch.bfloat16)
    q = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16)
    assert _decode_case([dict(bits=bits, k=k, v=v, first_seq=0, n_seqs=1, stride=1)], q, Hkv) <= 1.0


def test_decode_d256_shared_prefix_bf16_output():
    g = torch.Generator().manual_seed(256)
    A, Hq, Hkv = 3, 8, 2
    pk = torch.randn(1, Hkv, 400, D, generator=g).to(torch.bfloat16)
    pv = torch.randn(1, Hkv, 400, D, generator=g).to(torch.bfloat16)
    tk = torch.randn(A, Hkv, 120, D, generator=g).to(torch.bfloat16)
    tv = torch.randn(A, Hkv, 120, D, generator=g).to(torch.bfloat16)
    q = torch.randn(A, Hq, D, generator=g).to(torch.bfloat16)
    worst = _decode_case([dict(bits=2, k=pk, v=pv, first_seq=0, n_seqs=A),
                          dict(bits=4, k=tk, v=tv, first_seq=0, n_seqs=1, stride=1)], q, Hkv,
                         out_dtype=torch.bfloat16)
    assert worst <= 1.0


def test_append_d256():
    """The append step encodes the new row like the oracle and attends over it."""
    g = torch.Generator().manual_seed(9)
    B, Hkv, Hq, T = 2, 2, 4, 300
    k = torch.randn(B, Hkv, T + 1, D, generator=g).to(torch.float16)
    v = torch.randn(B, Hkv, T + 1, D, generator=g).to(torch.float16)
    q = torch.randn(B, Hq, D, generator=g).to(torch.float16)
    gc, oc = tq.Codec(D, 3, 128, 21), oracle.Codec(D, 3, 128, 21)
    cache = gc.alloc(B, Hkv, _cap(T + 1))
    gc.encode_kv(k[:, :, :T].to(DEV), v[:, :, :T].to(DEV), cache)
    segs = [tq.Segment(cache, T, b, 1, codes_batch=b) for b in range(B)]
    need = tq.tq_decode_append_workspace_bytes(segs, B, Hq, Hkv)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=DEV)
    out = torch.empty(B, Hq, D, dtype=torch.float32, device=DEV)
    tq.tq_decode_append(segs, k[:, :, T].contiguous().to(DEV), v[:, :, T].contiguous().to(DEV), q.to(DEV), B, Hq,
                        Hkv, out, ws)
    torch.cuda.synchronize()
    outc = out.cpu().numpy()
    kg, vg = cache.k.cpu().numpy(), cache.v.cpu().numpy()
    for b in range(B):
        for h in range(Hkv):
            ek = oc.encode(k[b, h].double().numpy(), h, True)
            ev = oc.encode(v[b, h].double().numpy(), h, False)
            pu.compare_k(kg[b, h, T:T + 1], oc.encode(k[b, h, T:T + 1].double().numpy(), h, True), oc, {})
            pu.compare_v(vg[b, h, T:T + 1], oc.encode(v[b, h, T:T + 1].double().numpy(), h, False), oc, {})
            for j in range(h * 2, h * 2 + 2):
                ref = oracle.attention(q[b, j].double().numpy(), [(oc, h, ek["rows"], ev["rows"])])
                assert np.max(np.abs(outc[b, j] - ref)) <= pu.ATTN_ABS
