"""The append step (tq_decode_append): a decode step that first encodes this
step's new key/value rows into each sequence's private tail, then attends
over the grown cache (bitpolar MultiHeadKvCache::push_token followed by
attention; fib-quant README, "Streaming KV encoder").

Checked against the oracle on the same seeded inputs:
  * the appended rows against the oracle's encode of those rows (codes and
    QJL signs bit-exact outside the 1e-5 boundary band, norms within 1e-4);
  * the step's output against oracle attention over oracle-encoded history
    plus the oracle-encoded new rows (2e-3 absolute);
and for self-consistency, the step's output is bitwise the output of
tq_decode_attention over the cache after the append (same codes, same plan).
"""
import numpy as np
import pytest
import torch

import oracle
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("kv_cache_vector_10_b200")

DEV = "cuda"


def _oracle_rows(oc, x, h, is_key):
    return oc.encode(x.double().cpu().numpy(), h, is_key)


@pytest.mark.parametrize("bits,dtype,Hq,Hkv,T", [(4, torch.float16, 4, 4, 200), (3, torch.bfloat16, 8, 2, 383),
                                                 (2, torch.bfloat16, 8, 4, 95), (5, torch.float32, 4, 4, 31),
                                                 (4, torch.float16, 4, 2, 0)])
def test_append_step_matches_oracle(bits, dtype, Hq, Hkv, T):
    g = torch.Generator().manual_seed(bits * 1000 + T)
    B, d = 3, 128
    k = (torch.randn(B, Hkv, T + 1, d, generator=g) * 1.5).to(dtype)
    v = torch.randn(B, Hkv, T + 1, d, generator=g).to(dtype)
    q = torch.randn(B, Hq, d, generator=g).to(dtype)
    gc, oc = tq.Codec(d, bits, 128, 11), oracle.Codec(d, bits, 128, 11)
    cap = (T + 1 + 15) // 16 * 16
    cache = gc.alloc(B, Hkv, cap)
    if T:
        gc.encode_kv(k[:, :, :T].to(DEV), v[:, :, :T].to(DEV), cache)
    segs = [tq.Segment(cache, T, b, 1, codes_batch=b) for b in range(B)]
    out = tq.decode_append(segs, k[:, :, T].to(DEV), v[:, :, T].to(DEV), q.to(DEV), Hkv, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert all(s.n_tokens == T + 1 for s in segs)
    assert gc.status() == (0, 0)
    rep = {}
    kg, vg = cache.k.cpu().numpy(), cache.v.cpu().numpy()
    for b in range(B):
        for h in range(Hkv):
            pu.compare_k(kg[b, h, T:T + 1], _oracle_rows(oc, k[b, h, T:T + 1], h, True), oc, rep)
            pu.compare_v(vg[b, h, T:T + 1], _oracle_rows(oc, v[b, h, T:T + 1], h, False), oc, rep)
    # the append step is a decode over the grown cache
    out2 = tq.decode_attention(segs, q.to(DEV), Hkv, out_dtype=torch.float32)
    assert torch.equal(out, out2)
    # against oracle attention over oracle codes (history + new row)
    G = Hq // Hkv
    outc = out.cpu().numpy()
    for b in range(B):
        for h in range(Hkv):
            ek = _oracle_rows(oc, k[b, h], h, True)
            ev = _oracle_rows(oc, v[b, h], h, False)
            for j in range(h * G, (h + 1) * G):
                ref = oracle.attention(q[b, j].double().numpy(), [(oc, h, ek["rows"], ev["rows"])])
                assert np.max(np.abs(outc[b, j] - ref)) <= pu.ATTN_ABS


def test_append_shared_prefix_tails_only():
    """A prefix shared by 3 sequences (bits 2) plus private tails (bits 4): the
    new rows go to the tails; the prefix codes are untouched."""
    g = torch.Generator().manual_seed(9)
    A, Hq, Hkv, d, P, Tt = 3, 8, 2, 128, 150, 60
    pk = torch.randn(1, Hkv, P, d, generator=g).to(torch.bfloat16)
    pv = torch.randn(1, Hkv, P, d, generator=g).to(torch.bfloat16)
    tk = torch.randn(A, Hkv, Tt + 1, d, generator=g).to(torch.bfloat16)
    tv = torch.randn(A, Hkv, Tt + 1, d, generator=g).to(torch.bfloat16)
    q = torch.randn(A, Hq, d, generator=g).to(torch.bfloat16)
    pc, tc = tq.Codec(d, 2, 128, 42), tq.Codec(d, 4, 128, 42)
    opc, otc = oracle.Codec(d, 2, 128, 42), oracle.Codec(d, 4, 128, 42)
    pcache, tcache = pc.alloc(1, Hkv, 160), tc.alloc(A, Hkv, 64)
    pc.encode_kv(pk.to(DEV), pv.to(DEV), pcache)
    tc.encode_kv(tk[:, :, :Tt].to(DEV), tv[:, :, :Tt].to(DEV), tcache)
    before = pcache.k.clone(), pcache.v.clone()
    segs = [tq.Segment(pcache, P, 0, A)] + [tq.Segment(tcache, Tt, a, 1, codes_batch=a) for a in range(A)]
    out = tq.decode_append(segs, tk[:, :, Tt].to(DEV), tv[:, :, Tt].to(DEV), q.to(DEV), Hkv,
                           out_dtype=torch.float32).cpu().numpy()
    assert segs[0].n_tokens == P and all(s.n_tokens == Tt + 1 for s in segs[1:])
    assert torch.equal(before[0], pcache.k) and torch.equal(before[1], pcache.v)
    rep = {}
    for a in range(A):
        for h in range(Hkv):
            pu.compare_k(tcache.k[a, h, Tt:Tt + 1].cpu().numpy(), _oracle_rows(otc, tk[a, h, Tt:Tt + 1], h, True),
                         otc, rep)
            pu.compare_v(tcache.v[a, h, Tt:Tt + 1].cpu().numpy(), _oracle_rows(otc, tv[a, h, Tt:Tt + 1], h, False),
                         otc, rep)
    G = Hq // Hkv
    for h in range(Hkv):
        epk, epv = _oracle_rows(opc, pk[0, h], h, True), _oracle_rows(opc, pv[0, h], h, False)
        for a in range(A):
            etk, etv = _oracle_rows(otc, tk[a, h], h, True), _oracle_rows(otc, tv[a, h], h, False)
            for j in range(h * G, (h + 1) * G):
                ref = oracle.attention(q[a, j].double().numpy(), [(opc, h, epk["rows"], epv["rows"]),
                                                                  (otc, h, etk["rows"], etv["rows"])])
                assert np.max(np.abs(out[a, j] - ref)) <= pu.ATTN_ABS


def test_append_codes_equal_bulk_encode():
    """The append step's codes equal tq_encode_kv's codes for the same rows,
    except decisions within float rounding of a boundary (counted; the oracle
    band covers them)."""
    g = torch.Generator().manual_seed(21)
    B, H, d, T = 4, 8, 128, 48
    k = torch.randn(B, H, T + 1, d, generator=g).to(torch.float16)
    v = torch.randn(B, H, T + 1, d, generator=g).to(torch.float16)
    q = torch.randn(B, H, d, generator=g).to(torch.float16)
    gc = tq.Codec(d, 4, 128, 3)
    c1, c2 = gc.alloc(B, H, 64), gc.alloc(B, H, 64)
    gc.encode_kv(k.to(DEV), v.to(DEV), c1)                       # all T + 1 rows in bulk
    gc.encode_kv(k[:, :, :T].to(DEV), v[:, :, :T].to(DEV), c2)
    segs = [tq.Segment(c2, T, b, 1, codes_batch=b) for b in range(B)]
    tq.decode_append(segs, k[:, :, T].to(DEV), v[:, :, T].to(DEV), q.to(DEV), H)
    torch.cuda.synchronize()
    kb, ka = c1.k[:, :, T].cpu().numpy(), c2.k[:, :, T].cpu().numpy()
    vb, va = c1.v[:, :, T].cpu().numpy(), c2.v[:, :, T].cpu().numpy()
    code_k = kb.shape[-1] - 8
    dk = (kb[..., :code_k] != ka[..., :code_k]).any(-1)
    dv = (vb[..., :-4] != va[..., :-4]).any(-1)
    assert int(dk.sum() + dv.sum()) <= 2, (int(dk.sum()), int(dv.sum()))
    nk_b, nk_a = kb[..., code_k:].copy().view(np.float32), ka[..., code_k:].copy().view(np.float32)
    assert np.allclose(nk_b[~dk], nk_a[~dk], rtol=1e-5, atol=0)
    nv_b, nv_a = vb[..., -4:].copy().view(np.float32), va[..., -4:].copy().view(np.float32)
    assert np.allclose(nv_b[~dv], nv_a[~dv], rtol=1e-5, atol=0)


def test_append_nonfinite_row_and_errors():
    g = torch.Generator().manual_seed(4)
    B, H, d = 2, 2, 128
    gc = tq.Codec(d, 3, 128, 5)
    cache = gc.alloc(B, H, 32)
    k = torch.randn(B, H, 20, d, generator=g, device="cpu").to(DEV)
    gc.encode_kv(k, k, cache)
    kn = torch.randn(B, H, d, generator=g).to(DEV)
    kn[1, 0, 7] = float("nan")
    q = torch.randn(B, 2 * H, d, generator=g).to(DEV)
    segs = [tq.Segment(cache, 20, b, 1, codes_batch=b) for b in range(B)]
    tq.decode_append(segs, kn, kn, q, H)
    assert gc.status() == (2, 0)                 # the key row and the value row
    kh, vh = gc.dequantize(cache, 21)
    assert float(kh[1, 0, 20].abs().max()) == 0.0 and float(vh[1, 0, 20].abs().max()) == 0.0
    tq.tq_reset_status(gc.ctx)
    # a shared segment is not a private tail: nowhere to append
    shared = [tq.Segment(cache, 21, 0, B)]
    with pytest.raises(tq.TQError, match="DIM_MISMATCH"):
        tq.decode_append(shared, kn, kn, q, H)
    # a full tail
    full = [tq.Segment(cache, 32, b, 1, codes_batch=b) for b in range(B)]
    with pytest.raises(tq.TQError, match="DIM_MISMATCH"):
        tq.decode_append(full, kn, kn, q, H)
    # two private tails for one sequence
    two = [tq.Segment(cache, 5, 0, 1, codes_batch=0), tq.Segment(cache, 5, 0, 1, codes_batch=1),
           tq.Segment(cache, 5, 1, 1, codes_batch=1)]
    with pytest.raises(tq.TQError, match="DIM_MISMATCH"):
        tq.decode_append(two, kn, kn, q, H)
