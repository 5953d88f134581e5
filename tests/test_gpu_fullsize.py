"""Parity at the benchmark workloads' own sizes, in the launch configuration
bench.py times, checked against the CPU oracle on sampled heads.

The whole workload is encoded and decoded on the GPU exactly as the bench
does it (same generators, same codecs, same segments, same output type);
the oracle then encodes the sampled (sequence, kv head) rows itself and
attends over its own codes.  Codes and QJL signs must be bit-exact outside
the 1e-5 boundary band; attention outputs within 2e-3 (plus the rounding to
the output type, at most half an ulp of it).  The decode reads the GPU's
codes, the oracle its own, so a boundary-band flip in the encode is part of
the error allowed here, as in the other end-to-end cases.
"""
import numpy as np
import pytest
import torch

import oracle
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("kv_cache_vector_10_b200")
from kv_cache_vector_10_b200 import workloads  # noqa: E402

DEV = "cuda"
D = M = 128


def _check_rows(cache, oc, enc_k, enc_v, b, h, T, rep):
    kg = cache.k[b, h, :T].cpu().numpy()
    vg = cache.v[b, h, :T].cpu().numpy()
    pu.compare_k(kg, enc_k, oc, rep)
    pu.compare_v(vg, enc_v, oc, rep)


def _check_out(out, ref, b, j):
    err = np.abs(out[b, j].float().cpu().numpy() - ref)
    tol = pu.attn_tolerance(ref, out.dtype)
    assert np.all(err <= tol), (b, j, float(np.max(err / tol)))


def test_mha_decode_full_size_sampled_heads():
    """batch 8 x 32 heads x 4096 tokens, fp16, bits 4; (b, h) = (0, 0) and (6, 21)."""
    w = workloads.mha_decode(device=DEV, data_seed=2)
    B, H, T, _ = w["k"].shape
    gc = tq.Codec(D, w["bits"], M, w["seed"])
    cache = gc.alloc(B, H, T)
    gc.encode_kv(w["k"], w["v"], cache)
    segs = [tq.Segment(cache, T, b, 1, codes_batch=b) for b in range(B)]
    out = torch.empty(B, H, D, dtype=w["q"].dtype, device=DEV)
    ws = torch.empty(max(tq.tq_decode_workspace_bytes(segs, B, H, H), 16), dtype=torch.uint8, device=DEV)
    tq.tq_decode_attention(segs, w["q"], B, H, H, out, ws)
    torch.cuda.synchronize()
    oc = oracle.Codec(D, w["bits"], M, w["seed"])
    rep = {}
    for b, h in ((0, 0), (6, 21)):
        ek = oc.encode(w["k"][b, h].double().cpu().numpy(), h, True)
        ev = oc.encode(w["v"][b, h].double().cpu().numpy(), h, False)
        _check_rows(cache, oc, ek, ev, b, h, T, rep)
        ref = oracle.attention(w["q"][b, h].double().cpu().numpy(), [(oc, h, ek["rows"], ev["rows"])])
        _check_out(out, ref, b, h)
    print("flips:", rep)


@pytest.mark.parametrize("variant", ["haar", "f16norms"])
def test_mha_decode_variants_full_size_sampled_heads(variant):
    """The multi-head workload under the Haar-QR rotation (the TMA-fed
    encoders with sqrt(d) Q in two binary16 pieces) and with binary16 key
    norms, as bench.py times them; (b, h) = (1, 3) and (7, 30)."""
    w = workloads.mha_decode(device=DEV, data_seed=4)
    B, H, T, _ = w["k"].shape
    kw = dict(rotation="haar") if variant == "haar" else dict(norms="f16")
    gc = tq.Codec(D, w["bits"], M, w["seed"], **kw)
    cache = gc.alloc(B, H, T)
    gc.encode_kv(w["k"], w["v"], cache)
    segs = [tq.Segment(cache, T, b, 1, codes_batch=b) for b in range(B)]
    out = torch.empty(B, H, D, dtype=w["q"].dtype, device=DEV)
    ws = torch.empty(max(tq.tq_decode_workspace_bytes(segs, B, H, H), 16), dtype=torch.uint8, device=DEV)
    tq.tq_decode_attention(segs, w["q"], B, H, H, out, ws)
    torch.cuda.synchronize()
    assert gc.status() == (0, 0)
    oc = oracle.Codec(D, w["bits"], M, w["seed"], **kw)
    rep = {}
    for b, h in ((1, 3), (7, 30)):
        ek = oc.encode(w["k"][b, h].double().cpu().numpy(), h, True)
        ev = oc.encode(w["v"][b, h].double().cpu().numpy(), h, False)
        _check_rows(cache, oc, ek, ev, b, h, T, rep)
        ref = oracle.attention(w["q"][b, h].double().cpu().numpy(), [(oc, h, ek["rows"], ev["rows"])])
        _check_out(out, ref, b, h)
    print("flips:", rep)


def test_gqa_decode_full_size_sampled_heads():
    """batch 4, 32 query heads over 8 kv heads, 32768 tokens, bf16, bits 2;
    (b, h_kv) = (0, 0) and (3, 5), all 4 query heads of each."""
    w = workloads.gqa_decode(device=DEV, data_seed=3)
    B, Hkv, T, _ = w["k"].shape
    Hq = w["q"].shape[1]
    G = Hq // Hkv
    gc = tq.Codec(D, w["bits"], M, w["seed"])
    cache = gc.alloc(B, Hkv, T)
    gc.encode_kv(w["k"], w["v"], cache)
    segs = [tq.Segment(cache, T, b, 1, codes_batch=b) for b in range(B)]
    out = torch.empty(B, Hq, D, dtype=w["q"].dtype, device=DEV)
    ws = torch.empty(max(tq.tq_decode_workspace_bytes(segs, B, Hq, Hkv), 16), dtype=torch.uint8, device=DEV)
    tq.tq_decode_attention(segs, w["q"], B, Hq, Hkv, out, ws)
    torch.cuda.synchronize()
    oc = oracle.Codec(D, w["bits"], M, w["seed"])
    rep = {}
    for b, h in ((0, 0), (3, 5)):
        ek = oc.encode(w["k"][b, h].double().cpu().numpy(), h, True)
        ev = oc.encode(w["v"][b, h].double().cpu().numpy(), h, False)
        _check_rows(cache, oc, ek, ev, b, h, T, rep)
        for j in range(h * G, (h + 1) * G):
            ref = oracle.attention(w["q"][b, j].double().cpu().numpy(), [(oc, h, ek["rows"], ev["rows"])])
            _check_out(out, ref, b, j)
    print("flips:", rep)


def test_shared_prefix_full_size_sampled_heads():
    """16 agents; prefix 4096 tokens at bits 2 shared by all, tails of 1024 at
    bits 4; 32 query heads over 8 kv heads, bf16; agents 0 and 11 on kv heads
    2 and 7 (4 query heads each, so 64 queries share every prefix tile)."""
    w = workloads.shared_prefix(device=DEV, data_seed=5)
    A, Hq = w["q"].shape[:2]
    Hkv = w["n_kv_heads"]
    P, Tt = w["prefix_k"].shape[2], w["tail_k"].shape[2]
    G = Hq // Hkv
    pc = tq.Codec(D, w["prefix_bits"], M, w["seed"])
    tc = tq.Codec(D, w["tail_bits"], M, w["seed"])
    pcache = pc.alloc(1, Hkv, P)
    tcache = tc.alloc(A, Hkv, Tt)
    pc.encode_kv(w["prefix_k"], w["prefix_v"], pcache)
    tc.encode_kv(w["tail_k"], w["tail_v"], tcache)
    segs = [tq.Segment(pcache, P, 0, A)] + [tq.Segment(tcache, Tt, a, 1, codes_batch=a) for a in range(A)]
    out = torch.empty(A, Hq, D, dtype=w["q"].dtype, device=DEV)
    ws = torch.empty(max(tq.tq_decode_workspace_bytes(segs, A, Hq, Hkv), 16), dtype=torch.uint8, device=DEV)
    tq.tq_decode_attention(segs, w["q"], A, Hq, Hkv, out, ws)
    torch.cuda.synchronize()
    opc = oracle.Codec(D, w["prefix_bits"], M, w["seed"])
    otc = oracle.Codec(D, w["tail_bits"], M, w["seed"])
    rep = {}
    for h in (2, 7):
        epk = opc.encode(w["prefix_k"][0, h].double().cpu().numpy(), h, True)
        epv = opc.encode(w["prefix_v"][0, h].double().cpu().numpy(), h, False)
        _check_rows(pcache, opc, epk, epv, 0, h, P, rep)
        for a in (0, 11):
            etk = otc.encode(w["tail_k"][a, h].double().cpu().numpy(), h, True)
            etv = otc.encode(w["tail_v"][a, h].double().cpu().numpy(), h, False)
            _check_rows(tcache, otc, etk, etv, a, h, Tt, rep)
            for j in range(h * G, (h + 1) * G):
                ref = oracle.attention(w["q"][a, j].double().cpu().numpy(),
                                       [(opc, h, epk["rows"], epv["rows"]), (otc, h, etk["rows"], etv["rows"])])
                _check_out(out, ref, a, j)
    print("flips:", rep)


def test_bulk_encode_full_size_sampled_layers():
    """32 layers x 8 kv heads x 8192 tokens, bf16; bits 4 on layers 0, 1, 30,
    31 and bits 3 on 2..29, encoded by the same three calls as the bench;
    layer 1 head 3 (bits 4) and layer 17 head 6 (bits 3) against the oracle."""
    w = workloads.bulk_encode(device=DEV, data_seed=4)
    L, H, T, _ = w["k"].shape
    c3 = tq.Codec(D, 3, M, w["seed"])
    c4 = tq.Codec(D, 4, M, w["seed"])
    cache3 = c3.alloc(28, H, T)
    cache4a = c4.alloc(2, H, T)
    cache4b = c4.alloc(2, H, T)
    for codec, cache, sl in ((c4, cache4a, slice(0, 2)), (c3, cache3, slice(2, 30)), (c4, cache4b, slice(30, 32))):
        codec.encode_kv(w["k"][sl], w["v"][sl], cache)
    torch.cuda.synchronize()
    rep = {}
    for layer, h, bits, cache, slot in ((1, 3, 4, cache4a, 1), (17, 6, 3, cache3, 15)):
        oc = oracle.Codec(D, bits, M, w["seed"])
        ek = oc.encode(w["k"][layer, h].double().cpu().numpy(), h, True)
        ev = oc.encode(w["v"][layer, h].double().cpu().numpy(), h, False)
        _check_rows(cache, oc, ek, ev, slot, h, T, rep)
    print("flips:", rep)


def test_mha_split_full_size_sampled_heads():
    """The multi-head data with each head's channels ordered by RMS over its
    keys and split into 64 outlier channels at bits 4 (m 64) and 64 normal
    channels at bits 3 (m 64), encoded and decoded as bench.py does it;
    (b, h) = (2, 9) and (5, 26)."""
    w = workloads.mha_decode(device=DEV, data_seed=2)
    B, H, T, _ = w["k"].shape
    order = w["k"].float().pow(2).mean(dim=(0, 2)).argsort(dim=-1, descending=True)
    idx = order[None, :, None, :]
    k = torch.gather(w["k"], 3, idx.expand_as(w["k"])).contiguous()
    v = torch.gather(w["v"], 3, idx.expand_as(w["v"])).contiguous()
    q = torch.gather(w["q"], 2, order[None].expand_as(w["q"])).contiguous()
    go, gn = tq.Codec(64, 4, 64, w["seed"]), tq.Codec(64, 3, 64, w["seed"] + 1000)
    co, cn = go.alloc(B, H, T), gn.alloc(B, H, T)
    go.encode_kv(k[..., :64], None, co)
    gn.encode_kv(k[..., 64:], None, cn)
    go.encode_kv(None, v[..., :64], co)
    gn.encode_kv(None, v[..., 64:], cn)
    out = tq.decode_split(go, co, gn, cn, T, q)
    torch.cuda.synchronize()
    assert go.status() == (0, 0) and gn.status() == (0, 0)
    oo, on = oracle.Codec(64, 4, 64, w["seed"]), oracle.Codec(64, 3, 64, w["seed"] + 1000)
    rep = {}
    for b, h in ((2, 9), (5, 26)):
        kb, vb = k[b, h].double().cpu().numpy(), v[b, h].double().cpu().numpy()
        eko, evo = oo.encode(kb[:, :64], h, True), oo.encode(vb[:, :64], h, False)
        ekn, evn = on.encode(kb[:, 64:], h, True), on.encode(vb[:, 64:], h, False)
        _check_rows(co, oo, eko, evo, b, h, T, rep)
        _check_rows(cn, on, ekn, evn, b, h, T, rep)
        ref = oracle.attention_split(q[b, h].double().cpu().numpy(), (oo, h, eko["rows"], evo["rows"]),
                                     (on, h, ekn["rows"], evn["rows"]))
        _check_out(out, ref, b, h)
    print("flips:", rep)


def test_mha_append_full_size_sampled_heads():
    """batch 8 x 32 heads, 4096 cached tokens encoded in bulk, then the step
    that appends token 4096 and attends over 4097, as bench.py times it; the
    appended rows and the outputs of (b, h) = (3, 4) and (6, 31)."""
    w = workloads.mha_decode(device=DEV, data_seed=2, n_tokens=4097)
    B, H, T1, _ = w["k"].shape
    T = T1 - 1
    gc = tq.Codec(D, w["bits"], M, w["seed"])
    cache = gc.alloc(B, H, T + 16)
    gc.encode_kv(w["k"][:, :, :T], w["v"][:, :, :T], cache)
    segs = [tq.Segment(cache, T, b, 1, codes_batch=b) for b in range(B)]
    out = tq.decode_append(segs, w["k"][:, :, T], w["v"][:, :, T], w["q"], H)
    torch.cuda.synchronize()
    assert gc.status() == (0, 0)
    oc = oracle.Codec(D, w["bits"], M, w["seed"])
    rep = {}
    for b, h in ((3, 4), (6, 31)):
        ek = oc.encode(w["k"][b, h].double().cpu().numpy(), h, True)
        ev = oc.encode(w["v"][b, h].double().cpu().numpy(), h, False)
        _check_rows(cache, oc, ek, ev, b, h, T1, rep)
        ref = oracle.attention(w["q"][b, h].double().cpu().numpy(), [(oc, h, ek["rows"], ev["rows"])])
        _check_out(out, ref, b, h)
    print("flips:", rep)
