"""GPU (libtq, sm_100a) versus the CPU oracle on the same seeded inputs.

Codes and QJL signs must be bit-exact except where the oracle's
pre-quantization value lies within 1e-5 of a decision boundary (counted);
dequantized vectors and scores within 1e-4 relative; attention outputs within
2e-3 absolute.  Scores, dequantization and decode are checked on codes the
oracle produced (uploaded to the device) so those comparisons see identical
codes; encode is checked against the oracle's own encode.  Sizes span
several tiles and ragged tails; every call goes through the C ABI.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("kv_cache_vector_10_b200")
from kv_cache_vector_10_b200 import workloads  # noqa: E402

DEV = "cuda"


def _codec_pair(d, bits, m, seed):
    return tq.Codec(d, bits, m, seed), oracle.Codec(d, bits, m, seed)


def _cap(T):
    return max(16, (T + 15) // 16 * 16)


def _encode_and_compare(k, v, d, bits, m, seed, token_offset=0, report=None):
    report = {} if report is None else report
    B, H, T, _ = k.shape
    gc, oc = _codec_pair(d, bits, m, seed)
    cache = gc.alloc(B, H, _cap(T + token_offset))
    gc.encode_kv(k.to(DEV), v.to(DEV), cache, token_offset)
    torch.cuda.synchronize()
    ek = pu.oracle_encode(oc, k, True)
    ev = pu.oracle_encode(oc, v, False)
    kg = cache.k.cpu().numpy()
    vg = cache.v.cpu().numpy()
    for b in range(B):
        for h in range(H):
            pu.compare_k(kg[b, h, token_offset:token_offset + T], ek[b][h], oc, report)
            pu.compare_v(vg[b, h, token_offset:token_offset + T], ev[b][h], oc, report)
    return gc, oc, cache, ek, ev, report


# ------------------------------------------------------------------- encode

def test_encode_single_head_workload():
    w = workloads.single_head(device=DEV)
    rep = {}
    _encode_and_compare(w["k"], w["v"], 128, 3, 128, 42, report=rep)
    print("flips:", rep)
    assert rep["k_rows_flipped"] <= 5


@pytest.mark.parametrize("bits", [2, 3, 4, 5])
@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
def test_encode_bits_dtypes_ragged(bits, dtype):
    g = torch.Generator().manual_seed(bits * 10 + int(dtype.itemsize))
    k = (torch.randn(2, 3, 333, 128, generator=g) * 2).to(dtype)
    v = torch.randn(2, 3, 333, 128, generator=g).to(dtype)
    _encode_and_compare(k, v, 128, bits, 128, 7 + bits)


@pytest.mark.parametrize("d,m", [(64, 64), (64, 256), (128, 32), (128, 256), (128, 96)])
def test_encode_dims_and_projections(d, m):
    g = torch.Generator().manual_seed(d + m)
    k = torch.randn(1, 2, 300, d, generator=g)
    v = torch.randn(1, 2, 300, d, generator=g)
    _encode_and_compare(k, v, d, 3, m, 1234)


def test_encode_strided_input_and_token_offset():
    g = torch.Generator().manual_seed(5)
    base = torch.randn(2, 200, 4, 128, generator=g, dtype=torch.float32).to(torch.bfloat16)   # [B, T, H, d]
    k = base.permute(0, 2, 1, 3)          # [B, H, T, d] view with token stride H*d
    v = (base * 0.5).permute(0, 2, 1, 3)
    gc, oc = _codec_pair(128, 4, 128, 99)
    cache = gc.alloc(2, 4, 512)
    kd = base.to(DEV).permute(0, 2, 1, 3)
    vd = (base * 0.5).to(DEV).permute(0, 2, 1, 3)
    gc.encode_kv(kd, vd, cache, 37)
    torch.cuda.synchronize()
    ek = pu.oracle_encode(oc, k, True)
    ev = pu.oracle_encode(oc, v, False)
    rep = {}
    for b in range(2):
        for h in range(4):
            pu.compare_k(cache.k[b, h, 37:237].cpu().numpy(), ek[b][h], oc, rep)
            pu.compare_v(cache.v[b, h, 37:237].cpu().numpy(), ev[b][h], oc, rep)
    # rows outside [37, 237) untouched
    assert int(cache.k[:, :, :37].abs().sum()) == 0 and int(cache.v[:, :, 237:].abs().sum()) == 0


def test_encode_deterministic():
    w = workloads.single_head(device=DEV, n_tokens=512)
    gc = tq.Codec(128, 3, 128, 42)
    c1, c2 = gc.alloc(1, 1, 512), gc.alloc(1, 1, 512)
    gc.encode_kv(w["k"], w["v"], c1)
    gc.encode_kv(w["k"], w["v"], c2)
    assert torch.equal(c1.k, c2.k) and torch.equal(c1.v, c2.v)


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
def test_encode_nonfinite_and_zero_rows(dtype):
    k = torch.randn(1, 2, 40, 128)
    v = torch.randn(1, 2, 40, 128)
    k[0, 0, 3, 5] = float("nan")
    k[0, 1, 7] = 0.0
    v[0, 1, 9, 0] = float("inf")
    v[0, 0, 11] = 0.0
    gc, oc, cache, ek, ev, rep = _encode_and_compare(k.to(dtype), v.to(dtype), 128, 3, 128, 3)
    n, flags = gc.status()
    assert n == 2 and flags == 0
    kh, vh = gc.dequantize(cache, 40)
    assert float(kh[0, 0, 3].abs().max()) == 0.0 and float(vh[0, 1, 9].abs().max()) == 0.0
    tq.tq_reset_status(gc.ctx)
    assert gc.status() == (0, 0)


@pytest.mark.parametrize("scale", [2.0 ** -18, 2.0 ** -10, 2.0 ** 13])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_encode_16bit_extreme_magnitudes(scale, dtype):
    """16-bit rows go through the tensor-core chunk transforms with the row in
    its own type: binary16 subnormals (2^-18), rows mixing subnormal and
    normal entries (2^-10) and rows near the binary16 maximum (2^13) encode
    like the oracle."""
    g = torch.Generator().manual_seed(int(math.log2(scale)) + 40)
    k = (torch.randn(1, 2, 260, 128, generator=g) * scale).to(dtype)
    v = (torch.randn(1, 2, 260, 128, generator=g) * scale).to(dtype)
    for d in (128, 64):
        gc, *_ , rep = _encode_and_compare(k[..., :d].contiguous(), v[..., :d].contiguous(), d, 4, 64, 21)
        assert gc.status() == (0, 0)
        assert rep.get("k_rows_flipped", 0) <= 3 and rep.get("v_index_flips", 0) <= 3, rep


@pytest.mark.parametrize("bits", [2, 3, 4, 5])
def test_encode_power_of_two_scaling_and_tiny_rows(bits):
    """Scaling fp32 input by 2^40 or 2^-40 scales every fp32 step of the encoder
    exactly, so the codes are identical and the stored norms scale by the same
    power of two.  Rows whose rotated sum of squares d|x|^2 falls below the
    smallest normal float are encoded exactly like zero rows, without being
    counted as non-finite."""
    g = torch.Generator().manual_seed(77 + bits)
    k = torch.randn(1, 2, 150, 128, generator=g)
    v = torch.randn(1, 2, 150, 128, generator=g)
    gc = tq.Codec(128, bits, 128, 5)
    out = []
    for s in (1.0, 2.0 ** 40, 2.0 ** -40, 2.0 ** -75, 0.0):
        c = gc.alloc(1, 2, 160)
        gc.encode_kv((k * s).to(DEV), (v * s).to(DEV), c)
        out.append((c.k[:, :, :150].cpu().numpy(), c.v[:, :, :150].cpu().numpy()))
    torch.cuda.synchronize()
    assert gc.status() == (0, 0)
    base_k, base_v = out[0]
    for (kk, vv), s in zip(out[1:3], (2.0 ** 40, 2.0 ** -40)):
        assert np.array_equal(kk[..., :-8], base_k[..., :-8]) and np.array_equal(vv[..., :-4], base_v[..., :-4])
        kn = kk[..., -8:].copy().view(np.float32)
        vn = vv[..., -4:].copy().view(np.float32)
        assert np.array_equal(kn, (base_k[..., -8:].copy().view(np.float32) * np.float32(s)))
        assert np.array_equal(vn, (base_v[..., -4:].copy().view(np.float32) * np.float32(s)))
    tiny, zero = out[3], out[4]
    assert np.array_equal(tiny[0], zero[0]) and np.array_equal(tiny[1], zero[1])
    assert not zero[0][..., -8:].any() and not zero[1][..., -4:].any()


def test_encode_empty_and_single_token():
    gc = tq.Codec(128, 4, 128, 1)
    cache = gc.alloc(1, 1, 16)
    k = torch.randn(1, 1, 0, 128, device=DEV)
    gc.encode_kv(k, k, cache)
    assert int(cache.k.sum()) == 0
    k1 = torch.randn(1, 1, 1, 128)
    _encode_and_compare(k1, k1 * 3, 128, 4, 128, 1)


# ------------------------------------------------------- scores / dequantize

@pytest.mark.parametrize("bits", [2, 3, 4, 5])
def test_dequantize_matches_oracle(bits):
    g = torch.Generator().manual_seed(bits)
    k = torch.randn(1, 2, 200, 128, generator=g) * 3
    v = torch.randn(1, 2, 200, 128, generator=g)
    gc, oc = _codec_pair(128, bits, 128, 11)
    ek, ev = pu.oracle_encode(oc, k, True), pu.oracle_encode(oc, v, False)
    cache = gc.alloc(1, 2, 208)
    pu.upload_rows(cache.k, ek, 200)
    pu.upload_rows(cache.v, ev, 200)
    kh, vh = gc.dequantize(cache, 200)
    for h in range(2):
        rk = oc.dequant(ek[0][h]["rows"], h, True)
        rv = oc.dequant(ev[0][h]["rows"], h, False)
        assert np.all(np.abs(kh[0, h].cpu().numpy() - rk) <= pu.vec_tolerance(rk))
        assert np.all(np.abs(vh[0, h].cpu().numpy() - rv) <= pu.vec_tolerance(rv))


@pytest.mark.parametrize("bits,d,m", [(2, 128, 128), (3, 128, 128), (4, 128, 128), (5, 128, 64), (3, 64, 64)])
def test_scores_match_oracle(bits, d, m):
    g = torch.Generator().manual_seed(bits + d)
    B, Hkv, Hq, T = 2, 2, 4, 300
    k = torch.randn(B, Hkv, T, d, generator=g)
    q = torch.randn(B, Hq, d, generator=g)
    gc, oc = _codec_pair(d, bits, m, 21)
    ek = pu.oracle_encode(oc, k, True)
    cache = gc.alloc(B, Hkv, _cap(T))
    pu.upload_rows(cache.k, ek, T)
    s = gc.attention_scores(cache, q.to(DEV), T).cpu().numpy()
    for b in range(B):
        for j in range(Hq):
            h = j // (Hq // Hkv)
            ref = oc.scores(q[b, j].double().numpy(), ek[b][h]["rows"], h)
            kh = oc.dequant(ek[b][h]["rows"], h, True)
            tol = pu.scores_tolerance(ref, q[b, j].double().numpy(), kh)
            assert np.all(np.abs(s[b, j] - ref) <= tol), float(np.max(np.abs(s[b, j] - ref) / tol))


def test_single_head_scores_workload():
    """The single-head workload: 4 queries scored against 1024 keys."""
    w = workloads.single_head(device=DEV)
    gc, oc = _codec_pair(128, 3, 128, 42)
    ek = pu.oracle_encode(oc, w["k"], True)
    cache = gc.alloc(1, 1, 1024)
    pu.upload_rows(cache.k, ek, 1024)
    s = gc.attention_scores(cache, w["q"], 1024).cpu().numpy()
    kh = oc.dequant(ek[0][0]["rows"], 0, True)
    for j in range(4):
        qq = w["q"][0, j].double().cpu().numpy()
        ref = oc.scores(qq, ek[0][0]["rows"], 0)
        assert np.all(np.abs(s[0, j] - ref) <= pu.scores_tolerance(ref, qq, kh))


# ------------------------------------------------------------------- decode

def _oracle_attention_out(q, seg_specs, b, j, G):
    """seg_specs: list of (oracle codec, encK, encV, codes_batch, first_seq, n_seqs, T)."""
    h = j // G
    segs = []
    for oc, ek, ev, cb, fs, ns, T in seg_specs:
        if fs <= b < fs + ns:
            segs.append((oc, h, ek[cb][h]["rows"][:T], ev[cb][h]["rows"][:T]))
    return oracle.attention(q[b, j].double().cpu().numpy(), segs)


def _run_decode_case(specs, q, Hkv, out_dtype=torch.float32):
    """specs: list of dict(codec_bits, k [Bc,H,T,d], v, first_seq, n_seqs, codes_batch)."""
    B, Hq, d = q.shape
    G = Hq // Hkv
    gsegs, osegs, keep = [], [], []
    for sp in specs:
        gc, oc = _codec_pair(d, sp["bits"], 128, sp.get("seed", 42))
        kk, vv = sp["k"], sp["v"]
        Bc, H, T, _ = kk.shape
        ek, ev = pu.oracle_encode(oc, kk, True), pu.oracle_encode(oc, vv, False)
        cache = gc.alloc(Bc, H, _cap(T))
        pu.upload_rows(cache.k, ek, T)
        pu.upload_rows(cache.v, ev, T)
        keep += [gc, cache]
        for cb in range(Bc):
            fs, ns = sp["first_seq"] + cb * sp.get("stride", 0), sp["n_seqs"]
            gsegs.append(tq.Segment(cache, T, fs, ns, codes_batch=cb))
            osegs.append((oc, ek, ev, cb, fs, ns, T))
    out = tq.decode_attention(gsegs, q.to(DEV), Hkv, out_dtype=out_dtype).float().cpu().numpy()
    worst = 0.0           # largest error as a multiple of the tolerance (ATTN_ABS for float32)
    for b in range(B):
        for j in range(Hq):
            ref = _oracle_attention_out(q, osegs, b, j, G)
            ratio = np.max(np.abs(out[b, j] - ref) / pu.attn_tolerance(ref, out_dtype))
            worst = max(worst, ratio * pu.ATTN_ABS)
    return worst


def test_decode_single_head_workload():
    w = workloads.single_head(device="cpu")
    worst = _run_decode_case([dict(bits=3, k=w["k"], v=w["v"], first_seq=0, n_seqs=1)], w["q"], 1)
    assert worst <= pu.ATTN_ABS, worst


@pytest.mark.parametrize("Hq,Hkv,bits,T", [(4, 4, 4, 1000), (8, 4, 3, 777), (8, 2, 2, 700), (6, 2, 5, 300),
                                          (4, 1, 3, 1)])
def test_decode_mha_gqa(Hq, Hkv, bits, T):
    g = torch.Generator().manual_seed(Hq * 100 + T)
    B = 3
    k = torch.randn(B, Hkv, T, 128, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, T, 128, generator=g).to(torch.bfloat16)
    q = torch.randn(B, Hq, 128, generator=g).to(torch.bfloat16)
    worst = _run_decode_case([dict(bits=bits, k=k, v=v, first_seq=0, n_seqs=1, stride=1)], q, Hkv)
    assert worst <= pu.ATTN_ABS, worst


def test_decode_shared_prefix_and_tails():
    """A prefix at bits 2 shared by 3 sequences plus private tails at bits 4."""
    g = torch.Generator().manual_seed(77)
    A, Hq, Hkv = 3, 8, 2
    pk = torch.randn(1, Hkv, 300, 128, generator=g).to(torch.bfloat16)
    pv = torch.randn(1, Hkv, 300, 128, generator=g).to(torch.bfloat16)
    tk = torch.randn(A, Hkv, 100, 128, generator=g).to(torch.bfloat16)
    tv = torch.randn(A, Hkv, 100, 128, generator=g).to(torch.bfloat16)
    q = torch.randn(A, Hq, 128, generator=g).to(torch.bfloat16)
    worst = _run_decode_case([dict(bits=2, k=pk, v=pv, first_seq=0, n_seqs=A),
                              dict(bits=4, k=tk, v=tv, first_seq=0, n_seqs=1, stride=1)], q, Hkv)
    assert worst <= pu.ATTN_ABS, worst


def test_decode_bf16_output_and_empty_segment():
    g = torch.Generator().manual_seed(3)
    k = torch.randn(2, 2, 90, 128, generator=g)
    v = torch.randn(2, 2, 90, 128, generator=g)
    q = torch.randn(2, 4, 128, generator=g)
    worst = _run_decode_case([dict(bits=3, k=k, v=v, first_seq=0, n_seqs=1, stride=1)], q, 2,
                             out_dtype=torch.bfloat16)
    assert worst <= pu.ATTN_ABS, worst


def test_decode_end_to_end_from_gpu_encode():
    """GPU encode -> GPU decode against oracle encode -> oracle attention."""
    w = workloads.gqa_decode(device=DEV, batch=2, n_tokens=1500)
    Hkv, Hq = 8, 32
    gc, oc = _codec_pair(128, 2, 128, 42)
    cache = gc.alloc(2, Hkv, 1504)
    gc.encode_kv(w["k"], w["v"], cache)
    segs = [tq.Segment(cache, 1500, b, 1, codes_batch=b) for b in range(2)]
    out = tq.decode_attention(segs, w["q"], Hkv, out_dtype=torch.float32).cpu().numpy()
    for b in range(2):
        for j in (0, 5, 31):
            h = j // 4
            ek = oc.encode(w["k"][b, h].double().cpu().numpy(), h, True)
            ev = oc.encode(w["v"][b, h].double().cpu().numpy(), h, False)
            ref = oracle.attention(w["q"][b, j].double().cpu().numpy(), [(oc, h, ek["rows"], ev["rows"])])
            assert np.max(np.abs(out[b, j] - ref)) <= pu.ATTN_ABS


# ------------------------------------------------------------------ errors

def test_argument_errors():
    gc = tq.Codec(128, 3, 128, 1)
    cache = gc.alloc(1, 2, 32)
    k = torch.randn(1, 2, 40, 128, device=DEV)
    with pytest.raises(tq.TQError, match="DIM_MISMATCH"):
        gc.encode_kv(k, k, cache)                 # beyond capacity
    with pytest.raises(tq.TQError, match="DIM_MISMATCH"):
        gc.encode_kv(k[:, :, :10], k[:, :, :10], cache, token_offset=25)
    mis = torch.randn(2 * 40 * 128 + 1, device=DEV)[1:].view(1, 2, 40, 128)   # 4-byte aligned only
    with pytest.raises(tq.TQError, match="ALIGN"):
        tq.tq_encode_kv(gc.ctx, mis, None, 1, 2, 10, cache)
    seg = [tq.Segment(cache, 16, 0, 1)]
    q = torch.randn(2, 4, 128, device=DEV)
    with pytest.raises(tq.TQError, match="DIM_MISMATCH"):
        tq.decode_attention(seg, q, 2)            # sequence 1 not covered
    ws = torch.empty(16, dtype=torch.uint8, device=DEV)
    with pytest.raises(tq.TQError, match="WORKSPACE"):
        tq.tq_decode_attention(seg, q[:1], 1, 4, 2, torch.empty(1, 4, 128, device=DEV), ws)


@pytest.mark.parametrize("rotation,out_dtype", [("hadamard", torch.float32), ("haar", torch.bfloat16),
                                                ("hadamard", torch.float16)])
def test_decode_direct_output_equals_combined(rotation, out_dtype):
    """When every sequence has one segment and the plan does not split it, the
    decode kernel writes the output itself (one launch fewer); adding an
    empty segment per sequence forces the combine step, which must give the
    same values (for one split it is the same o / l)."""
    g = torch.Generator().manual_seed(17)
    B, H, Hq, T, d = 8, 32, 32, 700, 128       # 256 (sequence, kv head) items: one split each
    k = torch.randn(B, H, T, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, H, T, d, generator=g).to(torch.bfloat16)
    q = torch.randn(B, Hq, d, generator=g).to(torch.bfloat16)
    gc = tq.Codec(d, 4, 128, 5, rotation=rotation)
    cache = gc.alloc(B, H, 704)
    gc.encode_kv(k.to(DEV), v.to(DEV), cache)
    segs = [tq.Segment(cache, T, b, 1, codes_batch=b) for b in range(B)]
    with_empty = segs + [tq.Segment(cache, 0, b, 1, codes_batch=b) for b in range(B)]
    assert tq.tq_decode_launch_count(segs, B, Hq, H) == 2              # query prep + decode
    assert tq.tq_decode_launch_count(with_empty, B, Hq, H) == 3        # + combine
    out1 = tq.decode_attention(segs, q.to(DEV), H, out_dtype=out_dtype)
    out2 = tq.decode_attention(with_empty, q.to(DEV), H, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2)
    # and against the oracle on a few (sequence, head) pairs
    oc = oracle.Codec(d, 4, 128, 5, rotation=rotation)
    for b, j in ((0, 0), (5, 17), (7, 31)):
        ek = oc.encode(k[b, j].double().numpy(), j, True)
        ev = oc.encode(v[b, j].double().numpy(), j, False)
        ref = oracle.attention(q[b, j].double().numpy(), [(oc, j, ek["rows"], ev["rows"])])
        assert np.all(np.abs(out1[b, j].float().cpu().numpy() - ref) <= pu.attn_tolerance(ref, out_dtype))
