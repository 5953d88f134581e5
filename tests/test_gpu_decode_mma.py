"""Tensor-core decode (tq_decode_mma_kernel): segments whose staged code tiles
serve many queries (a prefix shared by many sequences, wide query-head
groups) are scored and summed on the tensor cores.

Each case uploads the oracle's own codes, so no encode decision differs, and
compares the GPU output with the oracle's attention over those codes, within
the 2e-3 output tolerance (plus half an ulp of a 16-bit output type).  Cases
run on the path the planner picks (16 or more queries per kv head go to the
tensor cores), or are forced onto it (TQ_DECODE_PATH=mma) or off it
(TQ_DECODE_PATH=lut).
"""
import numpy as np
import pytest
import torch

import oracle
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("kv_cache_vector_10_b200")

DEV = "cuda"


def _cap(T):
    return max(16, (T + 15) // 16 * 16)


def _set_path(monkeypatch, path):
    if path is None:
        monkeypatch.delenv("TQ_DECODE_PATH", raising=False)
    else:
        monkeypatch.setenv("TQ_DECODE_PATH", path)


def _build(specs, d, m, norms="f32", rotation="hadamard"):
    """specs: dict(bits, k [Bc, H, T, d], v, first_seq, n_seqs, stride).
    Returns the GPU segments (with what keeps their buffers alive) and the
    oracle's view of them."""
    gsegs, osegs, keep = [], [], []
    for sp in specs:
        seed = sp.get("seed", 42)
        gc = tq.Codec(d, sp["bits"], m, seed, rotation=rotation, norms=norms)
        oc = oracle.Codec(d, sp["bits"], m, seed, rotation=rotation, norms=norms)
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
    return gsegs, osegs, keep


def _oracle_out(q, osegs, b, j, G):
    h = j // G
    segs = [(oc, h, ek[cb][h]["rows"][:T], ev[cb][h]["rows"][:T])
            for oc, ek, ev, cb, fs, ns, T in osegs if fs <= b < fs + ns]
    return oracle.attention(q[b, j].double().cpu().numpy(), segs)


def _check(out, q, osegs, Hkv, out_dtype, pairs=None):
    """Largest error over the checked (sequence, query head) pairs, as a
    multiple of the tolerance."""
    B, Hq, _ = q.shape
    G = Hq // Hkv
    o = out.float().cpu().numpy()
    worst = 0.0
    for b, j in (pairs if pairs is not None else [(b, j) for b in range(B) for j in range(Hq)]):
        ref = _oracle_out(q, osegs, b, j, G)
        worst = max(worst, float(np.max(np.abs(o[b, j] - ref) / pu.attn_tolerance(ref, out_dtype))))
    return worst


def _decode(gsegs, q, Hkv, out_dtype=torch.float32):
    return tq.decode_attention(gsegs, q.to(DEV), Hkv, out_dtype=out_dtype)


def _rand(g, shape, dtype=torch.bfloat16, scale=1.0):
    return (torch.randn(*shape, generator=g) * scale).to(dtype)


def test_shared_prefix_many_sequences(monkeypatch):
    """16 sequences share a 1000-token prefix at bits 2 (64 queries per kv
    head: the tensor cores) and own 100-token tails at bits 4 (4 queries: the
    lookup tables).  The same step forced onto the lookup tables agrees with
    the oracle too, and differs from the tensor-core output in its rounding,
    which shows the two paths ran."""
    g = torch.Generator().manual_seed(101)
    A, Hq, Hkv, d = 16, 8, 2, 128
    specs = [dict(bits=2, k=_rand(g, (1, Hkv, 1000, d)), v=_rand(g, (1, Hkv, 1000, d)), first_seq=0, n_seqs=A),
             dict(bits=4, k=_rand(g, (A, Hkv, 100, d)), v=_rand(g, (A, Hkv, 100, d)), first_seq=0, n_seqs=1,
                  stride=1)]
    q = _rand(g, (A, Hq, d))
    gsegs, osegs, keep = _build(specs, d, 128)
    _set_path(monkeypatch, None)
    out_mma = _decode(gsegs, q, Hkv)
    _set_path(monkeypatch, "lut")
    out_lut = _decode(gsegs, q, Hkv)
    torch.cuda.synchronize()
    assert _check(out_mma, q, osegs, Hkv, torch.float32) <= 1.0
    assert _check(out_lut, q, osegs, Hkv, torch.float32) <= 1.0
    assert not torch.equal(out_mma, out_lut)
    assert float((out_mma - out_lut).abs().max()) <= 2 * pu.ATTN_ABS


@pytest.mark.parametrize("bits", [2, 3, 4, 5])
@pytest.mark.parametrize("d,m", [(128, 128), (128, 64), (64, 128), (64, 64)])
def test_bits_and_dims(monkeypatch, bits, d, m):
    """A 333-token prefix shared by 5 sequences (20 queries per kv head) plus
    37-token tails, every bit width, head_dim and projection count the
    tensor-core decode takes."""
    g = torch.Generator().manual_seed(bits * 1000 + d + m)
    A, Hq, Hkv = 5, 8, 2
    specs = [dict(bits=bits, k=_rand(g, (1, Hkv, 333, d)), v=_rand(g, (1, Hkv, 333, d)), first_seq=0, n_seqs=A),
             dict(bits=bits, k=_rand(g, (A, Hkv, 37, d)), v=_rand(g, (A, Hkv, 37, d)), first_seq=0, n_seqs=1,
                  stride=1, seed=7)]
    q = _rand(g, (A, Hq, d))
    gsegs, osegs, keep = _build(specs, d, m)
    _set_path(monkeypatch, None)
    out = _decode(gsegs, q, Hkv)
    assert _check(out, q, osegs, Hkv, torch.float32) <= 1.0


def test_more_than_128_queries(monkeypatch):
    """40 sequences x 4 query heads = 160 queries per kv head: two query
    blocks per tile."""
    g = torch.Generator().manual_seed(5)
    A, Hq, Hkv, d = 40, 8, 2, 128
    specs = [dict(bits=3, k=_rand(g, (1, Hkv, 200, d)), v=_rand(g, (1, Hkv, 200, d)), first_seq=0, n_seqs=A),
             dict(bits=3, k=_rand(g, (A, Hkv, 20, d)), v=_rand(g, (A, Hkv, 20, d)), first_seq=0, n_seqs=1,
                  stride=1, seed=3)]
    q = _rand(g, (A, Hq, d))
    gsegs, osegs, keep = _build(specs, d, 128)
    _set_path(monkeypatch, None)
    out = _decode(gsegs, q, Hkv)
    pairs = [(b, j) for b in (0, 17, 31, 39) for j in range(Hq)]
    assert _check(out, q, osegs, Hkv, torch.float32, pairs) <= 1.0


@pytest.mark.parametrize("T", [1, 16, 63, 64, 65, 130, 1000])
def test_token_counts_forced(monkeypatch, T):
    """Single private segments forced onto the tensor cores: one token, a
    partial tile, exact tiles, a ragged last tile, several splits."""
    g = torch.Generator().manual_seed(T)
    B, Hq, Hkv, d = 2, 8, 2, 128
    specs = [dict(bits=4, k=_rand(g, (B, Hkv, T, d), torch.float16), v=_rand(g, (B, Hkv, T, d), torch.float16),
                  first_seq=0, n_seqs=1, stride=1)]
    q = _rand(g, (B, Hq, d), torch.float16)
    gsegs, osegs, keep = _build(specs, d, 128)
    _set_path(monkeypatch, "mma")
    out = _decode(gsegs, q, Hkv, torch.float16)
    assert _check(out, q, osegs, Hkv, torch.float16) <= 1.0


def test_direct_output_wide_group(monkeypatch):
    """One sequence, 32 query heads over one kv head, 50 tokens: one unsplit
    segment, so the kernel writes the bf16 output itself."""
    g = torch.Generator().manual_seed(50)
    B, Hq, Hkv, d = 1, 32, 1, 128
    specs = [dict(bits=3, k=_rand(g, (B, Hkv, 50, d)), v=_rand(g, (B, Hkv, 50, d)), first_seq=0, n_seqs=1,
                  stride=1)]
    q = _rand(g, (B, Hq, d))
    gsegs, osegs, keep = _build(specs, d, 128)
    _set_path(monkeypatch, None)
    assert tq.tq_decode_launch_count(gsegs, B, Hq, Hkv) == 2   # query preparation + decode
    out = _decode(gsegs, q, Hkv, torch.bfloat16)
    assert _check(out, q, osegs, Hkv, torch.bfloat16) <= 1.0


def test_binary16_norms(monkeypatch):
    g = torch.Generator().manual_seed(16)
    A, Hq, Hkv, d = 8, 8, 2, 128
    specs = [dict(bits=4, k=_rand(g, (1, Hkv, 400, d)), v=_rand(g, (1, Hkv, 400, d)), first_seq=0, n_seqs=A)]
    q = _rand(g, (A, Hq, d))
    gsegs, osegs, keep = _build(specs, d, 128, norms="f16")
    _set_path(monkeypatch, None)
    out = _decode(gsegs, q, Hkv)
    assert _check(out, q, osegs, Hkv, torch.float32) <= 1.0


def test_rescaled_running_max(monkeypatch):
    """Key norms that grow along the prefix and large queries: the scores'
    maximum rises tile after tile by far more than the rescale threshold, so
    the running maximum and the TMEM output are rescaled many times."""
    g = torch.Generator().manual_seed(8)
    A, Hq, Hkv, d, T = 8, 8, 2, 128, 700
    ramp = torch.linspace(0.2, 3.0, T).view(1, 1, T, 1)
    k = (torch.randn(1, Hkv, T, d, generator=g) * ramp).to(torch.bfloat16)
    v = _rand(g, (1, Hkv, T, d))
    q = _rand(g, (A, Hq, d), scale=6.0)
    specs = [dict(bits=4, k=k, v=v, first_seq=0, n_seqs=A)]
    gsegs, osegs, keep = _build(specs, d, 128)
    _set_path(monkeypatch, None)
    out = _decode(gsegs, q, Hkv)
    assert _check(out, q, osegs, Hkv, torch.float32) <= 1.0


def test_haar_rotation_stays_on_tables(monkeypatch):
    """The Haar rotation's output rotation is dense; its many-query segments
    use the lookup-table decode, with the same results."""
    g = torch.Generator().manual_seed(12)
    A, Hq, Hkv, d = 8, 8, 2, 128
    specs = [dict(bits=3, k=_rand(g, (1, Hkv, 300, d)), v=_rand(g, (1, Hkv, 300, d)), first_seq=0, n_seqs=A)]
    q = _rand(g, (A, Hq, d))
    gsegs, osegs, keep = _build(specs, d, 128, rotation="haar")
    _set_path(monkeypatch, None)
    out = _decode(gsegs, q, Hkv)
    assert _check(out, q, osegs, Hkv, torch.float32) <= 1.0


def test_append_wide_group(monkeypatch):
    """An append step on private tails with 16 query heads per kv head (the
    tensor-core decode waits for the new rows before reading any)."""
    g = torch.Generator().manual_seed(21)
    B, Hq, Hkv, d, T, bits = 2, 32, 2, 128, 150, 3
    k = _rand(g, (B, Hkv, T + 1, d))
    v = _rand(g, (B, Hkv, T + 1, d))
    q = _rand(g, (B, Hq, d))
    gc, oc = tq.Codec(d, bits, 128, 11), oracle.Codec(d, bits, 128, 11)
    cache = gc.alloc(B, Hkv, _cap(T + 1))
    gc.encode_kv(k[:, :, :T].to(DEV), v[:, :, :T].to(DEV), cache)
    segs = [tq.Segment(cache, T, b, 1, codes_batch=b) for b in range(B)]
    _set_path(monkeypatch, None)
    out = tq.decode_append(segs, k[:, :, T].to(DEV), v[:, :, T].to(DEV), q.to(DEV), Hkv,
                           out_dtype=torch.float32).cpu().numpy()
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hkv):
            ek = oc.encode(k[b, h].double().numpy(), h, True)
            ev = oc.encode(v[b, h].double().numpy(), h, False)
            for j in range(h * G, (h + 1) * G):
                ref = oracle.attention(q[b, j].double().numpy(), [(oc, h, ek["rows"], ev["rows"])])
                assert np.max(np.abs(out[b, j] - ref)) <= pu.ATTN_ABS


def test_two_prefixes_different_bits(monkeypatch):
    """Two prefixes shared by 12 sequences at bits 2 and 3 (two tensor-core
    launches) plus private tails at bits 4 (the byte tables): every output
    merges three segments."""
    g = torch.Generator().manual_seed(33)
    A, Hq, Hkv, d = 12, 8, 2, 128
    specs = [dict(bits=2, k=_rand(g, (1, Hkv, 300, d)), v=_rand(g, (1, Hkv, 300, d)), first_seq=0, n_seqs=A),
             dict(bits=3, k=_rand(g, (1, Hkv, 200, d)), v=_rand(g, (1, Hkv, 200, d)), first_seq=0, n_seqs=A, seed=9),
             dict(bits=4, k=_rand(g, (A, Hkv, 40, d)), v=_rand(g, (A, Hkv, 40, d)), first_seq=0, n_seqs=1,
                  stride=1, seed=5)]
    q = _rand(g, (A, Hq, d))
    gsegs, osegs, keep = _build(specs, d, 128)
    _set_path(monkeypatch, None)
    # query preparation, tails, two tensor-core launches, combine
    assert tq.tq_decode_launch_count(gsegs, A, Hq, Hkv) == 5
    out = _decode(gsegs, q, Hkv)
    pairs = [(b, j) for b in (0, 5, 11) for j in range(Hq)]
    assert _check(out, q, osegs, Hkv, torch.float32, pairs) <= 1.0


def test_two_prefixes_same_bits_one_launch(monkeypatch):
    """Two prefixes at bits 3 from codecs with different seeds, each shared
    by a different half of the batch: one tensor-core launch covers both,
    each CTA with its own segment's rotation signs, codebooks and S."""
    g = torch.Generator().manual_seed(34)
    B, Hq, Hkv, d = 16, 8, 2, 128
    specs = [dict(bits=3, k=_rand(g, (1, Hkv, 250, d)), v=_rand(g, (1, Hkv, 250, d)), first_seq=0, n_seqs=8, seed=1),
             dict(bits=3, k=_rand(g, (1, Hkv, 180, d)), v=_rand(g, (1, Hkv, 180, d)), first_seq=8, n_seqs=8, seed=2)]
    q = _rand(g, (B, Hq, d))
    gsegs, osegs, keep = _build(specs, d, 128)
    _set_path(monkeypatch, None)
    assert tq.tq_decode_launch_count(gsegs, B, Hq, Hkv) == 3   # query preparation, one decode, combine
    out = _decode(gsegs, q, Hkv)
    pairs = [(b, j) for b in (0, 7, 8, 15) for j in range(Hq)]
    assert _check(out, q, osegs, Hkv, torch.float32, pairs) <= 1.0


@pytest.mark.parametrize("d,m", [(256, 128), (128, 192)])
def test_many_queries_outside_the_tensor_core_shapes(monkeypatch, d, m):
    """head_dim 256 or 192 projections with 20 queries per kv head: the
    planner keeps these segments on the byte tables, same results."""
    g = torch.Generator().manual_seed(d + m)
    A, Hq, Hkv = 5, 8, 2
    specs = [dict(bits=3, k=_rand(g, (1, Hkv, 150, d)), v=_rand(g, (1, Hkv, 150, d)), first_seq=0, n_seqs=A)]
    q = _rand(g, (A, Hq, d))
    gsegs, osegs, keep = _build(specs, d, m)
    _set_path(monkeypatch, None)
    out = _decode(gsegs, q, Hkv)
    assert _check(out, q, osegs, Hkv, torch.float32) <= 1.0
