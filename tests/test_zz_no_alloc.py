"""The allocation-free decode entry point (tq_decode_attention_static).

Some callers cannot allocate device memory (a plug-in whose host application
owns every device allocation, a serving loop that must not call cudaMalloc
on the decode path); for them the library keeps its decode scratch in a
fixed array compiled into libtq.so.  This checks, through the C ABI, that
two consecutive calls of that entry point give the same outputs as the
workspace-taking tq_decode_attention.  Both build the same plan and launch
the same kernels on the same data, so the outputs must be identical, bit for
bit (the parity tests hold tq_decode_attention itself to the oracle).  It
lives in its own file, collected last.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("kv_cache_vector_10_b200")


def _case(seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    B, Hq, Hkv, T, d = 3, 8, 2, 700, 128
    k = torch.randn(B, Hkv, T, d, generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn(B, Hkv, T, d, generator=g, device="cuda").to(torch.bfloat16)
    q = torch.randn(B, Hq, d, generator=g, device="cuda").to(torch.bfloat16)
    return k, v, q


def test_static_scratch_decode_matches_workspace_decode():
    codec = tq.Codec(128, 3, 128, 42)
    tq.tq_ensure_heads(codec.ctx, 2)           # building tables allocates; do it up front
    for call, seed in enumerate((11, 12)):     # two calls in a row share the scratch array
        k, v, q = _case(seed)
        cache = codec.alloc(3, 2, 704)
        codec.encode_kv(k, v, cache)
        segs = [tq.Segment(cache, 700, b, 1, codes_batch=b) for b in range(3)]
        ref = tq.decode_attention(segs, q, 2, out_dtype=torch.float32)
        out = torch.full_like(ref, float("nan"))
        tq.tq_decode_attention_static(segs, q, 3, 8, 2, out)
        torch.cuda.synchronize()
        assert torch.isfinite(out).all(), call
        assert torch.equal(out, ref), (call, float((out - ref).abs().max()))


def test_static_scratch_shared_prefix_on_tensor_cores():
    """A prefix shared by 8 sequences (32 queries per kv head: the tensor-core
    decode) plus private tails (the byte tables): the same identity."""
    g = torch.Generator(device="cuda").manual_seed(5)
    A, Hq, Hkv, d = 8, 8, 2, 128
    pc, tc = tq.Codec(d, 2, 128, 42), tq.Codec(d, 4, 128, 42)
    tq.tq_ensure_heads(pc.ctx, Hkv)
    tq.tq_ensure_heads(tc.ctx, Hkv)
    pk = torch.randn(1, Hkv, 500, d, generator=g, device="cuda").to(torch.bfloat16)
    pv = torch.randn(1, Hkv, 500, d, generator=g, device="cuda").to(torch.bfloat16)
    tk = torch.randn(A, Hkv, 60, d, generator=g, device="cuda").to(torch.bfloat16)
    tv = torch.randn(A, Hkv, 60, d, generator=g, device="cuda").to(torch.bfloat16)
    q = torch.randn(A, Hq, d, generator=g, device="cuda").to(torch.bfloat16)
    pcache, tcache = pc.alloc(1, Hkv, 512), tc.alloc(A, Hkv, 64)
    pc.encode_kv(pk, pv, pcache)
    tc.encode_kv(tk, tv, tcache)
    segs = [tq.Segment(pcache, 500, 0, A)] + [tq.Segment(tcache, 60, a, 1, codes_batch=a) for a in range(A)]
    ref = tq.decode_attention(segs, q, Hkv, out_dtype=torch.float32)
    out = torch.full_like(ref, float("nan"))
    tq.tq_decode_attention_static(segs, q, A, Hq, Hkv, out)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    assert torch.equal(out, ref), float((out - ref).abs().max())


def test_static_scratch_rejects_oversized_calls():
    codec = tq.Codec(128, 2, 128, 1)
    cache = codec.alloc(1, 1, 16)
    B = 2048                                   # one shared segment, many sequences
    segs = [tq.Segment(cache, 16, 0, B)]
    q = torch.zeros(B, 64, 128, device="cuda")
    tq.tq_ensure_heads(codec.ctx, 1)
    assert tq.tq_decode_workspace_bytes(segs, B, 64, 1) > (8 << 20)
    with pytest.raises(tq.TQError, match="LIMIT"):
        tq.tq_decode_attention_static(segs, q, B, 64, 1, torch.empty_like(q))
