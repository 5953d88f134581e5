"""Decode steps captured in a CUDA graph and replayed: the split-K decode
(including its dependent launches and, for several segments, the combine
step; the shared prefix goes to the tensor-core decode) and the append step
replay to the same bytes as eager calls on the same inputs, also after the
query is updated in place."""
import pytest
import torch

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("kv_cache_vector_10_b200")

DEV = "cuda"


def _cache(B, H, T, bits, seed, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    codec = tq.Codec(128, bits, 128, seed)
    cache = codec.alloc(B, H, (T + 15) // 16 * 16)
    codec.encode_kv(torch.randn(B, H, T, 128, generator=g).to(dtype).to(DEV),
                    torch.randn(B, H, T, 128, generator=g).to(dtype).to(DEV), cache)
    return codec, cache


@pytest.mark.parametrize("shared", [False, True])
def test_decode_graph_replay_matches_eager(shared):
    B, H, Hq, T = 4, 8, 32, 1500
    codec, cache = _cache(B, H, T, 3, 5)
    segs = [tq.Segment(cache, T, b, 1, codes_batch=b) for b in range(B)]
    if shared:   # a shared prefix at another bit width: two decode launches and the combine
        _, pre = _cache(1, H, 700, 2, 6)
        segs = [tq.Segment(pre, 700, 0, B)] + segs
    g = torch.Generator().manual_seed(7)
    q_static = torch.randn(B, Hq, 128, generator=g).to(torch.bfloat16).to(DEV)
    ws = torch.empty(max(tq.tq_decode_workspace_bytes(segs, B, Hq, H), 16), dtype=torch.uint8, device=DEV)
    out_static = torch.empty(B, Hq, 128, dtype=torch.float32, device=DEV)
    # eager once (also builds every head table before capture)
    tq.tq_decode_attention(segs, q_static, B, Hq, H, out_static, ws)
    torch.cuda.synchronize()
    ref1 = out_static.clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            tq.tq_decode_attention(segs, q_static, B, Hq, H, out_static, ws)
    torch.cuda.current_stream().wait_stream(s)
    out_static.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out_static, ref1)
    # new query in place: the replay must use it
    q_static.copy_(torch.randn(B, Hq, 128, generator=g).to(torch.bfloat16))
    graph.replay()
    torch.cuda.synchronize()
    got = out_static.clone()
    tq.tq_decode_attention(segs, q_static, B, Hq, H, out_static, ws)
    torch.cuda.synchronize()
    assert torch.equal(got, out_static) and not torch.equal(got, ref1)


def test_append_graph_replay_appends_like_eager():
    """A captured append step writes the new rows and attends like the eager
    call (the graph replays with the segment lengths it was captured with)."""
    B, H, Hq, T = 2, 4, 8, 300
    codec, cache = _cache(B, H, T, 4, 11, torch.float16)
    codec2, cache2 = _cache(B, H, T, 4, 11, torch.float16)     # identical twin for the eager run
    g = torch.Generator().manual_seed(3)
    kn = torch.randn(B, H, 128, generator=g).to(torch.float16).to(DEV)
    vn = torch.randn(B, H, 128, generator=g).to(torch.float16).to(DEV)
    q = torch.randn(B, Hq, 128, generator=g).to(torch.float16).to(DEV)
    segs = [tq.Segment(cache, T, b, 1, codes_batch=b) for b in range(B)]
    segs2 = [tq.Segment(cache2, T, b, 1, codes_batch=b) for b in range(B)]
    ws = torch.empty(tq.tq_decode_append_workspace_bytes(segs, B, Hq, H), dtype=torch.uint8, device=DEV)
    out = torch.empty(B, Hq, 128, dtype=torch.float32, device=DEV)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            tq.tq_decode_append(segs, kn, vn, q, B, Hq, H, out, ws)
    torch.cuda.current_stream().wait_stream(s)
    graph.replay()
    torch.cuda.synchronize()
    ref = tq.decode_append(segs2, kn, vn, q, H, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    assert torch.equal(cache.k[:, :, :T + 1], cache2.k[:, :, :T + 1])
    assert torch.equal(cache.v[:, :, :T + 1], cache2.v[:, :, :T + 1])
