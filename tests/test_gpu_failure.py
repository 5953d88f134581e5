"""Failure detection on the GPU without a fault: a bounded wait made to run
out on purpose (an mbarrier phase that nothing completes) is reported in the
context's status word; while the flag is set the context's key-encode and
decode kernels skip their work; clearing it makes the context usable again,
with results identical to a fresh context's."""
import pytest
import torch

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("kv_cache_vector_10_b200")

DEV = "cuda"


def test_bounded_wait_timeout_is_reported_and_cleared():
    g = torch.Generator().manual_seed(1)
    x = torch.randn(1, 2, 300, 128, generator=g).to(DEV)
    q = torch.randn(1, 4, 128, generator=g).to(DEV)
    gc = tq.Codec(128, 3, 128, 5)
    ref = tq.Codec(128, 3, 128, 5)
    c_ref = ref.alloc(1, 2, 304)
    ref.encode_kv(x, x, c_ref)
    out_ref = tq.decode_attention([tq.Segment(c_ref, 300, 0, 1)], q, 2, out_dtype=torch.float32)

    tq.tq_selftest_wait_timeout(gc.ctx, 2000)           # 2 ms bound, nothing arrives
    n, flags = gc.status()
    assert n == 0 and flags & 1
    cache = gc.alloc(1, 2, 304)
    gc.encode_kv(x, x, cache)                            # skipped: keys stay untouched
    torch.cuda.synchronize()
    assert int(cache.k.abs().sum()) == 0
    assert gc.status()[1] & 1                            # the flag stays until cleared

    tq.tq_reset_status(gc.ctx)
    assert gc.status() == (0, 0)
    gc.encode_kv(x, x, cache)
    out = tq.decode_attention([tq.Segment(cache, 300, 0, 1)], q, 2, out_dtype=torch.float32)
    assert gc.status() == (0, 0)
    assert torch.equal(cache.k, c_ref.k) and torch.equal(cache.v, c_ref.v)
    assert torch.equal(out, out_ref)


def test_selftest_rejects_bad_timeouts():
    gc = tq.Codec(128, 3, 128, 5)
    for bad in (0, 100001):
        with pytest.raises(tq.TQError, match="TQ_ERR_LIMIT"):
            tq.tq_selftest_wait_timeout(gc.ctx, bad)
