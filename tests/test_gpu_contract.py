"""API-contract tests in the shape of bitpolar's kv_cache.rs unit tests
(bitpolar 0.3.3 src/kv_cache.rs, mod tests): push/len, score count equals
cache length, decoded value shape, positive compression ratio, clear,
multi-head push and score shape.  The page's config is head_dim 8, bits 4,
projections 16, seed 42; the GPU path supports head_dim 64/128 and
projections multiples of 32, so these use head_dim 64, projections 32."""
import pytest
import torch

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("kv_cache_vector_10_b200")


def _cache(heads=1):
    return tq.KvCache(heads, 64, 4, 32, 42, capacity=64)


def test_push_and_len():
    c = _cache()
    assert c.is_empty()
    c.push(torch.full((1, 64), 0.1, device="cuda"), torch.full((1, 64), 0.2, device="cuda"))
    assert len(c) == 1


def test_attention_scores_shape():
    c = _cache()
    for _ in range(5):
        c.push(torch.full((1, 64), 0.1, device="cuda"), torch.full((1, 64), 0.2, device="cuda"))
    s = c.attention_scores(torch.full((1, 64), 0.1, device="cuda"))
    assert s.shape == (1, 5)


def test_decode_values_shape():
    c = _cache()
    c.push(torch.full((1, 64), 0.1, device="cuda"), torch.full((1, 64), 0.2, device="cuda"))
    v = c.decode_values()
    assert v.shape == (1, 1, 64)


def test_compression_ratio_positive():
    c = _cache()
    c.push(torch.full((1, 64), 0.5, device="cuda"), torch.full((1, 64), 0.3, device="cuda"))
    assert c.compression_ratio() > 0.0


def test_clear():
    c = _cache()
    c.push(torch.full((1, 64), 0.1, device="cuda"), torch.full((1, 64), 0.2, device="cuda"))
    c.clear()
    assert c.is_empty()


def test_multi_head_push_and_len_and_scores_shape():
    c = _cache(4)
    c.push(torch.full((4, 64), 0.1, device="cuda"), torch.full((4, 64), 0.2, device="cuda"))
    assert len(c) == 1
    c2 = _cache(2)
    c2.push(torch.full((2, 64), 0.1, device="cuda"), torch.full((2, 64), 0.2, device="cuda"))
    s = c2.attention_scores(torch.full((2, 64), 0.1, device="cuda"))
    assert s.shape == (2, 1)


def test_contract_errors():
    with pytest.raises(tq.TQError, match="EMPTY"):
        tq.KvCache(0, 64, 4, 32, 42)
    c = _cache(2)
    with pytest.raises(tq.TQError, match="DIM_MISMATCH"):
        c.push(torch.zeros(3, 64, device="cuda"), torch.zeros(3, 64, device="cuda"))
    with pytest.raises(tq.TQError, match="ZERO_DIM"):
        tq.KvCache(1, 0, 4, 32, 42)
    with pytest.raises(tq.TQError, match="BITS"):
        tq.KvCache(1, 64, 9, 32, 42)
    with pytest.raises(tq.TQError, match="ZERO_PROJ"):
        tq.KvCache(1, 64, 4, 0, 42)
