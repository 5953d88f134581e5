"""Seeded synthetic workload generators: reproducible, shaped like the
configurations they stand for, with the stated value distributions."""
import torch

from kv_cache_vector_10_b200 import workloads as W


def test_reproducible_and_seed_sensitive():
    a = W.single_head(n_tokens=64)
    b = W.single_head(n_tokens=64)
    c = W.single_head(n_tokens=64, data_seed=9)
    assert torch.equal(a["k"], b["k"]) and torch.equal(a["q"], b["q"])
    assert not torch.equal(a["k"], c["k"])


def test_shapes_and_dtypes_small():
    m = W.mha_decode(batch=2, heads=4, n_tokens=64)
    assert m["k"].shape == (2, 4, 64, 128) and m["k"].dtype == torch.float16 and m["q"].shape == (2, 4, 128)
    g = W.gqa_decode(batch=2, q_heads=8, kv_heads=2, n_tokens=64)
    assert g["k"].shape == (2, 2, 64, 128) and g["k"].dtype == torch.bfloat16 and g["q"].shape == (2, 8, 128)
    s = W.shared_prefix(agents=3, prefix_tokens=32, tail_tokens=16, q_heads=8, kv_heads=2)
    assert s["prefix_k"].shape == (1, 2, 32, 128) and s["tail_k"].shape == (3, 2, 16, 128)
    bl = W.bulk_encode(layers=4, heads=2, n_tokens=16)
    assert bl["layer_bits"] == [4, 4, 4, 4] and bl["k"].shape == (4, 2, 16, 128)
    assert W.BULK_LAYER_BITS == [4, 4] + [3] * 28 + [4, 4]


def test_distributions():
    g = W.gqa_decode(batch=1, q_heads=4, kv_heads=1, n_tokens=4096)
    nrm = g["k"].float().norm(dim=-1)
    assert 0.49 <= float(nrm.min()) and float(nrm.max()) <= 2.02          # per-token norm ~ U[0.5, 2]
    m = W.mha_decode(batch=1, heads=2, n_tokens=4096)
    ch = m["k"].float().abs().mean(dim=2)[0]                              # per-(head, channel) scale
    ratio = ch.max(dim=-1).values / ch.median(dim=-1).values
    assert float(ratio.min()) > 5.0                                        # outlier channels x10
