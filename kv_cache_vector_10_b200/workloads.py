"""Seeded synthetic inputs for the five benchmark / parity workloads.

Only random-number generation and tensor shaping live here -- none of the
codec's arithmetic.  Both the tests (which hand the same tensors to the CPU
oracle and to the CUDA path) and bench.py use these generators.  Tensors are
drawn on the requested device with a torch.Generator seeded per tensor, so a
workload is reproducible on any machine with the same device type.

Workloads (head_dim 128, projections 128 throughout):
  single_head     bits 3, seed 42: 1024 keys and values iid N(0,1) fp32, 4 queries.
  mha_decode      bits 4: batch 8, 32 heads, 4096 tokens, fp16; every (head,
                  channel) scaled by exp(N(0, 0.5)), 4 channels per head
                  (seeded permutation) scaled x10; one query per sequence.
  gqa_decode      bits 2: batch 4, 32 query heads over 8 kv heads, 32768
                  tokens, bf16; each token g/|g| * u, g ~ N(0, I), u ~ U[0.5, 2].
  bulk_encode     32 layers x 8 kv heads x 8192 tokens, bf16 N(0,1); bits 3 on
                  layers 2..29 and bits 4 on layers 0, 1, 30, 31.
  shared_prefix   one 4096-token prefix at bits 2 + 16 private tails of 1024
                  tokens at bits 4; 32 query heads over 8 kv heads, bf16 N(0,1);
                  16 agents, one decode step each.
"""
from __future__ import annotations

import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal(shape, seed: int, dtype=torch.float32, device="cpu") -> torch.Tensor:
    return torch.randn(*shape, generator=_gen(seed, device), device=device, dtype=torch.float32).to(dtype)


def uniform(shape, seed: int, lo: float, hi: float, device="cpu") -> torch.Tensor:
    u = torch.rand(*shape, generator=_gen(seed, device), device=device, dtype=torch.float32)
    return lo + (hi - lo) * u


def single_head(device="cpu", n_tokens: int = 1024, n_queries: int = 4, data_seed: int = 1):
    """keys/values [1, 1, T, 128] fp32; queries [1, 4, 128] fp32 (4 query heads on one kv head)."""
    k = normal((1, 1, n_tokens, 128), data_seed * 1000 + 1, device=device)
    v = normal((1, 1, n_tokens, 128), data_seed * 1000 + 2, device=device)
    q = normal((1, n_queries, 128), data_seed * 1000 + 3, device=device)
    return dict(k=k, v=v, q=q, bits=3, seed=42, head_dim=128, projections=128)


def _channel_scales(heads: int, d: int, seed: int, device) -> torch.Tensor:
    s = torch.exp(normal((heads, d), seed, device=device) * 0.5)
    g = _gen(seed + 7, device)
    for h in range(heads):
        idx = torch.randperm(d, generator=g, device=device)[:4]
        s[h, idx] *= 10.0
    return s


def mha_decode(device="cpu", batch: int = 8, heads: int = 32, n_tokens: int = 4096, data_seed: int = 2,
               dtype=torch.float16):
    sc = _channel_scales(heads, 128, data_seed * 1000 + 9, device)[None, :, None, :]
    k = (normal((batch, heads, n_tokens, 128), data_seed * 1000 + 1, device=device) * sc).to(dtype)
    v = (normal((batch, heads, n_tokens, 128), data_seed * 1000 + 2, device=device) * sc).to(dtype)
    q = normal((batch, heads, 128), data_seed * 1000 + 3, dtype=dtype, device=device)
    return dict(k=k, v=v, q=q, bits=4, seed=42, head_dim=128, projections=128, n_kv_heads=heads)


def _unit_times_uniform(shape, seed: int, device):
    g = normal(shape, seed, device=device)
    g = g / g.norm(dim=-1, keepdim=True)
    return g * uniform(shape[:-1] + (1,), seed + 5, 0.5, 2.0, device=device)


def gqa_decode(device="cpu", batch: int = 4, q_heads: int = 32, kv_heads: int = 8, n_tokens: int = 32768,
               data_seed: int = 3, dtype=torch.bfloat16):
    k = _unit_times_uniform((batch, kv_heads, n_tokens, 128), data_seed * 1000 + 1, device).to(dtype)
    v = _unit_times_uniform((batch, kv_heads, n_tokens, 128), data_seed * 1000 + 2, device).to(dtype)
    q = normal((batch, q_heads, 128), data_seed * 1000 + 3, dtype=dtype, device=device)
    return dict(k=k, v=v, q=q, bits=2, seed=42, head_dim=128, projections=128, n_kv_heads=kv_heads)


BULK_LAYER_BITS = [4, 4] + [3] * 28 + [4, 4]


def bulk_encode(device="cpu", layers: int = 32, heads: int = 8, n_tokens: int = 8192, data_seed: int = 4,
                dtype=torch.bfloat16):
    """keys/values [layers, heads, T, 128]; layer l uses BULK_LAYER_BITS[l] (first and last two at 4)."""
    k = normal((layers, heads, n_tokens, 128), data_seed * 1000 + 1, dtype=dtype, device=device)
    v = normal((layers, heads, n_tokens, 128), data_seed * 1000 + 2, dtype=dtype, device=device)
    bits = [4 if (l < 2 or l >= layers - 2) else 3 for l in range(layers)]
    return dict(k=k, v=v, layer_bits=bits, seed=42, head_dim=128, projections=128)


def shared_prefix(device="cpu", agents: int = 16, prefix_tokens: int = 4096, tail_tokens: int = 1024,
                  q_heads: int = 32, kv_heads: int = 8, data_seed: int = 5, dtype=torch.bfloat16):
    pk = normal((1, kv_heads, prefix_tokens, 128), data_seed * 1000 + 1, dtype=dtype, device=device)
    pv = normal((1, kv_heads, prefix_tokens, 128), data_seed * 1000 + 2, dtype=dtype, device=device)
    tk = normal((agents, kv_heads, tail_tokens, 128), data_seed * 1000 + 3, dtype=dtype, device=device)
    tv = normal((agents, kv_heads, tail_tokens, 128), data_seed * 1000 + 4, dtype=dtype, device=device)
    q = normal((agents, q_heads, 128), data_seed * 1000 + 5, dtype=dtype, device=device)
    return dict(prefix_k=pk, prefix_v=pv, tail_k=tk, tail_v=tv, q=q, prefix_bits=2, tail_bits=4, seed=42,
                head_dim=128, projections=128, n_kv_heads=kv_heads)
