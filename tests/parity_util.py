"""Helpers for GPU-vs-oracle parity tests.

The unpacker here reads the documented packed row formats (include/tq.h)
with numpy bit operations; it shares no code with the oracle or with the
CUDA path.  Expected values always come from the oracle run on the same
seeded inputs; GPU outputs are only ever compared, never fed to the oracle.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle

BAND = 1e-5          # decisions within this distance of a boundary may differ
REL = 1e-4           # dequantized vectors, scores, stored norms
ATTN_ABS = 2e-3      # attention outputs


def attn_tolerance(ref: np.ndarray, out_dtype) -> np.ndarray:
    """Per-element bound on |out - ref| for attention outputs written in
    `out_dtype`: ATTN_ABS on the value before it is rounded to the output
    type, plus the rounding itself, at most half an ulp of that type at
    |ref| + ATTN_ABS (no slack for float32 outputs)."""
    ref = np.abs(np.asarray(ref, dtype=np.float64)) + ATTN_ABS
    if out_dtype == torch.float32:
        return np.full_like(ref, ATTN_ABS)
    mant = {torch.bfloat16: 8, torch.float16: 11}[out_dtype]
    _, e = np.frexp(ref)                     # ref in [2^(e-1), 2^e)
    half_ulp = np.ldexp(1.0, e - 1 - mant)   # ulp 2^(e-1-(mant-1)), halved
    if out_dtype == torch.float16:
        half_ulp = np.maximum(half_ulp, 2.0 ** -25)   # binary16 subnormal spacing / 2
    return ATTN_ABS + half_ulp


def unpack_k(rows: np.ndarray, d: int, bk: int, m: int, norms: str = "f32"):
    """rows [N, k_row_bytes] uint8 -> idx [N, d], bits [N, m], ns [N], gamma [N].
    norms "f16": the tail is n_s, gamma as binary16 (one 32-bit word)."""
    rows = np.ascontiguousarray(rows)
    N = rows.shape[0]
    pb = d // 8
    bits = np.unpackbits(rows[:, : bk * pb + m // 8], axis=1, bitorder="little")
    idx = np.zeros((N, d), dtype=np.int64)
    for p in range(bk):
        idx |= bits[:, p * d:(p + 1) * d].astype(np.int64) << p
    sg = bits[:, bk * d: bk * d + m].astype(np.int64)
    nb = 4 if norms == "f16" else 8
    tail = rows[:, bk * pb + m // 8: bk * pb + m // 8 + nb].copy().view(np.float16 if norms == "f16" else np.float32)
    return idx, sg, tail[:, 0].astype(np.float64), tail[:, 1].astype(np.float64)


def norm_slack(ref: np.ndarray, norms: str) -> np.ndarray:
    """Extra tolerance of a stored norm: one binary16 step at the oracle's
    value when norms are binary16 (the kernel rounds its fp32 norm, the
    oracle its fp64 norm), else 0."""
    if norms != "f16":
        return np.zeros_like(ref)
    return np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64)


def unpack_v(rows: np.ndarray, d: int, bv: int):
    rows = np.ascontiguousarray(rows)
    N = rows.shape[0]
    nb = bv * d // 8
    bits = np.unpackbits(rows[:, :nb], axis=1, bitorder="little").astype(np.int64).reshape(N, d, bv)
    idx = np.zeros((N, d), dtype=np.int64)
    for k in range(bv):
        idx |= bits[:, :, k] << k
    ns = rows[:, nb:nb + 4].copy().view(np.float32)[:, 0].astype(np.float64)
    return idx, ns


def _near_boundary(z: np.ndarray, beta: np.ndarray) -> np.ndarray:
    zz = np.where(np.isfinite(z), z, 1e30)
    return np.min(np.abs(zz[..., None] - beta[None, None, :]), axis=-1) < BAND


def compare_k(gpu_rows, ora, codec: oracle.Codec, report: dict):
    """Compare packed key rows.  ora: dict from Codec.encode(..., is_key=True)."""
    d, m, bk = codec.d, codec.m, codec.bits - 1
    norms = getattr(codec, "norms", "f32")
    gi, gb, gns, gg = unpack_k(gpu_rows, d, bk, m, norms)
    oi, ob, ons, og = unpack_k(ora["rows"], d, bk, m, norms)
    near = _near_boundary(ora["z"], codec.bk)
    bad_idx = (gi != oi) & ~near
    assert not bad_idx.any(), f"key index mismatch outside the boundary band at rows {np.nonzero(bad_idx.any(1))[0][:10]}"
    flipped = (gi != oi).any(axis=1)
    report["k_index_flips"] = report.get("k_index_flips", 0) + int((gi != oi).sum())
    # sign bits: rows without index flips and with a non-degenerate residual
    pn = ora["pn"]
    ok_rows = ~flipped & np.isfinite(pn).all(axis=1) & (og > 1e-6 * np.maximum(ons, 1e-30))
    near_p = np.abs(pn) < BAND
    bad_sign = (gb != ob) & ~near_p & ok_rows[:, None]
    assert not bad_sign.any(), f"QJL sign mismatch at rows {np.nonzero(bad_sign.any(1))[0][:10]}"
    report["k_sign_flips"] = report.get("k_sign_flips", 0) + int(((gb != ob) & ok_rows[:, None]).sum())
    report["k_rows_flipped"] = report.get("k_rows_flipped", 0) + int(flipped.sum())
    nf = ~flipped
    assert np.all(np.abs(gns[nf] - ons[nf]) <= REL * np.abs(ons[nf]) + norm_slack(ons[nf], norms) + 1e-30), \
        "n_s mismatch"
    assert np.all(np.abs(gg[nf] - og[nf]) <= REL * np.maximum(np.abs(og[nf]), 1e-3 * ons[nf]) +
                  norm_slack(og[nf], norms) + 1e-30), "gamma mismatch"
    return report


def compare_v(gpu_rows, ora, codec: oracle.Codec, report: dict):
    d, bv = codec.d, codec.bits
    gi, gns = unpack_v(gpu_rows, d, bv)
    oi, ons = unpack_v(ora["rows"], d, bv)
    near = _near_boundary(ora["z"], codec.bv)
    bad = (gi != oi) & ~near
    assert not bad.any(), f"value index mismatch outside the band at rows {np.nonzero(bad.any(1))[0][:10]}"
    flipped = (gi != oi).any(axis=1)
    report["v_index_flips"] = report.get("v_index_flips", 0) + int((gi != oi).sum())
    nf = ~flipped
    assert np.all(np.abs(gns[nf] - ons[nf]) <= REL * np.abs(ons[nf]) + 1e-30), "value n_s mismatch"
    return report


def oracle_encode(codec: oracle.Codec, x: torch.Tensor, is_key: bool):
    """x [B, H, T, d] (any float dtype, any device) -> per (b, h) oracle results."""
    xs = x.detach().to("cpu", torch.float64).numpy()
    B, H, T, _ = xs.shape
    return [[codec.encode(xs[b, h], h, is_key) for h in range(H)] for b in range(B)]


def upload_rows(cache_tensor: torch.Tensor, enc, T: int):
    """Write oracle rows into a PackedCache buffer [B, H, cap, row]."""
    B, H = len(enc), len(enc[0])
    host = cache_tensor.cpu()
    for b in range(B):
        for h in range(H):
            host[b, h, :T] = torch.from_numpy(enc[b][h]["rows"])
    cache_tensor.copy_(host)


def scores_tolerance(ref: np.ndarray, q: np.ndarray, khat: np.ndarray) -> np.ndarray:
    d = q.shape[-1]
    scale = np.linalg.norm(q) * np.linalg.norm(khat, axis=-1) / d
    return REL * np.maximum(np.abs(ref), scale)


def vec_tolerance(ref: np.ndarray) -> np.ndarray:
    d = ref.shape[-1]
    scale = np.linalg.norm(ref, axis=-1, keepdims=True) / math.sqrt(d)
    return REL * np.maximum(np.abs(ref), scale)
