"""Outlier/normal channel splitting (turboquant-plus-rs README, Modules:
outlier), GPU against the oracle: two codecs on the two channel groups of a
head (outliers first), one softmax over the tokens' total scores.  Codes are
uploaded from the oracle's encode so both sides score identical codes; the
output must agree within 2e-3 absolute.  The GPU encode of each group is the
ordinary tq_encode_kv on a channel slice, checked against the oracle too."""
import numpy as np
import pytest
import torch

import oracle
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

tq = pytest.importorskip("kv_cache_vector_10_b200")

DEV = "cuda"


def _case(bits_o, bits_n, rot_o, rot_n, d_o=64, d_n=64, B=2, Hq=4, Hkv=2, T=333, dtype=torch.bfloat16, seed=0):
    g = torch.Generator().manual_seed(seed)
    d = d_o + d_n
    scale = torch.cat([torch.full((d_o,), 5.0), torch.ones(d_n)])
    k = (torch.randn(B, Hkv, T, d, generator=g) * scale).to(dtype)
    v = torch.randn(B, Hkv, T, d, generator=g).to(dtype)
    q = torch.randn(B, Hq, d, generator=g).to(dtype)
    go, gn = tq.Codec(d_o, bits_o, 64, 7, rotation=rot_o), tq.Codec(d_n, bits_n, 64, 9, rotation=rot_n)
    oo, on = oracle.Codec(d_o, bits_o, 64, 7, rotation=rot_o), oracle.Codec(d_n, bits_n, 64, 9, rotation=rot_n)
    cap = (T + 15) // 16 * 16
    co, cn = go.alloc(B, Hkv, cap), gn.alloc(B, Hkv, cap)
    eko, evo = pu.oracle_encode(oo, k[..., :d_o], True), pu.oracle_encode(oo, v[..., :d_o], False)
    ekn, evn = pu.oracle_encode(on, k[..., d_o:], True), pu.oracle_encode(on, v[..., d_o:], False)
    for cache, ek, ev in ((co, eko, evo), (cn, ekn, evn)):
        pu.upload_rows(cache.k, ek, T)
        pu.upload_rows(cache.v, ev, T)
    out = tq.decode_split(go, co, gn, cn, T, q.to(DEV), out_dtype=torch.float32).cpu().numpy()
    G = Hq // Hkv
    for b in range(B):
        for j in range(Hq):
            h = j // G
            ref = oracle.attention_split(q[b, j].double().numpy(),
                                         (oo, h, eko[b][h]["rows"], evo[b][h]["rows"]),
                                         (on, h, ekn[b][h]["rows"], evn[b][h]["rows"]))
            assert np.max(np.abs(out[b, j] - ref)) <= pu.ATTN_ABS, (b, j, np.max(np.abs(out[b, j] - ref)))
    return k, v, go, gn, oo, on


@pytest.mark.parametrize("bits_o,bits_n", [(4, 3), (3, 2), (5, 4)])
def test_split_decode_matches_oracle(bits_o, bits_n):
    _case(bits_o, bits_n, "hadamard", "hadamard", seed=bits_o)


def test_split_decode_mixed_rotations_and_widths():
    """Groups of different widths (128 outlier channels + 64) and a Haar group."""
    _case(4, 2, "haar", "hadamard", d_o=128, d_n=64, Hq=2, Hkv=1, T=200, dtype=torch.float16, seed=11)


def test_split_encode_by_channel_slices_matches_oracle():
    """Each group is encoded by the ordinary encoder on a channel slice of the
    head (16-byte aligned strided view)."""
    g = torch.Generator().manual_seed(3)
    B, H, T = 2, 2, 150
    x = torch.randn(B, H, T, 128, generator=g).to(torch.float16)
    go, gn = tq.Codec(64, 4, 64, 7), tq.Codec(64, 3, 64, 9)
    oo, on = oracle.Codec(64, 4, 64, 7), oracle.Codec(64, 3, 64, 9)
    co, cn = go.alloc(B, H, 160), gn.alloc(B, H, 160)
    xd = x.to(DEV)
    go.encode_kv(xd[..., :64], xd[..., :64], co)
    gn.encode_kv(xd[..., 64:], xd[..., 64:], cn)
    rep = {}
    for b in range(B):
        for h in range(H):
            pu.compare_k(co.k[b, h, :T].cpu().numpy(), oo.encode(x[b, h, :, :64].double().numpy(), h, True), oo, rep)
            pu.compare_v(cn.v[b, h, :T].cpu().numpy(), on.encode(x[b, h, :, 64:].double().numpy(), h, False), on, rep)


def test_split_argument_errors():
    go, gn = tq.Codec(64, 4, 64, 7), tq.Codec(64, 3, 64, 9)
    co, cn = go.alloc(1, 2, 32), gn.alloc(1, 1, 32)
    q = torch.randn(1, 2, 128, device=DEV)
    with pytest.raises(tq.TQError, match="DIM_MISMATCH"):
        tq.decode_split(go, co, gn, cn, 10, q)             # different kv heads
    cn2 = gn.alloc(1, 2, 32)
    with pytest.raises(tq.TQError, match="DIM_MISMATCH"):
        tq.decode_split(go, co, gn, cn2, 40, q)            # beyond capacity
    with pytest.raises(tq.TQError, match="EMPTY"):
        tq.decode_split(go, co, gn, cn2, 0, q)
