#!/usr/bin/env python
"""Benchmark of the TurboQuant KV-cache hot path on B200.

A step is one pass of the whole hot path over one batch of synthetic input:
encode every key/value row of the batch into the packed cache (norm,
rotation, quantization, QJL signs, packing) and run one decode-attention
step for every query head over it (query preparation, split-K scoring from
the codes with online softmax and value accumulation, combine).  The
default workload is the multi-head decode case (batch 8, 32 heads, 4096
cached tokens, bits 4, fp16 K/V).  Other workloads: --workload gqa_decode |
shared_prefix | bulk_encode | single_head.

Prints ONE JSON line (rank 0).  `value` = KV tokens scored per second over
the whole job (sum over ranks of batch*heads*tokens per step / max-over-ranks
device time per step); for bulk_encode it is input GB/s.  `e2e` is the same
metric through the public API with host (pinned) inputs copied in and the
output copied back inside the timed region.  `roofline` is for the kernel
with the largest share of the step, timed live with CUDA events on the
launching stream.  `--impl reference` times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "compressed-KV decode: KV tokens scored/s; encode GB/s; % of HBM roofline"
D = 128
M = 128


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mha_decode",
                    choices=["mha_decode", "gqa_decode", "shared_prefix", "bulk_encode", "single_head",
                             "mha_append", "mha_decode_haar", "mha_split", "mha_decode_f16norms"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-workers", type=int, default=96, help="reference arm: at most this many processes")
    ap.add_argument("--ref-units", type=int, default=4, help="reference arm: oracle units per process per step")
    ap.add_argument("--cpu-single", action="store_true", help="CPU baseline single-threaded only")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip timing the other workloads in the same run (the `configs` key)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--graphs", action="store_true",
                    help="replay each piece from a captured CUDA graph instead of launching it eagerly")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


WORKLOAD_DESC = {
    "mha_decode": "mha_decode: batch 8, 32 query heads over 32 kv heads, 4096 tokens, d128, m128, bits 4 "
                  "(K 3+1, V 4), float16",
    "gqa_decode": "gqa_decode: batch 4, 32 query heads over 8 kv heads, 32768 tokens, d128, m128, bits 2 "
                  "(K 1+1, V 2), bfloat16",
    "shared_prefix": "shared_prefix: 16 agents, prefix 4096 tokens at bits 2 read once per kv head + 16 tails of "
                     "1024 tokens at bits 4, 32 q heads over 8 kv heads, d128, m128, bf16",
    "bulk_encode": "bulk_encode: 32 layers x 8 kv heads x 8192 tokens x d128, bf16; bits 3 on layers 2..29, bits 4 "
                   "on layers 0, 1, 30, 31; m128",
    "single_head": "single_head: batch 1, 4 query heads over 1 kv heads, 1024 tokens, d128, m128, bits 3 "
                   "(K 2+1, V 3), float32",
    "mha_append": "mha_append: batch 8, 32 query heads over 32 kv heads, 4096 cached tokens + 1 appended per "
                  "(sequence, kv head), d128, m128, bits 4 (K 3+1, V 4), float16",
    "mha_decode_f16norms": "mha_decode_f16norms: the mha_decode workload (batch 8, 32 heads, 4096 tokens, d128, "
                           "fp16, bits 4, m128) with binary16 key norms (68-byte key rows, 4.25 bits per key value)",
    "mha_decode_haar": "mha_decode_haar: the mha_decode workload with the Haar-QR rotation (batch 8, 32 heads, "
                       "4096 tokens, d128, m128, bits 4, float16)",
    "mha_split": "mha_split: the mha_decode data (batch 8, 32 heads, 4096 tokens, d128, fp16) split per head into "
                 "64 outlier channels (largest RMS) at bits 4 and 64 normal channels at bits 3 (3.5 index bits per "
                 "value), m64 per group",
}


STEP_DESC = {w: "encode all K/V rows + one decode step per query head"
             for w in ("mha_decode", "gqa_decode", "shared_prefix", "single_head", "mha_decode_haar",
                       "mha_decode_f16norms")}
STEP_DESC["bulk_encode"] = "encode all K/V rows of 32 layers"
STEP_DESC["mha_append"] = "append one token per (sequence, kv head) + one decode step per query head"
STEP_DESC["mha_split"] = "encode both channel groups of all K/V rows + one split decode step per query head"
L2_DESC = ("flushed (256 MiB write) before every timed piece, outside its CUDA events; "
           "ms_per_step = sum of the pieces")


def arm_config(workload):
    return {"workload": WORKLOAD_DESC[workload], "step": STEP_DESC[workload], "l2": L2_DESC}


# DRAM traffic of a piece: dram__bytes_read.sum + dram__bytes_write.sum summed
# over the piece's launches of one step (one ncu capture of every launch, caches
# flushed before each kernel, averaged over the captured steps), keyed by (piece, workload),
# with the SHA-1 of the source files holding those kernels when the counters
# were taken: once one of them changes the entry no longer applies (traffic:
# null).  Summaries: profiles/.
MEASURED_TRAFFIC = {
    ("encode_keys", "mha_decode"): (('tq_encode.cu', 'tq_internal.cuh'), "008f084c694e2a11b023fe06e61a5027e32563c1", 330782976),
    ("encode_values", "mha_decode"): (('tq_encode.cu', 'tq_internal.cuh'), "008f084c694e2a11b023fe06e61a5027e32563c1", 321204032),
    ("decode", "mha_decode"): (('tq_decode.cu', 'tq_decode_mma.cu', 'tq_aux.cu', 'tq_decode.cuh', 'tq_internal.cuh'), "a55d60bb799f47a9fa64595e143b436cb1e3a32a", 149267136),
    ("encode_keys", "gqa_decode"): (('tq_encode.cu', 'tq_internal.cuh'), "008f084c694e2a11b023fe06e61a5027e32563c1", 298793152),
    ("encode_values", "gqa_decode"): (('tq_encode.cu', 'tq_internal.cuh'), "008f084c694e2a11b023fe06e61a5027e32563c1", 292880512),
    ("decode", "gqa_decode"): (('tq_decode.cu', 'tq_decode_mma.cu', 'tq_aux.cu', 'tq_decode.cuh', 'tq_internal.cuh'), "a55d60bb799f47a9fa64595e143b436cb1e3a32a", 81083520),
    ("encode_keys", "bulk_encode"): (('tq_encode.cu', 'tq_internal.cuh'), "008f084c694e2a11b023fe06e61a5027e32563c1", 629477056),
    ("encode_values", "bulk_encode"): (('tq_encode.cu', 'tq_internal.cuh'), "008f084c694e2a11b023fe06e61a5027e32563c1", 616778560),
    ("encode_keys", "shared_prefix"): (('tq_encode.cu', 'tq_internal.cuh'), "008f084c694e2a11b023fe06e61a5027e32563c1", 43085248),
    ("encode_values", "shared_prefix"): (('tq_encode.cu', 'tq_internal.cuh'), "008f084c694e2a11b023fe06e61a5027e32563c1", 42974656),
    ("decode", "shared_prefix"): (('tq_decode.cu', 'tq_decode_mma.cu', 'tq_aux.cu', 'tq_decode.cuh', 'tq_internal.cuh'), "a55d60bb799f47a9fa64595e143b436cb1e3a32a", 27370688),
    ("decode_append", "mha_append"): (('tq_decode.cu', 'tq_decode_mma.cu', 'tq_aux.cu', 'tq_decode.cuh', 'tq_internal.cuh'), "a55d60bb799f47a9fa64595e143b436cb1e3a32a", 149690688),
    ("encode_keys", "mha_split"): (('tq_encode.cu', 'tq_internal.cuh'), "008f084c694e2a11b023fe06e61a5027e32563c1", 445315968),
    ("encode_values", "mha_split"): (('tq_encode.cu', 'tq_internal.cuh'), "008f084c694e2a11b023fe06e61a5027e32563c1", 436353792),
    ("decode_split", "mha_split"): (('tq_split.cu', 'tq_aux.cu', 'tq_decode.cuh', 'tq_internal.cuh'), "3deb5480f30ab8588392a6ac1abc822623297177", 152436800),
    ("encode_keys", "mha_decode_haar"): (('tq_encode.cu', 'tq_internal.cuh'), "008f084c694e2a11b023fe06e61a5027e32563c1", 333529664),
    ("encode_values", "mha_decode_haar"): (('tq_encode.cu', 'tq_internal.cuh'), "008f084c694e2a11b023fe06e61a5027e32563c1", 322862464),
    ("decode", "mha_decode_haar"): (('tq_decode.cu', 'tq_decode_mma.cu', 'tq_aux.cu', 'tq_decode.cuh', 'tq_internal.cuh'), "a55d60bb799f47a9fa64595e143b436cb1e3a32a", 153262400),
}


def measured_traffic(piece, workload):
    import hashlib
    ent = MEASURED_TRAFFIC.get((piece, workload))
    if not ent:
        return None
    files, sha, nbytes = ent
    h = hashlib.sha1()
    try:
        for src in files:
            with open(os.path.join(ROOT, "kv_cache_vector_10_b200", "csrc", src), "rb") as f:
                h.update(f.read())
    except OSError:
        return None
    return nbytes if h.hexdigest() == sha else None


def row_bytes(bits, norms="f32"):
    return (bits - 1) * D // 8 + M // 8 + (4 if norms == "f16" else 8), bits * D // 8 + 4


# ------------------------------------------------------------------ workloads

class Workload:
    """Device inputs, caches and the step of one workload.  A step is a list
    of pieces (one or more libtq calls each), bracketed by CUDA events on the
    launching stream: (name, algorithmic bytes, kernel launches)."""

    def __init__(self, name, device, rank=0):
        import torch

        import kv_cache_vector_10_b200 as tq
        from kv_cache_vector_10_b200 import workloads as W
        self.name, self.tq, self.torch = name, tq, torch
        seed_shift = 1000 * rank
        if name in ("mha_decode", "gqa_decode", "single_head", "mha_append", "mha_decode_haar", "mha_decode_f16norms"):
            if name in ("mha_decode", "mha_append", "mha_decode_haar", "mha_decode_f16norms"):
                w = W.mha_decode(device=device, data_seed=2 + seed_shift,
                                 n_tokens=4097 if name == "mha_append" else 4096)
            elif name == "gqa_decode":
                w = W.gqa_decode(device=device, data_seed=3 + seed_shift)
            else:
                w = W.single_head(device=device, data_seed=1 + seed_shift)
            self.w = w
            B, Hkv, T, _ = w["k"].shape
            Hq = w["q"].shape[1]
            bits = w["bits"]
            norms = "f16" if name == "mha_decode_f16norms" else "f32"
            kr, vr = row_bytes(bits, norms)
            es = w["k"].element_size()
            qb = B * Hq * D * 2 * w["q"].element_size()          # query in + output out
            self.codec = tq.Codec(D, bits, M, w["seed"], rotation="haar" if name == "mha_decode_haar" else "hadamard",
                                  norms=norms)
            self.B, self.Hq, self.Hkv = B, Hq, Hkv
            if name == "mha_append":
                T -= 1                                            # history; row T is the step's new row
                self.T = T
                self.cache = self.codec.alloc(B, Hkv, T + 16, device)
                self.codec.encode_kv(w["k"][:, :, :T], w["v"][:, :, :T], self.cache)   # set-up, untimed
                self.segments = [tq.Segment(self.cache, T, b, 1, codes_batch=b) for b in range(B)]
                self.inputs = dict(k_new=w["k"][:, :, T].contiguous(), v_new=w["v"][:, :, T].contiguous(),
                                   q=w["q"])
                self.tokens_scored = B * Hq * (T + 1)
                grown = [tq.Segment(self.cache, T + 1, b, 1, codes_batch=b) for b in range(B)]
                self.pieces = [("decode_append", B * Hkv * (T + 1) * (kr + vr) + B * Hkv * (2 * D * es + kr + vr)
                                + qb, tq.tq_decode_launch_count(grown, B, Hq, Hkv))]
            else:
                self.cache = self.codec.alloc(B, Hkv, (T + 15) // 16 * 16, device)
                self.segments = [tq.Segment(self.cache, T, b, 1, codes_batch=b) for b in range(B)]
                self.inputs = dict(k=w["k"], v=w["v"], q=w["q"])
                self.tokens_scored = B * Hq * T
                self.pieces = [("encode_keys", B * Hkv * T * (D * es + kr), 1),
                               ("encode_values", B * Hkv * T * (D * es + vr), 1),
                               ("decode", B * Hkv * T * (kr + vr) + qb,
                                tq.tq_decode_launch_count(self.segments, B, Hq, Hkv))]
        elif name == "mha_split":
            w = W.mha_decode(device=device, data_seed=2 + seed_shift)
            B, H, T, _ = w["k"].shape
            # channels ordered per head by RMS over the cached keys: outliers first
            order = w["k"].float().pow(2).mean(dim=(0, 2)).argsort(dim=-1, descending=True)   # [H, d]
            idx = order[None, :, None, :]
            k = torch.gather(w["k"], 3, idx.expand_as(w["k"])).contiguous()
            v = torch.gather(w["v"], 3, idx.expand_as(w["v"])).contiguous()
            q = torch.gather(w["q"], 2, order[None].expand_as(w["q"])).contiguous()
            self.codec_o = tq.Codec(64, 4, 64, w["seed"])
            self.codec_n = tq.Codec(64, 3, 64, w["seed"] + 1000)
            self.cache_o = self.codec_o.alloc(B, H, T, device)
            self.cache_n = self.codec_n.alloc(B, H, T, device)
            self.inputs = dict(k=k, v=v, q=q)
            self.B, self.Hq, self.Hkv, self.T = B, H, H, T
            self.tokens_scored = B * H * T
            es = k.element_size()
            ko, vo = 3 * 8 + 8 + 8, 4 * 8 + 4
            kn, vn = 2 * 8 + 8 + 8, 3 * 8 + 4
            qb = B * H * D * 2 * es
            self.pieces = [("encode_keys", B * H * T * (D * es + ko + kn), 2),
                           ("encode_values", B * H * T * (D * es + vo + vn), 2),
                           ("decode_split", B * H * T * (ko + kn + vo + vn) + qb, 5)]
        elif name == "shared_prefix":
            w = W.shared_prefix(device=device, data_seed=5 + seed_shift)
            self.w = w
            A, Hq = w["q"].shape[:2]
            Hkv = w["n_kv_heads"]
            P, Tt = w["prefix_k"].shape[2], w["tail_k"].shape[2]
            self.pcodec = tq.Codec(D, w["prefix_bits"], M, w["seed"])
            self.tcodec = tq.Codec(D, w["tail_bits"], M, w["seed"])
            self.pcache = self.pcodec.alloc(1, Hkv, P, device)
            self.tcache = self.tcodec.alloc(A, Hkv, Tt, device)
            self.segments = [tq.Segment(self.pcache, P, 0, A)] + \
                            [tq.Segment(self.tcache, Tt, a, 1, codes_batch=a) for a in range(A)]
            self.inputs = dict(pk=w["prefix_k"], pv=w["prefix_v"], tk=w["tail_k"], tv=w["tail_v"], q=w["q"])
            self.B, self.Hq, self.Hkv = A, Hq, Hkv
            self.tokens_scored = A * Hq * (P + Tt)
            pkr, pvr = row_bytes(w["prefix_bits"])
            tkr, tvr = row_bytes(w["tail_bits"])
            es = w["prefix_k"].element_size()
            self.pieces = [("encode_keys", Hkv * P * (D * es + pkr) + A * Hkv * Tt * (D * es + tkr), 2),
                           ("encode_values", Hkv * P * (D * es + pvr) + A * Hkv * Tt * (D * es + tvr), 2),
                           ("decode", Hkv * P * (pkr + pvr) + A * Hkv * Tt * (tkr + tvr) + 2 * A * Hq * D * es,
                            tq.tq_decode_launch_count(self.segments, A, Hq, Hkv))]
        elif name == "bulk_encode":
            w = W.bulk_encode(device=device, data_seed=4 + seed_shift)
            self.w = w
            L, H, T, _ = w["k"].shape
            self.c3 = tq.Codec(D, 3, M, w["seed"])
            self.c4 = tq.Codec(D, 4, M, w["seed"])
            self.cache3 = self.c3.alloc(28, H, T, device)
            self.cache4a = self.c4.alloc(2, H, T, device)
            self.cache4b = self.c4.alloc(2, H, T, device)
            self.inputs = dict(k=w["k"], v=w["v"])
            self.B, self.Hq, self.Hkv = L, H, H
            self.tokens_scored = 0
            es = w["k"].element_size()
            k3, v3 = row_bytes(3)
            k4, v4 = row_bytes(4)
            self.in_bytes = 2 * L * H * T * D * es
            self.pieces = [("encode_keys", L * H * T * D * es + H * T * (28 * k3 + 4 * k4), 3),
                           ("encode_values", L * H * T * D * es + H * T * (28 * v3 + 4 * v4), 3)]
        self.desc = WORKLOAD_DESC[name]
        self.out = None
        self.ws = None
        self.flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)   # 2x the L2

    def _decode(self, inp):
        torch, tq = self.torch, self.tq
        if self.out is None:
            need = tq.tq_decode_workspace_bytes(self.segments, self.B, self.Hq, self.Hkv)
            if self.name == "mha_append":
                need = tq.tq_decode_append_workspace_bytes(self.segments, self.B, self.Hq, self.Hkv)
            self.ws = torch.empty(max(need, 16), dtype=torch.uint8, device=inp["q"].device)
            self.out = torch.empty(self.B, self.Hq, D, dtype=inp["q"].dtype, device=inp["q"].device)
        if self.name == "mha_append":
            for sg in self.segments:          # every step appends at the same row T
                sg.n_tokens = self.T
            tq.tq_decode_append(self.segments, inp["k_new"], inp["v_new"], inp["q"], self.B, self.Hq, self.Hkv,
                                self.out, self.ws)
        else:
            tq.tq_decode_attention(self.segments, inp["q"], self.B, self.Hq, self.Hkv, self.out, self.ws)

    def _run_piece(self, name, inp):
        if name == "decode_split":
            if self.out is None:
                torch = self.torch
                need = self.tq.lib.tq_decode_split_workspace_bytes(self.codec_o.ctx, self.codec_n.ctx, self.B,
                                                                   self.Hq, self.T)
                self.ws = torch.empty(max(need, 16), dtype=torch.uint8, device=inp["q"].device)
            self.out = self.tq.decode_split(self.codec_o, self.cache_o, self.codec_n, self.cache_n, self.T, inp["q"],
                                            workspace=self.ws)
            return
        if name == "encode_keys" or name == "encode_values":
            side = "k" if name == "encode_keys" else "v"
            if self.name == "mha_split":
                x = inp[side]
                a = (x[..., :64], None) if side == "k" else (None, x[..., :64])
                self.codec_o.encode_kv(*a, self.cache_o)
                a = (x[..., 64:], None) if side == "k" else (None, x[..., 64:])
                self.codec_n.encode_kv(*a, self.cache_n)
                return
            if self.name == "shared_prefix":
                args_p = (inp["pk"], None) if side == "k" else (None, inp["pv"])
                args_t = (inp["tk"], None) if side == "k" else (None, inp["tv"])
                self.pcodec.encode_kv(*args_p, self.pcache)
                self.tcodec.encode_kv(*args_t, self.tcache)
            elif self.name == "bulk_encode":
                x = inp[side]
                for codec, cache, sl in ((self.c4, self.cache4a, slice(0, 2)), (self.c3, self.cache3, slice(2, 30)),
                                         (self.c4, self.cache4b, slice(30, 32))):
                    a = (x[sl], None) if side == "k" else (None, x[sl])
                    codec.encode_kv(*a, cache)
            else:
                a = (inp["k"], None) if side == "k" else (None, inp["v"])
                self.codec.encode_kv(*a, self.cache)
        else:
            self._decode(inp)

    def capture(self, inp):
        """Capture every piece on `inp` as a CUDA graph; later steps on the
        same input tensors replay them (the library's launches, dependent
        launches included, are graph-capturable).  Call after one eager step,
        which builds the head tables and workspaces."""
        torch = self.torch
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        self.graphs = {}
        with torch.cuda.stream(s):
            for name, _, _ in self.pieces:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=s):
                    self._run_piece(name, inp)
                self.graphs[name] = g
        torch.cuda.current_stream().wait_stream(s)
        self.graph_inp = inp

    def step(self, inp, events=None):
        """One step; events: two CUDA events per piece (start, end).  Returns
        the decode output (None for encode-only workloads)."""
        graphs = getattr(self, "graphs", None) if getattr(self, "graph_inp", None) is inp else None
        for i, (name, _, _) in enumerate(self.pieces):
            if self.flush is not None:
                self.flush.zero_()            # evict L2 before each piece (outside its events)
            if events:
                events[2 * i].record()
            if graphs:
                graphs[name].replay()
            else:
                self._run_piece(name, inp)
            if events:
                events[2 * i + 1].record()
        return self.out

    @property
    def launches(self):
        return sum(n for _, _, n in self.pieces)


def clock_sampler(device_index):
    """Samples SM clocks and throttle reasons every 200 ms until stopped."""
    q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")
    try:
        p = subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-lms", "200",
                              "-i", str(device_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
    except Exception:
        return None, []
    rows = []

    def rd():
        for line in p.stdout:
            rows.append([x.strip() for x in line.split(",")])
    t = threading.Thread(target=rd, daemon=True)
    t.start()
    return p, rows


def summarize_clocks(rows):
    sm = [float(r[1]) for r in rows if len(r) >= 9 and r[1].replace(".", "").isdigit()]
    mx = [float(r[2]) for r in rows if len(r) >= 9 and r[2].replace(".", "").isdigit()]
    reasons = set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for r in rows:
        if len(r) >= 9:
            for i, nm in enumerate(names):
                if r[5 + i].lower().startswith("active"):
                    reasons.add(nm)
    if not sm:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
    sm.sort()
    return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
            "samples": len(sm)}


# ------------------------------------------------------------- multi-rank
def max_over_ranks(x: float, world: int, device="cpu") -> float:
    """Max of a per-rank time over all ranks (every rank must call this)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, seconds: float) -> float:
    """Whole-job throughput of a weak-scaling run: every rank processes the
    same number of units; the job takes the slowest rank's time."""
    return world * units_per_rank / seconds


# ------------------------------------------------------------ CPU oracle arm

def load_workloads():
    """The seeded input generators, loaded from their file as a module of
    their own: importing them through the package would run its __init__,
    which maps libtq.so into a process that only runs the oracle."""
    import importlib.util
    name = "tq_workload_generators"
    if name in sys.modules:
        return sys.modules[name]
    spec = importlib.util.spec_from_file_location(name, os.path.join(ROOT, "kv_cache_vector_10_b200", "workloads.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    sys.modules[name] = mod
    return mod


def oracle_unit(wl_name, rank_seed=0):
    """One bounded CPU-oracle unit of the workload: returns (seconds, units, unit_name, sample_desc).

    Units are KV tokens scored (decode workloads) or input bytes (bulk_encode).
    rank_seed shifts the data seed, so parallel workers take different units."""
    import numpy as np
    import torch

    import oracle
    W = load_workloads()
    if wl_name == "bulk_encode":
        w = W.bulk_encode(device="cpu", layers=1, heads=1, n_tokens=1024, data_seed=4 + rank_seed)
        oc = oracle.Codec(D, 3, M, 42)
        k = w["k"][0, 0].double().numpy()
        v = w["v"][0, 0].double().numpy()
        t0 = time.perf_counter()
        oc.encode(k, 0, True)
        oc.encode(v, 0, False)
        dt = time.perf_counter() - t0
        return dt, 2 * 1024 * D * 2, "bytes", "1 layer x 1 head x 1024 tokens, bits 3, K+V encode"
    if wl_name == "shared_prefix":
        w = W.shared_prefix(device="cpu", agents=1, prefix_tokens=1024, tail_tokens=256, data_seed=5 + rank_seed)
        pc, tc = oracle.Codec(D, 2, M, 42), oracle.Codec(D, 4, M, 42)
        t0 = time.perf_counter()
        ekp = pc.encode(w["prefix_k"][0, 0].double().numpy(), 0, True)
        evp = pc.encode(w["prefix_v"][0, 0].double().numpy(), 0, False)
        ekt = tc.encode(w["tail_k"][0, 0].double().numpy(), 0, True)
        evt = tc.encode(w["tail_v"][0, 0].double().numpy(), 0, False)
        for j in range(4):
            oracle.attention(w["q"][0, j].double().numpy(),
                             [(pc, 0, ekp["rows"], evp["rows"]), (tc, 0, ekt["rows"], evt["rows"])])
        dt = time.perf_counter() - t0
        return dt, 4 * (1024 + 256), "tokens", "1 agent x 1 kv head (4 q heads), prefix 1024 + tail 256 tokens"
    if wl_name == "mha_split":
        w = W.mha_decode(device="cpu", batch=1, heads=1, n_tokens=512, data_seed=2 + rank_seed)
        order = w["k"][0, 0].pow(2).mean(dim=0).argsort(descending=True)
        k, v, q = (w["k"][0, 0][:, order].double().numpy(), w["v"][0, 0][:, order].double().numpy(),
                   w["q"][0, 0][order].double().numpy())
        oo, on = oracle.Codec(64, 4, 64, w["seed"]), oracle.Codec(64, 3, 64, w["seed"] + 1000)
        t0 = time.perf_counter()
        eko, evo = oo.encode(k[:, :64], 0, True), oo.encode(v[:, :64], 0, False)
        ekn, evn = on.encode(k[:, 64:], 0, True), on.encode(v[:, 64:], 0, False)
        oracle.attention_split(q, (oo, 0, eko["rows"], evo["rows"]), (on, 0, ekn["rows"], evn["rows"]))
        dt = time.perf_counter() - t0
        return dt, 512, "tokens", "1 kv head x 1 query head x 512 tokens: encode both channel groups + split decode"
    if wl_name == "mha_append":
        w = W.mha_decode(device="cpu", batch=1, heads=1, n_tokens=1025, data_seed=2 + rank_seed)
        oc = oracle.Codec(D, w["bits"], M, w["seed"])
        k, v = w["k"][0, 0].double().numpy(), w["v"][0, 0].double().numpy()
        ek, ev = oc.encode(k[:1024], 0, True), oc.encode(v[:1024], 0, False)     # the cached history
        t0 = time.perf_counter()
        nk, nv = oc.encode(k[1024:], 0, True), oc.encode(v[1024:], 0, False)
        oracle.attention(w["q"][0, 0].double().numpy(),
                         [(oc, 0, np.concatenate([ek["rows"], nk["rows"]]), np.concatenate([ev["rows"], nv["rows"]]))])
        dt = time.perf_counter() - t0
        return dt, 1025, "tokens", "1 kv head x 1 query head: append 1 token to 1024 + decode over 1025"
    if wl_name in ("mha_decode", "mha_decode_haar", "mha_decode_f16norms"):
        w = W.mha_decode(device="cpu", batch=1, heads=1, n_tokens=1024, data_seed=2 + rank_seed)
        G = 1
    elif wl_name == "gqa_decode":
        w = W.gqa_decode(device="cpu", batch=1, q_heads=4, kv_heads=1, n_tokens=1024, data_seed=3 + rank_seed)
        G = 4
    else:
        w = W.single_head(device="cpu", data_seed=1 + rank_seed)
        G = 4
    oc = oracle.Codec(D, w["bits"], M, w["seed"], rotation="haar" if wl_name == "mha_decode_haar" else "hadamard",
                      norms="f16" if wl_name == "mha_decode_f16norms" else "f32")
    T = w["k"].shape[2]
    t0 = time.perf_counter()
    ek = oc.encode(w["k"][0, 0].double().numpy(), 0, True)
    ev = oc.encode(w["v"][0, 0].double().numpy(), 0, False)
    for j in range(G):
        oracle.attention(w["q"][0, j].double().numpy(), [(oc, 0, ek["rows"], ev["rows"])])
    dt = time.perf_counter() - t0
    return dt, G * T, "tokens", f"1 kv head x {G} query head(s) x {T} tokens: encode K+V + decode"


def _oracle_loop(wl_name, seconds, worker):
    """Run oracle units of the workload for about `seconds` of CPU time
    (worker w takes data seeds shifted by 1000 w); returns (seconds, units,
    unit, desc, count)."""
    try:
        import torch
        torch.set_num_threads(1)
    except Exception:
        pass
    tot_t, tot_u, n = 0.0, 0, 0
    unit = desc = None
    while tot_t < seconds or n == 0:
        dt, u, unit, desc = oracle_unit(wl_name, rank_seed=1000 * worker + n)
        tot_t += dt
        tot_u += u
        n += 1
    return tot_t, tot_u, unit, desc, n


def host_cpu():
    """(usable cores, CPU model) of this host."""
    try:
        cores = len(os.sched_getaffinity(0))
    except Exception:
        cores = os.cpu_count() or 1
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return cores, model


def _baseline_entry(val, unit, cores, sample):
    if unit == "bytes":
        return {"value": val / 1e9, "unit": "GB/s in", "cores": cores, "kind": "oracle", "sample": sample}
    return {"value": val, "unit": "KV tokens scored/s", "cores": cores, "kind": "oracle", "sample": sample}


def cpu_baseline(wl_name, seconds, all_cores=True, max_workers=96):
    """The oracle timed on the host: single-threaded, and (all_cores) one
    process per core over independent (sequence, head) units, each process
    running its own units for about `seconds`; the all-core value is the sum
    of the processes' own rates (they run at the same time).  Processes are
    started with `spawn` (never forked from a process that used the GPU)."""
    ncores, model = host_cpu()
    t1, u1, unit, desc, n1 = _oracle_loop(wl_name, seconds, 0)
    single = _baseline_entry(u1 / t1, unit, 1, f"{n1} x ({desc}), {t1:.1f} s, single-threaded fp64 C oracle")
    single["cpu_model"] = model
    single["nproc"] = ncores
    if not all_cores or ncores <= 1:
        return single
    import concurrent.futures as cf
    import multiprocessing as mp
    workers = min(ncores, max_workers)
    with cf.ProcessPoolExecutor(max_workers=workers, mp_context=mp.get_context("spawn")) as ex:
        res = list(ex.map(_oracle_loop, [wl_name] * workers, [seconds] * workers, range(1, workers + 1)))
    rate = sum(u / t for t, u, _, _, _ in res)
    nall = sum(r[4] for r in res)
    tall = max(r[0] for r in res)
    multi = _baseline_entry(rate, unit, workers,
                            f"{workers} processes x about {tall:.1f} s each, {nall} units of ({desc}) in total, "
                            f"fp64 C oracle, one process per core over independent (sequence, head) units")
    multi["cpu_model"] = model
    multi["nproc"] = ncores
    multi["single_thread"] = single
    return multi


def _oracle_units(wl_name, n, seed0):
    """n oracle units of the workload (data seeds seed0, seed0 + 1, ...): (seconds, units, unit, desc);
    seconds counts the oracle's work only, not the input generation."""
    try:
        import torch
        torch.set_num_threads(1)
    except Exception:
        pass
    tot_t, tot_u = 0.0, 0
    unit = desc = None
    for i in range(n):
        dt, u, unit, desc = oracle_unit(wl_name, rank_seed=seed0 + i)
        tot_t += dt
        tot_u += u
    return tot_t, tot_u, unit, desc


def run_reference(args):
    """The oracle, as it stands, on the host's cores: one process per core
    (spawned), each step every process runs `--ref-units` oracle units of the
    workload on its own seeds.  A step's time is the slowest process's oracle
    time in that step (input generation excluded); value = all units / the
    sum of the step times.  Rank 0 alone runs it; other ranks exit without
    work."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import concurrent.futures as cf
    import multiprocessing as mp
    ncores, model = host_cpu()
    workers = max(1, min(ncores, args.ref_workers))
    per = max(1, args.ref_units)
    tot_t, tot_u, unit, desc = 0.0, 0, None, None
    with cf.ProcessPoolExecutor(max_workers=workers, mp_context=mp.get_context("spawn")) as ex:
        def one_step(i):
            seeds = [per * (workers * i + w) for w in range(workers)]
            res = list(ex.map(_oracle_units, [args.workload] * workers, [per] * workers, seeds))
            return max(r[0] for r in res), sum(r[1] for r in res), res[0][2], res[0][3]
        for i in range(args.warmup):
            one_step(i)
        for i in range(args.steps):
            dt, u, unit, desc = one_step(args.warmup + i)
            tot_t += dt
            tot_u += u
    val = tot_u / tot_t
    unit_name = "GB/s in" if unit == "bytes" else "KV tokens scored/s"
    if unit == "bytes":
        val /= 1e9
    sample = (f"{args.steps} timed steps; each step {workers} processes x {per} unit(s) of ({desc}), "
              f"fp64 C oracle, one process per core")
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": unit_name, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * tot_t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(arm_config(args.workload), oracle_sample=desc),
            "cpu_baseline": {"value": val, "unit": unit_name, "cores": workers, "kind": "oracle", "sample": sample,
                             "nproc": ncores, "cpu_model": model},
            "e2e": {"value": val, "unit": unit_name, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------ timing helpers

CONFIG_WORKLOADS = ["mha_decode", "gqa_decode", "bulk_encode", "shared_prefix"]


def piece_table(wl, piece_samples, hbm, peak_kind):
    """Per piece: mean, median and best of its event times, algorithmic bytes,
    achieved GB/s (from the mean) and the fraction of the HBM peak."""
    kernels = {}
    for (name, nbytes, nl), xs in zip(wl.pieces, piece_samples):
        srt = sorted(xs)
        ms = sum(xs) / len(xs)
        gbs = nbytes / (ms * 1e-3) / 1e9
        kernels[name] = {"ms": ms, "ms_median": srt[len(srt) // 2], "ms_best": srt[0], "iterations": len(xs),
                         "launches": nl, "algorithmic_bytes": nbytes, "achieved_gbs": gbs,
                         "frac_of_" + peak_kind + "_hbm": gbs / hbm,
                         "frac_best_of_" + peak_kind + "_hbm": nbytes / (srt[0] * 1e-3) / 1e9 / hbm,
                         "traffic": measured_traffic(name, wl.name)}
        if name.startswith("decode"):
            kernels[name]["kv_tokens_scored_per_s"] = wl.tokens_scored / (ms * 1e-3)
    return kernels


def time_config(name, dev, steps, warmup):
    """Time one workload's pieces (L2 flushed before each, CUDA events on the
    launching stream) over `steps` steps after `warmup`; returns its entry of
    the `configs` key.  The workload's tensors are released afterwards."""
    import torch
    wl = Workload(name, dev, 0)
    inp = wl.inputs
    for _ in range(warmup):
        wl.step(inp)
    torch.cuda.synchronize()
    n = len(wl.pieces)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * n)] for _ in range(steps)]
    for i in range(steps):
        wl.step(inp, evs[i])
    torch.cuda.synchronize()
    samples = [[e[2 * p].elapsed_time(e[2 * p + 1]) for e in evs] for p in range(n)]
    ms_step = sum(sum(x) / steps for x in samples)
    kernels = piece_table(wl, samples, 1.0, "unit")
    for k in kernels.values():           # fractions are filled in against the peak by the caller
        k.pop("frac_of_unit_hbm")
        k.pop("frac_best_of_unit_hbm")
    if name == "bulk_encode":
        value, unit = wl.in_bytes / (ms_step * 1e-3) / 1e9, "GB/s in"
    else:
        value, unit = wl.tokens_scored / (ms_step * 1e-3), "KV tokens scored/s"
    dom = max(kernels, key=lambda k: kernels[k]["ms"])
    out = {"workload": WORKLOAD_DESC[name], "step": STEP_DESC[name], "value": value, "unit": unit,
           "ms_per_step": ms_step, "steps": steps, "warmup": warmup, "dominant_kernel": dom, "kernels": kernels,
           "gpu_launches": wl.launches * steps}
    del wl, inp
    torch.cuda.empty_cache()
    return out


# -------------------------------------------------------------------- main

def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    wl = Workload(args.workload, dev, rank)
    inp = wl.inputs
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()

    for w in range(max(args.warmup, 3)):
        wl.step(inp)
        if w == 0 and args.graphs:
            wl.capture(inp)               # later warm-up and timed steps replay the graphs
    torch.cuda.synchronize()
    # timed region: every piece of every step between its own CUDA events on
    # the launching stream; L2 is flushed before each piece, outside them
    npieces = len(wl.pieces)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * npieces)] for _ in range(args.steps)]
    smi, rows = clock_sampler(dev.index)
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        wl.step(inp, evs[i])
    torch.cuda.synchronize()
    barrier()
    piece_samples = [[e[2 * p].elapsed_time(e[2 * p + 1]) for e in evs] for p in range(npieces)]
    piece_ms = [sum(x) / args.steps for x in piece_samples]
    ms_step = max_over_ranks(sum(piece_ms), world, dev)

    # the other workloads, each timed in the same run (one GPU only)
    configs = None
    if world == 1 and not args.no_configs:
        configs = {}
        for other in CONFIG_WORKLOADS:
            if other == args.workload:
                continue
            configs[other] = time_config(other, dev, max(args.steps, 50), max(args.warmup, 5))
    if smi is not None:
        time.sleep(0.25)
        smi.terminate()
    clocks = summarize_clocks(rows)

    # end to end through host buffers
    e2e = None
    if not args.no_e2e:
        host = {k: v.cpu().pin_memory() for k, v in inp.items()}
        dev_bufs = {k: torch.empty_like(v) for k, v in inp.items()}
        out_host = torch.empty(wl.B, wl.Hq, D, dtype=inp["q"].dtype).pin_memory() if "q" in inp else None
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = out_host.numel() * out_host.element_size() if out_host is not None else 0
        e_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(10)]

        def e2e_step(ev=None):
            if wl.flush is not None:
                wl.flush.zero_()
            if ev:
                ev[0].record()
            for k2, v2 in host.items():
                dev_bufs[k2].copy_(v2, non_blocking=True)
            saved = wl.flush
            wl.flush = None
            o = wl.step(dev_bufs)
            wl.flush = saved
            if out_host is not None:
                out_host.copy_(o, non_blocking=True)
            if ev:
                ev[1].record()
        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        barrier()
        n_e2e = max(3, min(args.steps, 10))
        for i in range(n_e2e):
            e2e_step(e_evs[i])
        torch.cuda.synchronize()
        e_ms = sum(e_evs[i][0].elapsed_time(e_evs[i][1]) for i in range(n_e2e)) / n_e2e
        e_ms = max_over_ranks(e_ms, world, dev)
        if wl.name == "bulk_encode":
            ev, eu = job_throughput(wl.in_bytes, world, e_ms * 1e-3) / 1e9, "GB/s in"
        else:
            ev, eu = job_throughput(wl.tokens_scored, world, e_ms * 1e-3), "KV tokens scored/s"
        e2e = {"value": ev, "unit": eu, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms}

    hbm, peak_kind = peaks()
    if wl.name == "bulk_encode":
        value, unit = job_throughput(wl.in_bytes, world, ms_step * 1e-3) / 1e9, "GB/s in"
    else:
        value, unit = job_throughput(wl.tokens_scored, world, ms_step * 1e-3), "KV tokens scored/s"
    kernels = piece_table(wl, piece_samples, hbm, peak_kind)
    dom = max(kernels, key=lambda k: kernels[k]["ms"])
    dk = kernels[dom]
    roofline = {"kernel": dom, "bound": "hbm", "achieved": dk["achieved_gbs"], "peak": hbm, "unit": "GB/s",
                "frac": dk["achieved_gbs"] / hbm, "peak_source": peak_kind + " (MEASURED_PEAKS.json hbm_gbs)",
                "traffic": measured_traffic(dom, wl.name)}
    line = {"metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": dict(arm_config(wl.name),
                           launch="each piece replayed from a captured CUDA graph" if args.graphs else "eager"),
            "roofline": roofline, "kernels": kernels, "gpu_launches": wl.launches * args.steps,
            "clocks": clocks, "e2e": e2e}
    if configs is not None:
        for c in configs.values():
            c["peak_gbs"] = hbm
            for k2, v2 in c["kernels"].items():
                v2["frac_of_" + peak_kind + "_hbm"] = v2["achieved_gbs"] / hbm
                v2["frac_best_of_" + peak_kind + "_hbm"] = v2["algorithmic_bytes"] / (v2["ms_best"] * 1e-3) / 1e9 / hbm
        line["configs"] = configs
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload, args.cpu_seconds, all_cores=not args.cpu_single)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
