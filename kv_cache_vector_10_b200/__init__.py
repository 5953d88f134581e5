"""kv_cache_vector_10_b200 -- TurboQuant KV-cache codec and compressed-KV
decode attention on NVIDIA B200 (sm_100a).

This module is a thin ctypes binding over ``lib/libtq.so`` (C ABI declared in
``include/tq.h``).  It only marshals arguments: tensors are passed as device
pointers (``tensor.data_ptr()``) together with torch's current CUDA stream;
every step of encode, scoring, dequantization and decode runs in the
library's kernels.  There is no CPU fallback: importing on a machine without
the built library raises, and calls on a non-sm_100 device fail with
``TQ_ERR_DEVICE``.

Names follow the C ABI (``tq_create``, ``tq_encode_kv``,
``tq_attention_scores``, ``tq_decode_attention``, ``tq_dequantize``).  The
``Codec`` / ``PackedCache`` / ``Segment`` classes are conveniences on top.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libtq.so")

TQ_OK = 0
TQ_F32, TQ_F16, TQ_BF16 = 0, 1, 2
TQ_KEYS, TQ_VALUES, TQ_BOTH = 0, 1, 2
TQ_ROT_HADAMARD, TQ_ROT_HAAR = 0, 1
ROTATIONS = {"hadamard": TQ_ROT_HADAMARD, "haar": TQ_ROT_HAAR}
TQ_NORMS_F32, TQ_NORMS_F16 = 0, 1
NORM_FORMATS = {"f32": TQ_NORMS_F32, "f16": TQ_NORMS_F16}
TQ_MAX_SEGMENTS = 64

STATUS_NAMES = {0: "TQ_OK", 1: "TQ_ERR_NULL", 2: "TQ_ERR_ZERO_DIM", 3: "TQ_ERR_DIM", 4: "TQ_ERR_BITS",
                5: "TQ_ERR_ZERO_PROJ", 6: "TQ_ERR_PROJ", 7: "TQ_ERR_EMPTY", 8: "TQ_ERR_DIM_MISMATCH",
                9: "TQ_ERR_WORKSPACE", 10: "TQ_ERR_ALIGN", 11: "TQ_ERR_CUDA", 12: "TQ_ERR_DEVICE",
                13: "TQ_ERR_LIMIT"}

EXPORTED = ["tq_create", "tq_create_ex", "tq_create_format", "tq_destroy", "tq_ensure_heads", "tq_row_bytes", "tq_packed_bytes", "tq_encode_kv",
            "tq_attention_scores", "tq_dequantize", "tq_decode_workspace_bytes", "tq_decode_launch_count",
            "tq_decode_attention",
            "tq_get_status", "tq_reset_status", "tq_status_string", "tq_last_cuda_error",
            "tq_decode_attention_static", "tq_decode_append", "tq_decode_append_workspace_bytes",
            "tq_selftest_wait_timeout", "tq_decode_attention_split", "tq_decode_split_workspace_bytes"]


class TQError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = f"{where}: {STATUS_NAMES.get(code, code)}"
        if code == 11 and _lib is not None:
            msg += f" ({_lib.tq_last_cuda_error().decode()})"
        super().__init__(msg)


class tq_codes(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("batch", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("capacity", ctypes.c_int64)]


class tq_segment(ctypes.Structure):
    _fields_ = [("ctx", ctypes.c_void_p), ("codes", tq_codes), ("codes_batch", ctypes.c_int32),
                ("first_seq", ctypes.c_int32), ("n_seqs", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("n_tokens", ctypes.c_int64)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python kv_cache_vector_10_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    V, I, I64, SZ, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_uint64
    sig = {
        "tq_create": (I, [I, I, I, U64, ctypes.POINTER(V)]),
        "tq_create_ex": (I, [I, I, I, U64, I, ctypes.POINTER(V)]),
        "tq_create_format": (I, [I, I, I, U64, I, I, ctypes.POINTER(V)]),
        "tq_destroy": (None, [V]),
        "tq_ensure_heads": (I, [V, I]),
        "tq_row_bytes": (I64, [V, I]),
        "tq_packed_bytes": (SZ, [V, I, I, I64, I]),
        "tq_encode_kv": (I, [V, V, V, I, I, I, I64, I64, I64, I64, ctypes.POINTER(tq_codes), I64, V]),
        "tq_attention_scores": (I, [V, ctypes.POINTER(tq_codes), V, I, I64, V, V]),
        "tq_dequantize": (I, [V, ctypes.POINTER(tq_codes), I64, V, V, V]),
        "tq_decode_workspace_bytes": (SZ, [ctypes.POINTER(tq_segment), I, I, I, I]),
        "tq_decode_launch_count": (I, [ctypes.POINTER(tq_segment), I, I, I, I]),
        "tq_decode_attention": (I, [ctypes.POINTER(tq_segment), I, V, I, I, I, I, V, I, V, SZ, V]),
        "tq_decode_attention_static": (I, [ctypes.POINTER(tq_segment), I, V, I, I, I, I, V, I, V]),
        "tq_decode_append": (I, [ctypes.POINTER(tq_segment), I, V, V, I, V, I, I, I, I, V, I, V, SZ, V]),
        "tq_decode_append_workspace_bytes": (SZ, [ctypes.POINTER(tq_segment), I, I, I, I]),
        "tq_get_status": (I, [V, V, ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(ctypes.c_uint32)]),
        "tq_reset_status": (I, [V, V]),
        "tq_selftest_wait_timeout": (I, [V, ctypes.c_uint32, V]),
        "tq_decode_split_workspace_bytes": (SZ, [V, V, I, I, I64]),
        "tq_decode_attention_split": (I, [V, ctypes.POINTER(tq_codes), V, ctypes.POINTER(tq_codes), I64, V, I, I, I,
                                          V, I, V, SZ, V]),
        "tq_status_string": (ctypes.c_char_p, [I]),
        "tq_last_cuda_error": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()
lib = _lib


def _check(code: int, where: str):
    if code != TQ_OK:
        raise TQError(code, where)


def _stream(stream=None):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(dt) -> int:
    import torch
    return {torch.float32: TQ_F32, torch.float16: TQ_F16, torch.bfloat16: TQ_BF16}[dt]


# ---------------------------------------------------------------- C ABI names

def tq_create(head_dim: int, bits: int, projections: int, seed: int) -> int:
    out = ctypes.c_void_p()
    _check(_lib.tq_create(head_dim, bits, projections, seed & 0xFFFFFFFFFFFFFFFF, ctypes.byref(out)), "tq_create")
    return out.value


def tq_create_ex(head_dim: int, bits: int, projections: int, seed: int, rotation: int) -> int:
    out = ctypes.c_void_p()
    _check(_lib.tq_create_ex(head_dim, bits, projections, seed & 0xFFFFFFFFFFFFFFFF, rotation, ctypes.byref(out)),
           "tq_create_ex")
    return out.value


def tq_create_format(head_dim: int, bits: int, projections: int, seed: int, rotation: int, key_norms: int) -> int:
    out = ctypes.c_void_p()
    _check(_lib.tq_create_format(head_dim, bits, projections, seed & 0xFFFFFFFFFFFFFFFF, rotation, key_norms,
                                 ctypes.byref(out)), "tq_create_format")
    return out.value


def tq_destroy(ctx: int) -> None:
    _lib.tq_destroy(ctx)


def tq_ensure_heads(ctx: int, n_heads: int) -> None:
    _check(_lib.tq_ensure_heads(ctx, n_heads), "tq_ensure_heads")


def tq_row_bytes(ctx: int, which: int) -> int:
    return _lib.tq_row_bytes(ctx, which)


def tq_packed_bytes(ctx: int, batch: int, n_kv_heads: int, capacity: int, which: int) -> int:
    return _lib.tq_packed_bytes(ctx, batch, n_kv_heads, capacity, which)


def tq_encode_kv(ctx: int, k, v, batch: int, n_kv_heads: int, n_tokens: int, codes: "PackedCache",
                 token_offset: int = 0, stream=None) -> None:
    """k, v: CUDA tensors [batch, n_kv_heads, n_tokens, d] (any strides with a
    contiguous last dim); either may be None."""
    ref = k if k is not None else v
    sb, sh, st, sd = ref.stride()
    if sd != 1:
        raise ValueError("last dimension must be contiguous")
    if k is not None and v is not None and (k.stride() != v.stride() or k.dtype != v.dtype):
        raise ValueError("k and v must share dtype and strides")
    c = codes.struct()
    _check(_lib.tq_encode_kv(ctx, k.data_ptr() if k is not None else None, v.data_ptr() if v is not None else None,
                             _dtype_code(ref.dtype), batch, n_kv_heads, n_tokens, sb, sh, st, ctypes.byref(c),
                             token_offset, _stream(stream)), "tq_encode_kv")


def tq_attention_scores(ctx: int, codes: "PackedCache", q, n_q_heads: int, n_tokens: int, scores, stream=None):
    c = codes.struct()
    _check(_lib.tq_attention_scores(ctx, ctypes.byref(c), q.data_ptr(), n_q_heads, n_tokens, scores.data_ptr(),
                                    _stream(stream)), "tq_attention_scores")


def tq_dequantize(ctx: int, codes: "PackedCache", n_tokens: int, k_hat=None, v_hat=None, stream=None):
    c = codes.struct()
    _check(_lib.tq_dequantize(ctx, ctypes.byref(c), n_tokens, k_hat.data_ptr() if k_hat is not None else None,
                              v_hat.data_ptr() if v_hat is not None else None, _stream(stream)), "tq_dequantize")


def _segment_array(segments):
    arr = (tq_segment * len(segments))()
    for i, s in enumerate(segments):
        arr[i].ctx = s.codec.ctx
        arr[i].codes = s.cache.struct()
        arr[i].codes_batch = s.codes_batch
        arr[i].first_seq = s.first_seq
        arr[i].n_seqs = s.n_seqs
        arr[i].n_tokens = s.n_tokens
    return arr


def tq_decode_workspace_bytes(segments, batch: int, n_q_heads: int, n_kv_heads: int) -> int:
    arr = _segment_array(segments)
    return _lib.tq_decode_workspace_bytes(arr, len(segments), batch, n_q_heads, n_kv_heads)


def tq_decode_launch_count(segments, batch: int, n_q_heads: int, n_kv_heads: int) -> int:
    """Kernels one decode call with these segments launches (host-only)."""
    arr = _segment_array(segments)
    return _lib.tq_decode_launch_count(arr, len(segments), batch, n_q_heads, n_kv_heads)


def tq_decode_attention(segments, q, batch: int, n_q_heads: int, n_kv_heads: int, out, workspace, stream=None):
    arr = _segment_array(segments)
    _check(_lib.tq_decode_attention(arr, len(segments), q.data_ptr(), _dtype_code(q.dtype), batch, n_q_heads,
                                    n_kv_heads, out.data_ptr(), _dtype_code(out.dtype), workspace.data_ptr(),
                                    workspace.numel() * workspace.element_size(), _stream(stream)),
           "tq_decode_attention")


def tq_decode_attention_static(segments, q, batch: int, n_q_heads: int, n_kv_heads: int, out, stream=None):
    """Decode attention with the library's built-in scratch array (no allocation,
    no workspace argument); see include/tq.h for its limits and sharing rules."""
    arr = _segment_array(segments)
    _check(_lib.tq_decode_attention_static(arr, len(segments), q.data_ptr(), _dtype_code(q.dtype), batch, n_q_heads,
                                           n_kv_heads, out.data_ptr(), _dtype_code(out.dtype), _stream(stream)),
           "tq_decode_attention_static")


def tq_decode_append_workspace_bytes(segments, batch: int, n_q_heads: int, n_kv_heads: int) -> int:
    arr = _segment_array(segments)
    return _lib.tq_decode_append_workspace_bytes(arr, len(segments), batch, n_q_heads, n_kv_heads)


def tq_decode_append(segments, k_new, v_new, q, batch: int, n_q_heads: int, n_kv_heads: int, out, workspace,
                     stream=None):
    arr = _segment_array(segments)
    if k_new.dtype != v_new.dtype:
        raise TQError(8, "tq_decode_append")
    _check(_lib.tq_decode_append(arr, len(segments), k_new.data_ptr(), v_new.data_ptr(), _dtype_code(k_new.dtype),
                                 q.data_ptr(), _dtype_code(q.dtype), batch, n_q_heads, n_kv_heads, out.data_ptr(),
                                 _dtype_code(out.dtype), workspace.data_ptr(),
                                 workspace.numel() * workspace.element_size(), _stream(stream)),
           "tq_decode_append")


def tq_get_status(ctx: int, stream=None):
    n = ctypes.c_uint64()
    f = ctypes.c_uint32()
    _check(_lib.tq_get_status(ctx, _stream(stream), ctypes.byref(n), ctypes.byref(f)), "tq_get_status")
    return n.value, f.value


def tq_selftest_wait_timeout(ctx: int, timeout_us: int, stream=None):
    """Make one bounded wait run out on purpose (see include/tq.h)."""
    _check(_lib.tq_selftest_wait_timeout(ctx, timeout_us, _stream(stream)), "tq_selftest_wait_timeout")


def tq_reset_status(ctx: int, stream=None):
    _check(_lib.tq_reset_status(ctx, _stream(stream)), "tq_reset_status")


# -------------------------------------------------------------- conveniences

class Codec:
    """A codec context: KvCacheConfig {head_dim, bits, projections, seed}, the
    rotation ("hadamard": FWHT with random signs; "haar": QR rotation) and the
    key-norm storage ("f32", or "f16": n_s and gamma as binary16)."""

    def __init__(self, head_dim: int, bits: int, projections: int, seed: int, rotation: str = "hadamard",
                 norms: str = "f32"):
        self.head_dim, self.bits, self.projections, self.seed = head_dim, bits, projections, seed
        self.rotation = rotation
        self.norms = norms
        self.ctx = tq_create_format(head_dim, bits, projections, seed, ROTATIONS[rotation], NORM_FORMATS[norms])
        self.k_row_bytes = tq_row_bytes(self.ctx, TQ_KEYS)
        self.v_row_bytes = tq_row_bytes(self.ctx, TQ_VALUES)

    def close(self):
        if self.ctx:
            tq_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def alloc(self, batch: int, n_kv_heads: int, capacity: int, device="cuda") -> "PackedCache":
        return PackedCache(self, batch, n_kv_heads, capacity, device)

    def encode_kv(self, k, v, cache: "PackedCache", token_offset: int = 0, stream=None):
        ref = k if k is not None else v
        B, H, T, _ = ref.shape
        tq_encode_kv(self.ctx, k, v, B, H, T, cache, token_offset, stream)

    def attention_scores(self, cache, q, n_tokens: int, stream=None):
        import torch
        B, Hq, _ = q.shape
        scores = torch.empty(B, Hq, n_tokens, dtype=torch.float32, device=q.device)
        tq_attention_scores(self.ctx, cache, q.float().contiguous(), Hq, n_tokens, scores, stream)
        return scores

    def dequantize(self, cache, n_tokens: int, keys: bool = True, values: bool = True, stream=None):
        import torch
        shp = (cache.batch, cache.n_kv_heads, n_tokens, self.head_dim)
        kh = torch.empty(shp, dtype=torch.float32, device=cache.k.device) if keys else None
        vh = torch.empty(shp, dtype=torch.float32, device=cache.k.device) if values else None
        tq_dequantize(self.ctx, cache, n_tokens, kh, vh, stream)
        return kh, vh

    def status(self, stream=None):
        return tq_get_status(self.ctx, stream)


class PackedCache:
    """Device buffers of packed K and V rows, [batch][n_kv_heads][capacity][row bytes]."""

    def __init__(self, codec: Codec, batch: int, n_kv_heads: int, capacity: int, device="cuda"):
        import torch
        if capacity % 16:
            raise ValueError("capacity must be a multiple of 16")
        self.codec, self.batch, self.n_kv_heads, self.capacity = codec, batch, n_kv_heads, capacity
        self.k = torch.zeros(batch, n_kv_heads, capacity, codec.k_row_bytes, dtype=torch.uint8, device=device)
        self.v = torch.zeros(batch, n_kv_heads, capacity, codec.v_row_bytes, dtype=torch.uint8, device=device)

    def struct(self) -> tq_codes:
        return tq_codes(self.k.data_ptr(), self.v.data_ptr(), self.batch, self.n_kv_heads, self.capacity)


class Segment:
    """Tokens [0, n_tokens) of batch slot `codes_batch` of `cache`, attended by
    sequences [first_seq, first_seq + n_seqs)."""

    def __init__(self, cache: PackedCache, n_tokens: int, first_seq: int, n_seqs: int = 1, codes_batch: int = 0):
        self.cache, self.codec = cache, cache.codec
        self.n_tokens, self.first_seq, self.n_seqs, self.codes_batch = n_tokens, first_seq, n_seqs, codes_batch


def decode_attention(segments, q, n_kv_heads: int, out_dtype=None, workspace=None, stream=None):
    """One decode step; q: [batch, n_q_heads, d] CUDA tensor."""
    import torch
    B, Hq, d = q.shape
    out = torch.empty(B, Hq, d, dtype=out_dtype or q.dtype, device=q.device)
    need = tq_decode_workspace_bytes(segments, B, Hq, n_kv_heads)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    tq_decode_attention(segments, q.contiguous(), B, Hq, n_kv_heads, out, workspace, stream)
    return out


def decode_append(segments, k_new, v_new, q, n_kv_heads: int, out_dtype=None, workspace=None, stream=None):
    """One decode step that first appends this step's rows: k_new, v_new
    [batch, n_kv_heads, d] go to token n_tokens of each sequence's private
    tail segment, which is then attended over n_tokens + 1 tokens.  The
    Segment objects are advanced (n_tokens += 1) after the call is enqueued."""
    import torch
    B, Hq, d = q.shape
    out = torch.empty(B, Hq, d, dtype=out_dtype or q.dtype, device=q.device)
    need = tq_decode_append_workspace_bytes(segments, B, Hq, n_kv_heads)
    if need == 0:
        raise TQError(8, "decode_append")
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    tq_decode_append(segments, k_new.contiguous(), v_new.contiguous(), q.contiguous(), B, Hq, n_kv_heads, out,
                     workspace, stream)
    for s in segments:
        if s.n_seqs == 1:
            s.n_tokens += 1
    return out


def decode_split(codec_o, cache_o, codec_n, cache_n, n_tokens: int, q, out_dtype=None, workspace=None,
                 stream=None):
    """Decode attention over an outlier/normal channel-split cache: q [batch,
    n_q_heads, d_o + d_n] with the outlier channels first; cache_o / cache_n
    hold the two groups' codes (codecs codec_o / codec_n)."""
    import torch
    B, Hq, d = q.shape
    out = torch.empty(B, Hq, d, dtype=out_dtype or q.dtype, device=q.device)
    need = _lib.tq_decode_split_workspace_bytes(codec_o.ctx, codec_n.ctx, B, Hq, n_tokens)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    qc = q.contiguous()
    co, cn = cache_o.struct(), cache_n.struct()
    _check(_lib.tq_decode_attention_split(codec_o.ctx, ctypes.byref(co), codec_n.ctx, ctypes.byref(cn), n_tokens,
                                          qc.data_ptr(), _dtype_code(qc.dtype), B, Hq, out.data_ptr(),
                                          _dtype_code(out.dtype), workspace.data_ptr(),
                                          workspace.numel() * workspace.element_size(), _stream(stream)),
           "tq_decode_attention_split")
    return out


class KvCache:
    """Multi-head compressed KV cache with the call shapes of bitpolar's
    KvCacheCompressor / MultiHeadKvCache (bitpolar 0.3.3 src/kv_cache.rs):
    push (append one or more tokens for every head), len / is_empty,
    attention_scores (pre-softmax, scaled by 1/sqrt(head_dim)),
    decode_values, compression_ratio (original fp32 bytes / packed bytes) and
    clear.  Head h uses seed + h.  Only bookkeeping lives here (the token
    count); every computation is a libtq call.  Batch 1; capacity fixed at
    construction (a multiple of 16)."""

    def __init__(self, num_heads: int, head_dim: int, bits: int, projections: int, seed: int,
                 capacity: int = 1024, device="cuda"):
        if num_heads <= 0:
            raise TQError(7, "KvCache")                      # TQ_ERR_EMPTY, bitpolar EmptyInput
        self.codec = Codec(head_dim, bits, projections, seed)
        self.num_heads, self.head_dim = num_heads, head_dim
        self.cache = self.codec.alloc(1, num_heads, capacity, device)
        self._len = 0

    def push(self, keys, values, stream=None):
        """keys, values: [num_heads, head_dim] (one token) or [num_heads, T, head_dim]."""
        k = keys if keys.dim() == 3 else keys[:, None, :]
        v = values if values.dim() == 3 else values[:, None, :]
        if k.shape[0] != self.num_heads or v.shape != k.shape or k.shape[-1] != self.head_dim:
            raise TQError(8, "KvCache.push")                 # TQ_ERR_DIM_MISMATCH
        self.codec.encode_kv(k[None].contiguous(), v[None].contiguous(), self.cache, self._len, stream)
        self._len += k.shape[1]

    def __len__(self):
        return self._len

    def is_empty(self) -> bool:
        return self._len == 0

    def attention_scores(self, queries, stream=None):
        """queries: [num_heads, head_dim] -> scores [num_heads, len]."""
        if queries.shape != (self.num_heads, self.head_dim):
            raise TQError(8, "KvCache.attention_scores")
        return self.codec.attention_scores(self.cache, queries[None], self._len, stream)[0]

    def decode_values(self, stream=None):
        """-> [num_heads, len, head_dim] reconstructed values."""
        _, vh = self.codec.dequantize(self.cache, self._len, keys=False, values=True, stream=stream)
        return vh[0]

    def compression_ratio(self) -> float:
        if self._len == 0:
            return 1.0
        original = 2 * self._len * self.num_heads * self.head_dim * 4
        packed = self._len * self.num_heads * (self.codec.k_row_bytes + self.codec.v_row_bytes)
        return original / packed

    def clear(self):
        self._len = 0
