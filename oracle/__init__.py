"""CPU oracle for the TurboQuant KV-cache codec (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the cpu_baseline /
reference arm of ``bench.py`` import this package.  The product package
``kv_cache_vector_10_b200`` never imports it.

The arithmetic lives in ``tq_oracle.c`` (plain fp64 C, see its header for the
passages each step follows); this module only compiles it with gcc, loads it
with ctypes and converts numpy arrays.  ``attention`` and the helpers below
add no arithmetic of their own beyond calling the C functions.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile tq_oracle.c into liboracle.so next to it (gcc, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-fPIC", "-shared",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Cfg(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int), ("bits", ctypes.c_int), ("m", ctypes.c_int),
                ("BK", ctypes.c_int), ("BV", ctypes.c_int), ("LK", ctypes.c_int),
                ("LV", ctypes.c_int), ("norm_correct", ctypes.c_int),
                ("ck", ctypes.c_double * 64), ("bk", ctypes.c_double * 64),
                ("cv", ctypes.c_double * 64), ("bv", ctypes.c_double * 64),
                ("rotation", ctypes.c_int), ("norm_f16", ctypes.c_int)]

ROTATIONS = {"hadamard": 0, "haar": 1}


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        _lib.tqo_splitmix64_next.restype = ctypes.c_uint64
        _lib.tqo_splitmix64_next.argtypes = [ctypes.POINTER(ctypes.c_uint64)]
        _lib.tqo_round_fp16.restype = ctypes.c_double
        _lib.tqo_round_fp16.argtypes = [ctypes.c_double]
        _lib.tqo_head_tables.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_uint64, ctypes.c_int, P, P]
        _lib.tqo_lloyd_max.restype = ctypes.c_int
        _lib.tqo_lloyd_max.argtypes = [ctypes.c_int, P, P]
        _lib.tqo_fwht.argtypes = [P, ctypes.c_int]
        _lib.tqo_rotate.argtypes = [ctypes.c_int, P, P, P]
        _lib.tqo_unrotate.argtypes = [ctypes.c_int, P, P, P]
        _lib.tqo_haar_matrix.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_uint64, ctypes.c_int, P]
        _lib.tqo_haar_gaussian.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_uint64, ctypes.c_int, P]
        _lib.tqo_rotate_dense.argtypes = [ctypes.c_int, P, P, P]
        _lib.tqo_unrotate_dense.argtypes = [ctypes.c_int, P, P, P]
        _lib.tqo_cfg_init.restype = ctypes.c_int
        _lib.tqo_cfg_init.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
        _lib.tqo_k_row_bytes.restype = ctypes.c_int
        _lib.tqo_k_row_bytes.argtypes = [ctypes.POINTER(_Cfg)]
        _lib.tqo_v_row_bytes.restype = ctypes.c_int
        _lib.tqo_v_row_bytes.argtypes = [ctypes.POINTER(_Cfg)]
        _lib.tqo_encode_block.restype = ctypes.c_int
        _lib.tqo_encode_block.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int, P, P, P, ctypes.c_int64,
                                          P, P, P, P, P]
        _lib.tqo_unpack_k.argtypes = [ctypes.POINTER(_Cfg), P, P, P, P, P]
        _lib.tqo_unpack_v.argtypes = [ctypes.POINTER(_Cfg), P, P, P]
        _lib.tqo_dequant_v.argtypes = [ctypes.POINTER(_Cfg), P, P, P]
        _lib.tqo_dequant_k.argtypes = [ctypes.POINTER(_Cfg), P, P, P, P]
        _lib.tqo_scores_fused.argtypes = [ctypes.POINTER(_Cfg), P, P, P, P, ctypes.c_int64, P]
        _lib.tqo_scores_dequant.argtypes = [ctypes.POINTER(_Cfg), P, P, P, P, ctypes.c_int64, P]
        _lib.tqo_attend.argtypes = [ctypes.c_int, P, P, P, P, P, P, P, P]
        _lib.tqo_attend_split.argtypes = [ctypes.POINTER(_Cfg), P, P, P, P, ctypes.POINTER(_Cfg), P, P, P, P,
                                          ctypes.c_int64, P, P]
        _lib.tqo_streaming_softmax_sum.argtypes = [ctypes.c_int64, ctypes.c_int, P, P, ctypes.c_int64, P]
        _lib.tqo_packed_bytes.restype = ctypes.c_int64
        _lib.tqo_packed_bytes.argtypes = [ctypes.POINTER(_Cfg), ctypes.c_int64]
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


# ----------------------------------------------------------------- primitives

def splitmix64_stream(seed: int, n: int) -> np.ndarray:
    lib = _load()
    st = ctypes.c_uint64(seed & 0xFFFFFFFFFFFFFFFF)
    return np.array([lib.tqo_splitmix64_next(ctypes.byref(st)) for _ in range(n)], dtype=np.uint64)


def round_fp16(x: float) -> float:
    return _load().tqo_round_fp16(float(x))


def lloyd_max(B: int):
    """Centroids (ascending) and boundaries of the 2^B-level Lloyd-Max quantizer of N(0,1)."""
    L = 1 << B
    c = np.zeros(64)
    b = np.zeros(64)
    got = _load().tqo_lloyd_max(B, _p(c), _p(b))
    assert got == L
    return c[:L].copy(), b[:L - 1].copy()


def fwht(v) -> np.ndarray:
    v = _f64(v).copy()
    _load().tqo_fwht(_p(v), v.shape[0])
    return v


def head_tables(d: int, m: int, seed: int, h: int):
    """Random signs [d] and the fp16-valued QJL matrix S [m, d] of head h."""
    signs = np.zeros(d)
    S = np.zeros((m, d))
    _load().tqo_head_tables(d, m, seed & 0xFFFFFFFFFFFFFFFF, h, _p(signs), _p(S))
    return signs, S


def haar_matrix(d: int, m: int, seed: int, h: int) -> np.ndarray:
    """The Haar rotation Q [d, d] of head h (QR of a seeded Gaussian matrix)."""
    Q = np.zeros((d, d))
    _load().tqo_haar_matrix(d, m, seed & 0xFFFFFFFFFFFFFFFF, h, _p(Q))
    return Q


def haar_gaussian(d: int, m: int, seed: int, h: int) -> np.ndarray:
    """The Gaussian matrix G [d, d] whose QR factor is head h's Haar rotation."""
    G = np.zeros((d, d))
    _load().tqo_haar_gaussian(d, m, seed & 0xFFFFFFFFFFFFFFFF, h, _p(G))
    return G


def rotate(rot, x) -> np.ndarray:
    """Pi x: rot is a head's signs [d] (Hadamard) or its matrix Q [d, d] (Haar)."""
    x = _f64(x)
    rot = _f64(rot)
    out = np.zeros_like(x)
    fn = _load().tqo_rotate_dense if rot.ndim == 2 else _load().tqo_rotate
    fn(x.shape[0], _p(rot), _p(x), _p(out))
    return out


def unrotate(rot, y) -> np.ndarray:
    """Pi^T y for a head's signs or Haar matrix."""
    y = _f64(y)
    rot = _f64(rot)
    out = np.zeros_like(y)
    fn = _load().tqo_unrotate_dense if rot.ndim == 2 else _load().tqo_unrotate
    fn(y.shape[0], _p(rot), _p(y), _p(out))
    return out


# ------------------------------------------------------------------- codec

NORM_FORMATS = {"f32": 0, "f16": 1}


class Codec:
    """One codec configuration (head_dim, bits, projections, seed, rotation,
    key-norm format) on the CPU; rotation is "hadamard" (FWHT with random
    signs) or "haar"; norms is "f32" or "f16" (key rows' n_s and gamma as
    binary16)."""

    def __init__(self, head_dim: int, bits: int, projections: int, seed: int, norm_correct: bool = True,
                 rotation: str = "hadamard", norms: str = "f32"):
        self.d, self.bits, self.m, self.seed = head_dim, bits, projections, seed
        self.rotation = rotation
        self.norms = norms
        self.cfg = _Cfg()
        if _load().tqo_cfg_init(ctypes.byref(self.cfg), head_dim, bits, projections, int(norm_correct)) != 0:
            raise ValueError("invalid oracle configuration")
        self.cfg.rotation = ROTATIONS[rotation]
        self.cfg.norm_f16 = NORM_FORMATS[norms]
        self.k_row_bytes = _lib.tqo_k_row_bytes(ctypes.byref(self.cfg))
        self.v_row_bytes = _lib.tqo_v_row_bytes(ctypes.byref(self.cfg))
        self._tables = {}

    @property
    def ck(self):
        return np.array(self.cfg.ck[: self.cfg.LK])

    @property
    def cv(self):
        return np.array(self.cfg.cv[: self.cfg.LV])

    @property
    def bk(self):
        return np.array(self.cfg.bk[: self.cfg.LK - 1])

    @property
    def bv(self):
        return np.array(self.cfg.bv[: self.cfg.LV - 1])

    def tables(self, h: int):
        """(rot, S) of head h: rot = the signs [d] (Hadamard) or Q [d, d] (Haar)."""
        if h not in self._tables:
            signs, S = head_tables(self.d, self.m, self.seed, h)
            rot = haar_matrix(self.d, self.m, self.seed, h) if self.rotation == "haar" else signs
            self._tables[h] = (rot, S)
        return self._tables[h]

    def encode(self, x, h: int, is_key: bool):
        """Encode rows x [T, d] of head h.

        Returns dict(rows=uint8 [T, row_bytes], z=[T, d], pn=[T, m] (keys),
        ns=[T], gamma=[T] (keys), nonfinite=int)."""
        x = _f64(x)
        T = x.shape[0]
        signs, S = self.tables(h)
        rb = self.k_row_bytes if is_key else self.v_row_bytes
        rows = np.zeros((T, rb), dtype=np.uint8)
        z = np.zeros((T, self.d))
        pn = np.zeros((T, self.m))
        ns = np.zeros(T)
        g = np.zeros(T)
        cnt = _lib.tqo_encode_block(ctypes.byref(self.cfg), int(is_key), _p(signs), _p(S), _p(x), T,
                                    _p(rows), _p(z), _p(pn), _p(ns), _p(g))
        out = dict(rows=rows, z=z, ns=ns, nonfinite=cnt)
        if is_key:
            out["pn"] = pn
            out["gamma"] = g
        return out

    def unpack_k(self, row):
        row = np.ascontiguousarray(row, dtype=np.uint8)
        idx = np.zeros(self.d, dtype=np.int32)
        bit = np.zeros(self.m, dtype=np.int32)
        ns = ctypes.c_double()
        g = ctypes.c_double()
        _lib.tqo_unpack_k(ctypes.byref(self.cfg), _p(row), _p(idx), _p(bit), ctypes.byref(ns), ctypes.byref(g))
        return idx, bit, ns.value, g.value

    def unpack_v(self, row):
        row = np.ascontiguousarray(row, dtype=np.uint8)
        idx = np.zeros(self.d, dtype=np.int32)
        ns = ctypes.c_double()
        _lib.tqo_unpack_v(ctypes.byref(self.cfg), _p(row), _p(idx), ctypes.byref(ns))
        return idx, ns.value

    def dequant(self, rows, h: int, is_key: bool) -> np.ndarray:
        rows = np.ascontiguousarray(rows, dtype=np.uint8)
        signs, S = self.tables(h)
        out = np.zeros((rows.shape[0], self.d))
        for t in range(rows.shape[0]):
            if is_key:
                _lib.tqo_dequant_k(ctypes.byref(self.cfg), _p(signs), _p(S), _p(rows[t]), _p(out[t]))
            else:
                _lib.tqo_dequant_v(ctypes.byref(self.cfg), _p(signs), _p(rows[t]), _p(out[t]))
        return out

    def scores(self, q, krows, h: int, fused: bool = True) -> np.ndarray:
        q = _f64(q)
        krows = np.ascontiguousarray(krows, dtype=np.uint8)
        signs, S = self.tables(h)
        T = krows.shape[0]
        out = np.zeros(T)
        fn = _lib.tqo_scores_fused if fused else _lib.tqo_scores_dequant
        fn(ctypes.byref(self.cfg), _p(signs), _p(S), _p(q), _p(krows), T, _p(out))
        return out

    def packed_bytes(self, n_rows: int) -> int:
        return _lib.tqo_packed_bytes(ctypes.byref(self.cfg), n_rows)


def attention(q, segments) -> np.ndarray:
    """Decode attention of one query over segments [(codec, h, krows, vrows), ...]
    concatenated along the token axis (softmax over all tokens)."""
    q = _f64(q)
    lib = _load()
    n = len(segments)
    d = segments[0][0].d
    keep = []
    cfgs = (ctypes.c_void_p * n)()
    sg = (ctypes.c_void_p * n)()
    Ss = (ctypes.c_void_p * n)()
    kr = (ctypes.c_void_p * n)()
    vr = (ctypes.c_void_p * n)()
    T = np.zeros(n, dtype=np.int64)
    for i, (codec, h, krows, vrows) in enumerate(segments):
        signs, S = codec.tables(h)
        krows = np.ascontiguousarray(krows, dtype=np.uint8)
        vrows = np.ascontiguousarray(vrows, dtype=np.uint8)
        keep += [krows, vrows]
        cfgs[i] = ctypes.cast(ctypes.byref(codec.cfg), ctypes.c_void_p)
        sg[i] = signs.ctypes.data
        Ss[i] = S.ctypes.data
        kr[i] = krows.ctypes.data
        vr[i] = vrows.ctypes.data
        T[i] = krows.shape[0]
    out = np.zeros(d)
    lib.tqo_attend(n, cfgs, sg, Ss, kr, vr, _p(T), _p(q), _p(out))
    return out


def streaming_softmax_sum(scores, vals, blk: int) -> np.ndarray:
    scores = _f64(scores)
    vals = _f64(vals)
    out = np.zeros(vals.shape[1])
    _load().tqo_streaming_softmax_sum(scores.shape[0], vals.shape[1], _p(scores), _p(vals), blk, _p(out))
    return out


def attention_split(q, part_o, part_n) -> np.ndarray:
    """Decode attention of one query q [d_o + d_n] over a split cache: part_x =
    (codec, h, krows, vrows) for the outlier group (channels first) and the
    normal group; both hold the same tokens."""
    q = _f64(q)
    (co, ho, ko, vo), (cn, hn, kn, vn) = part_o, part_n
    ro, So = co.tables(ho)
    rn, Sn = cn.tables(hn)
    ko, vo, kn, vn = (np.ascontiguousarray(a, dtype=np.uint8) for a in (ko, vo, kn, vn))
    out = np.zeros(co.d + cn.d)
    _load().tqo_attend_split(ctypes.byref(co.cfg), _p(_f64(ro)), _p(So), _p(ko), _p(vo), ctypes.byref(cn.cfg),
                             _p(_f64(rn)), _p(Sn), _p(kn), _p(vn), ko.shape[0], _p(q), _p(out))
    return out
