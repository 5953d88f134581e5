"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test checks the oracle (``oracle/``) against the pages' statements, a
closed form, a textbook table, an invariant or a brute-force computation,
chosen so that a dropped term, a wrong sign, a transposed operand or a
wrong index in the oracle makes at least one of them fail.  CPU only.
"""
import math
import os

import numpy as np
import pytest
from scipy import integrate, stats

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold_rows(name):
    with open(os.path.join(GOLD, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


def _hadamard(d):
    i = np.arange(d)
    pc = np.vectorize(lambda v: bin(v).count("1"))(i[:, None] & i[None, :])
    return np.where(pc % 2 == 0, 1.0, -1.0)


# --------------------------------------------------------------- PRNG / fp16

def test_splitmix64_published_sequence():
    want = [int(x, 16) for x in _gold_rows("splitmix64_seed0.txt")]
    got = [int(v) for v in oracle.splitmix64_stream(0, len(want))]
    assert got == want


def test_fp16_rounding_matches_ieee_binary16():
    rng = np.random.default_rng(3)
    xs = np.concatenate([rng.standard_normal(20000) * 4, rng.standard_normal(2000) * 1e-5,
                         [0.5 * 2.0 ** -24, 1.5 * 2.0 ** -24, 1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, 65504.0]])
    for x in xs:
        assert oracle.round_fp16(x) == float(np.float16(x))


def test_head_tables_distribution():
    """Signs are +-1 and balanced; S is fp16-valued and distributed as N(0,1)."""
    signs, S = oracle.head_tables(128, 128, 42, 0)
    assert set(np.unique(signs)) <= {-1.0, 1.0}
    assert abs(signs.mean()) < 0.35
    assert np.all(S.astype(np.float16).astype(np.float64) == S)
    flat = S.ravel()
    assert stats.kstest(flat, "norm").pvalue > 1e-3
    assert abs(flat.mean()) < 0.03 and abs(flat.var() - 1.0) < 0.05
    # heads differ (seed + h), same head is reproducible
    s1, S1 = oracle.head_tables(128, 128, 42, 1)
    s0b, S0b = oracle.head_tables(128, 128, 43, 0)
    assert not np.array_equal(S, S1)
    assert np.array_equal(S1, S0b) and np.array_equal(s1, s0b)   # seed+h wrapping add


@pytest.mark.parametrize("d,m,seed,h", [(16, 12, 77, 3), (128, 128, 42, 5), (8, 3, 2 ** 64 - 2, 4)])
def test_head_tables_draw_layout(d, m, seed, h):
    """Where each draw of the head's SplitMix64 stream (seed + h, wrapping)
    lands: draw j < d gives sign j from its top bit (set -> -1); the next
    draws, two at a time, give S row-major by Box-Muller, u1 = ((a>>11)+1)
    2^-53 from the first draw of the pair and u2 = (b>>11) 2^-53 from the
    second, cos to the even entry and sin to the odd one, each entry rounded
    to binary16 (numpy's IEEE conversion here).  A swapped u1/u2, a swapped
    cos/sin, another sign bit or a missing rounding fails."""
    signs, S = oracle.head_tables(d, m, seed, h)
    n = m * d
    u = [int(x) for x in oracle.splitmix64_stream((seed + h) % 2 ** 64, d + n + (n % 2))]
    for j in range(d):
        assert signs[j] == (-1.0 if u[j] >> 63 else 1.0)
    flat = S.ravel()
    for i in range(0, n, 2):
        a, b = u[d + i], u[d + i + 1]
        u1 = ((a >> 11) + 1) * 2.0 ** -53
        u2 = (b >> 11) * 2.0 ** -53
        rad = math.sqrt(-2.0 * math.log(u1))
        assert flat[i] == float(np.float16(rad * math.cos(2 * math.pi * u2)))
        if i + 1 < n:
            assert flat[i + 1] == float(np.float16(rad * math.sin(2 * math.pi * u2)))


# ------------------------------------------------------------------ codebook

def _unit_of_last_digit(text):
    return 10.0 ** -(len(text.split(".")[1]) if "." in text else 0)


def test_codebook_matches_textbook_table():
    for row in _gold_rows("lloyd_max_gaussian.txt"):
        B, cents, dist = [p.strip() for p in row.split("|")]
        B = int(B)
        c, _ = oracle.lloyd_max(B)
        pos = c[len(c) // 2:]
        toks = cents.split()
        assert len(toks) == len(pos)
        for got, tok in zip(pos, toks):
            assert abs(got - float(tok)) <= _unit_of_last_digit(tok) * 1.0000001, (B, got, tok)
        L = len(c)
        b = np.concatenate([[-np.inf], 0.5 * (c[:-1] + c[1:]), [np.inf]])
        D = sum(integrate.quad(lambda x, k=k: (x - c[k]) ** 2 * stats.norm.pdf(x), b[k], b[k + 1])[0]
                for k in range(L))
        # distortion of a Lloyd-Max fixed point: 1 - sum_k c_k^2 P(cell k)
        P = np.diff(stats.norm.cdf(b))
        assert abs(D - (1.0 - np.sum(c * c * P))) < 1e-9
        # the 1960 table's distortions carry their own rounding error (its
        # 16-level entry is 4e-6 low); compare them to 0.1 % relative
        assert abs(D - float(dist)) <= 1e-3 * float(dist), (B, D, dist)


def test_codebook_one_bit_closed_form():
    c, b = oracle.lloyd_max(1)
    assert abs(c[1] - math.sqrt(2 / math.pi)) < 1e-12 and c[0] == -c[1] and b[0] == 0.0


@pytest.mark.parametrize("B", [2, 3, 4, 5])
def test_codebook_is_lloyd_fixed_point(B):
    """Each centroid is the conditional mean of its cell (by numerical
    integration, independent of the oracle's erfc formulas); boundaries are
    midpoints; the codebook is antisymmetric."""
    c, b = oracle.lloyd_max(B)
    L = 1 << B
    assert np.all(np.diff(c) > 0)
    assert np.allclose(b, 0.5 * (c[:-1] + c[1:]), atol=0, rtol=1e-15)
    assert np.array_equal(c, -c[::-1])
    edges = np.concatenate([[-np.inf], b, [np.inf]])
    for k in range(L):
        num = integrate.quad(lambda x: x * stats.norm.pdf(x), edges[k], edges[k + 1], epsabs=1e-14)[0]
        den = integrate.quad(stats.norm.pdf, edges[k], edges[k + 1], epsabs=1e-14)[0]
        assert abs(num / den - c[k]) < 1e-9


# ------------------------------------------------------------------ rotation

@pytest.mark.parametrize("d", [2, 4, 8, 16, 32, 64, 128, 256])
def test_fwht_is_sylvester_hadamard(d):
    H = _hadamard(d)
    cols = np.stack([oracle.fwht(np.eye(d)[j]) for j in range(d)], axis=1)
    assert np.array_equal(cols, H)
    assert np.array_equal(H @ H, d * np.eye(d))


def test_rotation_orthonormal_and_dense_equivalent():
    d = 128
    rng = np.random.default_rng(5)
    signs, _ = oracle.head_tables(d, 8, 7, 3)
    Pi = _hadamard(d) @ np.diag(signs) / math.sqrt(d)
    for _ in range(10):
        x = rng.standard_normal(d) * rng.uniform(0.1, 10)
        y = oracle.rotate(signs, x)
        assert abs(np.linalg.norm(y) - np.linalg.norm(x)) < 1e-14 * np.linalg.norm(x)
        assert np.allclose(y, Pi @ x, atol=1e-13)
        assert np.allclose(oracle.unrotate(signs, y), x, atol=1e-13)
        assert np.allclose(oracle.unrotate(signs, x), Pi.T @ x, atol=1e-13)


# ------------------------------------------------------------ Haar rotation

def test_haar_gaussian_continues_the_head_stream():
    """G is filled by Box-Muller pairs drawn after the d sign draws and the
    (even) number of draws of S, from the head's stream (seed + h)."""
    d, m, seed, h = 16, 12, 77, 3
    G = oracle.haar_gaussian(d, m, seed, h)
    skip = d + m * d + (m * d) % 2
    u = oracle.splitmix64_stream(seed + h, skip + 4)[skip:].astype(object)
    for k in range(2):
        u1 = ((int(u[2 * k]) >> 11) + 1) * 2.0 ** -53
        u2 = (int(u[2 * k + 1]) >> 11) * 2.0 ** -53
        rad = math.sqrt(-2.0 * math.log(u1))
        assert abs(G.ravel()[2 * k] - rad * math.cos(2 * math.pi * u2)) < 1e-15
        assert abs(G.ravel()[2 * k + 1] - rad * math.sin(2 * math.pi * u2)) < 1e-15
    G128 = oracle.haar_gaussian(128, 128, 42, 0)
    assert stats.kstest(G128.ravel(), "norm").pvalue > 1e-3


@pytest.mark.parametrize("d", [8, 64, 128])
def test_haar_matrix_is_the_sign_fixed_qr_factor(d):
    """Q equals LAPACK's QR factor of the same G with the columns' signs set
    so that R has a positive diagonal; Q is orthogonal and Q^T G is upper
    triangular with a positive diagonal."""
    G = oracle.haar_gaussian(d, 32, 5, 1)
    Q = oracle.haar_matrix(d, 32, 5, 1)
    Qn, Rn = np.linalg.qr(G)
    Qn = Qn * np.sign(np.diag(Rn))[None, :]
    assert np.max(np.abs(Q - Qn)) < 1e-12
    assert np.max(np.abs(Q.T @ Q - np.eye(d))) < 1e-13
    R = Q.T @ G
    assert np.max(np.abs(np.tril(R, -1))) < 1e-12
    assert np.all(np.diag(R) > 0)


def test_haar_matrix_moments():
    """Haar on O(d): a column of Q is uniform on the sphere, so a squared
    entry is Beta(1/2, (d-1)/2) with mean 1/d; Q v is uniform for any fixed v."""
    d = 16
    sq, proj = [], []
    v = np.ones(d) / math.sqrt(d)
    for h in range(300):
        Q = oracle.haar_matrix(d, 8, 1234, h)
        sq.append(Q[:, 0] ** 2)
        proj.append((Q @ v)[3] ** 2)
    sq = np.concatenate(sq)
    assert abs(sq.mean() - 1.0 / d) < 4 * math.sqrt(2.0 * (d - 1) / (d * d * (d + 2))) / math.sqrt(len(sq) / d)
    assert stats.kstest(sq, stats.beta(0.5, (d - 1) / 2.0).cdf).pvalue > 1e-3
    assert stats.kstest(np.array(proj), stats.beta(0.5, (d - 1) / 2.0).cdf).pvalue > 1e-3
    # different heads differ
    assert not np.allclose(oracle.haar_matrix(d, 8, 1234, 0), oracle.haar_matrix(d, 8, 1234, 1))


def test_haar_rotation_is_the_dense_product():
    d = 128
    Q = oracle.haar_matrix(d, 128, 9, 2)
    rng = np.random.default_rng(8)
    for _ in range(5):
        x = rng.standard_normal(d) * rng.uniform(0.1, 10)
        assert np.allclose(oracle.rotate(Q, x), Q @ x, atol=1e-12)
        assert np.allclose(oracle.unrotate(Q, x), Q.T @ x, atol=1e-12)
        assert abs(np.linalg.norm(oracle.rotate(Q, x)) - np.linalg.norm(x)) < 1e-12 * np.linalg.norm(x)


# -------------------------------------------------------------- encode/QJL

def _independent_codes(codec, h, x, is_key):
    """Quantizer indices, n_s, residual and QJL bits recomputed in numpy from
    the method's definition, sharing only the head tables and codebook."""
    d = codec.d
    rot, S = codec.tables(h)
    n = np.linalg.norm(x)
    if codec.rotation == "haar":
        Pi = np.linalg.qr(oracle.haar_gaussian(d, codec.m, codec.seed, h))[0]
        Pi = Pi * np.sign(np.diag(np.linalg.qr(oracle.haar_gaussian(d, codec.m, codec.seed, h))[1]))[None, :]
    else:
        Pi = _hadamard(d) @ np.diag(rot) / math.sqrt(d)
    y = Pi @ x / n
    z = math.sqrt(d) * y
    c, b = (codec.ck, codec.bk) if is_key else (codec.cv, codec.bv)
    idx = np.sum(z[:, None] >= b[None, :], axis=1)
    yhat = c[idx] / math.sqrt(d)
    ns = n / np.linalg.norm(yhat)
    r = n * y - ns * yhat
    p = S @ r
    return idx, ns, r, p, z


@pytest.mark.parametrize("rotation", ["hadamard", "haar"])
@pytest.mark.parametrize("bits", [2, 3, 4, 5])
def test_encode_matches_independent_definition(bits, rotation):
    d, m = 64, 32
    codec = oracle.Codec(d, bits, m, 11, rotation=rotation)
    rng = np.random.default_rng(bits)
    x = rng.standard_normal((6, d)) * rng.uniform(0.2, 5, size=(6, 1))
    for is_key in (True, False):
        enc = codec.encode(x, 2, is_key)
        for t in range(x.shape[0]):
            idx, ns, r, p, z = _independent_codes(codec, 2, x[t], is_key)
            assert np.allclose(enc["z"][t], z, atol=1e-12)
            if is_key:
                gi, gb, gns, gg = codec.unpack_k(enc["rows"][t])
                assert np.array_equal(gi, idx)
                assert np.array_equal(gb, (p >= 0).astype(int))
                assert abs(gg - np.float32(np.linalg.norm(r))) <= 1e-6 * np.linalg.norm(r)
                assert np.allclose(enc["pn"][t], p / np.linalg.norm(r), atol=1e-12)
            else:
                gi, gns = codec.unpack_v(enc["rows"][t])
                assert np.array_equal(gi, idx)
            assert abs(gns - ns) <= 1e-6 * ns


def test_packed_layout_by_hand():
    """Raw bit positions of both packed formats, checked against indices
    recomputed in numpy: K plane p holds bit p of index j at byte p*d/8 +
    j/8, bit j%8; V holds index j's bit k at stream bit B_V*j + k."""
    d, m = 8, 16
    codec = oracle.Codec(d, 3, m, 1)     # K: 2 index bits + 16 sign bits, V: 3-bit fields
    rng = np.random.default_rng(12)
    x = rng.standard_normal((5, d))
    for is_key in (True, False):
        enc = codec.encode(x, 0, is_key)
        for t in range(5):
            idx, ns, r, p, z = _independent_codes(codec, 0, x[t], is_key)
            bits = np.unpackbits(enc["rows"][t], bitorder="little")
            if is_key:
                for j in range(d):
                    for pl in range(2):
                        assert bits[pl * d + j] == (idx[j] >> pl) & 1
                for i in range(m):
                    assert bits[2 * d + i] == int(p[i] >= 0)
                tail = enc["rows"][t][2 * d // 8 + m // 8:]
                assert tail.view(np.float32)[0] == np.float32(enc["ns"][t])
                assert tail.view(np.float32)[1] == np.float32(enc["gamma"][t])
            else:
                for j in range(d):
                    for k in range(3):
                        assert bits[3 * j + k] == (idx[j] >> k) & 1
                assert enc["rows"][t][3:].view(np.float32)[0] == np.float32(enc["ns"][t])
    assert codec.k_row_bytes == 2 * d // 8 + m // 8 + 8
    assert codec.v_row_bytes == 3 * d // 8 + 4


def _grid_indices(c, d, rng):
    """Indices whose counts follow the Gaussian cell probabilities, so the
    empirical second moment of C[idx] is close to the codebook's (1 - D)."""
    b = np.concatenate([[-np.inf], 0.5 * (c[:-1] + c[1:]), [np.inf]])
    P = np.diff(stats.norm.cdf(b))
    cnt = np.floor(P * d).astype(int)
    order = np.argsort(-(P * d - cnt))
    cnt[order[: d - cnt.sum()]] += 1
    return rng.permutation(np.repeat(np.arange(len(c)), cnt))


@pytest.mark.parametrize("rotation", ["hadamard", "haar"])
def test_special_case_exact_reconstruction(rotation):
    """x on the normalized codebook grid is reproduced exactly (norm
    correction) with zero residual, so scores are the exact inner products."""
    d, m = 128, 128
    rng = np.random.default_rng(9)
    for bits in (2, 3, 4):
        codec = oracle.Codec(d, bits, m, 100 + bits, rotation=rotation)
        signs, S = codec.tables(0)
        for is_key, c in ((True, codec.ck), (False, codec.cv)):
            L = len(c)
            for _ in range(3):
                # indices drawn so that the empirical second moment of C[idx] is
                # the codebook's, keeping every z inside its own cell
                idx = _grid_indices(c, d, rng)
                u = c[idx] / np.linalg.norm(c[idx])
                z = u * math.sqrt(d)
                lo = np.concatenate([[-np.inf], 0.5 * (c[:-1] + c[1:])])[idx]
                hi = np.concatenate([0.5 * (c[:-1] + c[1:]), [np.inf]])[idx]
                assert np.all((z > lo + 1e-6) & (z < hi - 1e-6))
                alpha = rng.uniform(0.5, 3.0)
                x = alpha * oracle.unrotate(signs, u)
                enc = codec.encode(x[None], 0, is_key)
                rec = codec.dequant(enc["rows"], 0, is_key)[0]
                if is_key:
                    assert enc["gamma"][0] < 1e-12 * alpha
                    # gamma is tiny, the QJL term vanishes: k_hat = x
                    assert np.allclose(rec, x, atol=1e-6 * alpha)
                    q = rng.standard_normal(d)
                    s = codec.scores(q, enc["rows"], 0)
                    assert abs(s[0] - q @ x / math.sqrt(d)) < 1e-6 * alpha * np.linalg.norm(q)
                else:
                    assert np.allclose(rec, x, atol=1e-6 * alpha)


def test_norm_correction_is_what_makes_grid_points_exact():
    """Without norm correction (n_s = n) the grid point is not reproduced:
    the special-case pin above depends on the correction step."""
    d = 128
    codec = oracle.Codec(d, 3, 128, 5, norm_correct=False)
    signs, _ = codec.tables(0)
    c = codec.cv
    idx = _grid_indices(c, d, np.random.default_rng(0))
    u = c[idx] / np.linalg.norm(c[idx])
    x = 2.0 * oracle.unrotate(signs, u)
    rec = codec.dequant(codec.encode(x[None], 0, False)["rows"], 0, False)[0]
    assert np.linalg.norm(rec - x) > 1e-2


# --------------------------------------------------------------------- QJL

def test_qjl_estimator_unbiased_and_variance_bound():
    """Over many seeds the TurboQuant inner-product estimate <q, k_hat> is
    unbiased for <q, x>, while the MSE stage alone is biased; the QJL error
    obeys Var <= (pi/2)/m ||q||^2 ||r||^2."""
    d, m, n_seeds = 64, 64, 4096
    rng = np.random.default_rng(123)
    x = rng.standard_normal(d)
    q = x + 0.3 * rng.standard_normal(d)     # correlated query: the MSE bias is visible
    errs, mse_errs, ratios = [], [], []
    for s in range(n_seeds):
        codec = oracle.Codec(d, 2, m, 1000 + 7919 * s)      # B_K = 1: large residual
        enc = codec.encode(x[None], 0, True)
        kh = codec.dequant(enc["rows"], 0, True)[0]
        signs, S = codec.tables(0)
        idx, bit, ns, g = codec.unpack_k(enc["rows"][0])
        mse_part = oracle.rotate(signs, q) @ (ns * codec.ck[idx] / math.sqrt(d))
        full = q @ kh
        errs.append(full - q @ x)
        mse_errs.append(mse_part - q @ x)
        r_ip = q @ x - mse_part
        ratios.append((full - mse_part - r_ip) ** 2 / (np.dot(q, q) * g * g))
    errs, mse_errs = np.array(errs), np.array(mse_errs)
    se = errs.std(ddof=1) / math.sqrt(n_seeds)
    assert abs(errs.mean()) < 4 * se
    se_m = mse_errs.std(ddof=1) / math.sqrt(n_seeds)
    assert abs(mse_errs.mean()) > 8 * se_m          # MSE-only is biased
    assert np.mean(ratios) <= (math.pi / 2) / m * 1.1


def test_qjl_rotated_frame_is_a_gaussian_projection():
    """S applied in the rotated frame equals (S Pi) applied to the original
    residual; S Pi has the law of an iid Gaussian matrix (row norms ~ sqrt(d))."""
    d, m = 64, 64
    codec = oracle.Codec(d, 3, m, 77)
    signs, S = codec.tables(0)
    Pi = _hadamard(d) @ np.diag(signs) / math.sqrt(d)
    rng = np.random.default_rng(1)
    r = rng.standard_normal(d)
    assert np.allclose(S @ (Pi @ r), (S @ Pi) @ r, atol=1e-12)
    SP = S @ Pi
    assert abs(np.mean(np.sum(SP * SP, axis=1)) / d - 1.0) < 0.1


# ------------------------------------------------------------ scores / attn

@pytest.mark.parametrize("rotation", ["hadamard", "haar"])
@pytest.mark.parametrize("cfg", [(8, 4, 16, 42), (128, 3, 128, 42), (64, 2, 32, 9), (128, 5, 64, 3)])
def test_scores_fused_equal_dequantized(cfg, rotation):
    d, bits, m, seed = cfg
    codec = oracle.Codec(d, bits, m, seed, rotation=rotation)
    rng = np.random.default_rng(d + bits)
    K = rng.standard_normal((16, d))
    enc = codec.encode(K, 1, True)
    for _ in range(3):
        q = rng.standard_normal(d)
        a = codec.scores(q, enc["rows"], 1, fused=True)
        b = codec.scores(q, enc["rows"], 1, fused=False)
        kh = codec.dequant(enc["rows"], 1, True)
        assert np.allclose(a, b, atol=1e-11)
        assert np.allclose(b, kh @ q / math.sqrt(d), atol=1e-11)


def test_streaming_softmax_equals_materialized():
    rng = np.random.default_rng(4)
    T, d = 1000, 16
    s = rng.standard_normal(T) * 3
    v = rng.standard_normal((T, d))
    p = np.exp(s - s.max())
    p /= p.sum()
    want = p @ v
    for blk in (1, 7, 64, 1000, 5000):
        assert np.allclose(oracle.streaming_softmax_sum(s, v, blk), want, atol=1e-13)


def test_attention_matches_brute_force_and_gqa_segments():
    d, m = 8, 16
    c1 = oracle.Codec(d, 4, m, 42)
    c2 = oracle.Codec(d, 2, m, 42)
    rng = np.random.default_rng(2)
    K1, V1 = rng.standard_normal((5, d)), rng.standard_normal((5, d))
    K2, V2 = rng.standard_normal((7, d)), rng.standard_normal((7, d))
    e = [c1.encode(K1, 0, True), c1.encode(V1, 0, False), c2.encode(K2, 0, True), c2.encode(V2, 0, False)]
    q = rng.standard_normal(d)
    got = oracle.attention(q, [(c1, 0, e[0]["rows"], e[1]["rows"]), (c2, 0, e[2]["rows"], e[3]["rows"])])
    kh = np.concatenate([c1.dequant(e[0]["rows"], 0, True), c2.dequant(e[2]["rows"], 0, True)])
    vh = np.concatenate([c1.dequant(e[1]["rows"], 0, False), c2.dequant(e[3]["rows"], 0, False)])
    s = kh @ q / math.sqrt(d)
    p = np.exp(s - s.max())
    p /= p.sum()
    assert np.allclose(got, p @ vh, atol=1e-12)


def test_attention_error_decreases_with_bits():
    d, m, T, n_seeds = 64, 64, 32, 64
    errs = {b: [] for b in (2, 3, 4, 5)}
    for s in range(n_seeds):
        rng = np.random.default_rng(500 + s)
        K, V = rng.standard_normal((T, d)), rng.standard_normal((T, d))
        q = rng.standard_normal(d)
        sc = K @ q / math.sqrt(d)
        p = np.exp(sc - sc.max())
        p /= p.sum()
        exact = p @ V
        for b in errs:
            codec = oracle.Codec(d, b, m, 77 + s)
            ek, ev = codec.encode(K, 0, True), codec.encode(V, 0, False)
            out = oracle.attention(q, [(codec, 0, ek["rows"], ev["rows"])])
            errs[b].append(np.linalg.norm(out - exact) / np.linalg.norm(exact))
    means = [np.mean(errs[b]) for b in (2, 3, 4, 5)]
    assert all(means[i] > means[i + 1] for i in range(3)), means


# ------------------------------------------------------------- edge cases

def test_degenerate_rows_and_nonfinite_count():
    d, m = 16, 16
    codec = oracle.Codec(d, 3, m, 3)
    x = np.zeros((3, d))
    x[1, 4] = np.nan
    x[2, :] = 1.0
    x[2, 3] = np.inf
    for is_key in (True, False):
        enc = codec.encode(x, 0, is_key)
        assert enc["nonfinite"] == 2
        for t in range(3):
            if is_key:
                idx, bit, ns, g = codec.unpack_k(enc["rows"][t])
                assert np.all(idx == len(codec.ck) // 2) and np.all(bit == 1) and ns == 0 and g == 0
            else:
                idx, ns = codec.unpack_v(enc["rows"][t])
                assert np.all(idx == len(codec.cv) // 2) and ns == 0
        assert np.allclose(codec.dequant(enc["rows"], 0, is_key), 0.0)


def test_determinism_same_seed_same_bytes():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((8, 128))
    a = oracle.Codec(128, 4, 128, 42).encode(x, 3, True)["rows"]
    b = oracle.Codec(128, 4, 128, 42).encode(x, 3, True)["rows"]
    c = oracle.Codec(128, 4, 128, 43).encode(x, 3, True)["rows"]
    assert np.array_equal(a, b) and not np.array_equal(a, c)


def test_scale_invariance_of_codes():
    """Indices and sign bits depend only on the direction; norms scale."""
    rng = np.random.default_rng(8)
    x = rng.standard_normal((4, 64))
    codec = oracle.Codec(64, 3, 32, 1)
    a = codec.encode(x, 0, True)
    b = codec.encode(x * 8.0, 0, True)
    pb = codec.k_row_bytes - 8
    assert np.array_equal(a["rows"][:, :pb], b["rows"][:, :pb])
    assert np.allclose(b["ns"], 8 * a["ns"], rtol=1e-14) and np.allclose(b["gamma"], 8 * a["gamma"], rtol=1e-12)


def test_compression_table_arithmetic():
    """The pages' ratios are 16 / bits-per-value; our formats follow the
    same accounting from their byte counts."""
    for row in _gold_rows("compression_formats.txt"):
        name, bpv, ratio = [p.strip() for p in row.split("|")]
        assert round(16.0 / float(bpv), 1) == float(ratio)
    for bits, bpv_ours in ((4, 4.375), (3, 3.375), (2, 2.375)):
        codec = oracle.Codec(128, bits, 128, 0)
        assert codec.packed_bytes(1) * 8 / (2 * 128) == bpv_ours


# ------------------------------------------------------ outlier splitting

def _split_parts(seed=3, T=60, bits=(4, 3)):
    rng = np.random.default_rng(seed)
    co, cn = oracle.Codec(64, bits[0], 64, 11), oracle.Codec(64, bits[1], 64, 29)
    K = rng.standard_normal((T, 128)) * np.r_[np.full(64, 4.0), np.ones(64)]
    V = rng.standard_normal((T, 128))
    eko, evo = co.encode(K[:, :64], 2, True), co.encode(V[:, :64], 2, False)
    ekn, evn = cn.encode(K[:, 64:], 2, True), cn.encode(V[:, 64:], 2, False)
    return rng, co, cn, (co, 2, eko["rows"], evo["rows"]), (cn, 2, ekn["rows"], evn["rows"])


def test_split_attention_is_softmax_over_the_concatenated_reconstruction():
    """Brute force: keys and values are the concatenations of the two groups'
    dequantized rows; scores q.k_hat / sqrt(128); one softmax over tokens."""
    rng, co, cn, po, pn = _split_parts()
    kh = np.concatenate([co.dequant(po[2], 2, True), cn.dequant(pn[2], 2, True)], axis=1)
    vh = np.concatenate([co.dequant(po[3], 2, False), cn.dequant(pn[3], 2, False)], axis=1)
    for _ in range(3):
        q = rng.standard_normal(128)
        s = kh @ q / math.sqrt(128)
        p = np.exp(s - s.max())
        p /= p.sum()
        assert np.allclose(oracle.attention_split(q, po, pn), p @ vh, atol=1e-12)


def test_split_scores_are_the_groups_scores_rescaled():
    """With q zero on the normal group, every token's split score is the outlier
    group's own score times sqrt(64 / 128): the attention equals a softmax of the
    group's scores scaled by 1/sqrt(2)."""
    rng, co, cn, po, pn = _split_parts(seed=5)
    q = np.r_[rng.standard_normal(64), np.zeros(64)]
    so = co.scores(q[:64], po[2], 2) * math.sqrt(64 / 128)
    p = np.exp(so - so.max())
    p /= p.sum()
    vh = np.concatenate([co.dequant(po[3], 2, False), cn.dequant(pn[3], 2, False)], axis=1)
    assert np.allclose(oracle.attention_split(q, po, pn), p @ vh, atol=1e-12)


def test_split_bits_per_value():
    """Channel-weighted bits: 64 outlier channels at b + 1 and 64 at b give b + 1/2
    index bits per value (the non-integer rates the module names)."""
    for b in (2, 3, 4):
        co, cn = oracle.Codec(64, b + 1, 64, 1), oracle.Codec(64, b, 64, 1)
        idx_bits = 64 * co.bits + 64 * cn.bits   # value rows: b index bits per coordinate
        assert idx_bits / 128 == b + 0.5
        assert co.v_row_bytes - 4 + cn.v_row_bytes - 4 == (64 * (b + 1) + 64 * b) // 8


# -------------------------------------------------- binary16 key norms (R11)

@pytest.mark.parametrize("rotation", ["hadamard", "haar"])
@pytest.mark.parametrize("bits", [2, 3, 4, 5])
def test_f16_norm_rows_are_f32_rows_with_ieee_rounded_norms(bits, rotation):
    """The binary16-norm key row is the fp32-norm row with its tail replaced
    by n_s and gamma rounded to binary16 by numpy's own IEEE conversion;
    value rows are unchanged."""
    rng = np.random.default_rng(bits)
    x = rng.standard_normal((24, 64)) * rng.uniform(0.01, 300.0, size=(24, 1))
    a = oracle.Codec(64, bits, 64, 5, rotation=rotation)
    b = oracle.Codec(64, bits, 64, 5, rotation=rotation, norms="f16")
    assert b.k_row_bytes == a.k_row_bytes - 4 and b.v_row_bytes == a.v_row_bytes
    ea, eb = a.encode(x, 1, True), b.encode(x, 1, True)
    body = a.k_row_bytes - 8
    assert np.array_equal(ea["rows"][:, :body], eb["rows"][:, :body])
    tail = eb["rows"][:, body:].copy().view(np.uint16)           # [T, 2] little-endian halves
    assert np.array_equal(tail[:, 0], ea["ns"].astype(np.float16).view(np.uint16))
    assert np.array_equal(tail[:, 1], ea["gamma"].astype(np.float16).view(np.uint16))
    assert np.array_equal(a.encode(x, 1, False)["rows"], b.encode(x, 1, False)["rows"])


def test_f16_norm_consumers_read_the_rounded_norms():
    """Dequantization and scores of binary16-norm rows equal those of the
    fp32-norm rows whose two norms are overwritten by the binary16-rounded
    values (exact in fp32)."""
    rng = np.random.default_rng(4)
    x = rng.standard_normal((16, 128)) * 3.0
    q = rng.standard_normal(128)
    a = oracle.Codec(128, 4, 128, 9)
    b = oracle.Codec(128, 4, 128, 9, norms="f16")
    ra, rb = a.encode(x, 0, True)["rows"].copy(), b.encode(x, 0, True)["rows"]
    body = a.k_row_bytes - 8
    nsg = ra[:, body:].copy().view(np.float32)
    ra[:, body:] = nsg.astype(np.float16).astype(np.float32).view(np.uint8).reshape(ra.shape[0], 8)
    assert np.allclose(b.dequant(rb, 0, True), a.dequant(ra, 0, True), rtol=0, atol=1e-13)
    assert np.allclose(b.scores(q, rb, 0), a.scores(q, ra, 0), rtol=0, atol=1e-12)
    assert np.allclose(b.scores(q, rb, 0, fused=False), b.scores(q, rb, 0), rtol=0, atol=1e-11)


def test_f16_norm_overflow_rows_are_degenerate_and_counted():
    """A key row whose n_s or gamma rounds to binary16 infinity (>= 65520) is
    stored as the zero row and counted; just below, it is kept."""
    rng = np.random.default_rng(6)
    u = rng.standard_normal(128)
    u /= np.linalg.norm(u)
    b = oracle.Codec(128, 3, 128, 2, norms="f16")
    zero = b.encode(np.zeros((1, 128)), 0, True)["rows"][0]
    big = b.encode(u[None] * 1e6, 0, True)
    assert big["nonfinite"] == 1 and np.array_equal(big["rows"][0], zero)
    ok = b.encode(u[None] * 3e4, 0, True)
    assert ok["nonfinite"] == 0 and not np.array_equal(ok["rows"][0], zero)
    idx, bit, ns, g = b.unpack_k(ok["rows"][0])
    assert ns == float(np.float16(ok["ns"][0])) and np.isfinite(ns)


def test_f16_norm_turbo4_key_rate():
    """Binary16 key norms give the pages' turbo4 rate for keys: 3 index planes
    + 128 sign bits + 2 x 16 bits over 128 values = 4.25 bits per value
    (turboquant-plus-rs "Compression formats"); fp32 norms give 4.5."""
    assert oracle.Codec(128, 4, 128, 0, norms="f16").k_row_bytes * 8 / 128 == 4.25
    assert oracle.Codec(128, 4, 128, 0).k_row_bytes * 8 / 128 == 4.5
