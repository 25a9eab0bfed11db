"""Pins of the CPU oracle against values fixed by definitions and mathematics.

None of these expected values comes from the oracle itself or from the GPU path:
they are IEEE tables (numpy's float16), hand-built blocks with hand-derived
values (tests/golden), exact integer / rational arithmetic on logical values,
closed forms and invariants.
"""
import glob
import math
import os
from fractions import Fraction as Fr

import numpy as np
import pytest

import blockpack as bp

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
QT = {"q8_0": 0, "q4_0": 1, "q4_k": 2, "q6_k": 3, "q5_k": 4, "f16": 5, "f32": 6}
BLOCK = {0: (32, 34), 1: (32, 18), 2: (256, 144), 3: (256, 210), 4: (256, 176), 5: (1, 2), 6: (1, 4)}
ALL = [0, 1, 2, 3, 4, 5, 6]


def integer_fields(qtype, rng):
    """Random fields whose weights are all integers (d = dmin = 1, or integer values)."""
    if qtype == 5:
        return {"bits": [bp.f16_bits(float(rng.integers(-50, 51)))]}
    if qtype == 6:
        return {"values": [float(rng.integers(-50, 51))]}
    f = bp.random_fields(qtype, rng)
    f["d"] = bp.f16_bits(1.0)
    if qtype in (2, 4):
        f["dmin"] = bp.f16_bits(1.0)
    return f


# ------------------------------------------------------------------ fp16

def test_f16_decode_all_patterns(orc):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float32)          # IEEE binary16 -> binary32 (library)
    got = np.array([orc.f16_to_f32(int(b)) for b in bits], dtype=np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))   # incl. signed zeros, subnormals


def test_f16_encode_round_to_nearest_even(orc):
    rng = np.random.default_rng(1)
    finite = np.arange(65536, dtype=np.uint32).astype(np.uint16).view(np.float16)
    finite = finite[np.isfinite(finite)].astype(np.float32)
    # exact fp16 values, midpoints between neighbours (ties), values just off the midpoints,
    # random values across the whole range including subnormals and overflow
    srt = np.unique(finite.astype(np.float64))
    mids = ((srt[1:] + srt[:-1]) / 2).astype(np.float32)
    mids = mids[mids.astype(np.float64) == (srt[1:] + srt[:-1]) / 2]      # keep exact midpoints
    near = np.concatenate([np.nextafter(mids, np.float32(np.inf)), np.nextafter(mids, np.float32(-np.inf))])
    rnd = (rng.standard_normal(20000) * np.exp2(rng.uniform(-30, 20, 20000))).astype(np.float32)
    edge = np.array([65504, 65519.996, 65520, 65536, 1e9, 2.0 ** -25, 2.0 ** -25 * 1.0001, 2.0 ** -24 * 1.5,
                     5.96e-8, 6.1e-5, -0.0, 0.0], dtype=np.float32)
    x = np.concatenate([finite, mids, near, rnd, edge, -edge])
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)           # numpy casts with round-to-nearest-even
    got = np.array([orc.f32_to_f16(float(v)) for v in x], dtype=np.uint16)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(x[i]), hex(got[i]), hex(ref[i])) for i in bad[:5]]


# ------------------------------------------------------------ golden blocks

@pytest.mark.parametrize("path", sorted(glob.glob(os.path.join(GOLDEN, "*_blocks.txt"))),
                         ids=lambda p: os.path.basename(p))
def test_golden_blocks(orc, path):
    qtype = QT[os.path.basename(path).rsplit("_blocks", 1)[0]]
    be, bb = BLOCK[qtype]
    blocks = bp.parse_golden(path)
    assert blocks
    for title, raw, expect in blocks:
        assert len(raw) == bb and len(expect) == be, title
        got = orc.dequant(qtype, np.frombuffer(raw, dtype=np.uint8), 1, be)[0]
        want = np.array([float(v) for v in expect], dtype=np.float32)
        assert np.array_equal(got, want), (title, got[:16], want[:16])


# -------------------------------------------------- round trip of random blocks

@pytest.mark.parametrize("qtype", ALL)
def test_dequant_round_trip(orc, qtype):
    """pack(logical fields) -> oracle dequant == exact value of d/scale/min/code, bit for bit."""
    rng = np.random.default_rng(10 + qtype)
    be, bb = BLOCK[qtype]
    nblk = 24 if be > 1 else 4096
    fields = [bp.random_fields(qtype, rng) for _ in range(nblk)]
    # plus extreme fields: largest codes and scales, subnormal d
    ext = bp.random_fields(qtype, rng)
    ext["d"] = 0x0003
    if qtype == 2:
        ext["sc"][:] = 63
        ext["m"][:] = 63
        ext["q"][:] = 15
    if qtype == 3:
        ext["sc"][:] = -128
        ext["q"][:] = 0
    if qtype == 4:
        ext["sc"][:] = 63
        ext["m"][:] = 63
        ext["q"][:] = 31
    if qtype == 5:
        ext = {"bits": [0x0001]}            # smallest subnormal
        fields.append({"bits": [0x7BFF]})   # largest finite
        fields.append({"bits": [0x8000]})   # negative zero
    if qtype == 6:
        ext = {"values": [np.float32(1e-45)]}   # smallest fp32 subnormal
    fields.append(ext)
    raw = b"".join(bp.pack(qtype, f) for f in fields)
    got = orc.dequant(qtype, np.frombuffer(raw, dtype=np.uint8), 1, be * len(fields))[0]
    want = np.array([float(v) for f in fields for v in bp.logical_weights(qtype, f)], dtype=np.float32)
    assert np.array_equal(got, want)


# ------------------------------------------------------------------ GEMV

@pytest.mark.parametrize("qtype", ALL)
def test_gemv_exact_integers(orc, qtype):
    """d = dmin = 1 and integer x: every product and sum is an integer, so y is exact."""
    rng = np.random.default_rng(20 + qtype)
    be, bb = BLOCK[qtype]
    rows, nb = 5, (3 if be > 1 else 96)
    cols = nb * be
    W = np.zeros((rows, nb * bb), dtype=np.uint8)
    wint = np.zeros((rows, cols), dtype=np.int64)
    for r in range(rows):
        for b in range(nb):
            f = integer_fields(qtype, rng)
            W[r, b * bb:(b + 1) * bb] = np.frombuffer(bp.pack(qtype, f), dtype=np.uint8)
            wint[r, b * be:(b + 1) * be] = [int(v) for v in bp.logical_weights(qtype, f)]
    x = rng.integers(-9, 10, cols)
    y = orc.gemv(qtype, W, rows, cols, x.astype(np.float32))
    want = wint @ x                                  # exact integer matmul, rows x cols
    assert np.array_equal(y.astype(np.int64), want)
    assert np.array_equal(y, want.astype(np.float32))


def test_gemv_one_hot_picks_column(orc):
    """x = e_k selects column k of W: a transposed operand or wrong row stride fails."""
    rng = np.random.default_rng(3)
    rows, cols = 7, 64
    fields = [[bp.random_fields(0, rng) for _ in range(2)] for _ in range(rows)]
    W = np.frombuffer(b"".join(bp.pack(0, f) for rf in fields for f in rf), dtype=np.uint8).reshape(rows, -1)
    dense = np.array([[float(v) for f in rf for v in bp.logical_weights(0, f)] for rf in fields])
    for k in (0, 31, 32, 63):
        x = np.zeros(cols, dtype=np.float32)
        x[k] = 1.0
        assert np.array_equal(orc.gemv(0, W, rows, cols, x), dense[:, k].astype(np.float32))


@pytest.mark.parametrize("qtype", ALL)
def test_gemv_matches_exact_rational(orc, qtype):
    """Double accumulation of exact products: result is the exact dot product to ~1 ulp of fp32."""
    rng = np.random.default_rng(30 + qtype)
    be, bb = BLOCK[qtype]
    rows, nb = 3, (2 if be > 1 else 64)
    cols = nb * be
    fields = [[bp.random_fields(qtype, rng) for _ in range(nb)] for _ in range(rows)]
    W = np.frombuffer(b"".join(bp.pack(qtype, f) for rf in fields for f in rf), dtype=np.uint8)
    x = rng.standard_normal(cols).astype(np.float32)
    y = orc.gemv(qtype, W.reshape(rows, -1), rows, cols, x)
    for r in range(rows):
        w = [v for f in fields[r] for v in bp.logical_weights(qtype, f)]
        exact = sum(Fr(float(np.float32(wk))) * Fr(float(xk)) for wk, xk in zip(w, x))
        ulp = np.spacing(np.float32(abs(float(exact)))) if exact != 0 else np.float32(1e-45)
        assert abs(float(y[r]) - float(exact)) <= float(ulp), (r, float(y[r]), float(exact))


def test_gemv_rejects_bad_cols(orc):
    with pytest.raises(ValueError):
        orc.gemv(2, np.zeros(144, dtype=np.uint8), 1, 128, np.zeros(128, dtype=np.float32))


# --------------------------------------------------------------- RMSNorm

def test_rmsnorm_constant_vector(orc):
    """x = c * 1: y_i = w_i * c / sqrt(c^2 + eps)."""
    n, eps = 4096, 1e-5
    w = np.linspace(0.9, 1.1, n).astype(np.float32)
    for c in (3.0, -0.25, 1e-3):
        y = orc.rmsnorm(np.full(n, c, dtype=np.float32), w, eps)
        want = w.astype(np.float64) * c / math.sqrt(c * c + float(np.float32(eps)))
        assert np.allclose(y, want, rtol=1e-6, atol=0)


def test_rmsnorm_three_four(orc):
    y = orc.rmsnorm(np.array([3, 4], dtype=np.float32), np.array([1, 2], dtype=np.float32), 0.0)
    r = math.sqrt(12.5)
    assert np.allclose(y, [3 / r, 8 / r], rtol=1e-7)


# ------------------------------------------------------------------ RoPE

def test_rope_identity_at_pos_zero(orc):
    rng = np.random.default_rng(4)
    q = rng.standard_normal(4 * 128).astype(np.float32)
    k = rng.standard_normal(2 * 128).astype(np.float32)
    q2, k2 = orc.rope(q, k, 4, 2, 128, 0, 5e5)
    assert np.array_equal(q2, q) and np.array_equal(k2, k)


def test_rope_preserves_pair_norms(orc):
    rng = np.random.default_rng(5)
    q = rng.standard_normal(8 * 128).astype(np.float32)
    k = rng.standard_normal(2 * 128).astype(np.float32)
    for pos in (1, 17, 4096, 8192):
        q2, k2 = orc.rope(q, k, 8, 2, 128, pos, 5e5)
        for a, b in ((q, q2), (k, k2)):
            n0 = np.hypot(a[0::2].astype(np.float64), a[1::2])
            n1 = np.hypot(b[0::2].astype(np.float64), b[1::2])
            assert np.allclose(n1, n0, rtol=1e-6)


def test_rope_quarter_turn_and_unit_angle(orc):
    """head_dim 4, theta = 4/pi^2, pos 1: pair 1 turns by theta^-1/2 = pi/2, pair 0 by 1 rad."""
    theta = 4.0 / math.pi ** 2
    a, b, c, d = 0.5, -2.0, 3.0, 1.25
    q = np.array([a, b, c, d], dtype=np.float32)
    q2, _ = orc.rope(q, np.zeros(4, dtype=np.float32), 1, 1, 4, 1, theta)
    assert np.allclose(q2[2:], [-d, c], atol=1e-6)                        # (c, d) -> (-d, c)
    assert np.allclose(q2[:2], [a * math.cos(1) - b * math.sin(1), a * math.sin(1) + b * math.cos(1)], atol=1e-6)


def test_rope_composes_as_rotation(orc):
    """rope(p1) then rope(p2) == rope(p1 + p2) (rotations by angles that add)."""
    rng = np.random.default_rng(6)
    q = rng.standard_normal(2 * 64).astype(np.float32)
    k = rng.standard_normal(64).astype(np.float32)
    qa, ka = orc.rope(q, k, 2, 1, 64, 300, 1e4)
    qb, kb = orc.rope(qa, ka, 2, 1, 64, 123, 1e4)
    qc, kc = orc.rope(q, k, 2, 1, 64, 423, 1e4)
    assert np.allclose(qb, qc, atol=3e-6) and np.allclose(kb, kc, atol=3e-6)


# --------------------------------------------------------------- softmax

def test_softmax_closed_form_and_sum(orc):
    y = orc.softmax(np.array([0.0, math.log(2.0)], dtype=np.float32))
    assert np.allclose(y, [1 / 3, 2 / 3], rtol=1e-6)
    rng = np.random.default_rng(7)
    x = (np.round(rng.standard_normal(128256) * 8 * 1024) / 1024).astype(np.float32)
    y = orc.softmax(x)
    assert abs(float(np.sum(y, dtype=np.float64)) - 1.0) < 1e-5
    assert np.allclose(orc.softmax(x + np.float32(1024.0)), y, rtol=1e-6, atol=1e-30)   # exact shift: invariance, no overflow
    assert np.argmax(y) == np.argmax(x)


# ---------------------------------------------------------------- SwiGLU

def test_swiglu_special_values(orc):
    g = np.array([0.0, 1.0, 30.0, -30.0], dtype=np.float32)
    u = np.array([5.0, 1.0, 2.0, 2.0], dtype=np.float32)
    out = orc.swiglu(g, u)
    assert out[0] == 0.0
    assert math.isclose(out[1], math.e / (1 + math.e), rel_tol=1e-7)       # silu(1) = 1 / (1 + e^-1)
    assert math.isclose(out[2], 60.0, rel_tol=1e-7)                          # silu(g) -> g for large g
    assert abs(out[3]) < 1e-10                                               # silu(g) -> 0 for very negative g


# ------------------------------------------------------------- attention

def _f16(a):
    return np.asarray(a, dtype=np.float16).view(np.uint16)


def test_attention_single_position_returns_v(orc):
    hd, max_ctx = 16, 4
    rng = np.random.default_rng(8)
    kc = _f16(rng.standard_normal((2, max_ctx, hd)))
    vc = _f16(rng.standard_normal((2, max_ctx, hd)))
    q = rng.standard_normal(4 * hd).astype(np.float32)
    out = orc.attn_decode(q, kc, vc, 4, 2, hd, 1, max_ctx).reshape(4, hd)
    v = vc.view(np.float16).astype(np.float32)
    for h in range(4):
        assert np.array_equal(out[h], v[h // 2, 0])                           # GQA: head h reads kv head h // 2


def test_attention_one_hot_values_give_probabilities(orc):
    """V[t] = e_t turns the output into the softmax weights; K chosen so scores are known."""
    hd, n_ctx, max_ctx = 8, 6, 8
    kc = np.zeros((1, max_ctx, hd), dtype=np.float16)
    vc = np.zeros((1, max_ctx, hd), dtype=np.float16)
    for t in range(n_ctx):
        kc[0, t, 0] = t * 0.5
        vc[0, t, t] = 1.0
    kc[0, n_ctx:, 0] = 100.0            # positions past n_ctx must not be read
    vc[0, n_ctx:, :] = 100.0
    a = 2.0
    q = np.zeros(hd, dtype=np.float32)
    q[0] = a
    out = orc.attn_decode(q, kc.view(np.uint16), vc.view(np.uint16), 1, 1, hd, n_ctx, max_ctx)
    s = [a * t * 0.5 / math.sqrt(hd) for t in range(n_ctx)]
    z = sum(math.exp(v) for v in s)
    want = [math.exp(v) / z for v in s] + [0.0] * (hd - n_ctx)
    assert np.allclose(out, want, rtol=1e-6, atol=1e-7)
    assert abs(float(np.sum(out, dtype=np.float64)) - 1.0) < 1e-6


def test_attention_group_mapping(orc):
    """4 q heads over 2 kv heads: heads 0,1 read group 0, heads 2,3 read group 1."""
    hd, max_ctx = 4, 2
    kc = np.zeros((2, max_ctx, hd), dtype=np.float16)
    vc = np.zeros((2, max_ctx, hd), dtype=np.float16)
    vc[0, :, 0] = 1.0
    vc[1, :, 1] = 1.0
    q = np.ones(4 * hd, dtype=np.float32)
    out = orc.attn_decode(q, kc.view(np.uint16), vc.view(np.uint16), 4, 2, hd, 2, max_ctx).reshape(4, hd)
    assert np.array_equal(out, [[1, 0, 0, 0], [1, 0, 0, 0], [0, 1, 0, 0], [0, 1, 0, 0]])
