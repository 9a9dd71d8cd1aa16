"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these compares the oracle with itself: each check uses an independent
route (a library routine, a closed form, brute force, exact rational
arithmetic, or a hand derivation stored under tests/golden/).
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def sylvester_by_popcount(n=32):
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    pc = np.vectorize(lambda v: bin(int(v)).count("1"))(i & j)
    return np.where(pc % 2 == 0, 1.0, -1.0)


# ----------------------------------------------------------------------------
# Hadamard
# ----------------------------------------------------------------------------

def test_fwht_of_unit_vectors_gives_sylvester_columns():
    eye = np.eye(32, dtype=np.float32)
    cols = np.stack([oracle.fwht32(eye[j]) for j in range(32)], axis=1)
    assert np.array_equal(cols, sylvester_by_popcount())
    assert np.array_equal(cols, scipy.linalg.hadamard(32).astype(np.float32))


def test_hadamard_is_orthogonal_times_32():
    eye = np.eye(32, dtype=np.float32)
    H = np.stack([oracle.fwht32(eye[j]) for j in range(32)], axis=1).astype(np.float64)
    assert np.array_equal(H @ H.T, 32.0 * np.eye(32))


def test_fwht_matches_library_matmul_when_sums_are_exact():
    rng = np.random.default_rng(1)
    v = rng.integers(-1000, 1000, size=(64, 32)).astype(np.float32)
    got = oracle.fwht32(v.ravel()).reshape(64, 32)
    want = v.astype(np.float64) @ scipy.linalg.hadamard(32).T.astype(np.float64)
    assert np.array_equal(got.astype(np.float64), want)


def test_fwht_all_equal_block():
    for val in [1.0, -3.5, 0.15625, 1e-20, 6e30]:
        got = oracle.fwht32(np.full(32, val, np.float32))
        assert got[0] == np.float32(32 * np.float64(np.float32(val)))
        assert np.all(got[1:] == 0)


def test_fwht_twice_is_32_times_identity_on_exact_values():
    rng = np.random.default_rng(2)
    v = rng.integers(-64, 64, size=32).astype(np.float32)
    assert np.array_equal(oracle.fwht32(oracle.fwht32(v)), 32 * v)


def test_fwht_fp32_rounding_matches_stagewise_numpy_float32():
    # each butterfly output is one binary32 rounding: numpy float32 adds in
    # the same pairing order reproduce it; a different order generally not.
    rng = np.random.default_rng(3)
    v = (rng.standard_normal(32) * np.exp2(rng.integers(-20, 20, 32))).astype(np.float32)
    w = v.copy()
    h = 1
    while h < 32:
        out = w.copy()
        for i in range(32):
            if i & h:
                continue
            out[i] = np.float32(w[i] + w[i + h])
            out[i + h] = np.float32(w[i] - w[i + h])
        w = out
        h <<= 1
    assert np.array_equal(oracle.fwht32(v), w)


# ----------------------------------------------------------------------------
# BF16 rounding
# ----------------------------------------------------------------------------

def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(4)
    bits = rng.integers(0, 2**32, size=20000, dtype=np.uint64).astype(np.uint32)
    # force many exact ties and near-ties
    bits[:4000] = (bits[:4000] & 0xFFFF0000) | 0x8000
    bits[4000:6000] = (bits[4000:6000] & 0xFFFF0000) | 0x7FFF
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    got = oracle.f32_to_bf16(f)
    want = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)


# ----------------------------------------------------------------------------
# E2M1 and E8M0
# ----------------------------------------------------------------------------

def test_e2m1_table_matches_golden():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "e2m1_values.txt"))
            if l.strip() and not l.startswith("#")]
    for code, val in rows:
        got = oracle.e2m1_decode(int(code))
        assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val))


def brute_force_e2m1(a: float) -> int:
    """Nearest of the 8 magnitudes, ties to the even code, saturating."""
    s = 8 if math.copysign(1.0, a) < 0 else 0
    m = abs(a)
    if m >= 6.0:  # saturation; below 6 the float64 distances are exact
        return s | 7
    d = np.abs(E2M1_GRID - m)
    best = np.flatnonzero(d == d.min())
    if best.size > 1:
        best = best[best % 2 == 0]
    return s | int(best[0])


def test_e2m1_encode_exhaustive_over_bf16():
    bits = np.arange(65536, dtype=np.uint32)
    f32 = (bits << 16).view(np.float32)
    ok = np.isfinite(f32)
    vals = f32[ok].astype(np.float64)
    ok = np.ones(vals.size, bool)
    for v in vals[ok]:
        assert oracle.e2m1_encode(v) == brute_force_e2m1(v), v


def test_e2m1_tie_points():
    for t, want in [(0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6),
                    (6.0, 7), (7.99, 7), (-0.25, 8), (-0.1, 8), (-5.0, 14)]:
        assert oracle.e2m1_encode(t) == want, t


def test_e8m0_defining_property():
    # For every positive finite binary32 exponent and a few mantissas, the
    # scale X = 2^(c-127) puts amax/X in [4, 8) unless clamped at c = 0.
    for e in range(-149, 128):
        for mant in [1.0, 1.3, 1.5, 1.999999]:
            a = np.float32(mant * 2.0 ** e)
            if not np.isfinite(a) or a == 0:
                continue
            c = oracle.e8m0_from_amax(a)
            assert 0 <= c <= 254          # an E8M0 code (255 is NaN); tiny amax clamps to 0
            r = Fraction(float(a)) / Fraction(2) ** (c - 127)
            assert r < 8
            if c > 0:
                assert r >= 4
            else:
                assert Fraction(float(a)) < Fraction(2) ** (-127 + 3)
    assert oracle.e8m0_from_amax(0.0) == 0
    assert oracle.e8m0_from_amax(float("inf")) == 255
    assert oracle.e8m0_from_amax(float("nan")) == 255


def test_round_trip_every_code_every_scale():
    # A block holding every code once (and 6 to fix the scale) quantises back
    # to itself for every scale code whose values are representable.
    codes = np.array(list(range(16)) + [7] * 16)
    for c in range(0, 253):
        vals = np.array([np.ldexp(oracle.e2m1_decode(int(k)), c - 127) for k in codes])
        f = vals.astype(np.float32)
        assert np.array_equal(f.astype(np.float64), vals)
        q, s = oracle.mx_quantize_blocks(f)
        assert s[0] == c
        got = oracle.unpack_codes(q)
        assert np.array_equal(got, codes), c


def test_idempotent_on_representable_random_blocks():
    rng = np.random.default_rng(5)
    for _ in range(300):
        c = int(rng.integers(1, 250))
        codes = rng.integers(0, 16, size=32)
        codes[rng.integers(0, 32)] = 7  # amax code fixes the scale
        vals = np.array([np.ldexp(oracle.e2m1_decode(int(k)), c - 127) for k in codes], np.float32)
        q, s = oracle.mx_quantize_blocks(vals)
        deq = oracle.dequantize(q.reshape(1, 16), s.reshape(1, 1))[0]
        assert np.array_equal(deq, vals.astype(np.float64))


def test_zero_and_negative_zero_blocks():
    q, s = oracle.mx_quantize_blocks(np.zeros(32, np.float32))
    assert s[0] == 0 and np.all(q == 0)
    q, s = oracle.mx_quantize_blocks(-np.zeros(32, np.float32))
    assert s[0] == 0 and np.all(q == 0x88)


def test_random_blocks_against_brute_force():
    rng = np.random.default_rng(6)
    for _ in range(200):
        v = (rng.standard_normal(32) * np.exp2(rng.integers(-30, 30))).astype(np.float32)
        q, s = oracle.mx_quantize_blocks(v)
        c = int(s[0])
        amax = float(np.max(np.abs(v)))
        r = Fraction(amax) / Fraction(2) ** (c - 127)
        assert 4 <= r < 8
        want = [brute_force_e2m1(float(np.ldexp(np.float64(x), 127 - c))) for x in v]
        assert np.array_equal(oracle.unpack_codes(q), np.array(want))


# ----------------------------------------------------------------------------
# Activation and weight paths
# ----------------------------------------------------------------------------

def _pattern(name):
    if name == "ones":
        return np.ones(32, np.float32)
    if name == "alt":
        return np.array([(-1.0) ** i for i in range(32)], np.float32)
    if name == "neg":
        return -np.ones(32, np.float32)
    if name == "zero":
        return np.zeros(32, np.float32)
    if name == "spike3":
        v = np.zeros(32, np.float32)
        v[0] = 3.0
        return v
    raise ValueError(name)


def test_hand_derived_blocks():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "hand_blocks.txt"))
            if l.strip() and not l.startswith("#")]
    assert len(rows) == 6
    for name, d, pat, scale, b0, brest in rows:
        x = synth.to_bf16_bits(_pattern(pat)[None, :])
        D = np.full(32, float(d), np.float32)
        q, s = oracle.quantize_act(x, D)
        assert int(s[0, 0]) == int(scale), name
        assert int(q[0, 0]) == int(b0, 16), name
        assert np.all(q[0, 1:] == int(brest, 16)), name


def test_activation_steps_follow_definition():
    # the rotated activations, re-derived with numpy float32 and torch bf16
    rng = np.random.default_rng(7)
    M, K = 3, 96
    x = synth.to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32) * 4)
    D = (np.exp(rng.standard_normal(K)) * np.sign(rng.standard_normal(K))).astype(np.float32)
    r = (np.float32(1.0) / D).astype(np.float32)
    xs = synth.bf16_bits_to_f32(synth.to_bf16_bits(synth.bf16_bits_to_f32(x) * r))
    H = scipy.linalg.hadamard(32).astype(np.float64)
    u = oracle.act_rotate(x, D)
    uf = synth.bf16_bits_to_f32(u).astype(np.float64)
    ref = (xs.reshape(M, K // 32, 32).astype(np.float64) @ H.T).reshape(M, K)
    # BF16 output of an FP32 butterfly: within one bf16 ulp of the exact rotation
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    assert np.all(np.abs(uf - ref) <= ulp + 1e-30)


def test_unquantised_transform_preserves_the_layer():
    # pins R1 (x/D with W*D) and R2 (H H^T = 32 I, 1/32 afterwards)
    rng = np.random.default_rng(8)
    M, N, K = 5, 7, 128
    x = synth.to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    W = rng.standard_normal((N, K)).astype(np.float32)
    D = (np.exp(rng.standard_normal(K)) * np.where(rng.random(K) < 0.3, -1, 1)).astype(np.float32)
    got = oracle.transform_f64(x, D, W)
    want = oracle.linear_f64(x, W)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_unquantised_linear_is_the_library_matmul():
    # the reference layer x . W^T against numpy's binary64 matmul (independent of
    # the oracle's own loops); a transposed operand or a dropped row fails it
    rng = np.random.default_rng(18)
    M, N, K = 6, 9, 96
    x = synth.to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    W = rng.standard_normal((N, K)).astype(np.float32)
    want = oracle.bf16_to_f64(x) @ W.astype(np.float64).T
    got = oracle.linear_f64(x, W)
    assert got.shape == (M, N)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_weight_path_definition():
    rng = np.random.default_rng(9)
    N, K = 4, 64
    W = rng.standard_normal((N, K)).astype(np.float32)
    D = np.exp(rng.standard_normal(K)).astype(np.float32)
    q, s = oracle.quantize_weights(W, D)
    t = (W * D).astype(np.float32)
    tt = np.stack([oracle.fwht32(row) for row in t])
    q2, s2 = oracle.mx_quantize_blocks(tt)
    assert np.array_equal(q.ravel(), q2) and np.array_equal(s.ravel(), s2)
    # no bf16 rounding on the weight side: compare with an exact rotation
    tb = t.reshape(N, K // 32, 32).astype(np.float64)
    ref = (tb @ scipy.linalg.hadamard(32).T).reshape(N, K)
    # five binary32 roundings per output: |err| <= 5 * 2^-24 * sum |t| of the block
    bound = np.repeat(5 * 2.0 ** -24 * np.abs(tb).sum(axis=2), 32, axis=1)
    assert np.all(np.abs(tt - ref) <= bound)


# ----------------------------------------------------------------------------
# Exact block-scaled GEMM
# ----------------------------------------------------------------------------

def fraction_to_bf16_bits(v: Fraction) -> int:
    """Correct RNE rounding of an exact rational to bf16 (independent code)."""
    if v == 0:
        return 0
    sign = 0x8000 if v < 0 else 0
    a = abs(v)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    lsb = e - 7 if e >= -126 else -133
    q = a / Fraction(2) ** lsb
    fl = math.floor(q)
    rem = q - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    if lsb == -133:
        bits = fl
    else:
        bits = ((e + 127) << 7) + (fl - 128)
    bits = min(bits, 0x7F80)
    return sign | bits


def exact_y(qa, sa, qw, sw, div=32):
    M, K = qa.shape[0], qa.shape[1] * 2
    N = qw.shape[0]
    ca, cw = oracle.unpack_codes(qa), oracle.unpack_codes(qw)
    out = np.zeros((M, N), np.uint16)
    for m in range(M):
        for n in range(N):
            s = Fraction(0)
            for k in range(K):
                s += (Fraction(oracle.e2m1_decode(int(ca[m, k])))
                      * Fraction(2) ** (int(sa[m, k // 32]) - 127)
                      * Fraction(oracle.e2m1_decode(int(cw[n, k])))
                      * Fraction(2) ** (int(sw[n, k // 32]) - 127))
            out[m, n] = fraction_to_bf16_bits(s / div)
    return out


@pytest.mark.parametrize("spread", ["narrow", "wide", "extreme"])
def test_exact_gemm_against_rationals(spread):
    rng = np.random.default_rng({"narrow": 10, "wide": 11, "extreme": 12}[spread])
    M, N, K = 3, 4, 96
    qa = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    qw = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    if spread == "narrow":
        sa = rng.integers(120, 135, size=(M, K // 32), dtype=np.uint8)
        sw = rng.integers(115, 125, size=(N, K // 32), dtype=np.uint8)
    elif spread == "wide":
        sa = rng.integers(60, 200, size=(M, K // 32), dtype=np.uint8)
        sw = rng.integers(60, 200, size=(N, K // 32), dtype=np.uint8)
    else:
        sa = rng.choice(np.array([0, 1, 254, 127, 2], np.uint8), size=(M, K // 32))
        sw = rng.choice(np.array([0, 254, 130, 3], np.uint8), size=(N, K // 32))
    got = oracle.gemm(qa, sa, qw, sw)
    assert np.array_equal(got, exact_y(qa, sa, qw, sw))
    rows, cols = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
    at = oracle.gemm_at(qa, sa, qw, sw, rows.ravel(), cols.ravel())
    assert np.array_equal(at, got.ravel())


@pytest.mark.parametrize("spread", ["narrow", "wide", "extreme"])
def test_plain_exact_gemm_against_rationals(spread):
    # plain MXFP4 product: the same exact sum, rounded once to bf16, no 2^-5
    rng = np.random.default_rng({"narrow": 20, "wide": 21, "extreme": 22}[spread])
    M, N, K = 3, 4, 96
    qa = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    qw = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    if spread == "narrow":
        sa = rng.integers(120, 135, size=(M, K // 32), dtype=np.uint8)
        sw = rng.integers(115, 125, size=(N, K // 32), dtype=np.uint8)
    elif spread == "wide":
        sa = rng.integers(60, 200, size=(M, K // 32), dtype=np.uint8)
        sw = rng.integers(60, 200, size=(N, K // 32), dtype=np.uint8)
    else:
        sa = rng.choice(np.array([0, 1, 254, 127, 2], np.uint8), size=(M, K // 32))
        sw = rng.choice(np.array([0, 254, 130, 3], np.uint8), size=(N, K // 32))
    got = oracle.gemm_plain(qa, sa, qw, sw)
    assert np.array_equal(got, exact_y(qa, sa, qw, sw, div=1))
    rows, cols = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
    assert np.array_equal(oracle.gemm_at_plain(qa, sa, qw, sw, rows.ravel(), cols.ravel()), got.ravel())


def test_plain_linear_is_exact_on_representable_operands():
    # Values that are E2M1 codes times a power of two with the block amax in
    # [4, 8) x 2^k quantise losslessly, so the plain layer reduces to the
    # correctly rounded exact product x . W^T.
    rng = np.random.default_rng(23)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    M, N, K = 3, 5, 64
    def representable(rows):
        v = rng.choice(grid, size=(rows, K)) * rng.choice([-1, 1], size=(rows, K))
        v[:, ::32] = 6.0 * rng.choice([-1, 1], size=(rows, K // 32))  # fixes each block's amax
        scale = 2.0 ** rng.integers(-6, 4, size=(rows, K // 32))
        return v * np.repeat(scale, 32, axis=1)
    x = representable(M)
    W = representable(N)
    xb = synth.to_bf16_bits(x.astype(np.float32))
    assert np.array_equal(synth.bf16_bits_to_f32(xb).astype(np.float64), x)  # exact in bf16 too
    y = oracle.dense_mm_plain(xb, W.astype(np.float32))
    for m in range(M):
        for n in range(N):
            s = sum((Fraction(x[m, k]) * Fraction(W[n, k]) for k in range(K)), Fraction(0))
            assert y[m, n] == fraction_to_bf16_bits(s), (m, n)


def test_plain_grouped_replicated_banks_equal_dense():
    p = synth.dense(40, 256, 48, seed=3)
    W = np.stack([p.W[0]] * 3)
    st, yg = oracle.grouped_mm_plain(p.x, W, np.array([10, 0, 30], np.int64), 1)
    assert st == 0
    assert np.array_equal(yg, oracle.dense_mm_plain(p.x, p.W[0]))


def _pack(codes):
    codes = np.asarray(codes, np.uint8)
    return (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)


def test_exact_gemm_subnormal_outputs():
    # one product 1.5 x 1.0 per output, scales chosen so that 2^-5 times it lands
    # in BF16's subnormal range (last bit 2^-133): 1.5 x 2^(64+65-259) = 12 x 2^-133
    # exactly, and 1.5 x 2^(64+62-259) = 1.5 x 2^-133, a tie between 1 and 2 units
    # that rounds to the even 2
    qa = np.zeros((1, 16), np.uint8)
    qa[0, 0] = 3                      # code 3 = 1.5 (element 0, low nibble)
    qw = np.zeros((2, 16), np.uint8)
    qw[:, 0] = 2                      # code 2 = 1.0
    sa = np.array([[64]], np.uint8)
    sw = np.array([[65], [62]], np.uint8)
    y = oracle.gemm(qa, sa, qw, sw)
    unit = Fraction(2) ** -133
    for n, s_w in enumerate((65, 62)):
        exact = Fraction(3, 2) * Fraction(2) ** (64 + s_w - 254 - 5)
        q = exact / unit
        units = int(q) + (1 if (q - int(q) > Fraction(1, 2) or (q - int(q) == Fraction(1, 2) and int(q) % 2)) else 0)
        assert y[0, n] == units        # BF16 subnormal bits = number of 2^-133 units
    assert list(y[0]) == [0x000C, 0x0002]


def test_plain_grouped_rows_use_the_named_expert():
    # type-2 list with one-row ranges, a repeated expert and an empty entry: each
    # range equals the plain dense product with the expert it names
    p = synth.grouped(40, 4, 64, 32, seed=8, dist="uniform", group_list_type=1)
    gl = np.array([[2, 1], [0, 0], [3, 38], [2, 1]], np.int64)
    st, y = oracle.grouped_mm_plain(p.x, p.W, gl, 2)
    assert st == oracle.OK
    r0 = 0
    for e, n in gl:
        if n:
            assert np.array_equal(y[r0:r0 + n], oracle.dense_mm_plain(p.x[r0:r0 + n], p.W[e])), (e, n)
        r0 += n


def test_exact_gemm_cancellation_and_ties():
    # +1 and -1 against +1, +1: the sum cancels to exactly +0
    ca = np.zeros((1, 32), int); cw = np.zeros((1, 32), int)
    ca[0, :2] = [0x2, 0xA]; cw[0, :2] = [0x2, 0x2]
    s127 = np.full((1, 1), 127, np.uint8)
    assert oracle.gemm(_pack(ca), s127, _pack(cw), s127)[0, 0] == 0
    # 8 * (4 * 1) + 0.5 * 0.5 * 2^-1 = 32 + 1/8; / 32 = 1 + 2^-8: a tie between
    # bf16 1.0 and 1 + 2^-7 -> even -> 1.0; one more tiny term breaks the tie upward
    ca = np.zeros((1, 64), int); cw = np.zeros((1, 64), int)
    ca[0, :8] = 6; cw[0, :8] = 2
    ca[0, 32] = 1; cw[0, 32] = 1
    sa = np.array([[127, 126]], np.uint8); sw = np.array([[127, 127]], np.uint8)
    assert oracle.gemm(_pack(ca), sa, _pack(cw), sw)[0, 0] == 0x3F80
    ca[0, 33] = 1; cw[0, 33] = 1
    sa2 = np.array([[127, 100]], np.uint8)
    ca2 = ca.copy(); ca2[0, 32] = 0; ca2[0, 33] = 0
    # exact tie again but via block 1 at a much smaller scale plus the tie term
    ca3 = np.zeros((1, 96), int); cw3 = np.zeros((1, 96), int)
    ca3[0, :8] = 6; cw3[0, :8] = 2
    ca3[0, 32] = 1; cw3[0, 32] = 1
    ca3[0, 64] = 1; cw3[0, 64] = 1
    sa3 = np.array([[127, 126, 60]], np.uint8); sw3 = np.array([[127, 127, 127]], np.uint8)
    assert oracle.gemm(_pack(ca3), sa3, _pack(cw3), sw3)[0, 0] == 0x3F81
    ca3[0, 64] = 9  # the tiny term negative: just below the tie -> 1.0
    assert oracle.gemm(_pack(ca3), sa3, _pack(cw3), sw3)[0, 0] == 0x3F80


# ----------------------------------------------------------------------------
# Grouped form
# ----------------------------------------------------------------------------

def test_group_list_validation_rules():
    M = 10
    assert oracle.group_offsets([3, 7, 10], 0, M)[0] == oracle.OK
    assert oracle.group_offsets([3, 4, 3], 1, M)[0] == oracle.OK
    assert oracle.group_offsets([3, 2, 10], 0, M)[0] == oracle.ERR_GROUP_LIST_INVALID  # decreasing
    assert oracle.group_offsets([-1, 2, 10], 0, M)[0] == oracle.ERR_GROUP_LIST_INVALID
    assert oracle.group_offsets([3, -1, 8], 1, M)[0] == oracle.ERR_GROUP_LIST_INVALID
    assert oracle.group_offsets([3, 7, 9], 0, M)[0] == oracle.ERR_GROUP_LIST_INVALID  # != M
    assert oracle.group_offsets([3, 4, 4], 1, M)[0] == oracle.ERR_GROUP_LIST_INVALID
    assert oracle.group_offsets([3, 7, 10], 3, M)[0] == oracle.ERR_GROUP_LIST_TYPE
    # type 2: [E, 2] rows of (group index, group size); sizes add up along M
    assert oracle.group_offsets([[2, 3], [0, 7], [1, 0]], 2, M)[0] == oracle.OK
    assert oracle.group_offsets([[2, 3], [0, 6], [1, 0]], 2, M)[0] == oracle.ERR_GROUP_LIST_INVALID  # sum != M
    assert oracle.group_offsets([[3, 3], [0, 7], [1, 0]], 2, M)[0] == oracle.ERR_GROUP_LIST_INVALID  # index >= E
    assert oracle.group_offsets([[2, 3], [-1, 7], [1, 0]], 2, M)[0] == oracle.ERR_GROUP_LIST_INVALID
    assert oracle.group_offsets([[2, -3], [0, 13], [1, 0]], 2, M)[0] == oracle.ERR_GROUP_LIST_INVALID
    assert oracle.group_offsets(np.zeros(1025, np.int64), 1, 0)[0] == oracle.ERR_TOO_MANY_GROUPS
    st, off = oracle.group_offsets([0, 0, 4, 4, 10], 0, M)
    assert st == oracle.OK and list(off) == [0, 0, 0, 4, 4, 10]


def test_grouped_cumsum_equals_counts_and_replicated_banks_equal_dense():
    p = synth.grouped(96, 4, 64, 48, seed=3, dist="uniform", group_list_type=1)
    st1, y1 = oracle.grouped_mm(p.x, p.D, p.W, p.group_list, 1)
    st0, y0 = oracle.grouped_mm(p.x, p.D, p.W, np.cumsum(p.group_list), 0)
    assert st0 == st1 == oracle.OK and np.array_equal(y0, y1)
    # replicated banks: every expert has expert 0's W and D
    Wr = np.repeat(p.W[:1], 4, axis=0)
    Dr = np.repeat(p.D[:1], 4, axis=0)
    st, yr = oracle.grouped_mm(p.x, Dr, Wr, p.group_list, 1)
    assert st == oracle.OK
    assert np.array_equal(yr, oracle.dense_mm(p.x, p.D[0], p.W[0]))


def test_grouped_type2_rows_use_the_named_expert():
    # type 2 names each range's expert: permuting the experts and naming them in the
    # list gives the same output as the counts form on the original order
    p = synth.grouped(80, 4, 64, 32, seed=6, dist="uniform", group_list_type=1)
    perm = np.array([2, 0, 3, 1])
    Wp, Dp = np.empty_like(p.W), np.empty_like(p.D)
    Wp[perm], Dp[perm] = p.W, p.D  # expert g now lives at index perm[g]
    gl2 = np.stack([perm, p.counts]).T.astype(np.int64)
    st2, y2 = oracle.grouped_mm(p.x, Dp, Wp, gl2, 2)
    st1, y1 = oracle.grouped_mm(p.x, p.D, p.W, p.counts.astype(np.int64), 1)
    assert st1 == st2 == oracle.OK and np.array_equal(y1, y2)
    # an expert named twice and one never named
    gl3 = np.array([[1, 30], [1, 20], [3, 30], [0, 0]], np.int64)
    st3, y3 = oracle.grouped_mm(p.x, p.D, p.W, gl3, 2)
    assert st3 == oracle.OK
    assert np.array_equal(y3[:50], oracle.dense_mm(p.x[:50], p.D[1], p.W[1]))
    assert np.array_equal(y3[50:], oracle.dense_mm(p.x[50:], p.D[3], p.W[3]))


def test_grouped_weight_list_equals_the_stacked_weights():
    # npu_grouped_matmul's weight given as a list (one tensor per expert) is the
    # same layer as the stacked [E, N, K] weight: the list form is written as one
    # dense call per entry, the stacked form is the C grouped routine
    p = synth.grouped(120, 5, 64, 32, seed=8, dist="zipf", group_list_type=1)
    W_list = [np.ascontiguousarray(p.W[e]) for e in range(p.E)]
    gl2 = np.ascontiguousarray(np.stack([np.array([4, 0, 2, 2, 1]), p.counts]).T.astype(np.int64))
    for gl, t in [(p.counts.astype(np.int64), 1), (np.cumsum(p.counts).astype(np.int64), 0), (gl2, 2)]:
        st_l, y_l = oracle.grouped_mm_list(p.x, p.D, W_list, gl, t)
        st_s, y_s = oracle.grouped_mm(p.x, p.D, p.W, gl, t)
        assert st_l == st_s == oracle.OK
        assert np.array_equal(y_l, y_s), t
    bad = p.counts.astype(np.int64).copy()
    bad[0] += 1
    assert oracle.grouped_mm_list(p.x, p.D, W_list, bad, 1)[0] == oracle.ERR_GROUP_LIST_INVALID


def test_grouped_rows_use_their_own_expert():
    p = synth.grouped(64, 3, 64, 32, seed=4, dist="uniform", group_list_type=1)
    st, y = oracle.grouped_mm(p.x, p.D, p.W, p.group_list, 1)
    assert st == oracle.OK
    off = np.concatenate([[0], np.cumsum(p.counts)])
    for g in range(3):
        rows = slice(off[g], off[g + 1])
        assert np.array_equal(y[rows], oracle.dense_mm(p.x[rows], p.D[g], p.W[g]))


def test_grouped_empty_groups():
    p = synth.grouped(40, 4, 64, 32, seed=5, dist="uniform", group_list_type=1)
    counts = np.array([0, 40, 0, 0], np.int64)
    st, y = oracle.grouped_mm(p.x, p.D, p.W, counts, 1)
    assert st == oracle.OK
    assert np.array_equal(y, oracle.dense_mm(p.x, p.D[1], p.W[1]))


def test_grouped_one_row_groups():
    # groups of a single row at the start, middle and end, around empty ones:
    # each row equals the dense product with its own expert
    p = synth.grouped(40, 5, 64, 32, seed=7, dist="uniform", group_list_type=1)
    counts = np.array([1, 0, 38, 0, 1], np.int64)
    st, y = oracle.grouped_mm(p.x, p.D, p.W, counts, 1)
    assert st == oracle.OK
    off = np.concatenate([[0], np.cumsum(counts)])
    for g in range(5):
        if counts[g]:
            want = oracle.dense_mm(p.x[off[g]:off[g + 1]], p.D[g], p.W[g])
            assert np.array_equal(y[off[g]:off[g + 1]], want), g


# ----------------------------------------------------------------------------
# Whole-layer sanity: the method's accuracy direction
# ----------------------------------------------------------------------------

def test_macaq_beats_plain_mxfp4_on_outlier_activations():
    # Direction stated by the accuracy section (native error > MACAQ error);
    # the size of the ratio on synthetic data is not pinned.
    p = synth.dense(32, 256, 64, seed=0)
    ref = oracle.linear_f64(p.x, p.W[0])
    y = synth.bf16_bits_to_f32(oracle.dense_mm(p.x, p.D[0], p.W[0])).astype(np.float64)
    yp = synth.bf16_bits_to_f32(oracle.dense_mm_plain(p.x, p.W[0])).astype(np.float64)
    nmse = lambda a: float(np.sum((a - ref) ** 2) / np.sum(ref ** 2))
    assert nmse(y) < nmse(yp)
    assert nmse(y) < 0.05


# ----------------------------------------------------------------------------
# Epilogue: bias and act_type (npu_grouped_matmul, parameters bias and act_type)
# ----------------------------------------------------------------------------

ACTS = [oracle.ACT_RELU, oracle.ACT_GELU_TANH, oracle.ACT_FAST_GELU, oracle.ACT_SILU]


def test_activations_match_library_routines():
    v = np.linspace(-12.0, 12.0, 4001)
    t = torch.from_numpy(v)
    assert np.array_equal(oracle.act(v, oracle.ACT_RELU), np.maximum(v, 0.0))
    np.testing.assert_allclose(oracle.act(v, oracle.ACT_GELU_TANH),
                               torch.nn.functional.gelu(t, approximate="tanh").numpy(), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(oracle.act(v, oracle.ACT_SILU), torch.nn.functional.silu(t).numpy(),
                               rtol=1e-13, atol=1e-15)
    assert np.array_equal(oracle.act(v, oracle.ACT_NONE), v)


def test_activations_odd_part_is_the_identity():
    # f(v) - f(-v) == v for every sigmoid- or tanh-gated form v * g(v) with
    # g(v) + g(-v) == 1: a dropped factor, a wrong sign or a missing 0.5 breaks it
    v = np.linspace(-30.0, 30.0, 6001)
    for a in (oracle.ACT_RELU, oracle.ACT_GELU_TANH, oracle.ACT_FAST_GELU, oracle.ACT_SILU):
        np.testing.assert_allclose(oracle.act(v, a) - oracle.act(-v, a), v, rtol=1e-12, atol=1e-12)


def test_gelu_forms_approximate_the_exact_gelu():
    # exact GELU v * Phi(v) from the error function; the tanh form is within
    # 1e-3 of it, the 1.702-sigmoid form (FAST_GELU reading) within 2.5e-2
    v = np.linspace(-8.0, 8.0, 3201)
    exact = np.array([x * 0.5 * (1.0 + math.erf(x / math.sqrt(2.0))) for x in v])
    assert np.max(np.abs(oracle.act(v, oracle.ACT_GELU_TANH) - exact)) < 1e-3
    assert np.max(np.abs(oracle.act(v, oracle.ACT_FAST_GELU) - exact)) < 2.5e-2
    # and the sigmoid slope: FAST_GELU'(0) = 1/2 like GELU, second derivative 1.702/2
    h = 1e-4
    d2 = (oracle.act(np.array([h]), 4)[0] - 2 * 0.0 + oracle.act(np.array([-h]), 4)[0]) / h ** 2
    assert abs(d2 - 1.702 / 2) < 1e-6


def test_f64_to_bf16_rounds_once_to_nearest_even():
    # every positive finite bf16 value and the midpoints between neighbours
    bits = np.arange(1, 0x7f80, dtype=np.uint32)
    vals = (bits << 16).view(np.float32).astype(np.float64)
    assert np.array_equal(oracle.f64_to_bf16(vals), bits.astype(np.uint16))
    assert np.array_equal(oracle.f64_to_bf16(-vals), (bits | 0x8000).astype(np.uint16))
    lo, hi = vals[:-1], vals[1:]
    mid = (lo + hi) / 2                          # exact in binary64
    even = np.where(bits[:-1] % 2 == 0, bits[:-1], bits[1:]).astype(np.uint16)
    assert np.array_equal(oracle.f64_to_bf16(mid), even)
    up = np.nextafter(mid, np.inf)
    dn = np.nextafter(mid, -np.inf)
    assert np.array_equal(oracle.f64_to_bf16(up), bits[1:].astype(np.uint16))
    assert np.array_equal(oracle.f64_to_bf16(dn), bits[:-1].astype(np.uint16))
    assert oracle.f64_to_bf16(np.array([2.0 ** 128]))[0] == 0x7f80
    assert oracle.f64_to_bf16(np.array([-0.0]))[0] == 0x8000


def test_epilogue_on_zero_activations_is_act_of_bias():
    # x = 0 makes every code and the exact sum zero, so y = RNE_bf16(act(bias)):
    # the bias is added in output units (after the 2^-5), then the activation
    rng = np.random.default_rng(11)
    K, N = 256, 64
    x = np.zeros((4, K), np.uint16)
    D = np.ones(K, np.float32)
    W = rng.standard_normal((N, K)).astype(np.float32)
    bias = (rng.standard_normal(N) * 3).astype(np.float32)
    for a in [oracle.ACT_NONE] + ACTS:
        y = oracle.dense_mm_ex(x, D, W, bias, a)
        ref = np.array([oracle.act(np.array([float(b)]), a)[0] for b in bias])
        assert np.array_equal(y, np.broadcast_to(oracle.f64_to_bf16(ref), y.shape)), a


def test_epilogue_without_bias_agrees_with_the_plain_product():
    # relu commutes with rounding to bf16, and a zero bias changes nothing
    p = synth.dense(24, 512, 48, seed=3)
    qa, sa = oracle.quantize_act(p.x, p.D[0])
    qw, sw = oracle.quantize_weights(p.W[0], p.D[0])
    y = oracle.gemm(qa, sa, qw, sw)
    yv = synth.bf16_bits_to_f32(y).astype(np.float64)
    assert np.array_equal(oracle.gemm_ex(qa, sa, qw, sw, np.zeros(48, np.float32), 0), y)
    relu = oracle.gemm_ex(qa, sa, qw, sw, None, oracle.ACT_RELU)
    assert np.array_equal(synth.bf16_bits_to_f32(relu).astype(np.float64), np.maximum(yv, 0.0))
    rows, cols = np.array([0, 5, 23]), np.array([47, 0, 13])
    b = np.linspace(-1, 1, 48).astype(np.float32)
    full = oracle.gemm_ex(qa, sa, qw, sw, b, oracle.ACT_SILU)
    assert np.array_equal(oracle.gemm_at_ex(qa, sa, qw, sw, rows, cols, b, oracle.ACT_SILU), full[rows, cols])


def test_epilogue_refuses_act_type_3_and_unknown_values():
    qa = np.zeros((1, 16), np.uint8)
    sa = np.zeros((1, 1), np.uint8)
    for a in (3, 6, -1):
        with pytest.raises(AssertionError):
            oracle.gemm_ex(qa, sa, qa, sa, None, a)


def test_grouped_epilogue_uses_each_experts_bias():
    # replicated weight banks with per-expert biases: entry g's rows equal the
    # dense product with bias g
    rng = np.random.default_rng(5)
    M, K, N, E = 40, 256, 32, 3
    p = synth.dense(M, K, N, seed=9)
    W = np.repeat(p.W, E, axis=0)
    D = np.repeat(p.D, E, axis=0)
    bias = rng.standard_normal((E, N)).astype(np.float32)
    counts = np.array([10, 0, 30], np.int64)
    st, y = oracle.grouped_mm_ex(p.x, D, W, counts, 1, bias, oracle.ACT_GELU_TANH)
    assert st == oracle.OK
    off = np.concatenate([[0], np.cumsum(counts)])
    for g in range(E):
        if counts[g]:
            ref = oracle.dense_mm_ex(p.x[off[g]:off[g + 1]], p.D[0], p.W[0], bias[g], oracle.ACT_GELU_TANH)
            assert np.array_equal(y[off[g]:off[g + 1]], ref)


def test_grouped_type2_bias_follows_the_named_expert():
    # type-2 rows name their expert; with replicated banks the bias is the only
    # thing that differs between experts, so each range must carry the bias of
    # the expert it names (not of its position in the list)
    rng = np.random.default_rng(6)
    M, K, N, E = 45, 256, 32, 4
    p = synth.dense(M, K, N, seed=10)
    W = np.repeat(p.W, E, axis=0)
    D = np.repeat(p.D, E, axis=0)
    bias = rng.standard_normal((E, N)).astype(np.float32)
    gl = np.array([[3, 10], [3, 5], [0, 0], [1, 30]], np.int64)   # expert 3 twice, expert 2 never
    st, y = oracle.grouped_mm_ex(p.x, D, W, gl, 2, bias, oracle.ACT_SILU)
    assert st == oracle.OK
    r0 = 0
    for e, n in gl:
        ref = oracle.dense_mm_ex(p.x[r0:r0 + n], p.D[0], p.W[0], bias[e], oracle.ACT_SILU)
        assert np.array_equal(y[r0:r0 + n], ref)
        r0 += n


# ----------------------------------------------------------------------------
# Offline calibration of D (reading R16: D = clamp(sqrt(max|x| / max|W|), 1e-2, 1e2))
# ----------------------------------------------------------------------------

def test_calibration_equalises_the_channel_ranges():
    # the defining property of the square-root rule: after x / D and W * D both
    # sides of every channel have the same range, sqrt(max|x| max|W|)
    p = synth.dense(200, 512, 96, seed=13)
    st, D = oracle.calibrate_d(p.x, p.W)
    assert st == oracle.OK
    a = np.abs(synth.bf16_bits_to_f32(p.x).astype(np.float64)).max(axis=0)
    w = np.abs(p.W[0].astype(np.float64)).max(axis=0)
    d = D[0].astype(np.float64)
    free = (d > 1e-2) & (d < 1e2)
    assert free.mean() > 0.9
    np.testing.assert_allclose((a / d)[free], (w * d)[free], rtol=2.5e-7)
    np.testing.assert_allclose((a / d)[free], np.sqrt(a * w)[free], rtol=1.5e-7)


def test_calibration_special_cases():
    K, N, T = 256, 8, 4
    x = np.zeros((T, K), np.float32)
    W = np.zeros((N, K), np.float32)
    x[:, 1] = 1.0                  # w = 0 < a             -> 1e2
    W[:, 2] = 1.0                  # a = 0 < w             -> clamp(0) = 1e-2
    x[:, 3], W[:, 3] = 2.0 ** 20, 2.0 ** -20   # a / w = 2^40 -> clamp 1e2
    x[:, 4], W[:, 4] = 2.0 ** -20, 2.0 ** 20   # a / w = 2^-40 -> clamp 1e-2
    x[:, 5], W[:, 5] = 9.0, 1.0                # sqrt(9) = 3 exactly
    x[2, 6], W[5, 6] = -16.0, -4.0             # magnitudes: sqrt(4) = 2
    st, D = oracle.calibrate_d(synth.to_bf16_bits(x), W)
    assert st == oracle.OK
    expect = np.ones(K, np.float32)            # column 0 and the rest: a = w = 0 -> 1
    expect[[1, 2, 3, 4, 5, 6]] = [1e2, 1e-2, 1e2, 1e-2, 3.0, 2.0]
    assert np.array_equal(D[0], expect.astype(np.float32))


def test_calibration_scales_with_the_square_root_of_the_activation_range():
    p = synth.dense(64, 256, 32, seed=17)
    xf = synth.bf16_bits_to_f32(p.x)
    _, D1 = oracle.calibrate_d(p.x, p.W)
    _, D4 = oracle.calibrate_d(synth.to_bf16_bits(xf * 4.0), p.W)   # exact in bf16
    free = (D1 > 2e-2) & (D1 < 50)
    assert np.array_equal(D4[free], (D1 * 2)[free])


def test_calibration_takes_each_experts_rows():
    # type 2 names the expert of each row range; an expert named twice is
    # calibrated on both of its ranges, an expert never named gets D = 1
    rng = np.random.default_rng(19)
    E, K, N = 4, 256, 16
    xf = rng.standard_normal((60, K)).astype(np.float32)
    xf[:, 7] *= 50
    xb = synth.to_bf16_bits(xf)
    W = rng.standard_normal((E, N, K)).astype(np.float32)
    gl = np.array([[2, 20], [0, 15], [2, 25], [3, 0]], np.int64)
    st, D = oracle.calibrate_d(xb, W, gl, 2)
    assert st == oracle.OK
    _, D2 = oracle.calibrate_d(np.concatenate([xb[:20], xb[35:60]]), W[2])
    _, D0 = oracle.calibrate_d(xb[20:35], W[0])
    assert np.array_equal(D[2], D2[0]) and np.array_equal(D[0], D0[0])
    assert np.array_equal(D[1], np.ones(K, np.float32)) and np.array_equal(D[3], np.ones(K, np.float32))
    # counts and cumulative sums give the same factors
    counts = np.array([10, 0, 30, 20], np.int64)
    _, Dc = oracle.calibrate_d(xb, W, counts, 1)
    _, Ds = oracle.calibrate_d(xb, W, np.cumsum(counts), 0)
    assert np.array_equal(Dc, Ds)
    assert oracle.calibrate_d(xb, W, np.array([10, 0, 30, 19], np.int64), 1)[0] == oracle.ERR_GROUP_LIST_INVALID


def test_calibration_reproduces_the_generator_factors():
    # the workload generator states the same rule independently (dense, and
    # grouped with Zipf-skewed counts including empty experts)
    p = synth.dense(128, 1024, 256, seed=0)
    st, D = oracle.calibrate_d(p.x, p.W)
    assert st == oracle.OK and np.array_equal(D, p.D)
    g = synth.grouped(2048, 32, 512, 64, seed=1, dist="zipf", group_list_type=0)
    st, D = oracle.calibrate_d(g.x, g.W, g.group_list, g.group_list_type)
    assert st == oracle.OK and np.array_equal(D, g.D)


# ----------------------------------------------------------------------------
# FP8 (E4M3) output: OCP FP8 E4M3, round to nearest even, saturating at 448
# ----------------------------------------------------------------------------

def _e4m3_library_values():
    import torch
    return torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()


def test_e4m3_decode_matches_the_library_format_for_every_code():
    ours = oracle.e4m3_decode(np.arange(256))
    lib = _e4m3_library_values()
    nan = np.isnan(lib)
    assert np.array_equal(nan, np.isnan(ours)) and nan.sum() == 2          # 0x7f and 0xff
    assert np.array_equal(ours[~nan], lib[~nan])
    assert ours[0x7e] == 448.0 and ours[1] == 2.0 ** -9 and ours[0x08] == 2.0 ** -6


def test_e4m3_encode_round_trips_every_code():
    vals = oracle.e4m3_decode(np.arange(256))
    codes = np.arange(256)
    keep = ~np.isnan(vals)
    assert np.array_equal(oracle.f64_to_e4m3(vals[keep]), codes[keep])


def test_e4m3_encode_is_the_nearest_code_ties_to_even_brute_force():
    lib = _e4m3_library_values()
    finite = np.flatnonzero(~np.isnan(lib))
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.uniform(-460, 460, 20000), rng.standard_normal(20000) * np.exp2(rng.integers(-12, 6, 20000)),
                        (lib[finite][:-1] + np.diff(lib[finite])) / 2])   # include midpoints (ties)
    v = v[np.isfinite(v)]
    got = oracle.f64_to_e4m3(v)
    for x, c in zip(v[:6000], got[:6000]):
        if abs(x) >= 448:
            assert c & 0x7f == 0x7e and (c >> 7) == int(np.signbit(x)), (x, c)
            continue
        d = np.abs(lib[finite] - x)
        best = finite[d == d.min()]
        if best.size > 1:                       # a tie: the even mantissa; the sign of zero follows x
            best = best[(best & 1) == 0]
            best = best[((best >> 7) == int(np.signbit(x))) | (lib[best] != 0)]
        assert c in set(best.tolist()) or (lib[c] == 0 and lib[best[0]] == 0), (x, c, best)


def test_e4m3_encode_matches_the_library_conversion_in_range():
    import torch
    rng = np.random.default_rng(1)
    v = (rng.standard_normal(50000) * np.exp2(rng.integers(-10, 8, 50000))).astype(np.float32)
    v = v[np.abs(v) < 440]
    lib = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.f64_to_e4m3(v.astype(np.float64)), lib)


def test_fp8_gemm_exact_where_the_product_is_representable():
    # one nonzero element per row of K = 32: activation code 2 (1.0) at scale 127,
    # weight codes 1..7 and 9..15 at scale 127 + k: y = w * 2^k / 32 * y_scale
    K, N = 32, 14
    qa = np.zeros((1, K // 2), np.uint8); qa[0, 0] = 2
    sa = np.full((1, 1), 127, np.uint8)
    w = [c for c in range(1, 16) if c != 8]
    qw = np.zeros((N, K // 2), np.uint8); qw[:, 0] = w
    sw = np.full((N, 1), 130, np.uint8)                  # 2^3
    y = oracle.gemm_fp8(qa, sa, qw, sw, y_scale=4.0)     # w * 8 / 32 * 4 = w
    want = oracle.f64_to_e4m3(np.array([oracle.e2m1_decode(c) for c in w]))
    assert np.array_equal(y[0], want)
    assert np.array_equal(oracle.e4m3_decode(y[0]), [oracle.e2m1_decode(c) for c in w])
    # saturation and RELU on the same values
    assert np.all(oracle.gemm_fp8(qa, sa, qw, sw, y_scale=1e4)[0] & 0x7f == 0x7e)
    yr = oracle.gemm_fp8(qa, sa, qw, sw, act_type=1, y_scale=4.0)[0]
    assert np.all(oracle.e4m3_decode(yr) == np.maximum([oracle.e2m1_decode(c) for c in w], 0.0))


def test_fp8_gemm_agrees_with_the_bf16_path_within_one_step():
    p = synth.dense(24, 256, 64, seed=5)
    qa, sa = oracle.quantize_act(p.x, p.D[0])
    qw, sw = oracle.quantize_weights(p.W[0], p.D[0])
    y16 = synth.bf16_bits_to_f32(oracle.gemm(qa, sa, qw, sw)).astype(np.float64)
    s = 100.0 / np.abs(y16).max()
    y8 = oracle.e4m3_decode(oracle.gemm_fp8(qa, sa, qw, sw, y_scale=s))
    step = np.exp2(np.floor(np.log2(np.maximum(np.abs(y16 * s), 2.0 ** -6))) - 3)
    assert np.all(np.abs(y8 - y16 * s) <= step)

