"""Pins for the oracle's other readings of the activation arithmetic.

The summary of the MACAQ page names a channel scaling by raw D and a BF16
Hadamard rotation without their working precision.  Reading 0 (R3: scale by
RN32(1/D), FP32 butterfly, one BF16 rounding) is the parity reference; the
oracle also implements 1 (true division by D), 2 (BF16 rounding at every
butterfly stage) and 3 (exact rotation, one rounding) to measure how often the
choice changes the codes.  Each reading is pinned here against arithmetic that
does not go through the oracle's own butterfly.
"""
import numpy as np
import pytest
import scipy.linalg

import oracle
import synth

R0, R1, R2, R3 = (oracle.READING_R3, oracle.READING_TRUE_DIVISION, oracle.READING_BF16_STAGES,
                  oracle.READING_EXACT_ROTATION)


def bf16(v):
    """RNE to BF16 through numpy float32 bit arithmetic (no oracle code)."""
    f = np.asarray(v, np.float32).view(np.uint32).astype(np.uint64)
    rounded = (f + 0x7FFF + ((f >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def to_f64(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32).astype(np.float64)


def test_reading_0_is_the_parity_reference():
    p = synth.dense(16, 512, 32, seed=8)
    assert np.array_equal(oracle.act_rotate_reading(p.x, p.D[0], R0), oracle.act_rotate(p.x, p.D[0]))
    c, s = oracle.quantize_act_reading(p.x, p.D[0], R0)
    c0, s0 = oracle.quantize_act(p.x, p.D[0])
    assert np.array_equal(c, c0) and np.array_equal(s, s0)


def test_scaling_steps_follow_float32_multiply_and_divide():
    # a single spike per block rotates exactly to +-xs in every position, so u[0]
    # shows the scaled value: RN32(x * RN32(1/D)) for R3, RN32(x / D) for reading 1.
    # With D = 0.3 the two land on different BF16 values for every x whose BF16
    # significand is 0x6d or 0x79 (the quotient lies next to a BF16 tie); other
    # significands agree after the rounding.
    exps = np.arange(0x70, 0x90, dtype=np.uint16)
    xb = np.concatenate([(exps << 7) | 0x6D, (exps << 7) | 0x79, (exps << 7) | 0x40,
                         0x8000 | (exps << 7) | 0x6D]).astype(np.uint16)
    n = xb.size
    K = 32 * n
    x = np.zeros((1, K), np.uint16)
    x[0, ::32] = xb
    D = np.full(K, 0.3, np.float32)
    xf = to_f64(xb).astype(np.float32)
    want0 = bf16(xf * (np.float32(1) / np.float32(0.3)))
    want1 = bf16(xf / np.float32(0.3))
    u0 = oracle.act_rotate_reading(x, D, R0)[0, ::32]
    u1 = oracle.act_rotate_reading(x, D, R1)[0, ::32]
    assert np.array_equal(u0, want0) and np.array_equal(u1, want1)
    differs = want0 != want1
    assert differs[:64].all() and not differs[64:96].any() and differs[96:].all()
    # the two readings agree when D is a power of two (1/D exact)
    D2 = np.full(K, 0.25, np.float32)
    assert np.array_equal(oracle.act_rotate_reading(x, D2, R0), oracle.act_rotate_reading(x, D2, R1))


def test_exact_rotation_is_the_hadamard_product_rounded_once():
    # reading 3 against a library matrix product: H (scipy, +-1) times the scaled
    # BF16 block in binary64, then one RNE to BF16
    p = synth.dense(8, 256, 16, seed=10)
    u3 = oracle.act_rotate_reading(p.x, p.D[0], R3)
    H = scipy.linalg.hadamard(32).astype(np.float64)
    xf = to_f64(p.x).astype(np.float32)
    r = (np.float32(1) / p.D[0].astype(np.float32)).astype(np.float32)
    xsb = to_f64(bf16(xf * r))
    want = oracle.f64_to_bf16((xsb.reshape(8, -1, 32) @ H.T).reshape(8, 256))
    assert np.array_equal(u3, want)


def test_bf16_stages_worked_example():
    # block [1, 2^-8, 2^-8, 0, ...] with D = 1.  The exact sum of all four is
    # 1 + 2^-7 (a BF16 value), so R3 and reading 3 give u[0] = 1.0078125.  With
    # BF16 stages: h = 1 rounds 1 + 2^-8 (a tie) to 1 and leaves 2^-8 + 0; h = 2
    # rounds 1 + 2^-8 to 1 again; every later stage adds zeros: u[0] = 1.
    K = 32
    x = np.zeros((1, K), np.uint16)
    x[0, 0] = bf16(1.0)
    x[0, 1] = bf16(2.0 ** -8)
    x[0, 2] = bf16(2.0 ** -8)
    D = np.ones(K, np.float32)
    assert to_f64(oracle.act_rotate_reading(x, D, R0))[0, 0] == 1.0078125
    assert to_f64(oracle.act_rotate_reading(x, D, R3))[0, 0] == 1.0078125
    assert to_f64(oracle.act_rotate_reading(x, D, R2))[0, 0] == 1.0


def test_bf16_stages_round_the_differences_too():
    # block [1, 2^-9, 2^-10, -2^-10, 0, ...], D = 1.  Row 3 of H is (+, -, -, +, ...),
    # so the exact u[3] = 1 - 2^-9 - 2^-10 - 2^-10 = 1 - 2^-8 (a BF16 value), which
    # R3's FP32 butterfly and reading 3 reach.  With BF16 stages the difference
    # 1 - 2^-9 at h = 1 is a tie between 1 - 2^-8 and 1 and goes to the even 1; at
    # h = 2, 1 - 2^-9 is again a tie and gives 1; later stages add zeros: u[3] = 1.
    K = 32
    x = np.zeros((1, K), np.uint16)
    x[0, :4] = bf16(np.array([1.0, 2.0 ** -9, 2.0 ** -10, -(2.0 ** -10)]))
    D = np.ones(K, np.float32)
    assert to_f64(oracle.act_rotate_reading(x, D, R0))[0, 3] == 1 - 2.0 ** -8
    assert to_f64(oracle.act_rotate_reading(x, D, R3))[0, 3] == 1 - 2.0 ** -8
    assert to_f64(oracle.act_rotate_reading(x, D, R2))[0, 3] == 1.0


@pytest.mark.parametrize("reading", [R1, R2, R3])
def test_readings_agree_when_every_partial_sum_is_exact_in_bf16(reading):
    # entries in {-1, 0, 1} and D = 1: every partial sum is an integer of magnitude
    # at most 32, exact in BF16, FP32 and binary64 alike
    rng = np.random.default_rng(11)
    v = rng.integers(-1, 2, size=(4, 256)).astype(np.float32)
    x = bf16(v)
    D = np.ones(256, np.float32)
    assert np.array_equal(oracle.act_rotate_reading(x, D, reading), oracle.act_rotate_reading(x, D, R0))


def test_unknown_reading_is_refused():
    x = np.zeros((1, 32), np.uint16)
    with pytest.raises(AssertionError):
        oracle.act_rotate_reading(x, np.ones(32, np.float32), 4)


def test_report_runs_and_reading_0_matches_itself():
    from oracle import readings_report
    res = readings_report.report(rows=2)
    assert len(res) == 5 * 4
    for r in res:
        assert 0.005 < r["nmse"] < 0.02
        if r["reading"].startswith("R3"):
            assert r["codes_differ"] == r["scales_differ"] == r["outputs_differ"] == 0.0
