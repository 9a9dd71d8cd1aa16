"""The form in which the kernels evaluate the gated activations, checked on the
host against the oracle's binary64 definitions.

The kernels compute v * sigmoid(a) as h + h * tanh(a / 2), h = v / 2, with the
FP32 argument rounded to FP16, a hardware tanh and the FP16 result widened to
FP32.  Here those steps are emulated with numpy: FP32 products and fused
multiply-adds (rounded once from binary64), RN to FP16, tanh in binary64
perturbed by a relative error of up to 2^-11 in the worst direction (the
approximation's own error), RN to FP16.  The emulation must stay within the
bound the library states (5e-4 |v| before the final BF16 rounding) for every
act_type, and with an exact tanh and no FP16 steps it must agree with the
oracle to FP32 rounding (the identity itself: a wrong constant, a missing
halving of a or a dropped h fails it).
"""
import math

import numpy as np
import pytest

import oracle

F32 = np.float32


def f32(x):
    return np.asarray(x, np.float64).astype(F32)


def fma32(a, b, c):
    # a*b is exact in binary64 for FP32 a, b (48 significant bits); one rounding to FP32
    return f32(a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64))


def half_angle(v, act):
    """a / 2 in FP32, as the kernels form it (v already FP32)."""
    c0 = F32(math.sqrt(2.0 / math.pi))
    c1 = F32(math.sqrt(2.0 / math.pi) * 0.044715)
    if act == oracle.ACT_GELU_TANH:   # a = 2u: a / 2 = u = v (c0 + c1 v^2)
        return f32(v * fma32(f32(v * v), np.full_like(v, c1), np.full_like(v, c0)))
    if act == oracle.ACT_FAST_GELU:   # a = 1.702 v
        return f32(F32(1.702 / 2) * v)
    if act == oracle.ACT_SILU:        # a = v
        return f32(F32(0.5) * v)
    raise ValueError(act)


def gated(v, act, rel_err=0.0, fp16=True):
    v = f32(v)
    u = half_angle(v, act)
    if fp16:
        with np.errstate(over="ignore"):  # RN to FP16 overflows to +-inf: tanh = +-1
            u = u.astype(np.float16).astype(np.float64)
    t = np.tanh(u.astype(np.float64)) * (1.0 + rel_err)
    t = np.clip(t, -1.0, 1.0)
    t = t.astype(np.float16).astype(F32) if fp16 else f32(t)
    h = f32(F32(0.5) * v)
    return fma32(h, t, h).astype(np.float64)


GRID = np.concatenate([np.linspace(-60.0, 60.0, 240001),
                       np.geomspace(1e-6, 1e4, 20001), -np.geomspace(1e-6, 1e4, 20001)])
GATED = [oracle.ACT_GELU_TANH, oracle.ACT_FAST_GELU, oracle.ACT_SILU]


@pytest.mark.parametrize("act", GATED)
def test_half_angle_form_is_the_activation(act):
    v = f32(GRID).astype(np.float64)
    ref = oracle.act(v, act)
    got = gated(GRID, act, fp16=False)
    # FP32 steps only: a few FP32 roundings of |v|-sized quantities
    assert np.all(np.abs(got - ref) <= 4e-7 * np.abs(v) + 1e-37)


@pytest.mark.parametrize("act", GATED)
@pytest.mark.parametrize("rel_err", [0.0, 2.0 ** -11, -(2.0 ** -11)])
def test_half_precision_tanh_stays_within_the_stated_bound(act, rel_err):
    v = f32(GRID).astype(np.float64)
    ref = oracle.act(v, act)
    got = gated(GRID, act, rel_err=rel_err)
    err = np.abs(got - ref)
    assert np.all(err <= 5e-4 * np.abs(v) + 1e-37), float(np.max(err / np.maximum(np.abs(v), 1e-300)))


def test_large_arguments_saturate_to_the_limits():
    # FP16 overflow of u (|v| > ~122 for GELU_TANH) gives tanh = +-1: y = v or 0
    v = np.array([200.0, -200.0, 1e4, -1e4])
    for act in GATED:
        got = gated(v, act)
        assert np.array_equal(got, np.where(v > 0, f32(v), 0.0)), act
