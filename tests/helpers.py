"""Shared test helpers: moving seeded inputs to the GPU and comparing outputs.

Tolerance on BF16 outputs (compared with the oracle's correctly rounded y):
  * cosine similarity >= 0.99999;
  * every |y - y_ref| <= 1e-2 * rms(y_ref) + ulp_bf16(y_ref).
The stated bar is max-abs <= 1e-2 * rms(y).  The one-ulp term admits the one
rounding-boundary flip that FP32 accumulation in hardware order can cause
against an exactly rounded reference: at |y| ~ 4 rms a single BF16 ulp is
already 0.03 rms, so no non-exact FP32 accumulator can meet the bare bar on
large outputs.  The bare figure and the share within rtol = atol = 1/128 (the
MACAQ page's output check) are reported alongside.
"""
from __future__ import annotations

import numpy as np
import torch

import synth


def x_to_dev(xbits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(xbits).view(np.int16)).view(torch.bfloat16).cuda()


def y_to_bits(y: torch.Tensor) -> np.ndarray:
    return y.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f32_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126)
    return np.exp2(e - 7)


def compare(y_bits: np.ndarray, ref_bits: np.ndarray, label: str = "") -> dict:
    a = synth.bf16_bits_to_f32(y_bits).astype(np.float64).ravel()
    b = synth.bf16_bits_to_f32(ref_bits).astype(np.float64).ravel()
    assert np.all(np.isfinite(a)), f"{label}: non-finite output"
    rms = float(np.sqrt(np.mean(b * b))) if b.size else 0.0
    err = np.abs(a - b)
    denom = float(np.linalg.norm(a) * np.linalg.norm(b))
    cos = float(a @ b / denom) if denom > 0 else 1.0
    within = err <= (1 / 128) + (1 / 128) * np.abs(b)
    stats = {
        "cos": cos,
        "maxabs_over_rms": float(err.max() / rms) if rms > 0 else float(err.max()),
        "share_rtol_atol_1_128": float(within.mean()) if b.size else 1.0,
        "bit_exact_share": float(np.mean(y_bits.ravel() == ref_bits.ravel())) if b.size else 1.0,
        "n": int(b.size),
    }
    if b.size:
        assert cos >= 0.99999, (label, stats)
        bound = 1e-2 * rms + bf16_ulp(b)
        bad = np.flatnonzero(err > bound)
        assert bad.size == 0, (label, stats, bad[:5], a[bad[:5]], b[bad[:5]])
    return stats


def dequant_matmul_bf16(qa, sa, qw, sw) -> np.ndarray:
    """Oracle dequantisation + binary64 matmul (library primitive), then x 2^-5
    and BF16 rounding: the exact result up to binary64 rounding, for outputs
    too many for the exact integer oracle."""
    import oracle
    A = oracle.dequantize(qa, sa)
    B = oracle.dequantize(qw, sw)
    y = (A @ B.T) / 32.0
    return synth.to_bf16_bits(y.astype(np.float32))


def assert_mx_equal(codes, scales, ref_codes, ref_scales, label: str = ""):
    """Activation MX encodings compared bit-exactly: the E8M0 scales everywhere,
    the E2M1 codes of every block whose scale is finite.  A block whose scale is
    255 is NaN as a whole (OCP MX: a NaN scale makes every element of its block
    NaN), so its element codes carry no value.  Such blocks arise only where x/D
    leaves the binary32 range (inf - inf in the butterfly), and the signs of the
    NaN elements then follow each machine's NaN propagation (IEEE 754 leaves the
    sign of a NaN result unspecified): the GPU and the host differ there."""
    scales, ref_scales = np.asarray(scales), np.asarray(ref_scales)
    assert np.array_equal(scales, ref_scales), f"{label}: scales differ from the oracle"
    finite = ref_scales != 255
    c = np.asarray(codes).reshape(*finite.shape, 16)
    r = np.asarray(ref_codes).reshape(*finite.shape, 16)
    bad = np.argwhere((c != r).any(axis=-1) & finite)
    assert bad.size == 0, f"{label}: codes differ from the oracle in {len(bad)} blocks, first {bad[:3].tolist()}"



def compare_fp8(y8: np.ndarray, ref8: np.ndarray, label: str = "") -> dict:
    """FP8 (E4M3) outputs against the oracle's correctly rounded codes, with the
    bound of compare() carried over to the FP8 grid: each decoded value within
    1e-2 x rms of the oracle's decoded outputs (the kernels' FP32 accumulation
    order and their half-precision tanh in the gated activations) plus one E4M3
    step at the oracle's value (the GPU's FP32 result may land on the other side
    of a rounding boundary; the step is 2^-9 below the normal range), and the
    decoded outputs keep cosine >= 0.9999."""
    import oracle
    a = oracle.e4m3_decode(np.asarray(y8).ravel())
    b = oracle.e4m3_decode(np.asarray(ref8).ravel())
    assert not np.isnan(a).any(), f"{label}: NaN output"
    rms = float(np.sqrt(np.mean(b * b))) if b.size else 0.0
    step = np.exp2(np.floor(np.log2(np.maximum(np.abs(b), 2.0 ** -6))) - 3)
    bad = np.flatnonzero(np.abs(a - b) > 1e-2 * rms + step)
    denom = float(np.linalg.norm(a) * np.linalg.norm(b))
    cos = float(a @ b / denom) if denom > 0 else 1.0
    stats = {"cos": cos, "exact_share": float(np.mean(np.asarray(y8).ravel() == np.asarray(ref8).ravel())),
             "within_one_step_share": float(np.mean(np.abs(a - b) <= step)) if b.size else 1.0,
             "n": int(a.size)}
    assert bad.size == 0, (label, stats, bad[:5], a[bad[:5]], b[bad[:5]])
    assert cos >= 0.9999, (label, stats)
    return stats
