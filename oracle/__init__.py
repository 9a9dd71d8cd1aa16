"""Plain CPU oracle for the MACAQ W4A4 MXFP4 linear (dense and grouped).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this package.  It
shares no code with the CUDA library and never imports it.

The arithmetic lives in ``macaq_oracle.c`` (plain C, built with
``-ffp-contract=off`` so every float operation is one IEEE rounding); this
module only loads it with ctypes and marshals numpy arrays.  Every function
cites what it follows on the pages:

* "MACAQ W4A4 fused dense and grouped matmul for Ascend 950", summary: channel
  scaling, block-32 BF16 Hadamard rotation, MXFP4 activation quantisation,
  matmul with BF16 output; weight transform offline.
* same page, "Latency against existing native CANN operators": the MX
  quantisation is block32 E2M1, round-to-even, scale_alg=0.
* "torch_npu.npu_grouped_matmul", function description and the group_list /
  group_list_type parameters: grouped y_i = x_i @ weight_i.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "macaq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

OK = 0
ERR_SHAPE = -3
ERR_TOO_MANY_GROUPS = -6
ERR_GROUP_LIST_TYPE = -7
ERR_GROUP_LIST_INVALID = -10
ERR_ACT_TYPE = -13
# npu_grouped_matmul act_type values (3 is not supported on that page)
ACT_NONE, ACT_RELU, ACT_GELU_TANH, ACT_FAST_GELU, ACT_SILU = 0, 1, 2, 4, 5


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no FMA contraction, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math",
            "-fopenmp", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        # MACAQ_ORACLE_LIB: a test may load a deliberately mutated build instead,
        # to check that the pins catch each planted mistake
        lib = ctypes.CDLL(os.environ.get("MACAQ_ORACLE_LIB") or build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        sig = {
            "oracle_f32_to_bf16": (ctypes.c_uint16, [ctypes.c_float]),
            "oracle_bf16_to_f64": (ctypes.c_double, [ctypes.c_uint16]),
            "oracle_fwht32": (None, [P, P, I64]),
            "oracle_e8m0_from_amax": (I, [ctypes.c_float]),
            "oracle_e2m1_decode": (ctypes.c_double, [I]),
            "oracle_e2m1_encode": (I, [ctypes.c_double]),
            "oracle_mx_quantize_blocks": (None, [P, I64, P, P]),
            "oracle_act_rotate": (None, [P, P, I64, I64, P]),
            "oracle_quantize_act": (I, [P, P, I64, I64, P, P, I]),
            "oracle_quantize_weights": (I, [P, P, I64, I64, P, P, I]),
            "oracle_gemm": (I, [P, P, P, P, I64, I64, I64, P, I]),
            "oracle_gemm_at": (I, [P, P, P, P, I64, P, P, I64, P]),
            "oracle_gemm_plain": (I, [P, P, P, P, I64, I64, I64, P, I]),
            "oracle_gemm_at_plain": (I, [P, P, P, P, I64, P, P, I64, P]),
            "oracle_group_offsets": (I, [P, I, I64, I64, P]),
            "oracle_grouped_mm": (I, [P, P, P, P, I, I64, I64, I64, I64, P, I]),
            "oracle_grouped_mm_ex": (I, [P, P, P, P, I, I64, I64, I64, I64, P, I, P, I]),
            "oracle_gemm_ex": (I, [P, P, P, P, I64, I64, I64, P, I, P, I]),
            "oracle_gemm_at_ex": (I, [P, P, P, P, I64, P, P, I64, P, I, P]),
            "oracle_act_array": (None, [P, I64, I, P]),
            "oracle_calibrate_d": (I, [P, I64, P, I64, I64, I64, P, I, P]),
            "oracle_f64_to_bf16_array": (None, [P, I64, P]),
            "oracle_linear_f64": (None, [P, P, I64, I64, I64, P]),
            "oracle_transform_f64": (None, [P, P, P, I64, I64, I64, P]),
            "oracle_dequantize": (None, [P, P, I64, I64, P]),
            "oracle_quantize_plain": (I, [P, I64, I64, P, P]),
            "oracle_act_rotate_reading": (I, [P, P, I64, I64, I, P]),
            "oracle_num_threads": (I, []),
            "oracle_e4m3_decode": (ctypes.c_double, [I]),
            "oracle_f64_to_e4m3": (I, [ctypes.c_double]),
            "oracle_f64_to_e4m3_array": (None, [P, I64, P]),
            "oracle_gemm_fp8": (I, [P, P, P, P, I64, I64, I64, P, I, ctypes.c_double, P, I]),
        }
        for name, (res, args) in sig.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------
# element-level pieces
# --------------------------------------------------------------------------

def f32_to_bf16(v) -> np.ndarray:
    """binary32 -> bf16 bit pattern, round-to-nearest-even (the BF16 rounding
    the summary's "BF16 Hadamard rotation" implies)."""
    v = _c(v, np.float32).ravel()
    f = _L().oracle_f32_to_bf16
    return np.array([f(float(x)) for x in v], dtype=np.uint16)


def bf16_to_f64(h) -> np.ndarray:
    h = _c(h, np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def fwht32(v) -> np.ndarray:
    """Unnormalised block-32 Sylvester Hadamard transform in FP32 (summary:
    "block-32 BF16 Hadamard rotation"; butterfly order h = 1..16)."""
    v = _c(v, np.float32)
    assert v.size % 32 == 0
    out = np.empty_like(v)
    _L().oracle_fwht32(_p(v), _p(out), v.size // 32)
    return out


def e8m0_from_amax(amax: float) -> int:
    """Shared scale code, OCP MX scale_alg=0 (latency section: scale_alg=0)."""
    return int(_L().oracle_e8m0_from_amax(float(amax)))


def e2m1_encode(v: float) -> int:
    """E2M1 round-to-nearest-even with saturation (latency section: E2M1,
    round-to-even)."""
    return int(_L().oracle_e2m1_encode(float(v)))


def e2m1_decode(code: int) -> float:
    return float(_L().oracle_e2m1_decode(int(code)))


def mx_quantize_blocks(v) -> tuple[np.ndarray, np.ndarray]:
    """MX quantisation of consecutive 32-element blocks of fp32 values."""
    v = _c(v, np.float32).ravel()
    assert v.size % 32 == 0
    nb = v.size // 32
    codes = np.empty(nb * 16, np.uint8)
    scales = np.empty(nb, np.uint8)
    _L().oracle_mx_quantize_blocks(_p(v), nb, _p(codes), _p(scales))
    return codes, scales


def unpack_codes(codes: np.ndarray) -> np.ndarray:
    """[..., K/2] packed bytes -> [..., K] 4-bit codes (element 2j = low nibble)."""
    lo = codes & 0xF
    hi = codes >> 4
    return np.stack([lo, hi], axis=-1).reshape(*codes.shape[:-1], codes.shape[-1] * 2)


# --------------------------------------------------------------------------
# activation and weight paths
# --------------------------------------------------------------------------

def act_rotate(x_bf16: np.ndarray, D: np.ndarray) -> np.ndarray:
    """u = RNE_bf16(FWHT32(RNE_bf16(x * RN32(1/D)))) as bf16 bits [M, K]
    (summary: channel scaling, then block-32 BF16 Hadamard rotation)."""
    x = _c(x_bf16, np.uint16)
    D = _c(D, np.float32)
    M, K = x.shape
    u = np.empty_like(x)
    _L().oracle_act_rotate(_p(x), _p(D), M, K, _p(u))
    return u


READING_R3, READING_TRUE_DIVISION, READING_BF16_STAGES, READING_EXACT_ROTATION = 0, 1, 2, 3


def act_rotate_reading(x_bf16: np.ndarray, D: np.ndarray, reading: int) -> np.ndarray:
    """Rotated BF16 activations under reading 0 (R3, the parity reference) or
    one of the other plain readings of the summary's scaling and BF16 rotation:
    1 true division by D, 2 BF16 rounding at every butterfly stage, 3 exact
    rotation rounded once.  Used only to measure how often the reading matters."""
    x = _c(x_bf16, np.uint16)
    D = _c(D, np.float32)
    M, K = x.shape
    u = np.empty_like(x)
    st = _L().oracle_act_rotate_reading(_p(x), _p(D), M, K, int(reading), _p(u))
    assert st == OK, st
    return u


def quantize_act_reading(x_bf16: np.ndarray, D: np.ndarray, reading: int):
    """Activation codes [M, K/2] and scales [M, K/32] under `reading`: the
    rotation of act_rotate_reading, then the same E8M0 / E2M1 steps (R4, R5)."""
    u = act_rotate_reading(x_bf16, D, reading)
    M, K = u.shape
    codes, scales = mx_quantize_blocks(bf16_to_f64(u).astype(np.float32))
    return codes.reshape(M, K // 2), scales.reshape(M, K // 32)


def quantize_act(x_bf16: np.ndarray, D: np.ndarray, nthreads: int = 0):
    """Activation codes [M, K/2] and E8M0 scales [M, K/32] (summary: scaling,
    rotation, MXFP4 activation quantisation)."""
    x = _c(x_bf16, np.uint16)
    D = _c(D, np.float32)
    M, K = x.shape
    codes = np.empty((M, K // 2), np.uint8)
    scales = np.empty((M, K // 32), np.uint8)
    st = _L().oracle_quantize_act(_p(x), _p(D), M, K, _p(codes), _p(scales), nthreads)
    assert st == OK, st
    return codes, scales


def quantize_weights(W: np.ndarray, D: np.ndarray, nthreads: int = 0):
    """Offline weight codes/scales from FWHT32(RN32(W*D)) in FP32 (summary:
    weight transformation is offline).  W [N, K] or [E, N, K]; D [K] or [E, K]."""
    W = _c(W, np.float32)
    D = _c(D, np.float32)
    if W.ndim == 3:
        outs = [quantize_weights(W[e], D[e], nthreads) for e in range(W.shape[0])]
        return np.stack([o[0] for o in outs]), np.stack([o[1] for o in outs])
    N, K = W.shape
    codes = np.empty((N, K // 2), np.uint8)
    scales = np.empty((N, K // 32), np.uint8)
    st = _L().oracle_quantize_weights(_p(W), _p(D), N, K, _p(codes), _p(scales), nthreads)
    assert st == OK, st
    return codes, scales


def gemm(qa, sa, qw, sw, nthreads: int = 0) -> np.ndarray:
    """Exact block-scaled product, y = RNE_bf16(2^-5 * sum) as bf16 bits [M, N]
    (summary: matrix multiplication producing BF16 output)."""
    qa, sa, qw, sw = (_c(a, np.uint8) for a in (qa, sa, qw, sw))
    M, K = qa.shape[0], qa.shape[1] * 2
    N = qw.shape[0]
    y = np.empty((M, N), np.uint16)
    st = _L().oracle_gemm(_p(qa), _p(sa), _p(qw), _p(sw), M, N, K, _p(y), nthreads)
    assert st == OK, st
    return y


def gemm_at(qa, sa, qw, sw, rows, cols) -> np.ndarray:
    """Exact outputs at the given (row, col) pairs only."""
    qa, sa, qw, sw = (_c(a, np.uint8) for a in (qa, sa, qw, sw))
    K = qa.shape[1] * 2
    rows = _c(rows, np.int64)
    cols = _c(cols, np.int64)
    out = np.empty(rows.size, np.uint16)
    st = _L().oracle_gemm_at(_p(qa), _p(sa), _p(qw), _p(sw), K, _p(rows), _p(cols), rows.size,
                             _p(out))
    assert st == OK, st
    return out


def dense_mm(x_bf16, D, W, nthreads: int = 0) -> np.ndarray:
    """Whole dense MACAQ linear: bf16 bits [M, N]."""
    qa, sa = quantize_act(x_bf16, D, nthreads)
    qw, sw = quantize_weights(W, D, nthreads)
    return gemm(qa, sa, qw, sw, nthreads)


def _bias_ptr(bias):
    if bias is None:
        return None, None
    b = _c(bias, np.float32)
    return b, _p(b)


def act(v, act_type: int) -> np.ndarray:
    """npu_grouped_matmul's activation act_type (1 RELU, 2 GELU_TANH, 4 FAST_GELU,
    5 SILU, 0 none) applied in binary64."""
    v = _c(v, np.float64)
    out = np.empty_like(v)
    _L().oracle_act_array(_p(v), v.size, int(act_type), _p(out))
    return out


def f64_to_bf16(v) -> np.ndarray:
    """binary64 -> bf16 bits, round to nearest even (one rounding)."""
    v = _c(v, np.float64)
    out = np.empty(v.shape, np.uint16)
    _L().oracle_f64_to_bf16_array(_p(v), v.size, _p(out))
    return out


def gemm_ex(qa, sa, qw, sw, bias=None, act_type: int = 0, nthreads: int = 0) -> np.ndarray:
    """y = RNE_bf16(act(2^-5 * exact sum + bias[n])) as bf16 bits [M, N]
    (npu_grouped_matmul: y_i = x_i @ weight_i + bias_i, then act_type)."""
    qa, sa, qw, sw = (_c(a, np.uint8) for a in (qa, sa, qw, sw))
    M, K = qa.shape[0], qa.shape[1] * 2
    N = qw.shape[0]
    b, bp = _bias_ptr(bias)
    y = np.empty((M, N), np.uint16)
    st = _L().oracle_gemm_ex(_p(qa), _p(sa), _p(qw), _p(sw), M, N, K, bp, int(act_type), _p(y), nthreads)
    assert st == OK, st
    return y


def gemm_at_ex(qa, sa, qw, sw, rows, cols, bias=None, act_type: int = 0) -> np.ndarray:
    """gemm_ex at the given (row, col) pairs only."""
    qa, sa, qw, sw = (_c(a, np.uint8) for a in (qa, sa, qw, sw))
    K = qa.shape[1] * 2
    rows = _c(rows, np.int64)
    cols = _c(cols, np.int64)
    b, bp = _bias_ptr(bias)
    out = np.empty(rows.size, np.uint16)
    st = _L().oracle_gemm_at_ex(_p(qa), _p(sa), _p(qw), _p(sw), K, _p(rows), _p(cols), rows.size, bp,
                                int(act_type), _p(out))
    assert st == OK, st
    return out


def dense_mm_ex(x_bf16, D, W, bias=None, act_type: int = 0, nthreads: int = 0) -> np.ndarray:
    """Dense MACAQ linear with bias and activation: bf16 bits [M, N]."""
    qa, sa = quantize_act(x_bf16, D, nthreads)
    qw, sw = quantize_weights(W, D, nthreads)
    return gemm_ex(qa, sa, qw, sw, bias, act_type, nthreads)


def e4m3_decode(codes) -> np.ndarray:
    """Values of OCP FP8 E4M3 codes (binary64; NaN for S.1111.111)."""
    c = np.asarray(codes, dtype=np.int64)
    f = _L().oracle_e4m3_decode
    return np.array([f(int(v)) for v in c.ravel()], np.float64).reshape(c.shape)


def f64_to_e4m3(v) -> np.ndarray:
    """binary64 -> E4M3 codes: round to nearest even, saturating at +-448 (the FP8
    output format; OCP FP8 E4M3)."""
    v = _c(v, np.float64)
    out = np.empty(v.shape, np.uint8)
    _L().oracle_f64_to_e4m3_array(_p(v.ravel()), v.size, _p(out.reshape(-1)))
    return out


def gemm_fp8(qa, sa, qw, sw, bias=None, act_type: int = 0, y_scale: float = 1.0, nthreads: int = 0) -> np.ndarray:
    """FP8 (E4M3) output of the layer: E4M3(act(2^-5 * exact sum + bias) * y_scale), [M, N] codes."""
    qa, sa, qw, sw = (_c(a, np.uint8) for a in (qa, sa, qw, sw))
    M, N, K = qa.shape[0], qw.shape[0], qa.shape[1] * 2
    y = np.empty((M, N), np.uint8)
    b, bp = _bias_ptr(bias)
    st = _L().oracle_gemm_fp8(_p(qa), _p(sa), _p(qw), _p(sw), M, N, K, bp, int(act_type), float(y_scale), _p(y),
                              nthreads)
    assert st == OK, st
    return y


def group_offsets(group_list, group_list_type: int, M: int):
    """Row offsets [E+1] from group_list (npu_grouped_matmul, group_list and
    group_list_type).  Returns (status, offsets)."""
    gl = _c(group_list, np.int64)
    E = gl.shape[0] if group_list_type == 2 else gl.size  # type 2: [E, 2] rows of (expert, rows)
    off = np.zeros(max(E + 1, 2), np.int64)
    st = _L().oracle_group_offsets(_p(gl), int(group_list_type), E, M, _p(off))
    return int(st), off[:E + 1]


def grouped_mm(x_bf16, D, W, group_list, group_list_type: int, nthreads: int = 0):
    """Grouped MACAQ linear (npu_grouped_matmul, single x / single 3-D weight /
    single y).  Returns (status, y bf16 bits [M, N])."""
    x = _c(x_bf16, np.uint16)
    D = _c(D, np.float32)
    W = _c(W, np.float32)
    gl = _c(group_list, np.int64)
    M, K = x.shape
    E, N, _ = W.shape
    y = np.zeros((M, N), np.uint16)
    st = _L().oracle_grouped_mm(_p(x), _p(D), _p(W), _p(gl), int(group_list_type), E, M, N, K,
                                _p(y), nthreads)
    return int(st), y


def grouped_mm_list(x_bf16, D, W_list, group_list, group_list_type: int, nthreads: int = 0):
    """Grouped MACAQ linear with one weight tensor per expert (npu_grouped_matmul,
    parameter weight given as a list of tensors, the single-x / several-weight /
    single-y case of its constraints).  The rows of list entry j (group_list as in
    grouped_mm) are the dense MACAQ linear of the expert e the entry uses (e = j
    for types 0 and 1, the named index for type 2) with D[e] and W_list[e] [N, K].
    Written as that definition (one dense call per entry), independently of the
    C routine behind grouped_mm.  Returns (status, y bf16 bits [M, N])."""
    x = _c(x_bf16, np.uint16)
    D = _c(D, np.float32)
    M = x.shape[0]
    E = len(W_list)
    N = W_list[0].shape[0]
    st, off = group_offsets(group_list, group_list_type, M)
    y = np.zeros((M, N), np.uint16)
    if st != OK:
        return st, y
    gl = _c(group_list, np.int64)
    for j in range(E):
        a, b = int(off[j]), int(off[j + 1])
        e = int(gl[j, 0]) if group_list_type == 2 else j
        if b > a:
            y[a:b] = dense_mm(x[a:b], D[e], W_list[e], nthreads)
    return OK, y


def grouped_mm_ex(x_bf16, D, W, group_list, group_list_type: int, bias=None, act_type: int = 0,
                  nthreads: int = 0):
    """Grouped MACAQ linear with per-expert bias [E, N] and activation.
    Returns (status, y bf16 bits [M, N])."""
    x = _c(x_bf16, np.uint16)
    D = _c(D, np.float32)
    W = _c(W, np.float32)
    gl = _c(group_list, np.int64)
    M, K = x.shape
    E, N, _ = W.shape
    b, bp = _bias_ptr(bias)
    y = np.zeros((M, N), np.uint16)
    st = _L().oracle_grouped_mm_ex(_p(x), _p(D), _p(W), _p(gl), int(group_list_type), E, M, N, K, bp,
                                   int(act_type), _p(y), nthreads)
    return int(st), y


def calibrate_d(x_bf16, W, group_list=None, group_list_type: int = 1):
    """Offline channel factors D [E, K] from calibration activations x bf16 [T, K]
    and weights W fp32 [E, N, K] (reading R16).  Returns (status, D)."""
    x = _c(x_bf16, np.uint16)
    W = _c(W, np.float32)
    if W.ndim == 2:
        W = W[None]
    T, K = x.shape
    E, N, _ = W.shape
    gl = None if group_list is None else _c(group_list, np.int64)
    D = np.empty((E, K), np.float32)
    st = _L().oracle_calibrate_d(_p(x), T, _p(W), E, N, K, None if gl is None else _p(gl), int(group_list_type),
                                 _p(D))
    return int(st), D


def linear_f64(x_bf16, W) -> np.ndarray:
    x = _c(x_bf16, np.uint16)
    W = _c(W, np.float32)
    M, K = x.shape
    N = W.shape[0]
    out = np.empty((M, N), np.float64)
    _L().oracle_linear_f64(_p(x), _p(W), M, N, K, _p(out))
    return out


def transform_f64(x_bf16, D, W) -> np.ndarray:
    """((x/D)H).((W*D)H)^T / 32 in binary64, with no rounding to BF16 or MXFP4."""
    x = _c(x_bf16, np.uint16)
    D = _c(D, np.float32)
    W = _c(W, np.float32)
    M, K = x.shape
    N = W.shape[0]
    out = np.empty((M, N), np.float64)
    _L().oracle_transform_f64(_p(x), _p(D), _p(W), M, N, K, _p(out))
    return out


def dequantize(codes, scales) -> np.ndarray:
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    R, K = codes.shape[0], codes.shape[1] * 2
    out = np.empty((R, K), np.float64)
    _L().oracle_dequantize(_p(codes), _p(scales), R, K, _p(out))
    return out


def quantize_plain(v) -> tuple[np.ndarray, np.ndarray]:
    """Plain MXFP4 of [R, K] fp32 values, no D and no H (the pages' native
    baseline, npu_dynamic_mx_quant)."""
    v = _c(v, np.float32)
    R, K = v.shape
    codes = np.empty((R, K // 2), np.uint8)
    scales = np.empty((R, K // 32), np.uint8)
    st = _L().oracle_quantize_plain(_p(v), R, K, _p(codes), _p(scales))
    assert st == OK, st
    return codes, scales


def gemm_plain(qa, sa, qw, sw, nthreads: int = 0) -> np.ndarray:
    """Plain MXFP4 product: y = RNE_bf16(exact block-scaled sum), no 2^-5."""
    qa, sa, qw, sw = (_c(a, np.uint8) for a in (qa, sa, qw, sw))
    M, K = qa.shape[0], qa.shape[1] * 2
    N = qw.shape[0]
    y = np.empty((M, N), np.uint16)
    st = _L().oracle_gemm_plain(_p(qa), _p(sa), _p(qw), _p(sw), M, N, K, _p(y), nthreads)
    assert st == OK, st
    return y


def gemm_at_plain(qa, sa, qw, sw, rows, cols) -> np.ndarray:
    """Plain MXFP4 outputs at the given (row, col) pairs only."""
    qa, sa, qw, sw = (_c(a, np.uint8) for a in (qa, sa, qw, sw))
    K = qa.shape[1] * 2
    rows = _c(rows, np.int64)
    cols = _c(cols, np.int64)
    out = np.empty(rows.size, np.uint16)
    st = _L().oracle_gemm_at_plain(_p(qa), _p(sa), _p(qw), _p(sw), K, _p(rows), _p(cols), rows.size,
                                   _p(out))
    assert st == OK, st
    return out


def quantize_act_plain(x_bf16) -> tuple[np.ndarray, np.ndarray]:
    """Plain MXFP4 of BF16 activations (their exact FP32 values), no D and no H."""
    x = _c(x_bf16, np.uint16)
    return quantize_plain(bf16_to_f64(x).astype(np.float32))


def dense_mm_plain(x_bf16, W, nthreads: int = 0) -> np.ndarray:
    """Whole dense plain MXFP4 W4A4 linear (the native baseline): bf16 bits [M, N]."""
    qa, sa = quantize_act_plain(x_bf16)
    qw, sw = quantize_plain(W)
    return gemm_plain(qa, sa, qw, sw, nthreads)


def grouped_mm_plain(x_bf16, W, group_list, group_list_type: int, nthreads: int = 0):
    """Grouped plain MXFP4 linear: rows of group g against W[g].  Returns
    (status, y bf16 bits [M, N])."""
    x = _c(x_bf16, np.uint16)
    W = _c(W, np.float32)
    M = x.shape[0]
    E, N, _ = W.shape
    st, off = group_offsets(group_list, group_list_type, M)
    y = np.zeros((M, N), np.uint16)
    if st != OK:
        return st, y
    gl = _c(group_list, np.int64)
    for g in range(E):
        a, b = int(off[g]), int(off[g + 1])
        e = int(gl[g, 0]) if group_list_type == 2 else g
        if b > a:
            y[a:b] = dense_mm_plain(x[a:b], W[e], nthreads)
    return OK, y


def num_threads() -> int:
    return int(_L().oracle_num_threads())
