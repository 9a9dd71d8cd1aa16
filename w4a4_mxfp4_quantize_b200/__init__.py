"""B200-native MACAQ W4A4 MXFP4 linear (dense and grouped).

A thin Python binding over the C ABI in ``include/macaq.h`` (library
``libmacaq.so`` built in this directory).  This module only marshals
arguments: every step of the computation runs in the library's sm_100a
kernels.  PyTorch provides device memory and streams.  There is no CPU
fallback: without the built library or a B200, every call raises.

The operation (MACAQ page "MACAQ W4A4 fused dense and grouped matmul for
Ascend 950", summary): y = BF16(2^-5 * MXFP4(H(x/D)) . MXFP4(H(W*D))^T) with H
the block-32 Sylvester Hadamard rotation along K; grouped calls follow
torch_npu.npu_grouped_matmul's group_list / group_list_type.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_ROOT = os.path.dirname(_HERE)
_LIB_PATH = os.path.join(_HERE, "libmacaq.so")
_SRC = os.path.join(_HERE, "csrc", "macaq.cu")
_INCLUDE = os.path.join(_ROOT, "include")

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared"]

STATUS = {
    0: "MACAQ_OK", -1: "MACAQ_ERR_NULL", -2: "MACAQ_ERR_ALIGN", -3: "MACAQ_ERR_SHAPE",
    -4: "MACAQ_ERR_ARCH", -5: "MACAQ_ERR_ALIAS", -6: "MACAQ_ERR_TOO_MANY_GROUPS",
    -7: "MACAQ_ERR_GROUP_LIST_TYPE", -8: "MACAQ_ERR_CUDA", -9: "MACAQ_ERR_DEVICE_TIMEOUT",
    -10: "MACAQ_ERR_GROUP_LIST_INVALID", -11: "MACAQ_ERR_WORKSPACE", -12: "MACAQ_ERR_BAD_D",
    -13: "MACAQ_ERR_ACT_TYPE",
}

# npu_grouped_matmul act_type values accepted by the _ex calls (3 is not supported)
ACT_NONE, ACT_RELU, ACT_GELU_TANH, ACT_FAST_GELU, ACT_SILU = 0, 1, 2, 4, 5


class MacaqError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS.get(status, status)} ({status})")
        self.status = status


def _sources():
    d = os.path.join(_HERE, "csrc")
    return [os.path.join(d, f) for f in sorted(os.listdir(d))] + [os.path.join(_INCLUDE, "macaq.h")]


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libmacaq.so for sm_100a in-tree (nvcc cross-compiles without a GPU)."""
    newest = max(os.path.getmtime(f) for f in _sources())
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < newest:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["nvcc", *NVCC_FLAGS, "-I" + _INCLUDE, "-o", tmp, _SRC]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None
_lock = threading.Lock()

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_SIG = {
    "macaq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "macaq_abi_version": (ctypes.c_int, []),
    "macaq_weight_code_bytes": (ctypes.c_size_t, [_I64, _I64, _I64]),
    "macaq_weight_scale_bytes": (ctypes.c_size_t, [_I64, _I64, _I64]),
    "macaq_prepare_weights": (ctypes.c_int, [_P, _P, _I64, _I64, _I64, _P, _P, _P]),
    "macaq_workspace_bytes": (ctypes.c_size_t, [_I64, _I64, _I64, _I64]),
    "macaq_dense_mm": (ctypes.c_int, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P, ctypes.c_size_t, _P, _P]),
    "macaq_grouped_mm": (ctypes.c_int, [_P, _P, _P, _P, _P, ctypes.c_int, _I64, _P, _I64, _I64, _I64, _P,
                                        ctypes.c_size_t, _P, _P]),
    "macaq_dense_mm_ex": (ctypes.c_int, [_P, _P, _P, _P, _P, ctypes.c_int, _P, _I64, _I64, _I64, _P,
                                         ctypes.c_size_t, _P, _P]),
    "macaq_grouped_mm_ex": (ctypes.c_int, [_P, _P, _P, _P, _P, ctypes.c_int, _I64, _P, ctypes.c_int, _P, _I64,
                                           _I64, _I64, _P, ctypes.c_size_t, _P, _P]),
    "macaq_quantize_activations": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _P]),
    "macaq_export_weights": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, _P]),
    "macaq_mx_encode_blocks": (ctypes.c_int, [_P, _P, _P, _I64, _P]),
    "macaq_unfused_workspace_bytes": (ctypes.c_size_t, [_I64, _I64]),
    "macaq_dense_mm_noalloc": (ctypes.c_int, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _P]),
    "macaq_unfused_dense_mm": (ctypes.c_int, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P, ctypes.c_size_t,
                                              _P, _P]),
    "macaq_prepare_weights_plain": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _P]),
    "macaq_calibrate_d": (ctypes.c_int, [_P, _I64, _P, _I64, _I64, _I64, _P, ctypes.c_int, _P, _P]),
    "macaq_dense_mm_plain": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I64, _I64, _P, ctypes.c_size_t, _P, _P]),
    "macaq_grouped_mm_plain": (ctypes.c_int, [_P, _P, _P, _P, ctypes.c_int, _I64, _P, _I64, _I64, _I64, _P,
                                              ctypes.c_size_t, _P, _P]),
    "macaq_fused_plan": (ctypes.c_int, [_I64, _I64, _I64, _P, _P]),
    "macaq_fused_probe": (ctypes.c_int, [_P, _P, _P, _P, _P, _I64, _I64, _I64, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, _P, _P, _P, _P]),
    "macaq_test_wait_expiry": (ctypes.c_int, [_I64, _P, _P]),
    "macaq_prepare_weights_transposed": (ctypes.c_int, [_P, _P, _I64, _I64, _I64, _P, _P, _P]),
    "macaq_grouped_mm_list": (ctypes.c_int, [_P, _P, _P, _P, _P, ctypes.c_int, _I64, _P, ctypes.c_int, _P, _I64,
                                             _I64, _I64, _P, ctypes.c_size_t, _P, _P]),
    "macaq_dense_mm_fp8": (ctypes.c_int, [_P, _P, _P, _P, _P, ctypes.c_int, ctypes.c_float, _P, _I64, _I64, _I64,
                                          _P, ctypes.c_size_t, _P, _P]),
    "macaq_grouped_mm_fp8": (ctypes.c_int, [_P, _P, _P, _P, _P, ctypes.c_int, _I64, _P, ctypes.c_int,
                                            ctypes.c_float, _P, _I64, _I64, _I64, _P, ctypes.c_size_t, _P, _P]),
}


def lib() -> ctypes.CDLL:
    """The loaded C library; raises if it has not been built."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(_LIB_PATH):
                    raise RuntimeError(f"libmacaq.so is not built ({_LIB_PATH}); run "
                                       "w4a4_mxfp4_quantize_b200.build()")
                L = ctypes.CDLL(_LIB_PATH)
                for name, (res, args) in _SIG.items():
                    f = getattr(L, name)
                    f.restype = res
                    f.argtypes = args
                _lib = L
    return _lib


def exported_symbols() -> list[str]:
    return list(_SIG)


def _check(st: int, where: str):
    if st != 0:
        raise MacaqError(st, where)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _arg(t, name: str, dtype, ndim: int | None = None, min_numel: int = 0):
    """Element type, rank and size of an argument, checked before the call (the
    library reads min_numel elements of it; a wrong element type would make it
    read another tensor's bytes, or past the end)."""
    if t is None:
        return
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got shape {tuple(t.shape)}")
    if t.numel() < min_numel:
        raise ValueError(f"{name} holds {t.numel()} elements; the call reads {min_numel}")


def _weights_args(Wq, Ws, E: int, N: int, K: int):
    """Weight tile images: uint8, at least the bytes macaq_weight_*_bytes give
    (0 for a shape the library refuses, which it then reports itself)."""
    qb, sb = weight_bytes(E, N, K)
    _arg(Wq, "Wq", torch.uint8, min_numel=qb)
    _arg(Ws, "Ws", torch.uint8, min_numel=sb)


def _on(stream):
    """Allocations for a call (its output, workspace and result tensors) are made
    on the stream its kernels run on: the caching allocator then hands their
    memory to no other stream while those kernels may still use it, and the
    workspace's zero fill is ordered before them."""
    return torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()


def _require_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("expected contiguous CUDA tensors")


def _output(out, M: int, N: int, device):
    """The output tensor: the caller's (checked: bf16 [M, N]) or a new one."""
    if out is None:
        return torch.empty((M, N), dtype=torch.bfloat16, device=device)
    if out.dtype != torch.bfloat16 or tuple(out.shape) != (M, N):
        raise ValueError(f"out must be bfloat16 of shape {(M, N)}, got {out.dtype} {tuple(out.shape)}")
    return out


# ---------------------------------------------------------------------------
# workspace: scratch for the quantise-once and grouped paths.  Callers may pass
# their own (e.g. to capture calls in a CUDA graph); otherwise one buffer per
# (device, stream) is kept and grown on demand.
# ---------------------------------------------------------------------------
_ws: dict = {}


def workspace_bytes(M: int, N: int, K: int, E: int = 1) -> int:
    return int(lib().macaq_workspace_bytes(M, N, K, E))


def unfused_workspace_bytes(M: int, K: int) -> int:
    return int(lib().macaq_unfused_workspace_bytes(M, K))


def workspace(nbytes: int, device: torch.device, stream=None, given: torch.Tensor | None = None):
    if nbytes == 0:
        return None
    if given is not None:
        if given.numel() * given.element_size() < nbytes:
            raise MacaqError(-11, "workspace")
        return given
    s = stream if stream is not None else torch.cuda.current_stream(device)
    key = (device.index, s.cuda_stream)
    buf = _ws.get(key)
    if buf is None or buf.numel() < nbytes:
        with _on(stream):
            buf = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=device)
        _ws[key] = buf
    return buf


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


# ---------------------------------------------------------------------------
# public API
# ---------------------------------------------------------------------------

def weight_bytes(E: int, N: int, K: int) -> tuple[int, int]:
    L = lib()
    return int(L.macaq_weight_code_bytes(E, N, K)), int(L.macaq_weight_scale_bytes(E, N, K))


def prepare_weights(W: torch.Tensor, D: torch.Tensor, stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Offline: W fp32 [N, K] or [E, N, K], D fp32 [K] or [E, K] -> (Wq, Ws) tile images."""
    if W.dim() == 2:
        W = W.unsqueeze(0)
    if D.dim() == 1:
        D = D.unsqueeze(0)
    _arg(W, "W", torch.float32, ndim=3)
    E, N, K = W.shape
    _arg(D, "D", torch.float32, min_numel=E * K)
    _require_cuda(W, D)
    qb, sb = weight_bytes(E, N, K)
    if qb == 0:
        raise MacaqError(-3, "prepare_weights")
    with _on(stream):
        Wq = torch.empty(qb, dtype=torch.uint8, device=W.device)
        Ws = torch.empty(sb, dtype=torch.uint8, device=W.device)
    _check(lib().macaq_prepare_weights(_ptr(W), _ptr(D), E, N, K, _ptr(Wq), _ptr(Ws), _stream_ptr(stream)),
           "macaq_prepare_weights")
    return Wq, Ws


def prepare_weights_transposed(W_kn: torch.Tensor, D: torch.Tensor, stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Offline, from weights stored transposed: W_kn fp32 [K, N] or [E, K, N], D fp32
    [K] or [E, K] -> the same (Wq, Ws) as prepare_weights on the [E, N, K] weights."""
    if W_kn.dim() == 2:
        W_kn = W_kn.unsqueeze(0)
    if D.dim() == 1:
        D = D.unsqueeze(0)
    _arg(W_kn, "W_kn", torch.float32, ndim=3)
    E, K, N = W_kn.shape
    _arg(D, "D", torch.float32, min_numel=E * K)
    _require_cuda(W_kn, D)
    qb, sb = weight_bytes(E, N, K)
    if qb == 0:
        raise MacaqError(-3, "prepare_weights_transposed")
    with _on(stream):
        Wq = torch.empty(qb, dtype=torch.uint8, device=W_kn.device)
        Ws = torch.empty(sb, dtype=torch.uint8, device=W_kn.device)
    _check(lib().macaq_prepare_weights_transposed(_ptr(W_kn), _ptr(D), E, N, K, _ptr(Wq), _ptr(Ws),
                                                  _stream_ptr(stream)), "macaq_prepare_weights_transposed")
    return Wq, Ws


def grouped_mm_list(x: torch.Tensor, D: torch.Tensor, Wq_list, Ws_list, group_list: torch.Tensor,
                    group_list_type: int, N: int, out: torch.Tensor | None = None,
                    status: torch.Tensor | None = None, stream=None, ws: torch.Tensor | None = None,
                    bias: torch.Tensor | None = None, act_type: int = ACT_NONE) -> torch.Tensor:
    """Grouped MACAQ linear with one prepared weight pair per expert (npu_grouped_matmul's
    weight as a list): Wq_list[e], Ws_list[e] from prepare_weights on expert e's [N, K]."""
    _arg(x, "x", torch.bfloat16, ndim=2)
    _arg(group_list, "group_list", torch.int64)
    E = _groups(group_list, group_list_type)
    if len(Wq_list) != E or len(Ws_list) != E:
        raise ValueError(f"Wq_list and Ws_list need {E} entries, one per group_list entry")
    M, K = x.shape
    _arg(D, "D", torch.float32, min_numel=E * K)
    for e in range(E):
        _weights_args(Wq_list[e], Ws_list[e], 1, N, K)
    _arg(status, "status", torch.int32, min_numel=1)
    _require_cuda(x, D, group_list, out, status, *Wq_list, *Ws_list)
    _check_bias(bias, (E, N))
    with _on(stream):
        y = _output(out, M, N, x.device)
        # two separate device tables (each starts 16-byte aligned, as the C call requires)
        wq_table = torch.tensor([w.data_ptr() for w in Wq_list], dtype=torch.int64).to(x.device)
        ws_table = torch.tensor([w.data_ptr() for w in Ws_list], dtype=torch.int64).to(x.device)
    L = lib()
    ws = workspace(int(L.macaq_workspace_bytes(M, N, K, E)), x.device, stream, ws)
    _check(L.macaq_grouped_mm_list(_ptr(x), _ptr(D), _ptr(wq_table), _ptr(ws_table), _ptr(group_list),
                                   int(group_list_type), E, _ptr(bias), int(act_type), _ptr(y), M, N, K, _ptr(ws),
                                   _nbytes(ws), _ptr(status), _stream_ptr(stream)), "macaq_grouped_mm_list")
    return y


def dense_mm_fp8(x: torch.Tensor, D: torch.Tensor, Wq: torch.Tensor, Ws: torch.Tensor, N: int, y_scale: float,
                 bias: torch.Tensor | None = None, act_type: int = ACT_NONE, out: torch.Tensor | None = None,
                 status: torch.Tensor | None = None, stream=None, ws: torch.Tensor | None = None) -> torch.Tensor:
    """MACAQ linear with an FP8 output: E4M3 codes (uint8 [M, N]) of act(v + bias) * y_scale."""
    _dense_args(x, D, Wq, Ws, N, status)
    _require_cuda(x, D, Wq, Ws, out, status)
    M, K = x.shape
    _check_bias(bias, (N,))
    with _on(stream):
        y8 = torch.empty((M, N), dtype=torch.uint8, device=x.device) if out is None else out
    if y8.dtype != torch.uint8 or tuple(y8.shape) != (M, N):
        raise ValueError(f"out must be uint8 of shape {(M, N)}")
    L = lib()
    ws = workspace(int(L.macaq_unfused_workspace_bytes(M, K)), x.device, stream, ws)
    _check(L.macaq_dense_mm_fp8(_ptr(x), _ptr(D), _ptr(Wq), _ptr(Ws), _ptr(bias), int(act_type), float(y_scale),
                                _ptr(y8), M, N, K, _ptr(ws), _nbytes(ws), _ptr(status), _stream_ptr(stream)),
           "macaq_dense_mm_fp8")
    return y8


def grouped_mm_fp8(x: torch.Tensor, D: torch.Tensor, Wq: torch.Tensor, Ws: torch.Tensor, group_list: torch.Tensor,
                   group_list_type: int, N: int, y_scale: float, bias: torch.Tensor | None = None,
                   act_type: int = ACT_NONE, out: torch.Tensor | None = None, status: torch.Tensor | None = None,
                   stream=None, ws: torch.Tensor | None = None) -> torch.Tensor:
    """Grouped MACAQ linear with an FP8 output (E4M3 codes, uint8 [M, N])."""
    E = _grouped_args(x, D, Wq, Ws, group_list, group_list_type, N, status)
    _require_cuda(x, D, Wq, Ws, group_list, out, status)
    M, K = x.shape
    _check_bias(bias, (E, N))
    with _on(stream):
        y8 = torch.empty((M, N), dtype=torch.uint8, device=x.device) if out is None else out
    if y8.dtype != torch.uint8 or tuple(y8.shape) != (M, N):
        raise ValueError(f"out must be uint8 of shape {(M, N)}")
    L = lib()
    ws = workspace(int(L.macaq_workspace_bytes(M, N, K, E)), x.device, stream, ws)
    _check(L.macaq_grouped_mm_fp8(_ptr(x), _ptr(D), _ptr(Wq), _ptr(Ws), _ptr(group_list), int(group_list_type), E,
                                  _ptr(bias), int(act_type), float(y_scale), _ptr(y8), M, N, K, _ptr(ws),
                                  _nbytes(ws), _ptr(status), _stream_ptr(stream)), "macaq_grouped_mm_fp8")
    return y8


def _check_bias(bias, shape):
    if bias is None:
        return
    _require_cuda(bias)
    if bias.dtype != torch.float32 or tuple(bias.shape) != shape:
        raise ValueError(f"bias must be float32 of shape {shape}, got {bias.dtype} {tuple(bias.shape)}")


def calibrate_d(x_cal: torch.Tensor, W: torch.Tensor, group_list: torch.Tensor | None = None,
                group_list_type: int = 1, stream=None) -> torch.Tensor:
    """Offline: channel factors D fp32 [E, K] from calibration activations x_cal bf16
    [T, K] and weights W fp32 [N, K] or [E, N, K] (rows split by group_list when E > 1)."""
    if W.dim() == 2:
        W = W.unsqueeze(0)
    _arg(x_cal, "x_cal", torch.bfloat16, ndim=2)
    _arg(W, "W", torch.float32, ndim=3)
    _arg(group_list, "group_list", torch.int64)
    T, K = x_cal.shape
    E, N, KW = W.shape
    if KW != K:
        raise ValueError(f"W has {KW} input channels, x_cal {K}")
    _require_cuda(x_cal, W, group_list)
    with _on(stream):
        D = torch.empty((E, K), dtype=torch.float32, device=W.device)
    _check(lib().macaq_calibrate_d(_ptr(x_cal), T, _ptr(W), E, N, K, _ptr(group_list), int(group_list_type),
                                   _ptr(D), _stream_ptr(stream)), "macaq_calibrate_d")
    return D


def dense_mm(x: torch.Tensor, D: torch.Tensor, Wq: torch.Tensor, Ws: torch.Tensor, N: int,
             out: torch.Tensor | None = None, status: torch.Tensor | None = None, stream=None,
             ws: torch.Tensor | None = None, bias: torch.Tensor | None = None,
             act_type: int = ACT_NONE) -> torch.Tensor:
    """y [M, N] bf16 = MACAQ linear of x bf16 [M, K]; optional fp32 bias [N] and
    output activation act_type (npu_grouped_matmul's bias and act_type)."""
    _dense_args(x, D, Wq, Ws, N, status)
    _require_cuda(x, D, Wq, Ws, out, status)
    M, K = x.shape
    _check_bias(bias, (N,))
    with _on(stream):
        y = _output(out, M, N, x.device)
    L = lib()
    need = int(L.macaq_workspace_bytes(M, N, K, 1))
    ws = workspace(need, x.device, stream, ws)
    if bias is None and act_type == ACT_NONE:
        _check(L.macaq_dense_mm(_ptr(x), _ptr(D), _ptr(Wq), _ptr(Ws), _ptr(y), M, N, K, _ptr(ws),
                                _nbytes(ws), _ptr(status), _stream_ptr(stream)),
               "macaq_dense_mm")
    else:
        _check(L.macaq_dense_mm_ex(_ptr(x), _ptr(D), _ptr(Wq), _ptr(Ws), _ptr(bias), int(act_type), _ptr(y),
                                   M, N, K, _ptr(ws), _nbytes(ws), _ptr(status), _stream_ptr(stream)),
               "macaq_dense_mm_ex")
    return y


def _dense_args(x, D, Wq, Ws, N: int, status):
    _arg(x, "x", torch.bfloat16, ndim=2)
    K = x.shape[1]
    _arg(D, "D", torch.float32, min_numel=K)
    if Wq is not None:
        _weights_args(Wq, Ws, 1, N, K)
    _arg(status, "status", torch.int32, min_numel=1)


def _grouped_args(x, D, Wq, Ws, group_list, group_list_type: int, N: int, status) -> int:
    _arg(x, "x", torch.bfloat16, ndim=2)
    _arg(group_list, "group_list", torch.int64)
    E = _groups(group_list, group_list_type)
    K = x.shape[1]
    _arg(D, "D", torch.float32, min_numel=E * K)
    _weights_args(Wq, Ws, E, N, K)
    _arg(status, "status", torch.int32, min_numel=1)
    return E


def _groups(group_list: torch.Tensor, group_list_type: int) -> int:
    """Number of group_list entries: rows of the [E, 2] form for type 2."""
    if group_list_type == 2:
        if group_list.dim() != 2 or group_list.shape[1] != 2:
            raise MacaqError(-3, "group_list of type 2 must be [E, 2]")
        return int(group_list.shape[0])
    return group_list.numel()


def grouped_mm(x: torch.Tensor, D: torch.Tensor, Wq: torch.Tensor, Ws: torch.Tensor, group_list: torch.Tensor,
               group_list_type: int, N: int, out: torch.Tensor | None = None,
               status: torch.Tensor | None = None, stream=None, ws: torch.Tensor | None = None,
               bias: torch.Tensor | None = None, act_type: int = ACT_NONE) -> torch.Tensor:
    """Grouped MACAQ linear; group_list int64 on the device: [E] for type 0 (cumsum) and 1
    (counts), [E, 2] rows of (group index, group size) for type 2.  Optional fp32 bias
    [E, N] (per expert) and output activation act_type."""
    E = _grouped_args(x, D, Wq, Ws, group_list, group_list_type, N, status)
    _require_cuda(x, D, Wq, Ws, group_list, out, status)
    M, K = x.shape
    _check_bias(bias, (E, N))
    with _on(stream):
        y = _output(out, M, N, x.device)
    L = lib()
    need = int(L.macaq_workspace_bytes(M, N, K, E))
    ws = workspace(need, x.device, stream, ws)
    if bias is None and act_type == ACT_NONE:
        _check(L.macaq_grouped_mm(_ptr(x), _ptr(D), _ptr(Wq), _ptr(Ws), _ptr(group_list), int(group_list_type), E,
                                  _ptr(y), M, N, K, _ptr(ws), _nbytes(ws), _ptr(status),
                                  _stream_ptr(stream)),
               "macaq_grouped_mm")
    else:
        _check(L.macaq_grouped_mm_ex(_ptr(x), _ptr(D), _ptr(Wq), _ptr(Ws), _ptr(group_list), int(group_list_type),
                                     E, _ptr(bias), int(act_type), _ptr(y), M, N, K, _ptr(ws), _nbytes(ws),
                                     _ptr(status), _stream_ptr(stream)),
               "macaq_grouped_mm_ex")
    return y


def prepare_weights_plain(W: torch.Tensor, stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Offline, plain MXFP4 baseline: W fp32 [N, K] or [E, N, K] -> (Wq, Ws) tile images of W itself."""
    if W.dim() == 2:
        W = W.unsqueeze(0)
    _arg(W, "W", torch.float32, ndim=3)
    _require_cuda(W)
    E, N, K = W.shape
    qb, sb = weight_bytes(E, N, K)
    if qb == 0:
        raise MacaqError(-3, "prepare_weights_plain")
    with _on(stream):
        Wq = torch.empty(qb, dtype=torch.uint8, device=W.device)
        Ws = torch.empty(sb, dtype=torch.uint8, device=W.device)
    _check(lib().macaq_prepare_weights_plain(_ptr(W), E, N, K, _ptr(Wq), _ptr(Ws), _stream_ptr(stream)),
           "macaq_prepare_weights_plain")
    return Wq, Ws


def dense_mm_plain(x: torch.Tensor, Wq: torch.Tensor, Ws: torch.Tensor, N: int, out: torch.Tensor | None = None,
                   status: torch.Tensor | None = None, stream=None, ws: torch.Tensor | None = None) -> torch.Tensor:
    """Plain MXFP4 W4A4 baseline (no D, no Hadamard): y [M, N] bf16."""
    _dense_args(x, None, Wq, Ws, N, status)
    _require_cuda(x, Wq, Ws, out, status)
    M, K = x.shape
    with _on(stream):
        y = _output(out, M, N, x.device)
    L = lib()
    ws = workspace(int(L.macaq_workspace_bytes(M, N, K, 1)), x.device, stream, ws)
    _check(L.macaq_dense_mm_plain(_ptr(x), _ptr(Wq), _ptr(Ws), _ptr(y), M, N, K, _ptr(ws), _nbytes(ws),
                                  _ptr(status), _stream_ptr(stream)),
           "macaq_dense_mm_plain")
    return y


def grouped_mm_plain(x: torch.Tensor, Wq: torch.Tensor, Ws: torch.Tensor, group_list: torch.Tensor,
                     group_list_type: int, N: int, out: torch.Tensor | None = None,
                     status: torch.Tensor | None = None, stream=None, ws: torch.Tensor | None = None) -> torch.Tensor:
    """Grouped plain MXFP4 W4A4 baseline; group_list as in grouped_mm."""
    E = _grouped_args(x, None, Wq, Ws, group_list, group_list_type, N, status)
    _require_cuda(x, Wq, Ws, group_list, out, status)
    M, K = x.shape
    with _on(stream):
        y = _output(out, M, N, x.device)
    L = lib()
    ws = workspace(int(L.macaq_workspace_bytes(M, N, K, E)), x.device, stream, ws)
    _check(L.macaq_grouped_mm_plain(_ptr(x), _ptr(Wq), _ptr(Ws), _ptr(group_list), int(group_list_type), E,
                                    _ptr(y), M, N, K, _ptr(ws), _nbytes(ws), _ptr(status), _stream_ptr(stream)),
           "macaq_grouped_mm_plain")
    return y


def unfused_dense_mm(x: torch.Tensor, D: torch.Tensor, Wq: torch.Tensor, Ws: torch.Tensor, N: int,
                     out: torch.Tensor | None = None, status: torch.Tensor | None = None,
                     stream=None, ws: torch.Tensor | None = None) -> torch.Tensor:
    """Ablation: separate quantisation kernel, then the block-scaled GEMM."""
    _dense_args(x, D, Wq, Ws, N, status)
    _require_cuda(x, D, Wq, Ws, out, status)
    M, K = x.shape
    with _on(stream):
        y = _output(out, M, N, x.device)
    L = lib()
    need = int(L.macaq_unfused_workspace_bytes(M, K))
    ws = workspace(need, x.device, stream, ws)
    _check(L.macaq_unfused_dense_mm(_ptr(x), _ptr(D), _ptr(Wq), _ptr(Ws), _ptr(y), M, N, K, _ptr(ws),
                                    _nbytes(ws), _ptr(status), _stream_ptr(stream)),
           "macaq_unfused_dense_mm")
    return y


def dense_mm_noalloc(x: torch.Tensor, D: torch.Tensor, Wq: torch.Tensor, Ws: torch.Tensor, N: int,
                     out: torch.Tensor | None = None, status: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """Dense MACAQ linear using the library's fixed device scratch buffer
    instead of a caller workspace (for callers that cannot allocate)."""
    _dense_args(x, D, Wq, Ws, N, status)
    _require_cuda(x, D, Wq, Ws, out, status)
    M, K = x.shape
    with _on(stream):
        y = _output(out, M, N, x.device)
    _check(lib().macaq_dense_mm_noalloc(_ptr(x), _ptr(D), _ptr(Wq), _ptr(Ws), _ptr(y), M, N, K, _ptr(status),
                                        _stream_ptr(stream)), "macaq_dense_mm_noalloc")
    return y


def quantize_activations(x: torch.Tensor, D: torch.Tensor, stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Activation prologue alone: canonical codes [M, K/2] and E8M0 scales [M, K/32]."""
    _dense_args(x, D, None, None, 0, None)
    _require_cuda(x, D)
    M, K = x.shape
    with _on(stream):
        codes = torch.empty((M, K // 2), dtype=torch.uint8, device=x.device)
        scales = torch.empty((M, K // 32), dtype=torch.uint8, device=x.device)
    _check(lib().macaq_quantize_activations(_ptr(x), _ptr(D), _ptr(codes), _ptr(scales), M, K,
                                            _stream_ptr(stream)), "macaq_quantize_activations")
    return codes, scales


def fused_plan(M: int, N: int, K: int) -> tuple[int, int]:
    """(token tile, K split) that dense_mm's fused kernel uses for this shape (M <= 128)."""
    bt, s = ctypes.c_int(0), ctypes.c_int(0)
    _check(lib().macaq_fused_plan(M, N, K, ctypes.byref(bt), ctypes.byref(s)), "macaq_fused_plan")
    return bt.value, s.value


def fused_probe(x: torch.Tensor, D: torch.Tensor | None, Wq: torch.Tensor, Ws: torch.Tensor, N: int,
                token_tile: int, k_split: int, plain: bool = False, dump: bool = True, stream=None):
    """Test only: the fused kernel with a given plan; returns (y, codes, scales), the
    last two being its own activation operand tiles in canonical form (None
    without dump)."""
    _dense_args(x, None if plain else D, Wq, Ws, N, None)
    _require_cuda(x, D, Wq, Ws)
    M, K = x.shape
    with _on(stream):
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
        codes = torch.empty((M, K // 2), dtype=torch.uint8, device=x.device) if dump else None
        scales = torch.empty((M, K // 32), dtype=torch.uint8, device=x.device) if dump else None
    _check(lib().macaq_fused_probe(_ptr(x), None if plain else _ptr(D), _ptr(Wq), _ptr(Ws), _ptr(y), M, N, K,
                                   int(token_tile), int(k_split), int(bool(plain)), _ptr(codes), _ptr(scales),
                                   None, _stream_ptr(stream)), "macaq_fused_probe")
    return y, codes, scales


def run_wait_expiry(timeout_ns: int, stream=None) -> torch.Tensor:
    """Test only: run the kernels' bounded wait out on purpose; returns the device status word."""
    with _on(stream):
        status = torch.zeros(4, dtype=torch.int32, device="cuda")
    _check(lib().macaq_test_wait_expiry(int(timeout_ns), _ptr(status), _stream_ptr(stream)),
           "macaq_test_wait_expiry")
    return status


def export_weights(Wq: torch.Tensor, Ws: torch.Tensor, E: int, N: int, K: int,
                   stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Prepared tile images -> canonical codes [E, N, K/2] and scales [E, N, K/32]."""
    _weights_args(Wq, Ws, E, N, K)
    _require_cuda(Wq, Ws)
    with _on(stream):
        codes = torch.empty((E, N, K // 2), dtype=torch.uint8, device=Wq.device)
        scales = torch.empty((E, N, K // 32), dtype=torch.uint8, device=Wq.device)
    _check(lib().macaq_export_weights(_ptr(Wq), _ptr(Ws), _ptr(codes), _ptr(scales), E, N, K,
                                      _stream_ptr(stream)), "macaq_export_weights")
    return codes, scales


def mx_encode_blocks(v: torch.Tensor, stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """MX encoding (E8M0 + E2M1) of fp32 blocks of 32."""
    _arg(v, "v", torch.float32)
    _require_cuda(v)
    n = v.numel()
    with _on(stream):
        codes = torch.empty(n // 2, dtype=torch.uint8, device=v.device)
        scales = torch.empty(n // 32, dtype=torch.uint8, device=v.device)
    _check(lib().macaq_mx_encode_blocks(_ptr(v), _ptr(codes), _ptr(scales), n, _stream_ptr(stream)),
           "macaq_mx_encode_blocks")
    return codes, scales
