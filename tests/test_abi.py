"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol include/macaq.h declares, and refuses bad arguments by name
before touching the device.

The refusal tests pass made-up device addresses.  They rely on the library
refusing each call before any launch, so they run only in a process that sees
no CUDA device: where a GPU is visible, one test re-runs them in a child
process with CUDA_VISIBLE_DEVICES set empty.  A broken host check then ends in
a named CUDA error there, never in a kernel reading unmapped memory."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

import w4a4_mxfp4_quantize_b200 as mq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "macaq.h")


@pytest.fixture(scope="module")
def L():
    mq.build()
    return mq.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(macaq_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for need in ["macaq_prepare_weights", "macaq_dense_mm", "macaq_grouped_mm", "macaq_workspace_bytes",
                 "macaq_weight_code_bytes", "macaq_weight_scale_bytes", "macaq_quantize_activations",
                 "macaq_export_weights", "macaq_unfused_dense_mm", "macaq_status_string"]:
        assert need in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    assert set(declared_functions()) <= set(mq.exported_symbols()) | {"macaq_abi_version"}


def test_abi_version_and_status_strings(L):
    assert L.macaq_abi_version() == 5
    for code, name in mq.STATUS.items():
        assert L.macaq_status_string(code).decode() == name
    assert L.macaq_status_string(-99).decode() == "MACAQ_ERR_UNKNOWN"


def test_weight_sizes(L):
    assert L.macaq_weight_code_bytes(1, 1024, 1024) == 1024 * 512
    assert L.macaq_weight_scale_bytes(1, 1024, 1024) == 1024 * 32
    assert L.macaq_weight_code_bytes(2, 48, 256) == 2 * 256 * 128  # rows padded to 256 (image pairs)
    assert L.macaq_weight_scale_bytes(1, 384, 512) == 512 * 16     # three images and a zero fourth
    assert L.macaq_weight_code_bytes(1, 1000, 1024) == 0           # N % 16 != 0
    assert L.macaq_weight_code_bytes(1, 1024, 1000) == 0           # K % 256 != 0
    assert L.macaq_weight_code_bytes(1025, 1024, 1024) == 0        # E > 1024
    assert L.macaq_unfused_workspace_bytes(16, 1024) == 4096 + 128 * (512 + 32)


def _device_visible() -> bool:
    import torch
    return torch.cuda.is_available()


# every test below that passes made-up addresses carries this mark
hidden_device = pytest.mark.skipif(_device_visible(), reason="made-up device addresses: run with the device hidden")


def test_fake_address_refusals_run_with_the_device_hidden():
    if not _device_visible():
        pytest.skip("no device visible: the refusal tests run in this process")
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.abspath(__file__), "-x", "-q", "-p",
                        "no:cacheprovider", "-m", "not gpu", "-k", "by_name or no_gpu"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and "skipped" not in r.stdout.splitlines()[-1], r.stdout[-2000:]


P = ctypes.c_void_p
A, B, C, Dp, Y = (P(i << 32) for i in range(1, 6))


def dense(L, x=A, d=B, wq=C, ws=Dp, y=Y, M=16, N=1024, K=1024):
    return L.macaq_dense_mm(x, d, wq, ws, y, M, N, K, None, 0, None, None)


@hidden_device
def test_dense_refusals_by_name(L):
    assert dense(L, N=1000) == -3
    assert dense(L, K=1000) == -3
    assert dense(L, K=128) == -3
    assert dense(L, K=288) == -3                   # a whole number of 32-blocks, but not of 256-wide tiles
    assert dense(L, K=65536 + 256) == -3
    assert dense(L, N=65536 + 16) == -3
    assert dense(L, M=-1) == -3
    assert dense(L, x=None) == -1
    assert dense(L, y=None) == -1
    assert dense(L, x=P((1 << 32) + 8)) == -2
    assert dense(L, y=P(1 << 32)) == -5           # y overlaps x
    assert dense(L, M=0, x=None) == 0            # M = 0 is a no-op


@hidden_device
def test_grouped_refusals_by_name(L):
    gl = P(9 << 32)

    def g(E=4, t=1, glp=gl, N=1024, K=1024, M=64):
        return L.macaq_grouped_mm(A, B, C, Dp, glp, t, E, Y, M, N, K, None, 0, None, None)

    assert g(E=0) == -6
    assert g(E=1025) == -6
    assert g(t=3) == -7
    assert g(t=-1) == -7
    assert g(t=2) == -11  # type 2 is accepted; the missing workspace is the next refusal
    assert g(N=24) == -3
    assert g(glp=None) == -1
    assert g(glp=P((9 << 32) + 4)) == -2


@hidden_device
def test_epilogue_refusals_by_name(L):
    bias = P(11 << 32)

    def d(act=0, b=bias, M=16, N=1024):
        return L.macaq_dense_mm_ex(A, B, C, Dp, b, act, Y, M, N, 1024, None, 0, None, None)

    def g(act=0, b=bias, E=4):
        return L.macaq_grouped_mm_ex(A, B, C, Dp, P(9 << 32), 1, E, b, act, Y, 64, 1024, 1024, None, 0, None, None)

    for act in (3, 6, -1, 100):      # act_type 3 is "not supported" on the npu_grouped_matmul page
        assert d(act=act) == -13
        assert g(act=act) == -13
    assert d(b=P((11 << 32) + 4)) == -2           # bias not 16-byte aligned
    assert d(b=P((5 << 32) + 64)) == -5           # bias inside y ([16, 1024] bf16 at 5 << 32)
    assert g(b=P((5 << 32) + 4096), E=4) == -5
    assert d(act=3, M=0) == -13                   # refused even when there is nothing to compute
    assert g(act=2, b=None) == -11                # accepted; the missing workspace is the next refusal


@hidden_device
def test_calibration_refusals_by_name(L):
    x, W, D, gl = P(1 << 32), P(2 << 32), P(3 << 32), P(4 << 32)

    def c(x=x, T=1024, W=W, E=1, N=512, K=1024, gl=None, t=1, D=D):
        return L.macaq_calibrate_d(x, T, W, E, N, K, gl, t, D, None)

    assert c(E=0) == -6
    assert c(E=1025, gl=gl) == -6
    assert c(K=1000) == -3
    assert c(N=0) == -3
    assert c(T=-1) == -3
    assert c(E=4) == -1                 # a group list is needed for E > 1
    assert c(D=None) == -1
    assert c(E=4, gl=gl, t=3) == -7
    assert c(D=P((3 << 32) + 4)) == -2
    assert c(D=P((1 << 32) + 1024)) == -5   # D inside x


@hidden_device
def test_no_gpu_means_a_named_cuda_error_not_a_fallback(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("GPU present")
    assert dense(L) == -8
    assert L.macaq_dense_mm_ex(A, B, C, Dp, None, 5, Y, 16, 1024, 1024, None, 0, None, None) == -8


@hidden_device
def test_noalloc_refusals_by_name(L):
    # the size check of the fixed scratch buffer comes before any device access
    M, K, N = 65536, 1024, 128  # needs ~34 MiB of scratch, above the 8 MiB buffer
    assert L.macaq_dense_mm_noalloc(A, B, C, Dp, Y, M, N, K, None, None) == -11
    assert L.macaq_dense_mm_noalloc(A, B, C, Dp, Y, 16, 1000, 1024, None, None) == -3
    assert L.macaq_dense_mm_noalloc(None, B, C, Dp, Y, 16, 1024, 1024, None, None) == -1


@hidden_device
def test_probe_and_plan_refusals_by_name(L):
    import ctypes as ct
    bt, s = ct.c_int(0), ct.c_int(0)
    assert L.macaq_fused_plan(129, 1024, 1024, ct.byref(bt), ct.byref(s)) == -3   # fused kernel: M <= 128
    assert L.macaq_fused_plan(16, 1000, 1024, ct.byref(bt), ct.byref(s)) == -3
    assert L.macaq_fused_plan(16, 1024, 1024, None, ct.byref(s)) == -1

    def probe(M=16, bt=16, s=1, codes=P(12 << 32), scales=P(13 << 32), K=1024):
        return L.macaq_fused_probe(A, B, C, Dp, Y, M, 1024, K, bt, s, 0, codes, scales, None, None)

    assert probe(M=129) == -3
    assert probe(bt=48) == -3
    assert probe(s=3) == -3                    # 3 does not divide K/256 = 4
    assert probe(s=9, K=4608) == -3            # at most 8 CTAs per cluster
    assert probe(scales=None) == -1            # codes and scales come together
    assert probe(codes=P((12 << 32) + 8)) == -2
    assert probe(codes=P((5 << 32) + 64)) == -5   # codes inside y
    assert L.macaq_test_wait_expiry(10, P(12 << 32), None) == -3      # below 1 us
    assert L.macaq_test_wait_expiry(2 * 10 ** 9, P(12 << 32), None) == -3
    assert L.macaq_test_wait_expiry(10 ** 6, None, None) == -1


@hidden_device
def test_weight_list_and_transposed_refusals_by_name(L):
    gl, wql, wsl = P(9 << 32), P(14 << 32), P(15 << 32)

    def g(E=4, t=1, q=wql, w=wsl, act=0, N=1024):
        return L.macaq_grouped_mm_list(A, B, q, w, gl, t, E, None, act, Y, 64, N, 1024, None, 0, None, None)

    assert g(E=0) == -6
    assert g(t=3) == -7
    assert g(q=None) == -1
    assert g(w=P((15 << 32) + 8)) == -2           # the table itself must be 16-byte aligned
    assert g(q=P((5 << 32) + 64)) == -5           # a table inside y
    assert g(act=3) == -13
    assert g(N=24) == -3
    assert g() == -11                              # accepted; the missing workspace is the next refusal
    W, D, Wq, Ws = P(1 << 32), P(2 << 32), P(3 << 32), P(4 << 32)
    assert L.macaq_prepare_weights_transposed(W, D, 1, 1000, 1024, Wq, Ws, None) == -3
    assert L.macaq_prepare_weights_transposed(W, D, 0, 1024, 1024, Wq, Ws, None) == -6
    assert L.macaq_prepare_weights_transposed(None, D, 1, 1024, 1024, Wq, Ws, None) == -1
    assert L.macaq_prepare_weights_transposed(W, P((2 << 32) + 4), 1, 1024, 1024, Wq, Ws, None) == -2



@hidden_device
def test_fp8_output_refusals_by_name(L):
    y8 = P(5 << 32)

    def d(scale=1.0, act=0, y=y8, M=16, N=1024, ws=None, nws=0):
        return L.macaq_dense_mm_fp8(A, B, C, Dp, None, act, ctypes.c_float(scale), y, M, N, 1024, ws, nws, None,
                                    None)

    def g(scale=1.0, act=0, E=4):
        return L.macaq_grouped_mm_fp8(A, B, C, Dp, P(9 << 32), 1, E, None, act, ctypes.c_float(scale), y8, 64, 1024,
                                      1024, None, 0, None, None)

    for bad in (0.0, -1.0, float("inf"), float("nan")):
        assert d(scale=bad) == -3                 # the output scale must be finite and positive
        assert d(scale=bad, M=0) == -3            # refused even when there is nothing to compute
        assert g(scale=bad) == -3
    assert d(act=3) == -13
    assert g(act=3) == -13
    assert d(y=None) == -1
    assert d(y=P((5 << 32) + 8)) == -2            # the FP8 output starts 16-byte aligned like the others
    assert d(y=P((1 << 32) + 4096)) == -5         # y8 inside x
    assert d(N=24) == -3
    assert d() == -11                             # accepted; the missing workspace is the next refusal
    assert g() == -11
    assert d(M=0) == 0
