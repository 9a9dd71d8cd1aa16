"""The dense entry point for callers that cannot allocate device memory.

Some callers may not call cudaMalloc at all: code running where device
allocation is not permitted, or serving processes whose device memory is laid
out once up front and must not grow.  macaq_dense_mm_noalloc serves them: it
runs the quantise-once dense path with its scratch in a fixed buffer that the
library holds on each device.  These checks call it through the C ABI and
compare it with macaq_dense_mm, the entry point that takes a caller-provided
workspace, on two calls in a row with different inputs (the shared buffer keeps
the previous call's contents, so the second call must not depend on them):
identical outputs where both run the same kernels, the stated tolerance and
the oracle where macaq_dense_mm takes its fused kernel.  The refusal of sizes
beyond the buffer needs no device and is checked with the other host-side
refusals (tests/test_abi.py).

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
import w4a4_mxfp4_quantize_b200 as mq
from helpers import compare, f32_dev, x_to_dev, y_to_bits

pytestmark = pytest.mark.gpu


def _noalloc(L, x, D, Wq, Ws, y, M, N, K, status=None):
    P = ctypes.c_void_p
    s = torch.cuda.current_stream()
    return L.macaq_dense_mm_noalloc(P(x.data_ptr()), P(D.data_ptr()), P(Wq.data_ptr()), P(Ws.data_ptr()),
                                    P(y.data_ptr()), M, N, K, None if status is None else P(status.data_ptr()),
                                    P(s.cuda_stream))


def _oracle(p, xb):
    qa, sa = oracle.quantize_act(xb, p.D[0])
    qw, sw = oracle.quantize_weights(p.W[0], p.D[0])
    return oracle.gemm(qa, sa, qw, sw)


@pytest.mark.parametrize("M,K,N", [(300, 512, 272), (4096, 1024, 1024), (64, 3072, 1024)])
def test_noalloc_matches_workspace_entry_point_twice(M, K, N):
    mq.build()
    L = mq.lib()
    p = synth.dense(M, K, N, seed=7)
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    D = f32_dev(p.D[0])
    rng = np.random.default_rng(8)
    inputs = [p.x, synth.to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32) * 3)]
    for xb in inputs:  # two calls in a row on the shared buffer
        x = x_to_dev(xb)
        y_ref = mq.dense_mm(x, D, Wq, Ws, N)
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        assert _noalloc(L, x, D, Wq, Ws, y, M, N, K, status) == 0
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        if M > 128:
            # both entry points run the same two kernels: the outputs are identical
            assert np.array_equal(y_to_bits(y), y_to_bits(y_ref)), f"noalloc M={M} K={K} N={N}"
        else:
            # macaq_dense_mm runs the fused kernel here, a different FP32 summation order
            compare(y_to_bits(y), y_to_bits(y_ref), f"noalloc M={M} K={K} N={N}")
            compare(y_to_bits(y), _oracle(p, xb), f"noalloc M={M} K={K} N={N} vs oracle")


def test_noalloc_python_wrapper_equals_the_c_call():
    L = mq.lib()
    p = synth.dense(200, 512, 144, seed=9)
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    x, D = x_to_dev(p.x), f32_dev(p.D[0])
    y_c = torch.empty((p.M, p.N), dtype=torch.bfloat16, device="cuda")
    assert _noalloc(L, x, D, Wq, Ws, y_c, p.M, p.N, p.K) == 0
    y_py = mq.dense_mm_noalloc(x, D, Wq, Ws, p.N)
    torch.cuda.synchronize()
    assert np.array_equal(y_to_bits(y_py), y_to_bits(y_c))
    compare(y_to_bits(y_py), _oracle(p, p.x), "noalloc wrapper vs oracle")
