"""The dense entry point for callers that cannot allocate device memory.

Some callers may not call cudaMalloc at all: code running where device
allocation is not permitted, or serving processes whose device memory is laid
out once up front and must not grow.  macaq_dense_mm_noalloc serves them: it
runs the quantise-once dense path with its scratch in a fixed buffer that the
library holds on each device.  These checks call it through the C ABI and
compare it with macaq_dense_mm, the entry point that takes a caller-provided
workspace, on two calls in a row with different inputs (the shared buffer keeps
the previous call's contents, so the second call must not depend on them).

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

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
        compare(y_to_bits(y), y_to_bits(y_ref), f"noalloc M={M} K={K} N={N}")


def test_noalloc_refuses_sizes_beyond_its_buffer():
    L = mq.lib()
    M, K, N = 65536, 1024, 128  # needs ~34 MiB of scratch, above the 8 MiB buffer
    P = ctypes.c_void_p
    # the size check comes before any device access: distinct dummy addresses suffice
    st = L.macaq_dense_mm_noalloc(P(1 << 40), P(2 << 40), P(3 << 40), P(4 << 40), P(5 << 40), M, N, K, None, None)
    assert st == -11  # MACAQ_ERR_WORKSPACE, nothing launched
