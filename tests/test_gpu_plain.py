"""Plain MXFP4 W4A4 baseline on the GPU (no D, no Hadamard) against the oracle.

The baseline is the native comparison of the MACAQ page: activations and weights
quantised to MXFP4 directly, then the same block-scaled tensor-core product with
no 2^-5.  Weight preparation must be bit-exact; outputs are compared with the
oracle's exact product under the same tolerance as the MACAQ path.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import w4a4_mxfp4_quantize_b200 as mq
from helpers import compare, f32_dev, x_to_dev, y_to_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    mq.build()
    oracle.build()


def _export(Wq, Ws, E, N, K):
    codes, scales = mq.export_weights(Wq, Ws, E, N, K)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy()


@pytest.mark.parametrize("shape", [(1, 1024, 1024), (1, 48, 256), (3, 144, 512), (2, 384, 768)])
def test_plain_weight_prep_bit_exact(shape):
    E, N, K = shape
    rng = np.random.default_rng(E * 7 + N + K)
    W = (rng.standard_normal((E, N, K)) * 0.02).astype(np.float32)
    W[0, 0, :32] = 0.0                       # an all-zero block
    W[-1, -1, 32:64] *= 1e4                  # a large-range block
    Wq, Ws = mq.prepare_weights_plain(f32_dev(W))
    codes, scales = _export(Wq, Ws, E, N, K)
    for e in range(E):
        qc, qs = oracle.quantize_plain(W[e])
        assert np.array_equal(codes[e], qc), e
        assert np.array_equal(scales[e], qs), e


def _run_dense_plain(p: synth.Problem):
    Wq, Ws = mq.prepare_weights_plain(f32_dev(p.W))
    y = mq.dense_mm_plain(x_to_dev(p.x), Wq, Ws, p.N)
    torch.cuda.synchronize()
    return y_to_bits(y)


@pytest.mark.parametrize("M,K,N", [(1, 256, 16), (16, 1024, 1024), (5, 512, 48), (128, 1024, 2048),
                                   (129, 512, 256), (300, 1024, 160)])
def test_dense_plain_exact_oracle(M, K, N):
    # M <= 128 runs the fused kernel, larger M the quantise-once path
    p = synth.dense(M, K, N, seed=M + 2 * K + N)
    compare(_run_dense_plain(p), oracle.dense_mm_plain(p.x, p.W[0]), f"plain {M}x{K}x{N}")


def test_dense_plain_bit_exact_on_representable_operands():
    # losslessly quantisable operands and short K: the FP32 accumulation is exact,
    # so the GPU must return the oracle's correctly rounded result bit for bit
    rng = np.random.default_rng(31)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    M, N, K = 40, 128, 256

    def representable(rows):
        v = rng.choice(grid, size=(rows, K)) * rng.choice([-1, 1], size=(rows, K))
        v[:, ::32] = 6.0
        return v * np.repeat(2.0 ** rng.integers(-3, 3, size=(rows, K // 32)), 32, axis=1)

    x = synth.to_bf16_bits(representable(M).astype(np.float32))
    W = representable(N).astype(np.float32)
    Wq, Ws = mq.prepare_weights_plain(f32_dev(W))
    for m_rows in (M, 200):  # fused path and quantise-once path
        xx = np.concatenate([x] * (m_rows // M + 1))[:m_rows]
        y = mq.dense_mm_plain(x_to_dev(xx), Wq, Ws, N)
        torch.cuda.synchronize()
        assert np.array_equal(y_to_bits(y), oracle.dense_mm_plain(xx, W)), m_rows


def test_dense_plain_prefill_sampled():
    p = synth.config(2)[3]
    y = _run_dense_plain(p)
    qa, sa = oracle.quantize_act_plain(p.x)
    qw, sw = oracle.quantize_plain(p.W[0])
    rng = np.random.default_rng(9)
    rows = rng.integers(0, p.M, 3000)
    cols = rng.integers(0, p.N, 3000)
    compare(y[rows, cols], oracle.gemm_at_plain(qa, sa, qw, sw, rows, cols), p.name + " plain sampled")


def _run_grouped_plain(p: synth.Problem):
    Wq, Ws = mq.prepare_weights_plain(f32_dev(p.W))
    gl = torch.from_numpy(np.asarray(p.group_list, np.int64)).cuda()
    y = mq.grouped_mm_plain(x_to_dev(p.x), Wq, Ws, gl, p.group_list_type, p.N)
    torch.cuda.synchronize()
    return y_to_bits(y)


@pytest.mark.parametrize("T,E,K,N,dist,gtype", [(96, 4, 256, 128, "uniform", 1), (300, 16, 256, 64, "zipf", 0)])
def test_grouped_plain_exact_oracle(T, E, K, N, dist, gtype):
    p = synth.grouped(T, E, K, N, seed=T + 3 * E, dist=dist, group_list_type=gtype)
    st, want = oracle.grouped_mm_plain(p.x, p.W, p.group_list, p.group_list_type)
    assert st == 0
    compare(_run_grouped_plain(p), want, p.name + " plain")


def test_plain_needs_no_d_and_checks_its_arguments():
    p = synth.dense(16, 256, 128, seed=1)
    Wq, Ws = mq.prepare_weights_plain(f32_dev(p.W))
    with pytest.raises(mq.MacaqError):
        mq.dense_mm_plain(x_to_dev(p.x), Wq, Ws, 130)  # N % 16 != 0
    y = mq.dense_mm_plain(x_to_dev(p.x), Wq, Ws, p.N)
    torch.cuda.synchronize()
    assert y.shape == (16, 128)
