"""GPU parity of the output bias and activation (npu_grouped_matmul's bias and
act_type) against the CPU oracle, through the C ABI's _ex entry points.

The oracle adds the bias to 2^-5 times the exact block-scaled sum and applies
the activation in binary64, then rounds once to BF16; the kernels do the same
in FP32, the gated activations through a hardware half-precision tanh.  Outputs
are judged by the tolerance in tests/helpers.py, and the gated activations also
by their own error bound.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import w4a4_mxfp4_quantize_b200 as mq
from helpers import bf16_ulp, compare, f32_dev, x_to_dev, y_to_bits

pytestmark = pytest.mark.gpu

ACTS = [mq.ACT_NONE, mq.ACT_RELU, mq.ACT_GELU_TANH, mq.ACT_FAST_GELU, mq.ACT_SILU]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    mq.build()
    mq.lib()
    torch.cuda.init()


def _bias(N, seed, E=None):
    rng = np.random.default_rng(seed)
    shape = (N,) if E is None else (E, N)
    return (rng.standard_normal(shape) * 0.5).astype(np.float32)


@pytest.mark.parametrize("M,K,N", [(16, 1024, 1024), (100, 512, 272), (300, 768, 272), (1000, 512, 400)])
@pytest.mark.parametrize("act", ACTS)
@pytest.mark.parametrize("with_bias", [True, False])
def test_dense_bias_and_activation(M, K, N, act, with_bias):
    # M <= 128 runs the fused kernel, larger M the quantise-once GEMM
    if not with_bias and act == mq.ACT_NONE:
        pytest.skip("plain call: covered by the parity tests")
    p = synth.dense(M, K, N, seed=M + N + act)
    bias = _bias(N, seed=act) if with_bias else None
    x, D = x_to_dev(p.x), f32_dev(p.D[0])
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    y = mq.dense_mm(x, D, Wq, Ws, N, bias=None if bias is None else f32_dev(bias), act_type=act)
    torch.cuda.synchronize()
    qa, sa = oracle.quantize_act(p.x, p.D[0])
    qw, sw = oracle.quantize_weights(p.W[0], p.D[0])
    compare(y_to_bits(y), oracle.gemm_ex(qa, sa, qw, sw, bias, act), f"dense M={M} act={act} bias={with_bias}")


@pytest.mark.parametrize("act", [mq.ACT_GELU_TANH, mq.ACT_SILU])
def test_dense_prefill_shape_sampled(act):
    # M = 4096, K = 1024, N = 3072 (the prefill workload) with bias: sampled exact outputs
    p = synth.dense(4096, 1024, 3072, seed=21)
    bias = _bias(3072, seed=22)
    x, D = x_to_dev(p.x), f32_dev(p.D[0])
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    y = y_to_bits(mq.dense_mm(x, D, Wq, Ws, 3072, bias=f32_dev(bias), act_type=act))
    rng = np.random.default_rng(23)
    rows, cols = rng.integers(0, 4096, 4000), rng.integers(0, 3072, 4000)
    qa, sa = oracle.quantize_act(p.x[np.unique(rows)], p.D[0])
    ridx = np.searchsorted(np.unique(rows), rows)
    qw, sw = oracle.quantize_weights(p.W[0], p.D[0])
    ref = oracle.gemm_at_ex(qa, sa, qw, sw, ridx, cols, bias, act)
    compare(y[rows, cols], ref, f"prefill sampled act={act}")


@pytest.mark.parametrize("act", ACTS)
def test_grouped_bias_per_expert_and_activation(act):
    p = synth.grouped(300, 5, 512, 144, seed=4 + act, dist="uniform")
    bias = _bias(144, seed=act, E=5)
    x, D = x_to_dev(p.x), f32_dev(p.D)
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), D)
    gl = torch.from_numpy(p.group_list).cuda()
    y = mq.grouped_mm(x, D, Wq, Ws, gl, p.group_list_type, p.N, bias=f32_dev(bias), act_type=act)
    torch.cuda.synchronize()
    st, ref = oracle.grouped_mm_ex(p.x, p.D, p.W, p.group_list, p.group_list_type, bias, act)
    assert st == oracle.OK
    compare(y_to_bits(y), ref, f"grouped act={act}")


def test_grouped_type2_bias_follows_the_named_expert():
    # [E, 2] rows of (expert, rows): a repeated expert takes its own bias each time
    rng = np.random.default_rng(31)
    E, K, N = 4, 256, 128
    W = rng.standard_normal((E, N, K)).astype(np.float32) * 0.02
    D = np.ones((E, K), np.float32)
    gl = np.array([[2, 40], [0, 0], [2, 25], [3, 35]], np.int64)
    M = int(gl[:, 1].sum())
    xf = rng.standard_normal((M, K)).astype(np.float32)
    xb = synth.to_bf16_bits(xf)
    bias = _bias(N, seed=32, E=E)
    Wq, Ws = mq.prepare_weights(f32_dev(W), f32_dev(D))
    y = mq.grouped_mm(x_to_dev(xb), f32_dev(D), Wq, Ws, torch.from_numpy(gl).cuda(), 2, N,
                      bias=f32_dev(bias), act_type=mq.ACT_FAST_GELU)
    torch.cuda.synchronize()
    st, ref = oracle.grouped_mm_ex(xb, D, W, gl, 2, bias, mq.ACT_FAST_GELU)
    assert st == oracle.OK
    compare(y_to_bits(y), ref, "grouped type 2 bias")


def test_act_type_3_is_refused_without_launching():
    p = synth.dense(16, 256, 64, seed=1)
    x, D = x_to_dev(p.x), f32_dev(p.D[0])
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    y = torch.full((16, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mq.MacaqError) as e:
        mq.dense_mm(x, D, Wq, Ws, 64, out=y, act_type=3)
    assert e.value.status == -13
    torch.cuda.synchronize()
    assert bool((y == 7.0).all())


@pytest.mark.parametrize("M", [64, 1000])
@pytest.mark.parametrize("act", [mq.ACT_GELU_TANH, mq.ACT_FAST_GELU, mq.ACT_SILU])
def test_gated_activation_error_bound(M, act):
    # The gated forms are v sigmoid(a) = h + h tanh(a / 2), h = v / 2, with a hardware
    # half-precision tanh: the argument rounded to FP16 (relative 2^-11, times
    # tanh' <= 1 and |u| tanh'(u) <= 0.45), the approximation (~2^-11) and the FP16
    # result (2^-12 near 1) keep |tanh error| below ~1e-3, so |y - y_exact| <= 5e-4 |v|
    # before the BF16 rounding of each side (one ulp between them).  v is the
    # oracle's pre-activation value (bias included).
    K, N = 512, 400
    p = synth.dense(M, K, N, seed=40 + act)
    bias = _bias(N, seed=41)
    x, D = x_to_dev(p.x), f32_dev(p.D[0])
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    y = y_to_bits(mq.dense_mm(x, D, Wq, Ws, N, bias=f32_dev(bias), act_type=act))
    qa, sa = oracle.quantize_act(p.x, p.D[0])
    qw, sw = oracle.quantize_weights(p.W[0], p.D[0])
    v = synth.bf16_bits_to_f32(oracle.gemm_ex(qa, sa, qw, sw, bias, mq.ACT_NONE)).astype(np.float64)
    ref = synth.bf16_bits_to_f32(oracle.gemm_ex(qa, sa, qw, sw, bias, act)).astype(np.float64)
    got = synth.bf16_bits_to_f32(y).astype(np.float64)
    err = np.abs(got - ref)
    bound = 6e-4 * np.abs(v) + bf16_ulp(np.maximum(np.abs(got), np.abs(ref)))
    bad = np.flatnonzero(err > bound)
    assert bad.size == 0, (act, bad[:5], v.ravel()[bad[:5]], got.ravel()[bad[:5]], ref.ravel()[bad[:5]])
    # a large share agrees bit for bit: the error is a fraction of one BF16 ulp
    assert np.mean(got == ref) > 0.3
