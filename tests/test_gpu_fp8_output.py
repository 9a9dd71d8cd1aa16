"""FP8 (E4M3) output of the MACAQ linear on the GPU, through the C ABI.

The output option that feeds a following FP8 layer (npu_grouped_matmul's
output_dtype parameter; here its FP8 choice): y8 = E4M3(act(v + bias) * y_scale),
round to nearest even with saturation at +-448.  Compared with the oracle's
correctly rounded codes (the exact sum in binary64) with the BF16 tests' bound
carried over to the FP8 grid (tests/helpers.compare_fp8); without an activation
the codes themselves agree almost everywhere and lie within one E4M3 step.  The
dense call runs the fused kernel for M <= 128 (with and without a K split) and
the quantise-once pair above; the grouped call always the latter.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import w4a4_mxfp4_quantize_b200 as mq
from helpers import compare, compare_fp8, f32_dev, x_to_dev, y_to_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    mq.build()
    mq.lib()
    torch.cuda.init()


def _oracle_fp8(p, x_rows, D, W, bias, act, y_scale):
    qa, sa = oracle.quantize_act(x_rows, D)
    qw, sw = oracle.quantize_weights(W, D)
    return oracle.gemm_fp8(qa, sa, qw, sw, bias=bias, act_type=act, y_scale=y_scale)


@pytest.mark.parametrize("M,K,N,act", [(16, 1024, 256, 0), (300, 512, 272, 2), (129, 768, 144, 5), (64, 256, 48, 1),
                                        (32, 2048, 512, 2), (128, 1024, 384, 0)])
def test_dense_fp8_output_against_the_oracle(M, K, N, act):
    p = synth.dense(M, K, N, seed=M + N)
    bias = (np.random.default_rng(M).standard_normal(N) * 0.3).astype(np.float32) if act else None
    qa, sa = oracle.quantize_act(p.x, p.D[0])
    qw, sw = oracle.quantize_weights(p.W[0], p.D[0])
    y16 = synth.bf16_bits_to_f32(oracle.gemm_ex(qa, sa, qw, sw, bias, act)).astype(np.float64)
    y_scale = float(400.0 / max(np.abs(y16).max(), 1e-6))   # the largest output near the top of the range
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    y8 = mq.dense_mm_fp8(x_to_dev(p.x), f32_dev(p.D[0]), Wq, Ws, N, y_scale,
                         bias=None if bias is None else f32_dev(bias), act_type=act)
    torch.cuda.synchronize()
    ref = oracle.gemm_fp8(qa, sa, qw, sw, bias=bias, act_type=act, y_scale=y_scale)
    stats = compare_fp8(y8.cpu().numpy(), ref, f"dense fp8 {M}x{K}x{N} act {act}")
    if act == 0:  # scaling only: FP32 summation order is the one difference
        assert stats["exact_share"] >= 0.99 and stats["within_one_step_share"] == 1.0, stats


def test_dense_fp8_saturates_and_matches_the_bf16_call():
    # a scale that pushes part of the outputs past 448: those saturate to +-448,
    # the rest equal the E4M3 rounding of the BF16 call's values within one step
    p = synth.dense(256, 1024, 512, seed=3)
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    x, D = x_to_dev(p.x), f32_dev(p.D[0])
    y16 = mq.dense_mm(x, D, Wq, Ws, p.N).float().cpu().numpy().astype(np.float64)
    y_scale = float(900.0 / np.abs(y16).max())
    y8 = mq.dense_mm_fp8(x, D, Wq, Ws, p.N, y_scale).cpu().numpy()
    torch.cuda.synchronize()
    big = np.abs(y16 * y_scale) >= 464.0
    assert big.any() and np.all((y8[big] & 0x7F) == 0x7E)
    ours = oracle.e4m3_decode(y8[~big])
    want = y16[~big] * y_scale
    step = np.exp2(np.floor(np.log2(np.maximum(np.abs(want), 2.0 ** -6))) - 3)
    assert np.all(np.abs(ours - want) <= step)


@pytest.mark.parametrize("gtype", [1, 2])
def test_grouped_fp8_output_against_the_oracle(gtype):
    p = synth.grouped(200, 5, 512, 144, seed=17, dist="zipf", group_list_type=1)
    bias = (np.random.default_rng(4).standard_normal((p.E, p.N)) * 0.3).astype(np.float32)
    idx = np.array([4, 0, 2, 2, 1], np.int64) if gtype == 2 else np.arange(p.E)
    gl = np.ascontiguousarray(np.stack([idx, p.counts]).T.astype(np.int64)) if gtype == 2 else p.counts.astype(np.int64)
    y_scale = 37.0
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    y8 = mq.grouped_mm_fp8(x_to_dev(p.x), f32_dev(p.D), Wq, Ws, torch.from_numpy(gl).cuda(), gtype, p.N, y_scale,
                           bias=f32_dev(bias), act_type=mq.ACT_SILU).cpu().numpy()
    torch.cuda.synchronize()
    off = np.concatenate([[0], np.cumsum(p.counts)])
    for j in range(p.E):
        a, b = int(off[j]), int(off[j + 1])
        if b == a:
            continue
        e = int(idx[j])
        ref = _oracle_fp8(p, p.x[a:b], p.D[e], p.W[e], bias[e], mq.ACT_SILU, y_scale)
        compare_fp8(y8[a:b], ref, f"grouped fp8 type {gtype} entry {j}")


def test_fp8_refusals():
    p = synth.dense(32, 256, 64, seed=1)
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    for bad in (0.0, -1.0, float("inf"), float("nan")):
        with pytest.raises(mq.MacaqError) as e:
            mq.dense_mm_fp8(x_to_dev(p.x), f32_dev(p.D[0]), Wq, Ws, p.N, bad)
        assert e.value.status == -3
    with pytest.raises(mq.MacaqError) as e:
        mq.dense_mm_fp8(x_to_dev(p.x), f32_dev(p.D[0]), Wq, Ws, p.N, 1.0, act_type=3)
    assert e.value.status == -13


@pytest.mark.parametrize("M,K,N", [(16, 1024, 256), (96, 2048, 384)])
def test_fused_fp8_equals_the_e4m3_of_the_fused_bf16_values(M, K, N):
    # M <= 128 runs the fused kernel for both outputs (the same plan and summation
    # order): with y_scale = 1 the FP8 codes are the E4M3 rounding of the FP32 values
    # whose BF16 rounding the BF16 call returns, so decoding both and comparing them
    # within the larger of the two rounding steps must agree everywhere
    p = synth.dense(M, K, N, seed=M + 5)
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    x, D = x_to_dev(p.x), f32_dev(p.D[0])
    y16 = mq.dense_mm(x, D, Wq, Ws, N).float().cpu().numpy().astype(np.float64).ravel()
    y8 = mq.dense_mm_fp8(x, D, Wq, Ws, N, 1.0).cpu().numpy().ravel()
    torch.cuda.synchronize()
    dec = oracle.e4m3_decode(y8)
    big = np.abs(y16) >= 464.0
    assert np.all((y8[big] & 0x7F) == 0x7E)
    step = np.exp2(np.floor(np.log2(np.maximum(np.abs(y16[~big]), 2.0 ** -6))) - 3)
    assert np.all(np.abs(dec[~big] - y16[~big]) <= step)


def test_bf16_path_unchanged_next_to_fp8():
    # the GEMM carries both output forms: the BF16 call still matches the oracle exactly as before
    p = synth.dense(300, 512, 272, seed=9)
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    y = mq.dense_mm(x_to_dev(p.x), f32_dev(p.D[0]), Wq, Ws, p.N)
    torch.cuda.synchronize()
    qa, sa = oracle.quantize_act(p.x, p.D[0])
    qw, sw = oracle.quantize_weights(p.W[0], p.D[0])
    compare(y_to_bits(y), oracle.gemm(qa, sa, qw, sw), "bf16 beside fp8")
