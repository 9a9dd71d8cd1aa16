"""GPU parity of the offline D calibration (macaq_calibrate_d) with the CPU
oracle: bit-exact, since both sides take maxima of magnitudes and one IEEE
binary64 divide and square root per channel."""
import numpy as np
import pytest
import torch

import oracle
import synth
import w4a4_mxfp4_quantize_b200 as mq
from helpers import f32_dev, x_to_dev, y_to_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    mq.build()
    mq.lib()
    torch.cuda.init()


@pytest.mark.parametrize("T,K,N", [(1024, 1024, 2048), (1, 256, 16), (333, 3072, 1024)])
def test_dense_calibration_bit_exact(T, K, N):
    # 1,024 calibration tokens is the MACAQ page's pilot; 1 and 333 rows are edge cases
    p = synth.dense(T, K, N, seed=T + K)
    D = mq.calibrate_d(x_to_dev(p.x), f32_dev(p.W))
    st, ref = oracle.calibrate_d(p.x, p.W)
    assert st == oracle.OK
    assert np.array_equal(D.cpu().numpy(), ref)


def test_calibration_special_channels_bit_exact():
    K, N, T = 512, 16, 8
    rng = np.random.default_rng(3)
    x = rng.standard_normal((T, K)).astype(np.float32)
    W = rng.standard_normal((N, K)).astype(np.float32)
    x[:, 0] = 0.0; W[:, 0] = 0.0          # both zero
    W[:, 1] = 0.0                          # w = 0 < a
    x[:, 2] = 0.0                          # a = 0 < w
    x[:, 3] *= 2.0 ** 30                   # clamp high
    W[:, 4] *= 2.0 ** 30                   # clamp low
    xb = synth.to_bf16_bits(x)
    D = mq.calibrate_d(x_to_dev(xb), f32_dev(W))
    st, ref = oracle.calibrate_d(xb, W)
    assert st == oracle.OK
    assert np.array_equal(D.cpu().numpy(), ref)
    assert ref[0, 0] == 1.0 and ref[0, 1] == np.float32(1e2) and ref[0, 2] == np.float32(1e-2)


@pytest.mark.parametrize("gtype", [0, 1, 2])
def test_grouped_calibration_bit_exact(gtype):
    # Zipf-skewed experts (some empty); type 2 lists the experts in reverse order
    g = synth.grouped(3000, 24, 512, 96, seed=5, dist="zipf", group_list_type=1)
    counts = g.counts
    if gtype == 0:
        gl = np.cumsum(counts).astype(np.int64)
    elif gtype == 1:
        gl = counts.astype(np.int64)
    else:
        gl = np.stack([np.arange(24)[::-1], counts[::-1]], axis=1).astype(np.int64)
        # rows then follow the reversed order: reorder x to match
    x = g.x
    if gtype == 2:
        off = np.concatenate([[0], np.cumsum(counts)])
        x = np.concatenate([g.x[off[e]:off[e + 1]] for e in range(23, -1, -1)])
    D = mq.calibrate_d(x_to_dev(x), f32_dev(g.W), torch.from_numpy(gl).cuda(), gtype)
    st, ref = oracle.calibrate_d(x, g.W, gl, gtype)
    assert st == oracle.OK
    assert np.array_equal(D.cpu().numpy(), ref)
    assert np.array_equal(ref, g.D)        # the same factors the workload generator states


def test_invalid_group_list_is_refused_before_launch():
    g = synth.grouped(100, 4, 256, 32, seed=6)
    bad = torch.tensor([10, 20, 30, 39], dtype=torch.int64, device="cuda")   # 99 rows, not 100
    with pytest.raises(mq.MacaqError) as e:
        mq.calibrate_d(x_to_dev(g.x), f32_dev(g.W), bad, 1)
    assert e.value.status == -10


def test_calibrated_layer_end_to_end():
    # calibrate on the device, prepare the weights with that D, run the layer:
    # the same output as with the oracle's factors
    p = synth.dense(1024, 1024, 512, seed=8)
    x, W = x_to_dev(p.x), f32_dev(p.W)
    D = mq.calibrate_d(x, W)
    Wq, Ws = mq.prepare_weights(W, D)
    y = mq.dense_mm(x[:128].contiguous(), D[0], Wq, Ws, 512)
    st, Dref = oracle.calibrate_d(p.x, p.W)
    Wq2, Ws2 = mq.prepare_weights(W, f32_dev(Dref))
    y2 = mq.dense_mm(x[:128].contiguous(), f32_dev(Dref[0]), Wq2, Ws2, 512)
    torch.cuda.synchronize()
    assert np.array_equal(y_to_bits(y), y_to_bits(y2))
