"""The seeded input generator follows its stated recipe: x ~ N(0, 1) with
max(1, round(0.01 K)) outlier channels scaled by 20, rounded to BF16; W ~
N(0, 0.02); D the closed-form channel factor; Zipf(1.1) group counts with a
seeded 1/16 of the experts at probability 0; the workload shapes; and the same
seed giving the same tensors."""
import numpy as np
import pytest

import synth


@pytest.mark.parametrize("K,n_out", [(768, 8), (1024, 10), (2048, 20), (3072, 31), (64, 1)])
def test_outlier_channels(K, n_out):
    rng = np.random.default_rng(3)
    xb = synth.make_x(512, K, rng)
    assert xb.dtype == np.uint16 and xb.shape == (512, K)
    x = synth.bf16_bits_to_f32(xb).astype(np.float64)
    assert np.all(np.isfinite(x))
    sd = x.std(axis=0)
    out = sd > 5.0
    assert out.sum() == n_out
    assert np.all(np.abs(sd[out] / 20.0 - 1.0) < 0.15)    # scaled by 20
    assert np.all(np.abs(sd[~out] - 1.0) < 0.15)          # the rest N(0, 1)


def test_weights_spread():
    W = synth.make_w(2, 256, 512, np.random.default_rng(4))
    assert W.dtype == np.float32 and W.shape == (2, 256, 512)
    assert abs(W.std() / 0.02 - 1.0) < 0.01 and abs(W.mean()) < 1e-3


def test_same_seed_same_tensors():
    a, b, c = synth.dense(32, 256, 64, seed=5), synth.dense(32, 256, 64, seed=5), synth.dense(32, 256, 64, seed=6)
    assert np.array_equal(a.x, b.x) and np.array_equal(a.W, b.W) and np.array_equal(a.D, b.D)
    assert not np.array_equal(a.x, c.x)
    g1 = synth.grouped(300, 8, 256, 64, seed=2, dist="zipf", group_list_type=0)
    g2 = synth.grouped(300, 8, 256, 64, seed=2, dist="zipf", group_list_type=0)
    assert np.array_equal(g1.group_list, g2.group_list) and np.array_equal(g1.x, g2.x)


def test_zipf_counts_of_the_expert_workload():
    counts = synth.zipf_counts(8192, 128, np.random.default_rng(0))
    assert counts.dtype == np.int64 and counts.sum() == 8192
    assert (counts == 0).sum() >= 8                        # the 8 experts at probability 0
    # Zipf(1.1) over the remaining 120 ranks: the top expert holds about 1/H of the tokens
    ranks = np.arange(1, 129, dtype=np.float64)
    share = counts.max() / 8192
    assert 0.5 / np.sum(ranks ** -1.1) < share < 1.5 / np.sum(ranks[:120] ** -1.1)


def test_workload_shapes():
    (c0,) = synth.config(0)
    assert (c0.M, c0.K, c0.N, c0.E) == (16, 1024, 1024, 1)
    c1 = synth.config(1)
    assert [(p.M, p.K, p.N) for p in c1] == [(128, k, n) for k, n in synth.QWEN_PAIRS]
    for p in synth.config(3):
        assert (p.M, p.E, p.group_list_type) == (4096, 4, 1) and p.group_list.sum() == 4096
        assert p.D.shape == (4, p.K) and p.W.shape == (4, p.N, p.K)


def test_channel_factor_closed_form():
    # D = clamp(sqrt(max|x| / max|W|), 1e-2, 1e2) per channel, with the special cases
    xb = synth.to_bf16_bits(np.array([[4.0, 0.0, 0.0, 1e6], [-9.0, 0.0, 3.0, 0.0]], np.float32))
    W = np.array([[1.0, 0.0, 0.0, 1e-6], [-0.25, 0.0, 0.0, 0.0]], np.float32)
    D = synth.make_d(xb, W)
    assert D[0] == np.float32(3.0)                        # sqrt(9 / 1)
    assert D[1] == 1.0                                    # 0 / 0
    assert D[2] == np.float32(1e2)                        # w = 0 < a
    assert D[3] == np.float32(1e2)                        # sqrt(1e12) clamped
