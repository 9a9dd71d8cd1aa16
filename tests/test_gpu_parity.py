"""GPU parity of the CUDA path against the CPU oracle, through the C ABI.

Bit-exact: activation codes and E8M0 scales, prepared weight codes and
scales, and the MX conversion itself.  BF16 outputs: the tolerance described
in tests/helpers.py.  Every input is seeded and synthetic (synth).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import w4a4_mxfp4_quantize_b200 as mq
from helpers import assert_mx_equal, compare, dequant_matmul_bf16, f32_dev, x_to_dev, y_to_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    mq.build()
    mq.lib()
    torch.cuda.init()


# ----------------------------------------------------------------------------
# MX conversion (E8M0 + E2M1 with the hardware cvt) -- bit exact
# ----------------------------------------------------------------------------

def _gpu_mx(blocks: np.ndarray):
    q, s = mq.mx_encode_blocks(f32_dev(blocks.ravel()))
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().numpy()


def test_mx_encode_all_bf16_values_at_many_scales():
    bits = np.arange(65536, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    f = f[np.isfinite(f)]
    rng = np.random.default_rng(0)
    f = f[rng.permutation(f.size)]
    f = f[: f.size // 32 * 32]
    q, s = _gpu_mx(f)
    qo, so = oracle.mx_quantize_blocks(f)
    assert np.array_equal(s, so)
    assert np.array_equal(q, qo)


def test_mx_encode_tie_points_and_saturation_edges():
    rows = []
    for c in [0, 1, 2, 3, 60, 120, 127, 130, 200, 250, 252]:
        unit = np.ldexp(1.0, c - 127)
        vals = [6.0, -6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5,
                -5.0, 0.2499, 0.7501, 5.0001, 4.9999, 7.99, -7.99, 0.0, -0.0, 1e-40, -1e-40, 2.9999, 3.0001,
                1.2499, 1.7501, 0.5, 6.0]
        blk = np.array([v * unit for v in vals], np.float64).astype(np.float32)
        rows.append(blk)
    blocks = np.stack(rows)
    q, s = _gpu_mx(blocks)
    qo, so = oracle.mx_quantize_blocks(blocks)
    assert np.array_equal(s, so)
    assert np.array_equal(q, qo)


def test_mx_encode_random_wide_range_and_zero_blocks():
    rng = np.random.default_rng(1)
    v = (rng.standard_normal((4096, 32)) * np.exp2(rng.integers(-140, 120, (4096, 1)))).astype(np.float32)
    v[::97] = 0.0
    v[1::97] = -0.0
    v[2::97, :31] = 0.0
    q, s = _gpu_mx(v)
    qo, so = oracle.mx_quantize_blocks(v)
    assert np.array_equal(s, so)
    assert np.array_equal(q, qo)


# ----------------------------------------------------------------------------
# Activation prologue -- bit exact on codes and scales
# ----------------------------------------------------------------------------

def _gpu_act(x_bits, D):
    q, s = mq.quantize_activations(x_to_dev(x_bits), f32_dev(D))
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().numpy()


@pytest.mark.parametrize("cfg", [0, 1, 2])
def test_activation_codes_bit_exact_on_dense_configs(cfg):
    for p in synth.config(cfg):
        q, s = _gpu_act(p.x, p.D[0])
        qo, so = oracle.quantize_act(p.x, p.D[0])
        assert_mx_equal(q, s, qo, so, p.name)


def test_activation_codes_bit_exact_adversarial():
    rng = np.random.default_rng(2)
    M, K = 300, 512
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[0] = 1.0                        # all-equal blocks
    x[1] = 0.0                        # zero rows
    x[2] = -0.0
    x[3, ::2] = 1e-38                 # tiny values
    x[4] *= 1e30                      # huge values
    x[5] = np.where(np.arange(K) % 2, -1.0, 1.0)
    x[6:40] *= np.exp2(rng.integers(-40, 40, (34, 1)))
    xb = synth.to_bf16_bits(x)
    xb[7] = rng.integers(0, 65536, K, dtype=np.uint32).astype(np.uint16) & 0x7F7F  # random finite patterns
    D = np.exp(rng.standard_normal(K) * 2).astype(np.float32) * np.where(rng.random(K) < 0.3, -1, 1)
    D = D.astype(np.float32)
    q, s = _gpu_act(xb, D)
    qo, so = oracle.quantize_act(xb, D)
    assert_mx_equal(q, s, qo, so, "adversarial")


# ----------------------------------------------------------------------------
# Offline weight preparation -- bit exact
# ----------------------------------------------------------------------------

def _gpu_weights(W, D):
    E, N, K = W.shape
    Wq, Ws = mq.prepare_weights(f32_dev(W), f32_dev(D))
    q, s = mq.export_weights(Wq, Ws, E, N, K)
    torch.cuda.synchronize()
    return Wq, Ws, q.cpu().numpy(), s.cpu().numpy()


@pytest.mark.parametrize("shape", [(1, 1024, 1024), (1, 48, 256), (3, 144, 512), (2, 2048, 768)])
def test_weight_prep_bit_exact(shape):
    E, N, K = shape
    rng = np.random.default_rng(3)
    W = rng.normal(0, 0.02, shape).astype(np.float32)
    W[0, 0] = 0.0
    D = (np.exp(rng.standard_normal((E, K))) * np.where(rng.random((E, K)) < 0.2, -1, 1)).astype(np.float32)
    _, _, q, s = _gpu_weights(W, D)
    qo, so = oracle.quantize_weights(W, D)
    assert np.array_equal(s, so)
    assert np.array_equal(q, qo)


def test_prepare_rejects_bad_d():
    W = torch.zeros((1, 16, 256), device="cuda")
    D = torch.ones((1, 256), device="cuda")
    D[0, 7] = 0.0
    with pytest.raises(mq.MacaqError) as e:
        mq.prepare_weights(W, D)
    assert e.value.status == -12


# ----------------------------------------------------------------------------
# Dense fused linear -- tolerance on BF16 output
# ----------------------------------------------------------------------------

def _run_dense(p: synth.Problem, fn=None):
    fn = fn or mq.dense_mm
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    y = fn(x_to_dev(p.x), f32_dev(p.D[0]), Wq, Ws, p.N)
    torch.cuda.synchronize()
    return y_to_bits(y)


def _oracle_dense_full(p):
    qa, sa = oracle.quantize_act(p.x, p.D[0])
    qw, sw = oracle.quantize_weights(p.W[0], p.D[0])
    return oracle.gemm(qa, sa, qw, sw)


@pytest.mark.parametrize("M,K,N", [(1, 256, 16), (16, 256, 128), (5, 512, 48), (17, 1024, 144), (64, 768, 256),
                                   (100, 512, 384), (128, 256, 128), (129, 512, 256), (300, 1024, 160)])
def test_dense_small_shapes_exact_oracle(M, K, N):
    p = synth.dense(M, K, N, seed=M + K + N)
    compare(_run_dense(p), _oracle_dense_full(p), f"dense {M}x{K}x{N}")


@pytest.mark.parametrize("cfg", [0, 1])
def test_dense_configs_full_oracle(cfg):
    for p in synth.config(cfg):
        compare(_run_dense(p), _oracle_dense_full(p), p.name)


def _check_large(p: synth.Problem, y_bits: np.ndarray, n_samples: int = 3000):
    qa, sa = oracle.quantize_act(p.x, p.D[0])
    qw, sw = oracle.quantize_weights(p.W[0], p.D[0])
    rng = np.random.default_rng(7)
    rows = rng.integers(0, p.M, n_samples)
    cols = rng.integers(0, p.N, n_samples)
    exact = oracle.gemm_at(qa, sa, qw, sw, rows, cols)
    compare(y_bits[rows, cols], exact, p.name + " sampled exact")
    compare(y_bits, dequant_matmul_bf16(qa, sa, qw, sw), p.name + " full f64")


@pytest.mark.parametrize("i", [0, 1, 2, 3, 4])
def test_dense_prefill_config(i):
    p = synth.config(2)[i]
    _check_large(p, _run_dense(p))


def test_unfused_ablation_matches_oracle():
    for p in [synth.dense(16, 1024, 1024, 0), synth.dense(200, 512, 384, 1), synth.config(2)[1]]:
        y = _run_dense(p, mq.unfused_dense_mm)
        if p.M <= 256:
            compare(y, _oracle_dense_full(p), p.name + " unfused")
        else:
            _check_large(p, y)


def test_binding_rejects_wrong_output_tensor():
    p = synth.dense(16, 256, 64, 0)
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    x, D = x_to_dev(p.x), f32_dev(p.D[0])
    with pytest.raises(ValueError):
        mq.dense_mm(x, D, Wq, Ws, 64, out=torch.empty((16, 32), dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(ValueError):
        mq.dense_mm(x, D, Wq, Ws, 64, out=torch.empty((16, 64), dtype=torch.float32, device="cuda"))


def test_dense_zero_rows_is_noop():
    p = synth.dense(16, 256, 64, 0)
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    y = mq.dense_mm(x, f32_dev(p.D[0]), Wq, Ws, 64)
    assert y.shape == (0, 64)


def test_dense_on_a_side_stream_and_repeatable():
    p = synth.dense(96, 1024, 512, 5)
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    x, D = x_to_dev(p.x), f32_dev(p.D[0])
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        ys = [mq.dense_mm(x, D, Wq, Ws, p.N, stream=s) for _ in range(3)]
    s.synchronize()
    a = [y_to_bits(y) for y in ys]
    assert np.array_equal(a[0], a[1]) and np.array_equal(a[0], a[2])   # deterministic
    compare(a[0], _oracle_dense_full(p), "side stream")


def test_signed_d():
    p = synth.dense(40, 512, 128, 9)
    p.D = (p.D * np.where(np.arange(512) % 3 == 0, -1, 1)).astype(np.float32)
    compare(_run_dense(p), _oracle_dense_full(p), "signed D")


# ----------------------------------------------------------------------------
# Grouped
# ----------------------------------------------------------------------------

def _run_grouped(p: synth.Problem, gl=None, gtype=None, status=None):
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    gl = p.group_list if gl is None else gl
    gtype = p.group_list_type if gtype is None else gtype
    y = mq.grouped_mm(x_to_dev(p.x), f32_dev(p.D), Wq, Ws, torch.from_numpy(np.asarray(gl, np.int64)).cuda(),
                      gtype, p.N, status=status)
    torch.cuda.synchronize()
    return y


def _oracle_grouped(p):
    st, y = oracle.grouped_mm(p.x, p.D, p.W, p.group_list, p.group_list_type)
    assert st == 0
    return y


@pytest.mark.parametrize("T,E,K,N,dist,gtype", [(96, 4, 256, 128, "uniform", 1), (200, 5, 512, 144, "uniform", 0),
                                                 (300, 16, 256, 64, "zipf", 0), (64, 3, 1024, 256, "uniform", 1)])
def test_grouped_small_exact_oracle(T, E, K, N, dist, gtype):
    p = synth.grouped(T, E, K, N, seed=T + E, dist=dist, group_list_type=gtype)
    compare(y_to_bits(_run_grouped(p)), _oracle_grouped(p), p.name)


def test_grouped_empty_groups_first_last_consecutive():
    p = synth.grouped(120, 6, 256, 64, seed=11, dist="uniform", group_list_type=1)
    for counts in ([0, 0, 60, 0, 60, 0], [120, 0, 0, 0, 0, 0], [0, 0, 0, 0, 0, 120], [1, 0, 0, 118, 0, 1]):
        p.group_list = np.array(counts, np.int64)
        p.group_list_type = 1
        compare(y_to_bits(_run_grouped(p)), _oracle_grouped(p), f"grouped {counts}")


def test_grouped_cumsum_equals_counts():
    p = synth.grouped(150, 4, 512, 128, seed=12, dist="uniform", group_list_type=1)
    y1 = y_to_bits(_run_grouped(p))
    y0 = y_to_bits(_run_grouped(p, np.cumsum(p.group_list), 0))
    assert np.array_equal(y0, y1)


def test_grouped_replicated_banks_equal_dense():
    p = synth.grouped(256, 4, 1024, 256, seed=13, dist="uniform", group_list_type=1)
    p.W = np.repeat(p.W[:1], 4, axis=0)
    p.D = np.repeat(p.D[:1], 4, axis=0)
    yg = y_to_bits(_run_grouped(p))
    pd = synth.Problem(x=p.x, W=p.W[:1], D=p.D[:1], M=p.M, N=p.N, K=p.K)
    yd = _run_dense(pd)
    compare(yg, yd, "replicated banks vs dense")
    compare(yg, _oracle_dense_full(pd), "replicated banks vs oracle")


@pytest.mark.parametrize("gl,gtype", [([10, 5, 30], 0), ([10, -1, 21], 1), ([10, 10, 11], 1), ([10, 20, 29], 0),
                                      ([-3, 20, 30], 0), ([[0, 10], [3, 10], [1, 10]], 2),
                                      ([[0, 10], [2, 10], [1, 9]], 2), ([[0, 10], [-1, 10], [1, 10]], 2),
                                      ([[0, 40], [2, -10], [1, 0]], 2)])
def test_grouped_invalid_group_list_sets_status_and_leaves_y(gl, gtype):
    p = synth.grouped(30, 3, 256, 64, seed=14, dist="uniform", group_list_type=1)
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    y = torch.full((30, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    mq.grouped_mm(x_to_dev(p.x), f32_dev(p.D), Wq, Ws, torch.tensor(gl, dtype=torch.int64, device="cuda"), gtype,
                  64, out=y, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == -10
    assert bool(torch.all(y == 7.0))


@pytest.mark.parametrize("T,E,K,N", [(200, 5, 512, 144), (300, 16, 256, 256)])
def test_grouped_type2_named_experts(T, E, K, N):
    # type 2: [E, 2] rows of (group index, group size); the row ranges follow the
    # list order and use the named expert, which may repeat or never appear
    p = synth.grouped(T, E, K, N, seed=T + E + 1, dist="zipf", group_list_type=1)
    rng = np.random.default_rng(E)
    idx = rng.integers(0, E, E)
    idx[0] = idx[-1]                      # one expert named twice
    gl2 = np.ascontiguousarray(np.stack([idx, p.counts]).T.astype(np.int64))
    st, want = oracle.grouped_mm(p.x, p.D, p.W, gl2, 2)
    assert st == 0
    got = y_to_bits(_run_grouped(p, gl=gl2, gtype=2))
    compare(got, want, p.name + " type 2")


@pytest.mark.parametrize("which", [0, 1])
def test_grouped_config3(which):
    p = synth.config(3)[which]
    y = y_to_bits(_run_grouped(p))
    _check_grouped_sampled(p, y)


@pytest.mark.parametrize("which", [0, 1])
def test_grouped_config4(which):
    p = synth.config(4)[which]
    assert (p.counts == 0).sum() > 0          # some groups empty
    y = y_to_bits(_run_grouped(p))
    _check_grouped_sampled(p, y)


def _check_grouped_sampled(p, y, per_group=24):
    off = np.concatenate([[0], np.cumsum(p.counts)])
    rng = np.random.default_rng(5)
    got, want = [], []
    for g in range(p.E):
        if p.counts[g] == 0:
            continue
        rows = rng.integers(off[g], off[g + 1], per_group)
        cols = rng.integers(0, p.N, per_group)
        qa, sa = oracle.quantize_act(p.x[rows], p.D[g])
        qw, sw = oracle.quantize_weights(p.W[g][np.unique(cols)], p.D[g])
        idx = np.searchsorted(np.unique(cols), cols)
        want.append(oracle.gemm_at(qa, sa, qw, sw, np.arange(per_group), idx))
        got.append(y[rows, cols])
    compare(np.concatenate(got), np.concatenate(want), p.name + " sampled exact")


# ----------------------------------------------------------------------------
# Launch-level properties
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("M,K,N", [(16, 1024, 1024), (128, 3072, 1024), (512, 1024, 384)])
def test_graph_capture_replays_bit_identical(M, K, N):
    # calls do no host synchronisation: capture once, replay many times
    p = synth.dense(M, K, N, seed=21)
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    x, D = x_to_dev(p.x), f32_dev(p.D[0])
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    nb = mq.workspace_bytes(M, N, K)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda") if nb else None
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        mq.dense_mm(x, D, Wq, Ws, N, out=y, ws=ws)
    s.synchronize()
    first = y_to_bits(y)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        mq.dense_mm(x, D, Wq, Ws, N, out=y, ws=ws)
    for _ in range(100):
        y.fill_(0)
        g.replay()
    torch.cuda.synchronize()
    assert np.array_equal(y_to_bits(y), first)
    compare(first, _oracle_dense_full(p), "graph")


@pytest.mark.parametrize("M", [129, 255, 256, 1000])
def test_dense_quantise_once_path_ragged(M):
    p = synth.dense(M, 512, 272, seed=M)
    compare(_run_dense(p), _oracle_dense_full(p), f"two-kernel M={M}")


def _decode_activation_images(ws: np.ndarray, M: int, K: int):
    """Canonical codes [M, K/2] and scales [M, K/32] read back from the dense
    quantise-once workspace: 4096 reserved bytes, then one image per (128-row
    tile, 256-K tile) of 17408 bytes -- 16384 code bytes (row r at 128 r, its
    16-byte chunk for block c at (c ^ (r mod 8)) * 16) then 1024 scale bytes
    (block c of row r at 512 (c // 4) + 16 (r mod 32) + 4 (r // 32) + c mod 4)."""
    KT = K // 256
    tiles = (M + 127) // 128
    imgs = ws[4096:4096 + tiles * KT * 17408].reshape(tiles, KT, 17408)
    r = np.arange(128)[:, None]
    c = np.arange(8)[None, :]
    phys = (c ^ (r & 7))                                     # [128, 8] physical chunk of logical block c
    codes = imgs[:, :, :16384].reshape(tiles, KT, 128, 8, 16)
    codes = np.take_along_axis(codes, phys[None, None, :, :, None], axis=3)     # logical block order
    codes = codes.transpose(0, 2, 1, 3, 4).reshape(tiles * 128, K // 2)[:M]
    sf_idx = 512 * (c // 4) + 16 * (r % 32) + 4 * (r // 32) + (c % 4)           # [128, 8]
    scales = imgs[:, :, 16384:][:, :, sf_idx]                                  # [tiles, KT, 128, 8]
    scales = scales.transpose(0, 2, 1, 3).reshape(tiles * 128, K // 32)[:M]
    return codes, scales


@pytest.mark.parametrize("M,K,plain", [(300, 768, False), (4096, 1024, False), (1000, 512, True)])
def test_quantise_once_activation_images_bit_exact(M, K, plain):
    # the quantiser of the two-kernel path writes each row's codes and scales
    # into the GEMM's tile images; rows past M are never written (their output
    # rows are never stored), so only rows < M are compared
    p = synth.dense(M, K, 256, seed=7 + M)
    x = x_to_dev(p.x)
    ws = torch.zeros(mq.workspace_bytes(M, 256, K), dtype=torch.uint8, device="cuda")
    if plain:
        Wq, Ws = mq.prepare_weights_plain(f32_dev(p.W))
        mq.dense_mm_plain(x, Wq, Ws, 256, ws=ws)
        qa, sa = oracle.quantize_act_plain(p.x)
    else:
        D = f32_dev(p.D[0])
        Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
        mq.dense_mm(x, D, Wq, Ws, 256, ws=ws)
        qa, sa = oracle.quantize_act(p.x, p.D[0])
    torch.cuda.synchronize()
    codes, scales = _decode_activation_images(ws.cpu().numpy(), M, K)
    assert_mx_equal(codes, scales, qa, sa, f"images M={M} K={K}")


def test_max_rows_sampled():
    # the MACAQ page's maximum-row checks go to M = 65,536; one more row for a partial tile
    for M in (65536, 65537):
        rng = np.random.default_rng(M)
        K, N = 256, 128
        x = synth.to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
        W = rng.normal(0, 0.02, (1, N, K)).astype(np.float32)
        D = synth.make_d(x, W[0])[None, :]
        p = synth.Problem(x=x, W=W, D=D, M=M, N=N, K=K)
        _check_large(p, _run_dense(p), n_samples=2000)


@pytest.mark.parametrize("M", [64, 128, 512])
def test_dependent_calls_on_one_stream(M):
    # Calls overlap their set-up with the previous kernel (programmatic
    # dependent launch); inputs written by the previous call and outputs read
    # by it must still be ordered.  Chain: a -> y1 -> y2, then a write-after-read
    # (the third call overwrites `a`, which the first call read).
    K1, N1, N2 = 1024, 1024, 256  # square first layer: its output may overwrite its input buffer
    p1 = synth.dense(M, K1, N1, seed=31)
    p2 = synth.dense(M, N1, N2, seed=32)
    Wq1, Ws1 = mq.prepare_weights(f32_dev(p1.W), f32_dev(p1.D))
    Wq2, Ws2 = mq.prepare_weights(f32_dev(p2.W), f32_dev(p2.D))
    D1, D2 = f32_dev(p1.D[0]), f32_dev(p2.D[0])
    a = x_to_dev(p1.x)
    a_copy = a.clone()
    c = x_to_dev(synth.to_bf16_bits(np.random.default_rng(33).standard_normal((M, K1)).astype(np.float32)))
    torch.cuda.synchronize()
    # reference: one call at a time
    r1 = mq.dense_mm(a_copy, D1, Wq1, Ws1, N1); torch.cuda.synchronize()
    r2 = mq.dense_mm(r1, D2, Wq2, Ws2, N2); torch.cuda.synchronize()
    r3 = mq.dense_mm(c, D1, Wq1, Ws1, N1); torch.cuda.synchronize()
    # back to back on one stream, no host synchronisation
    y1 = torch.empty((M, N1), dtype=torch.bfloat16, device="cuda")
    y2 = torch.empty((M, N2), dtype=torch.bfloat16, device="cuda")
    for _ in range(3):
        mq.dense_mm(a, D1, Wq1, Ws1, N1, out=y1)
        mq.dense_mm(y1, D2, Wq2, Ws2, N2, out=y2)
        mq.dense_mm(c, D1, Wq1, Ws1, N1, out=a)    # overwrites the first call's input
        mq.dense_mm(a_copy, D1, Wq1, Ws1, N1, out=y1)  # restore the chain for the next iteration
        a.copy_(a_copy)
    torch.cuda.synchronize()
    assert np.array_equal(y_to_bits(y2), y_to_bits(r2))
    mq.dense_mm(a, D1, Wq1, Ws1, N1, out=y1)
    mq.dense_mm(c, D1, Wq1, Ws1, N1, out=a)
    torch.cuda.synchronize()
    assert np.array_equal(y_to_bits(y1), y_to_bits(r1))
    assert np.array_equal(y_to_bits(a), y_to_bits(r3))


@pytest.mark.parametrize("kind", ["dense", "grouped"])
def test_padding_rows_never_reach_the_output(kind):
    # The quantiser writes only real rows of the activation images; padding rows
    # keep whatever the workspace held.  Fill it with 0xFF (E8M0 255 = NaN scales,
    # E2M1 -6 codes) first: every output must stay finite and match the oracle.
    if kind == "dense":
        p = synth.dense(300, 512, 144, seed=41)       # ragged last row tile (44 rows)
        need = mq.workspace_bytes(p.M, p.N, p.K)
    else:
        p = synth.grouped(300, 6, 512, 144, seed=42, dist="zipf")
        need = mq.workspace_bytes(p.M, p.N, p.K, p.E)
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device="cuda")
    x = x_to_dev(p.x)
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    if kind == "dense":
        y = mq.dense_mm(x, f32_dev(p.D[0]), Wq, Ws, p.N, ws=ws)
        qa, sa = oracle.quantize_act(p.x, p.D[0])
        qw, sw = oracle.quantize_weights(p.W[0], p.D[0])
        ref = oracle.gemm(qa, sa, qw, sw)
    else:
        gl = torch.from_numpy(p.group_list).cuda()
        y = mq.grouped_mm(x, f32_dev(p.D), Wq, Ws, gl, p.group_list_type, p.N, ws=ws)
        st, ref = oracle.grouped_mm(p.x, p.D, p.W, p.group_list, p.group_list_type)
        assert st == oracle.OK
    torch.cuda.synchronize()
    assert bool(torch.isfinite(y.float()).all())
    compare(y_to_bits(y), ref, f"{kind} with a poisoned workspace")
