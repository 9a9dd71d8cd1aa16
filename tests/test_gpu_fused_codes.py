"""The activation codes and scales of the fused small-M kernel itself, bit-exact.

The fused kernel (dense M <= 128) quantises its activation tile straight into
shared memory, one 32-element block per prologue thread, so its codes never
reach global memory on the product path.  macaq_fused_probe runs that
kernel with a chosen plan (token tile, K split) and copies each activation
operand tile out of shared memory just before the tensor core reads it.  These
tests compare those tiles with the oracle's codes and E8M0 scales (MACAQ page,
summary; MX rule in "Latency against existing native CANN operators"), for
every plan the kernel can run on the headline workload's shapes, on ragged and
adversarial inputs, and for the plain MXFP4 prologue; the output of each probe
run is checked against the oracle too.  The device status word and the other
launch-level checks (the kernels' bounded wait run out on purpose, calls on a
stream other than the current one) are here as well.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import w4a4_mxfp4_quantize_b200 as mq
from helpers import assert_mx_equal, compare, f32_dev, x_to_dev, y_to_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    mq.build()
    mq.lib()
    torch.cuda.init()


def _plans(M: int, K: int):
    """(token tile, K split) of every plan of the fused kernel."""
    KT = K // 256
    for bt in (16, 32, 64, 128):
        for s in range(1, 9):
            if KT % s == 0:
                yield bt, s


def _probe_all_plans(p: synth.Problem, plain: bool = False, plans=None):
    """Every runnable plan of the fused kernel on problem p: its own codes and
    scales against the oracle's (bit-exact), its output against the oracle's
    (tolerance).  Returns the plans that ran."""
    x = x_to_dev(p.x)
    if plain:
        Wq, Ws = mq.prepare_weights_plain(f32_dev(p.W))
        D = None
        qa, sa = oracle.quantize_act_plain(p.x)
        qw, sw = oracle.quantize_plain(p.W[0])
        ref = oracle.gemm_plain(qa, sa, qw, sw)
    else:
        Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
        D = f32_dev(p.D[0])
        qa, sa = oracle.quantize_act(p.x, p.D[0])
        qw, sw = oracle.quantize_weights(p.W[0], p.D[0])
        ref = oracle.gemm(qa, sa, qw, sw)
    ran = []
    for bt, s in (plans if plans is not None else _plans(p.M, p.K)):
        try:
            y, codes, scales = mq.fused_probe(x, D, Wq, Ws, p.N, bt, s, plain=plain)
        except mq.MacaqError as e:
            assert e.status == -3, e     # a cluster the device cannot hold: refused by name
            continue
        torch.cuda.synchronize()
        label = f"{p.name or (p.M, p.K, p.N)} plan BT={bt} S={s}{' plain' if plain else ''}"
        assert_mx_equal(codes.cpu().numpy(), scales.cpu().numpy(), qa, sa, label)
        compare(y_to_bits(y), ref, label)
        ran.append((bt, s))
    return ran


@pytest.mark.parametrize("cfg", [0, 1])
def test_fused_kernel_codes_every_plan_on_headline_shapes(cfg):
    for p in synth.config(cfg):
        ran = _probe_all_plans(p)
        default = mq.fused_plan(p.M, p.N, p.K)
        assert default in ran, (p.name, default, ran)


@pytest.mark.parametrize("M,K,N", [(1, 256, 16), (5, 512, 48), (17, 1024, 144), (77, 768, 256), (100, 512, 384)])
def test_fused_kernel_codes_ragged_rows(M, K, N):
    p = synth.dense(M, K, N, seed=M + K)
    assert _probe_all_plans(p)


def test_fused_kernel_codes_adversarial():
    # the adversarial blocks of the quantiser test, through the fused kernel's prologue
    rng = np.random.default_rng(2)
    M, K, N = 100, 512, 128
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
    W = rng.normal(0, 0.02, (1, N, K)).astype(np.float32)
    p = synth.Problem(x=xb, W=W, D=D.astype(np.float32)[None, :], M=M, N=N, K=K)
    qa, sa = oracle.quantize_act(xb, p.D[0])
    Wq, Ws = mq.prepare_weights(f32_dev(W), f32_dev(p.D))
    for bt, s in [(16, 1), (16, 2), (32, 1), (64, 2), (128, 1)]:
        _, codes, scales = mq.fused_probe(x_to_dev(xb), f32_dev(p.D[0]), Wq, Ws, N, bt, s)
        torch.cuda.synchronize()
        assert_mx_equal(codes.cpu().numpy(), scales.cpu().numpy(), qa, sa, f"adversarial plan {(bt, s)}")


def test_fused_kernel_codes_plain_prologue():
    p = synth.dense(128, 1024, 256, seed=21)
    assert _probe_all_plans(p, plain=True, plans=[(16, 1), (16, 4), (32, 2), (64, 1), (128, 4)])


def test_fused_probe_without_copy_equals_dense_mm():
    p = synth.dense(128, 2048, 1024, seed=3)
    x, D = x_to_dev(p.x), f32_dev(p.D[0])
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    bt, s = mq.fused_plan(p.M, p.N, p.K)
    y_probe, codes, sc = mq.fused_probe(x, D, Wq, Ws, p.N, bt, s, dump=False)
    y = mq.dense_mm(x, D, Wq, Ws, p.N)
    torch.cuda.synchronize()
    assert codes is None and sc is None
    assert np.array_equal(y_to_bits(y_probe), y_to_bits(y))


# ----------------------------------------------------------------------------
# The grouped path's activation images (quantise-once into the workspace)
# ----------------------------------------------------------------------------

def _grouped_images(ws: np.ndarray, M: int, K: int, E: int):
    """Canonical codes / scales of every tile row of the grouped workspace's
    activation images, and the tile prefix gtp[E+1]: the workspace holds 4096
    reserved bytes, then goff int64[E+1], gtp int32[E+1], gexp int32[E], the
    valid flag and slab count, the slab table int4[ceil(M/32) + E] (each
    region starting on a 256-byte boundary), then the images of
    ceil(M/128) + E row tiles x K/256 K tiles, 17408 bytes each (the dense
    image layout)."""
    a256 = lambda n: (n + 255) // 256 * 256  # noqa: E731
    goff = 4096
    gtp = a256(goff + (E + 1) * 8)
    gexp = a256(gtp + (E + 1) * 4)
    valid = a256(gexp + E * 4)
    slabs = a256(valid + 16)
    act = a256(slabs + ((M + 31) // 32 + E) * 16)
    tiles = (M + 127) // 128 + E
    KT = K // 256
    tp = ws[gtp:gtp + (E + 1) * 4].view(np.int32).copy()
    imgs = ws[act:act + tiles * KT * 17408].reshape(tiles, KT, 17408)
    r = np.arange(128)[:, None]
    c = np.arange(8)[None, :]
    codes = imgs[:, :, :16384].reshape(tiles, KT, 128, 8, 16)
    codes = np.take_along_axis(codes, (c ^ (r & 7))[None, None, :, :, None], axis=3)
    codes = codes.transpose(0, 2, 1, 3, 4).reshape(tiles * 128, K // 2)
    sf_idx = 512 * (c // 4) + 16 * (r % 32) + 4 * (r // 32) + (c % 4)
    scales = imgs[:, :, 16384:][:, :, sf_idx].transpose(0, 2, 1, 3).reshape(tiles * 128, K // 32)
    return codes, scales, tp


@pytest.mark.parametrize("cfg,which", [(3, 0), (3, 1), (4, 0), (4, 1)])
def test_grouped_activation_images_bit_exact(cfg, which):
    # each list entry's rows are quantised with its expert's D into tiles that
    # start at its tile prefix; padding rows are never written, so only the
    # rows of the groups are compared
    p = synth.config(cfg)[which]
    x = x_to_dev(p.x)
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    ws = torch.zeros(mq.workspace_bytes(p.M, p.N, p.K, p.E), dtype=torch.uint8, device="cuda")
    gl = torch.from_numpy(p.group_list.astype(np.int64)).cuda()
    mq.grouped_mm(x, f32_dev(p.D), Wq, Ws, gl, p.group_list_type, p.N, ws=ws)
    torch.cuda.synchronize()
    codes, scales, tp = _grouped_images(ws.cpu().numpy(), p.M, p.K, p.E)
    off = np.concatenate([[0], np.cumsum(p.counts)])
    checked = 0
    for g in range(p.E):
        a, b = int(off[g]), int(off[g + 1])
        if b == a:
            continue
        qa, sa = oracle.quantize_act(p.x[a:b], p.D[g])
        rows = slice(int(tp[g]) * 128, int(tp[g]) * 128 + (b - a))
        assert_mx_equal(codes[rows], scales[rows], qa, sa, f"{p.name} group {g}")
        checked += b - a
    assert checked == p.M


def test_grouped_type2_activation_images_use_the_named_expert():
    p = synth.grouped(300, 6, 512, 128, seed=43, dist="zipf", group_list_type=1)
    idx = np.array([5, 0, 3, 3, 1, 2], np.int64)
    gl2 = np.ascontiguousarray(np.stack([idx, p.counts]).T.astype(np.int64))
    x = x_to_dev(p.x)
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    ws = torch.zeros(mq.workspace_bytes(p.M, p.N, p.K, p.E), dtype=torch.uint8, device="cuda")
    mq.grouped_mm(x, f32_dev(p.D), Wq, Ws, torch.from_numpy(gl2).cuda(), 2, p.N, ws=ws)
    torch.cuda.synchronize()
    codes, scales, tp = _grouped_images(ws.cpu().numpy(), p.M, p.K, p.E)
    off = np.concatenate([[0], np.cumsum(p.counts)])
    for j in range(p.E):
        a, b = int(off[j]), int(off[j + 1])
        if b == a:
            continue
        qa, sa = oracle.quantize_act(p.x[a:b], p.D[idx[j]])
        rows = slice(int(tp[j]) * 128, int(tp[j]) * 128 + (b - a))
        assert_mx_equal(codes[rows], scales[rows], qa, sa, f"type-2 entry {j}")


# ----------------------------------------------------------------------------
# Launch-level checks
# ----------------------------------------------------------------------------

def test_bounded_wait_expires_reports_timeout_and_the_context_stays_usable():
    # a wait on a barrier that nothing arrives on ends by its own limit (1 ms)
    # and reports MACAQ_ERR_DEVICE_TIMEOUT; nothing faults, traps or hangs
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    st = mq.run_wait_expiry(1_000_000)
    e1.record()
    torch.cuda.synchronize()
    assert int(st[0].item()) == -9
    assert e0.elapsed_time(e1) >= 0.9          # ms: the wait lasted its limit
    p = synth.dense(16, 512, 128, seed=5)
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    y = mq.dense_mm(x_to_dev(p.x), f32_dev(p.D[0]), Wq, Ws, p.N)
    torch.cuda.synchronize()
    qa, sa = oracle.quantize_act(p.x, p.D[0])
    qw, sw = oracle.quantize_weights(p.W[0], p.D[0])
    compare(y_to_bits(y), oracle.gemm(qa, sa, qw, sw), "after an expired wait")


@pytest.mark.parametrize("M", [64, 300])
def test_calls_on_a_stream_that_is_not_current(M):
    # outputs and workspace are allocated on the call's stream, not torch's
    # current one, while that current stream is kept busy
    p = synth.dense(M, 512, 256, seed=M + 1)
    x, D = x_to_dev(p.x), f32_dev(p.D[0])
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    mq._ws.clear()
    torch.cuda._sleep(20_000_000)            # the current stream stays busy for a while
    y = mq.dense_mm(x, D, Wq, Ws, p.N, stream=s)
    q, sc = mq.quantize_activations(x, D, stream=s)
    s.synchronize()
    torch.cuda.synchronize()
    qa, sa = oracle.quantize_act(p.x, p.D[0])
    qw, sw = oracle.quantize_weights(p.W[0], p.D[0])
    assert_mx_equal(q.cpu().numpy(), sc.cpu().numpy(), qa, sa, f"side stream M={M}")
    compare(y_to_bits(y), oracle.gemm(qa, sa, qw, sw), f"side stream M={M}")
