"""The rest of npu_grouped_matmul's grouped surface on the GPU, through the C ABI.

* Weight list (parameter weight as a list of tensors; the single-x /
  several-weight / single-y case of the page's constraints): one separately
  prepared weight pair per expert, passed as device tables of addresses.  The
  list call runs the same kernels as the stacked call, so the outputs must be
  identical; a small case is also compared with the oracle's list form.
* Transposed weights (the page's constraints allow the weight transposed):
  preparation from [E, K, N] gives the same tile images as from [E, N, K].
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
    mq.lib()
    torch.cuda.init()


def _per_expert_weights(p):
    """Each expert prepared on its own (separate allocations, in reverse order so
    that they are not laid out like the stacked images)."""
    Wq_l, Ws_l = [None] * p.E, [None] * p.E
    for e in reversed(range(p.E)):
        Wq_l[e], Ws_l[e] = mq.prepare_weights(f32_dev(p.W[e]), f32_dev(p.D[e]))
    return Wq_l, Ws_l


@pytest.mark.parametrize("T,E,K,N,gtype", [(200, 5, 512, 144, 1), (300, 16, 256, 256, 0), (96, 4, 1024, 128, 2)])
def test_weight_list_equals_stacked_and_oracle(T, E, K, N, gtype):
    p = synth.grouped(T, E, K, N, seed=T + E + 7, dist="zipf", group_list_type=1)
    if gtype == 2:
        idx = np.array([3, 1, 1, 0], np.int64)[:E]
        gl = np.ascontiguousarray(np.stack([idx, p.counts]).T.astype(np.int64))
    elif gtype == 0:
        gl = np.cumsum(p.counts).astype(np.int64)
    else:
        gl = p.counts.astype(np.int64)
    x, D = x_to_dev(p.x), f32_dev(p.D)
    glt = torch.from_numpy(gl).cuda()
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    Wq_l, Ws_l = _per_expert_weights(p)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y_s = mq.grouped_mm(x, D, Wq, Ws, glt, gtype, N)
    y_l = mq.grouped_mm_list(x, D, Wq_l, Ws_l, glt, gtype, N, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert np.array_equal(y_to_bits(y_l), y_to_bits(y_s))
    st, want = oracle.grouped_mm_list(p.x, p.D, [p.W[e] for e in range(E)], gl, gtype)
    assert st == oracle.OK
    compare(y_to_bits(y_l), want, f"weight list T={T} E={E} type {gtype}")


def test_weight_list_moe_shape_with_bias_and_activation():
    # the E = 128 Zipf workload's first projection, with a per-expert bias and GELU_TANH
    p = synth.config(4)[0]
    x, D = x_to_dev(p.x), f32_dev(p.D)
    glt = torch.from_numpy(p.group_list.astype(np.int64)).cuda()
    bias = f32_dev(np.random.default_rng(9).standard_normal((p.E, p.N)).astype(np.float32) * 0.5)
    Wq, Ws = mq.prepare_weights(f32_dev(p.W), f32_dev(p.D))
    Wq_l, Ws_l = _per_expert_weights(p)
    y_s = mq.grouped_mm(x, D, Wq, Ws, glt, p.group_list_type, p.N, bias=bias, act_type=mq.ACT_GELU_TANH)
    y_l = mq.grouped_mm_list(x, D, Wq_l, Ws_l, glt, p.group_list_type, p.N, bias=bias,
                             act_type=mq.ACT_GELU_TANH)
    torch.cuda.synchronize()
    assert np.array_equal(y_to_bits(y_l), y_to_bits(y_s))


def test_weight_list_entry_overlapping_y_is_refused_on_the_device():
    # The tables are read on the device only.  An entry that points into y is
    # refused there (status MACAQ_ERR_ALIAS, y left as it was).  The entry is a
    # real, aligned device buffer (y itself), so nothing here could read
    # unmapped memory whatever the check did.
    p = synth.grouped(64, 3, 256, 128, seed=5, dist="uniform", group_list_type=1)
    x, D = x_to_dev(p.x), f32_dev(p.D)
    glt = torch.from_numpy(p.counts.astype(np.int64)).cuda()
    Wq_l, Ws_l = _per_expert_weights(p)
    need = mq.weight_bytes(1, p.N, p.K)[0]
    y = torch.full((need // (2 * p.N) + 64, p.N), 7.0, dtype=torch.bfloat16, device="cuda")[:p.M]
    fake = y.view(torch.uint8).reshape(-1)  # y's own bytes posing as expert 1's code images
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    # two separate tables: each must start 16-byte aligned
    wq_table = torch.tensor([Wq_l[0].data_ptr(), fake.data_ptr(), Wq_l[2].data_ptr()], dtype=torch.int64).cuda()
    ws_table = torch.tensor([Ws_l[0].data_ptr(), Ws_l[1].data_ptr(), Ws_l[2].data_ptr()], dtype=torch.int64).cuda()
    ws = torch.zeros(mq.workspace_bytes(p.M, p.N, p.K, p.E), dtype=torch.uint8, device="cuda")
    import ctypes
    P = ctypes.c_void_p
    rc = mq.lib().macaq_grouped_mm_list(P(x.data_ptr()), P(D.data_ptr()), P(wq_table.data_ptr()),
                                        P(ws_table.data_ptr()), P(glt.data_ptr()), 1, p.E, None, 0,
                                        P(y.data_ptr()), p.M, p.N, p.K, P(ws.data_ptr()), ws.numel(),
                                        P(status.data_ptr()), P(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert rc == 0
    assert int(status.item()) == -5
    assert bool(torch.all(y == 7.0))


@pytest.mark.parametrize("E,N,K", [(1, 1024, 1024), (3, 144, 512), (2, 48, 256)])
def test_transposed_weight_preparation_gives_the_same_images(E, N, K):
    rng = np.random.default_rng(E * N + K)
    W = rng.normal(0, 0.02, (E, N, K)).astype(np.float32)
    D = (np.exp(rng.standard_normal((E, K))) * np.where(rng.random((E, K)) < 0.2, -1, 1)).astype(np.float32)
    Wq, Ws = mq.prepare_weights(f32_dev(W), f32_dev(D))
    Wq_t, Ws_t = mq.prepare_weights_transposed(f32_dev(np.ascontiguousarray(W.transpose(0, 2, 1))), f32_dev(D))
    torch.cuda.synchronize()
    assert torch.equal(Wq, Wq_t) and torch.equal(Ws, Ws_t)
    q, s = mq.export_weights(Wq_t, Ws_t, E, N, K)
    torch.cuda.synchronize()
    for e in range(E):
        qo, so = oracle.quantize_weights(W[e], D[e])
        assert np.array_equal(q.cpu().numpy()[e], qo) and np.array_equal(s.cpu().numpy()[e], so), e
