"""Argument checks of the Python binding that run before any device work:
element types, ranks and sizes are refused by name (CPU tensors suffice, the
device check comes last)."""
import pytest
import torch

import w4a4_mxfp4_quantize_b200 as mq


@pytest.fixture(scope="module", autouse=True)
def _lib():
    mq.build()
    mq.lib()


M, K, N, E = 16, 256, 64, 3


def dense_args(**kw):
    qb, sb = mq.weight_bytes(1, N, K)
    a = dict(x=torch.zeros((M, K), dtype=torch.bfloat16), D=torch.ones(K), Wq=torch.zeros(qb, dtype=torch.uint8),
             Ws=torch.zeros(sb, dtype=torch.uint8), N=N)
    a.update(kw)
    return a


def grouped_args(**kw):
    qb, sb = mq.weight_bytes(E, N, K)
    a = dict(x=torch.zeros((M, K), dtype=torch.bfloat16), D=torch.ones((E, K)),
             Wq=torch.zeros(qb, dtype=torch.uint8), Ws=torch.zeros(sb, dtype=torch.uint8),
             group_list=torch.tensor([5, 5, 6], dtype=torch.int64), group_list_type=1, N=N)
    a.update(kw)
    return a


@pytest.mark.parametrize("fn", [mq.dense_mm, mq.unfused_dense_mm, mq.dense_mm_noalloc])
@pytest.mark.parametrize("change,message", [
    (dict(x=torch.zeros((M, K), dtype=torch.float16)), "x must be torch.bfloat16"),
    (dict(x=torch.zeros((M, K), dtype=torch.float32)), "x must be torch.bfloat16"),
    (dict(x=torch.zeros((2, M, K), dtype=torch.bfloat16)), "x must have 2 dimensions"),
    (dict(D=torch.ones(K, dtype=torch.float64)), "D must be torch.float32"),
    (dict(D=torch.ones(K - 1)), "D holds"),
    (dict(Wq=torch.zeros(100, dtype=torch.uint8)), "Wq holds"),
    (dict(Ws=torch.zeros(8, dtype=torch.uint8)), "Ws holds"),
    (dict(Wq=torch.zeros(10 ** 6, dtype=torch.int8)), "Wq must be torch.uint8"),
    (dict(status=torch.zeros(1, dtype=torch.int64)), "status must be torch.int32"),
])
def test_dense_refusals(fn, change, message):
    with pytest.raises(ValueError, match=message):
        fn(**dense_args(**change))


def test_dense_valid_cpu_arguments_reach_the_device_check():
    with pytest.raises(ValueError, match="expected contiguous CUDA tensors"):
        mq.dense_mm(**dense_args())


@pytest.mark.parametrize("change,message", [
    (dict(group_list=torch.tensor([5, 5, 6], dtype=torch.int32)), "group_list must be torch.int64"),
    (dict(D=torch.ones((1, K))), "D holds"),
    (dict(Wq=torch.zeros(mq.weight_bytes(1, N, K)[0], dtype=torch.uint8)), "Wq holds"),
    (dict(x=torch.zeros((M, K), dtype=torch.float32)), "x must be torch.bfloat16"),
])
def test_grouped_refusals(change, message):
    with pytest.raises(ValueError, match=message):
        mq.grouped_mm(**grouped_args(**change))


def test_grouped_plain_refusals():
    a = grouped_args(group_list=torch.tensor([5, 5, 6], dtype=torch.int32))
    a.pop("D")
    with pytest.raises(ValueError, match="group_list must be torch.int64"):
        mq.grouped_mm_plain(**a)


def test_grouped_valid_cpu_arguments_reach_the_device_check():
    with pytest.raises(ValueError, match="expected contiguous CUDA tensors"):
        mq.grouped_mm(**grouped_args())


def test_shape_the_library_refuses_is_left_to_it():
    # N % 16 != 0: weight_bytes is 0, so no size check; the library's own shape
    # refusal (MacaqError -3 on a GPU) is what the caller sees there
    assert mq.weight_bytes(1, 130, K) == (0, 0)
    with pytest.raises(ValueError, match="expected contiguous CUDA tensors"):
        mq.dense_mm_plain(**{k: v for k, v in dense_args(N=130).items() if k != "D"})


def test_prepare_and_calibrate_refusals():
    with pytest.raises(ValueError, match="W must be torch.float32"):
        mq.prepare_weights(torch.zeros((N, K), dtype=torch.float64), torch.ones(K))
    with pytest.raises(ValueError, match="D holds"):
        mq.prepare_weights(torch.zeros((E, N, K)), torch.ones(K))   # one row of D for three experts
    with pytest.raises(ValueError, match="x_cal must be torch.bfloat16"):
        mq.calibrate_d(torch.zeros((8, K)), torch.zeros((N, K)))
    with pytest.raises(ValueError, match="input channels"):
        mq.calibrate_d(torch.zeros((8, K), dtype=torch.bfloat16), torch.zeros((N, 2 * K)))
    with pytest.raises(ValueError, match="v must be torch.float32"):
        mq.mx_encode_blocks(torch.zeros(64, dtype=torch.float64))
    with pytest.raises(ValueError, match="Wq holds"):
        mq.export_weights(torch.zeros(10, dtype=torch.uint8), torch.zeros(10, dtype=torch.uint8), 1, N, K)


def test_weight_list_and_transposed_refusals():
    qb, sb = mq.weight_bytes(1, N, K)
    a = grouped_args()
    wq = [torch.zeros(qb, dtype=torch.uint8) for _ in range(E)]
    wsc = [torch.zeros(sb, dtype=torch.uint8) for _ in range(E)]
    with pytest.raises(ValueError, match="need 3 entries"):
        mq.grouped_mm_list(a["x"], a["D"], wq[:2], wsc[:2], a["group_list"], 1, N)
    with pytest.raises(ValueError, match="Wq holds"):
        mq.grouped_mm_list(a["x"], a["D"], [torch.zeros(10, dtype=torch.uint8)] * E, wsc, a["group_list"], 1, N)
    with pytest.raises(ValueError, match="expected contiguous CUDA tensors"):
        mq.grouped_mm_list(a["x"], a["D"], wq, wsc, a["group_list"], 1, N)
    with pytest.raises(ValueError, match="W_kn must be torch.float32"):
        mq.prepare_weights_transposed(torch.zeros((K, N), dtype=torch.float64), torch.ones(K))



def test_fp8_output_refusals():
    with pytest.raises(ValueError, match="x must be torch.bfloat16"):
        mq.dense_mm_fp8(**dense_args(x=torch.zeros((M, K))), y_scale=1.0)
    with pytest.raises(ValueError, match="Wq holds"):
        mq.dense_mm_fp8(**dense_args(Wq=torch.zeros(100, dtype=torch.uint8)), y_scale=1.0)
    with pytest.raises(ValueError, match="expected contiguous CUDA tensors"):
        mq.dense_mm_fp8(**dense_args(), y_scale=1.0)
    with pytest.raises(ValueError, match="group_list must be torch.int64"):
        mq.grouped_mm_fp8(**grouped_args(group_list=torch.tensor([5, 5, 6], dtype=torch.int32)), y_scale=1.0)
    with pytest.raises(ValueError, match="expected contiguous CUDA tensors"):
        mq.grouped_mm_fp8(**grouped_args(), y_scale=1.0)
