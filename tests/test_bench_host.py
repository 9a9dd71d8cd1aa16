"""Host-side pieces of bench.py that need no GPU: the ALU bound of the activation
prologue and the CPU oracle figures (all cores, one thread, decoded GEMM)."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle  # noqa: E402
import synth  # noqa: E402


def test_alu_bound_is_lane_operations_over_issue_rate():
    # 4096 x 1024 elements x ~17 lane operations / (148 SMs x 128 lanes x 1965 MHz)
    t = bench.alu_bound_us(4096, 1024, 148)
    assert abs(t - 4096 * 1024 * bench.QUANT_LANE_OPS_PER_ELEMENT / (148 * 128 * 1965.0)) < 1e-12
    assert 1.8 < t < 2.0
    assert abs(bench.alu_bound_us(8192, 1024, 148) - 2 * t) < 1e-12
    assert abs(bench.alu_bound_us(4096, 1024, 74) - 2 * t) < 1e-12
    assert abs(bench.QUANT_LANE_OPS_PER_ELEMENT - 16.96875) < 1e-12


def test_cpu_oracle_detail_reports_one_thread_and_decoded_gemm_and_restores_threads():
    oracle.build()
    probs = [synth.dense(8, 256, 64, seed=s) for s in (1, 2)]
    cores = oracle.num_threads()
    v, el, threads, sample, prepared = bench.cpu_oracle_sample(probs, budget_s=0.2, rows=2)
    assert v > 0 and threads == cores and "2 of 8 rows" in sample
    d = bench.cpu_oracle_detail(probs, prepared, cores, budget_s=0.2)
    assert d["single_thread"]["cores"] == 1 and d["single_thread"]["value"] > 0
    assert d["dequant_f64_gemm"]["cores"] == cores and d["dequant_f64_gemm"]["value"] > 0
    assert oracle.num_threads() == cores


def test_decoded_gemm_equals_the_exact_oracle_gemm_on_these_operands():
    # the decoded binary64 product is exact here (few terms, short significands),
    # so it rounds to the oracle's BF16 output: the timed baseline computes the same layer
    oracle.build()
    p = synth.dense(4, 256, 32, seed=5)
    qw, sw = oracle.quantize_weights(p.W[0], p.D[0])
    qa, sa = oracle.quantize_act(p.x, p.D[0])
    dec = (oracle.dequantize(qa, sa) @ oracle.dequantize(qw, sw).T) * 2.0 ** -5
    assert np.array_equal(oracle.f64_to_bf16(dec), oracle.gemm(qa, sa, qw, sw))


def test_eager_series_alternates_two_distinct_activation_buffers():
    import types
    import torch
    seen = []
    fake = types.SimpleNamespace(dense_mm=lambda x, *a, **k: seen.append((x.data_ptr(), x.clone())))
    pp = object.__new__(bench.Prepared)
    pp.x = torch.arange(64, dtype=torch.float32).reshape(4, 16)
    pp.D = pp.Wq = pp.Ws = None
    pp.gl = None
    pp.p = types.SimpleNamespace(N=16)
    for i in range(4):
        pp.run_alloc(fake, None, alt=bool(i & 1))
    ptrs = [s[0] for s in seen]
    assert ptrs[0] == ptrs[2] and ptrs[1] == ptrs[3] and ptrs[0] != ptrs[1]
    assert all(torch.equal(s[1], pp.x) for s in seen)


def test_type2_list_covers_the_same_groups():
    import types
    import numpy as np
    import torch
    import synth
    p = synth.grouped(300, 16, 256, 64, seed=1, dist="zipf", group_list_type=0)
    calls = []
    fake = types.SimpleNamespace(grouped_mm=lambda x, D, Wq, Ws, gl, t, N, **k: calls.append((gl.clone(), t, N)))
    pp = object.__new__(bench.Prepared)
    pp.p, pp.x, pp.D, pp.Wq, pp.Ws, pp.ws = p, None, None, None, None, None
    pp.y = torch.empty(0)
    pp.run_type2(fake)
    gl, t, N = calls[0]
    assert t == 2 and N == p.N and tuple(gl.shape) == (p.E, 2) and gl.dtype == torch.int64
    rows = gl.numpy()
    assert np.array_equal(rows[:, 0], np.arange(p.E))
    assert np.array_equal(rows[:, 1], p.counts) and rows[:, 1].sum() == p.M
    # the type-0 list of the same problem gives the same row ranges
    assert np.array_equal(np.cumsum(rows[:, 1]), p.group_list)
