"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a temporary copy of oracle/macaq_oracle.c (the
oracle itself is never changed), builds it with the oracle's own flags, and runs
the host pin suites against that build: every mutant must fail at least one
pin.  An unmutated copy built the same way must pass, so a failure is the
planted mistake's and not the harness's.
"""
import concurrent.futures
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "macaq_oracle.c")
PINS = ["tests/test_oracle.py", "tests/test_oracle_readings.py"]

# the BF16 rounding step of the exact GEMM (the binary64 one beside it is alike)
BF_ROUND = "        q = (q << 1) | (uint32_t)wide_bit(&a, i);\n    if (L > 0) {\n        int round = wide_bit(&a, L - 1);\n        int sticky = wide_any_below(&a, L - 1);\n        if (round && (sticky || (q & 1)))"

# (name, text in the oracle, replacement[, occurrences replaced, default 1]):
# each a mistake someone could make
MUTANTS = [
    ("butterfly difference sign", "float b = v[i + h];\n            v[i] = a + b;\n            v[i + h] = a - b;",
     "float b = v[i + h];\n            v[i] = a + b;\n            v[i + h] = b - a;"),
    ("E8M0 offset of the largest E2M1 exponent", "int c = floor_log2 - 2 + 127;", "int c = floor_log2 - 1 + 127;"),
    ("E2M1 tie at 0.25 rounded up", "if (a <= 0.25)", "if (a < 0.25)"),
    ("E2M1 tie at 2.5 rounded up", "else if (a <= 2.5)", "else if (a < 2.5)"),
    ("activations multiplied by D", "float prod = bf16_bits_to_float(xrow[k]) * r;",
     "float prod = bf16_bits_to_float(xrow[k]) / r;"),
    ("no BF16 rounding of the scaled activations", "v[i] = bf16_bits_to_float(float_to_bf16_rne(prod));",
     "v[i] = prod;"),
    ("weights divided by D", "t[i] = W[n * K + k] * D[k];", "t[i] = W[n * K + k] / D[k];"),
    ("output scale 2^-4", "return gemm_exp(qa, sa, qw, sw, M, N, K, y, nthreads, -5);",
     "return gemm_exp(qa, sa, qw, sw, M, N, K, y, nthreads, -4);"),
    ("plain path keeps 2^-5", "return gemm_exp(qa, sa, qw, sw, M, N, K, y, nthreads, 0);",
     "return gemm_exp(qa, sa, qw, sw, M, N, K, y, nthreads, -5);"),
    ("counts read as cumulative sums", "        if (type == 0) {\n            if (v < off[g])",
     "        if (type == 1) {\n            if (v < off[g])"),
    ("calibration ratio inverted", "d = sqrt(a / w);", "d = sqrt(w / a);"),
    ("GELU cubic coefficient", "(v + 0.044715 * v * v * v)", "(v + 0.04715 * v * v * v)"),
    ("FAST_GELU slope", "return v / (1.0 + exp(-1.702 * v));", "return v / (1.0 + exp(-1.72 * v));"),
    ("BF16 ties rounded up", "if (dropped > 0x8000u || (dropped == 0x8000u && (keep & 1u)))",
     "if (dropped >= 0x8000u)"),
    ("type-2 rows use the list position, not the named expert",
     "int64_t e = type == 2 ? group_list[2 * g] : g;", "int64_t e = g;"),
    ("grouped bias taken by list position", "bias ? bias + e * N : NULL", "bias ? bias + g * N : NULL"),
    ("grouped activations scaled by expert 0's D", "oracle_quantize_act(x + r0 * K, D + e * K,",
     "oracle_quantize_act(x + r0 * K, D,"),
    ("weight scale dropped from the exact dot", "int E = (int)sa[b] + (int)sw[b] - 256;",
     "int E = (int)sa[b] + 127 - 256;"),
    ("code nibbles swapped in both exact dots", "int ca = (qa[k / 2] >> (4 * (k & 1))) & 15;",
     "int ca = (qa[k / 2] >> (4 * (1 - (k & 1)))) & 15;", 2),
    ("type-2 index bound off by one", "group_list[2 * g] >= E))", "group_list[2 * g] > E))"),
    ("calibration rows of a type-2 entry credited to its position",
     "int64_t e = (group_list && type == 2) ? group_list[2 * g] : g;", "int64_t e = g;"),
    ("calibration ignores an expert without rows", "            if (rows[e] == 0) {\n                D[e * K + k] = 1.0f;",
     "            if (rows[e] < 0) {\n                D[e * K + k] = 1.0f;"),
    ("calibration lower clamp 1e-3", "    if (d < 1e-2)\n        d = 1e-2;", "    if (d < 1e-3)\n        d = 1e-3;"),
    ("E8M0 not clamped at 0", "    if (c < 0)\n        c = 0;", "    if (c < -1)\n        c = 0;"),
    ("BF16 from binary64 ties away from zero", "double q = nearbyint(ldexp(a, -lsb));", "double q = round(ldexp(a, -lsb));"),
    ("weights not rotated", "            fwht32_f32(t);\n            double d[32];", "            double d[32];"),
    ("SILU as v sigmoid(2v)", "return v / (1.0 + exp(-v));", "return v / (1.0 + exp(-2.0 * v));"),
    ("true-division reading multiplies by the reciprocal",
     "float s = reading == 1 ? xf / D[k] : xf * (1.0f / D[k]);", "float s = xf * (1.0f / D[k]);"),
    ("BF16-stage reading rounds only the sums",
     "v[i + h] = oracle_bf16_to_f64(oracle_f64_to_bf16(a - c));", "v[i + h] = a - c;"),
    ("exact GEMM rounding without the sticky bit", BF_ROUND, BF_ROUND.replace("(sticky || (q & 1))", "(q & 1)")),
    ("exact GEMM ties away from zero", BF_ROUND, BF_ROUND.replace("round && (sticky || (q & 1))", "round")),
    ("exact GEMM without BF16 subnormals", "int lsb_exp = E >= -126 ? E - 7 : -133;", "int lsb_exp = E - 7;"),
    ("bias added after the activation",
     "            if (bias)\n                s += (double)bias[n];\n            y[m * N + n] = oracle_f64_to_bf16(oracle_act(s, act));",
     "            y[m * N + n] = oracle_f64_to_bf16(oracle_act(s, act) + (bias ? (double)bias[n] : 0.0));"),
    ("one-row groups skipped with the empty ones", "        if (r1 == r0)\n            continue;",
     "        if (r1 <= r0 + 1)\n            continue;"),
    ("block amax without the absolute value", "        float a = (float)fabs(v[i]);\n        if (a > amax || isnan(a))",
     "        float a = (float)v[i];\n        if (a > amax || isnan(a))"),
    ("codes packed high nibble first", "codes[j] = (uint8_t)(lo | (hi << 4));", "codes[j] = (uint8_t)(hi | (lo << 4));"),
    ("one D per block instead of per channel", "float r = 1.0f / D[k];                            /* RN32(1/D) */",
     "float r = 1.0f / D[32 * b];                       /* RN32(1/D) */"),
    ("RELU leaks negatives", "return v > 0.0 ? v : 0.0;", "return v > 0.0 ? v : 0.01 * v;"),
    ("calibration skips the last weight row", "            for (int64_t n = 0; n < N; n++) {\n                double v = fabs((double)W[(e * N + n) * K + k]);",
     "            for (int64_t n = 0; n + 1 < N; n++) {\n                double v = fabs((double)W[(e * N + n) * K + k]);"),
    ("calibration skips the last row of each group", "        for (int64_t r = off[g]; r < off[g + 1]; r++)",
     "        for (int64_t r = off[g]; r + 1 < off[g + 1]; r++)"),
]


def _build(text: str, out: str):
    with tempfile.NamedTemporaryFile("w", suffix=".c", delete=False) as f:
        f.write(text)
        c = f.name
    try:
        subprocess.check_call(["gcc", "-O2", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
                               "-shared", "-fPIC", "-o", out, c, "-lm"])
    finally:
        os.unlink(c)


def _run_pins(lib: str) -> int:
    env = dict(os.environ, MACAQ_ORACLE_LIB=lib, OMP_NUM_THREADS="2")
    return subprocess.run([sys.executable, "-m", "pytest", *PINS, "-x", "-q", "-p", "no:cacheprovider",
                           "-m", "not gpu"], cwd=ROOT, env=env, capture_output=True, timeout=600).returncode


def test_every_planted_mistake_fails_a_pin(tmp_path):
    src = open(SRC).read()
    jobs = [("control", None, None)] + MUTANTS
    libs = []
    for i, (name, old, new, *count) in enumerate(jobs):
        if old is not None:
            want = count[0] if count else 1
            assert src.count(old) == want, f"{name}: the text to mutate must occur {want} time(s)"
        lib = str(tmp_path / f"m{i}.so")
        _build(src if old is None else src.replace(old, new), lib)
        libs.append((name, lib))
    with concurrent.futures.ThreadPoolExecutor(max_workers=4) as ex:
        codes = list(ex.map(lambda nl: _run_pins(nl[1]), libs))
    assert codes[0] == 0, "the unmutated build must pass every pin"
    survivors = [name for (name, _), rc in zip(libs[1:], codes[1:]) if rc == 0]
    assert not survivors, f"mistakes no pin caught: {survivors}"


# Mistakes in the oracle's Python layer, planted in a copy of the package
PY_MUTANTS = [
    ("plain type-2 rows use the list position", "e = int(gl[g, 0]) if group_list_type == 2 else g", "e = g"),
    ("plain activations taken as their bit patterns", "return quantize_plain(bf16_to_f64(x).astype(np.float32))",
     "return quantize_plain(x.astype(np.float32))"),
    ("BF16 widening shifted by 15", "return (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)",
     "return (h.astype(np.uint32) << 15).view(np.float32).astype(np.float64)"),
    ("plain one-row groups skipped", "        if b > a:\n            y[a:b] = dense_mm_plain(", "        if b > a + 1:\n            y[a:b] = dense_mm_plain("),
    ("weight-list type-2 rows use the list position", "e = int(gl[j, 0]) if group_list_type == 2 else j", "e = j"),
    ("weight-list entries use expert 0's D", "y[a:b] = dense_mm(x[a:b], D[e], W_list[e], nthreads)",
     "y[a:b] = dense_mm(x[a:b], D[0], W_list[e], nthreads)"),
]


def _tree_copy(dst: str, init_text: str):
    import shutil
    ignore = shutil.ignore_patterns("__pycache__", "*.so", "*.so.tmp*")
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(dst, "oracle"), ignore=ignore)
    shutil.copytree(os.path.join(ROOT, "synth"), os.path.join(dst, "synth"), ignore=ignore)
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(dst, "tests", "golden"))
    for f in ["tests/conftest.py", *PINS, "pytest.ini"]:
        shutil.copy(os.path.join(ROOT, f), os.path.join(dst, f))
    with open(os.path.join(dst, "oracle", "__init__.py"), "w") as f:
        f.write(init_text)


def _run_pins_in(tree: str) -> int:
    env = dict(os.environ, OMP_NUM_THREADS="2", CUDA_VISIBLE_DEVICES="")
    env.pop("MACAQ_ORACLE_LIB", None)
    return subprocess.run([sys.executable, "-m", "pytest", *PINS, "-x", "-q", "-p", "no:cacheprovider",
                           "-m", "not gpu"], cwd=tree, env=env, capture_output=True, timeout=600).returncode


def test_every_planted_python_mistake_fails_a_pin(tmp_path):
    init = open(os.path.join(ROOT, "oracle", "__init__.py")).read()
    trees = []
    for i, (name, old, new) in enumerate([("control", None, None)] + PY_MUTANTS):
        if old is not None:
            assert init.count(old) == 1, f"{name}: the text to mutate must occur once"
        tree = str(tmp_path / f"t{i}")
        _tree_copy(tree, init if old is None else init.replace(old, new))
        trees.append((name, tree))
    with concurrent.futures.ThreadPoolExecutor(max_workers=4) as ex:
        codes = list(ex.map(lambda nt: _run_pins_in(nt[1]), trees))
    assert codes[0] == 0, "the unmutated copy must pass every pin"
    survivors = [name for (name, _), rc in zip(trees[1:], codes[1:]) if rc == 0]
    assert not survivors, f"mistakes no pin caught: {survivors}"


# Mistakes in the C boundary's host-side checks, planted in copies of the
# library source and caught by the device-free boundary tests.  Each mutant is a
# full nvcc build (about a minute), so this case runs only on request
# (MACAQ_ABI_MUTANTS=1).
ABI_SRC = os.path.join(ROOT, "w4a4_mxfp4_quantize_b200", "csrc", "macaq.cu")
ABI_TESTS = ["tests/test_abi.py", "tests/test_c_header.py"]
ABI_MUTANTS = [
    ("act_type 3 accepted", "bool act_supported(int act) { return act == 0 || act == 1 || act == 2 || act == 4 || act == 5; }",
     "bool act_supported(int act) { return act >= 0 && act <= 5; }"),
    ("K % 32 accepted", "return K >= 256 && K <= 65536 && K % 256 == 0 && N >= 16", "return K >= 256 && K <= 65536 && K % 32 == 0 && N >= 16"),
    ("N % 8 accepted", "N <= 65536 && N % 16 == 0;", "N <= 65536 && N % 8 == 0;"),
    ("alignment of x not checked", "if (!aligned16(x) || (!plain && !aligned16(D))", "if ((!plain && !aligned16(D))"),
    ("y overlapping x not refused", "if (overlaps(y, ybytes, x, static_cast<size_t>(M) * K * 2) ||", "if (false ||"),
    ("bias alignment not checked", "if (!aligned16(ep.bias)) return MACAQ_ERR_ALIGN;", ""),
    ("group_list_type -1 accepted", "if (group_list_type < 0 || group_list_type > 2) return MACAQ_ERR_GROUP_LIST_TYPE;",
     "if (group_list_type > 2) return MACAQ_ERR_GROUP_LIST_TYPE;"),
    ("weight rows padded to 128", "return static_cast<size_t>(E) * pad256(N) * (K / 2);",
     "return static_cast<size_t>(E) * ((N + 127) / 128 * 128) * (K / 2);"),
    ("status name of act_type refusal", 'case MACAQ_ERR_ACT_TYPE: return "MACAQ_ERR_ACT_TYPE";',
     'case MACAQ_ERR_ACT_TYPE: return "MACAQ_ERR_SHAPE";'),
]


def _abi_build_and_test(name: str, text: str, d: str) -> int:
    os.makedirs(d, exist_ok=True)
    src = os.path.join(d, "macaq.cu")
    with open(src, "w") as f:
        f.write(text)
    lib = os.path.join(d, "libmacaq.so")
    import w4a4_mxfp4_quantize_b200 as mq
    subprocess.check_call(["nvcc", *mq.NVCC_FLAGS, "-I" + os.path.join(ROOT, "include"),
                           "-I" + os.path.dirname(ABI_SRC), "-o", lib, src])
    code = ("import sys, pytest, w4a4_mxfp4_quantize_b200 as mq; mq._LIB_PATH = sys.argv[1]; "
            "sys.exit(pytest.main([*sys.argv[2:], '-x', '-q', '-p', 'no:cacheprovider', '-m', 'not gpu']))")
    # The boundary tests pass made-up device addresses; a mutant that lets one
    # through must meet a process that sees no device, never launch a kernel.
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    return subprocess.run([sys.executable, "-c", code, lib, *ABI_TESTS], cwd=ROOT, env=env, capture_output=True,
                          timeout=600).returncode


def _device_visible() -> bool:
    import torch
    return torch.cuda.is_available()


@pytest.mark.skipif(os.environ.get("MACAQ_ABI_MUTANTS") != "1", reason="nvcc builds; run with MACAQ_ABI_MUTANTS=1")
@pytest.mark.skipif(_device_visible(), reason="mutated host checks: run only where no device is visible")
def test_every_planted_boundary_mistake_fails_a_boundary_test(tmp_path):
    src = open(ABI_SRC).read()
    jobs = [("control", None, None)] + ABI_MUTANTS
    for name, old, _ in ABI_MUTANTS:
        assert src.count(old) == 1, f"{name}: the text to mutate must occur once"
    with concurrent.futures.ThreadPoolExecutor(max_workers=5) as ex:
        codes = list(ex.map(lambda ij: _abi_build_and_test(
            ij[1][0], src if ij[1][1] is None else src.replace(ij[1][1], ij[1][2]), str(tmp_path / f"a{ij[0]}")),
            enumerate(jobs)))
    assert codes[0] == 0, "the unmutated build must pass the boundary tests"
    survivors = [name for (name, _, _), rc in zip(jobs[1:], codes[1:]) if rc == 0]
    assert not survivors, f"mistakes no boundary test caught: {survivors}"
