"""How much the unpinned reading of the activation arithmetic matters.

The summary of the MACAQ page names a channel scaling by raw D and a BF16
Hadamard rotation without their working precision.  The oracle's parity
reference is R3 (scale by RN32(1/D), FP32 butterfly, one BF16 rounding); it also
implements three other plain readings (true division by D, BF16 rounding at
every butterfly stage, exact rotation rounded once).  This script quantises the
synthetic M = 4096 activations of the five projections (a row sample) under each
reading and reports, against R3: the share of E2M1 codes and E8M0 scales that
differ, the share of BF16 layer outputs that differ (exact block-scaled GEMM
against the same MXFP4 weights), and each reading's NMSE against the
unquantised binary64 layer.

    python oracle/readings_report.py [rows]

Test infrastructure: it calls only the oracle and the seeded input generators.
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402

NAMES = {oracle.READING_R3: "R3 (reference)", oracle.READING_TRUE_DIVISION: "true division by D",
         oracle.READING_BF16_STAGES: "BF16 at every butterfly stage",
         oracle.READING_EXACT_ROTATION: "exact rotation, one rounding"}


def report(rows: int = 64) -> list[dict]:
    out = []
    for p in synth.config(2):
        x = p.x[:rows]
        D = p.D[0]
        qw, sw = oracle.quantize_weights(p.W[0], D)
        ref = oracle.linear_f64(x, p.W[0])
        base = None
        for reading in NAMES:
            qa, sa = oracle.quantize_act_reading(x, D, reading)
            y = oracle.gemm(qa, sa, qw, sw)
            yf = oracle.bf16_to_f64(y)
            nmse = float(np.sum((yf - ref) ** 2) / np.sum(ref ** 2))
            if base is None:
                base = (oracle.unpack_codes(qa), sa, y)
            out.append({
                "problem": p.name, "reading": NAMES[reading],
                "codes_differ": float(np.mean(oracle.unpack_codes(qa) != base[0])),
                "scales_differ": float(np.mean(sa != base[1])),
                "outputs_differ": float(np.mean(y != base[2])),
                "nmse": nmse,
            })
    return out


def main():
    rows = int(sys.argv[1]) if len(sys.argv) > 1 else 64
    res = report(rows)
    print(f"rows per projection: {rows}")
    print("| projection | reading | codes differ | scales differ | outputs differ | NMSE vs unquantised |")
    print("|---|---|---|---|---|---|")
    for r in res:
        print(f"| {r['problem']} | {r['reading']} | {100 * r['codes_differ']:.3f} % | "
              f"{100 * r['scales_differ']:.3f} % | {100 * r['outputs_differ']:.2f} % | {r['nmse']:.5f} |")


if __name__ == "__main__":
    main()
