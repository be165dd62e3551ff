"""Write tests/golden/oracle_small.json from the CPU oracle alone.

No page prints a worked example for these formats, so the only stored
expected values are the oracle's own, on tiny seeded cases; they guard the
oracle against silent drift (a change to its arithmetic must regenerate this
file and say, in its commit message, which passage or reading justifies it).
Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from bit_quantized_gemm_quant_b200 import inputs  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small.json")


def case_q4_0(seed=0, M=2, N=3, K=64):
    g = inputs.generator(seed)
    w = inputs.weights_fp32(N, K, g).numpy()
    x = inputs.activations_bf16(M, K, g).view(dtype=__import__("torch").int16).numpy().view(np.uint16)
    wq, d = oracle.q4_0_quantize(w)
    wb = oracle.q4_0_dequantize(wq, d)
    y, a, _ = oracle.matmul_ref(x, wb, nthreads=1)
    return {"fmt": "q4_0", "seed": seed, "M": M, "N": N, "K": K, "group_size": 32, "bits": 4,
            "w_f32_hex": [f"{v:08x}" for v in w.view(np.uint32).ravel()],
            "x_bf16_hex": [f"{v:04x}" for v in x.ravel()],
            "wq_hex": wq.tobytes().hex(), "scales_f16_hex": [f"{v:04x}" for v in d.ravel()],
            "w_bf16_hex": [f"{v:04x}" for v in wb.ravel()],
            "y": [float(v) for v in y.ravel()], "a": [float(v) for v in a.ravel()]}


def case_affine(bits, seed=0, M=2, N=3, K=128, G=64):
    import torch
    g = inputs.generator(seed)
    w = inputs.weights_bf16_valued(N, K, g).numpy()
    x = inputs.activations_bf16(M, K, g).view(torch.int16).numpy().view(np.uint16)
    wq, s, b = oracle.affine_quantize(w, G, bits)
    wb = oracle.affine_dequantize(wq, s, b, G, bits)
    y, a, _ = oracle.matmul_ref(x, wb, nthreads=1)
    return {"fmt": f"affine{bits}", "seed": seed, "M": M, "N": N, "K": K, "group_size": G, "bits": bits,
            "w_f32_hex": [f"{v:08x}" for v in w.view(np.uint32).ravel()],
            "x_bf16_hex": [f"{v:04x}" for v in x.ravel()],
            "wq_hex": [f"{v:08x}" for v in wq.ravel()],
            "scales_bf16_hex": [f"{v:04x}" for v in s.ravel()],
            "biases_bf16_hex": [f"{v:04x}" for v in b.ravel()],
            "w_bf16_hex": [f"{v:04x}" for v in wb.ravel()],
            "y": [float(v) for v in y.ravel()], "a": [float(v) for v in a.ravel()]}


def main():
    cases = [case_q4_0(), case_affine(4), case_affine(8)]
    with open(OUT, "w") as f:
        json.dump({"written_by": "tests/golden/make_golden.py (CPU oracle only)", "cases": cases}, f,
                  indent=0)
    print(OUT)


if __name__ == "__main__":
    main()
