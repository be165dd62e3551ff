"""The oracle still reproduces the stored small cases written by
tests/golden/make_golden.py (guards against silent drift of its arithmetic)."""
import json
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "oracle_small.json")


def _u(hexes, dtype):
    return np.array([int(h, 16) for h in hexes], dtype=dtype)


def test_oracle_reproduces_stored_cases():
    with open(GOLDEN) as f:
        cases = json.load(f)["cases"]
    assert {c["fmt"] for c in cases} == {"q4_0", "affine4", "affine8"}
    for c in cases:
        M, N, K = c["M"], c["N"], c["K"]
        w = _u(c["w_f32_hex"], np.uint32).view(np.float32).reshape(N, K)
        x = _u(c["x_bf16_hex"], np.uint16).reshape(M, K)
        if c["fmt"] == "q4_0":
            wq, d = oracle.q4_0_quantize(w)
            assert wq.tobytes().hex() == c["wq_hex"]
            assert np.array_equal(d.ravel(), _u(c["scales_f16_hex"], np.uint16))
            wb = oracle.q4_0_dequantize(wq, d)
        else:
            wq, s, b = oracle.affine_quantize(w, c["group_size"], c["bits"])
            assert np.array_equal(wq.ravel(), _u(c["wq_hex"], np.uint32))
            assert np.array_equal(s.ravel(), _u(c["scales_bf16_hex"], np.uint16))
            assert np.array_equal(b.ravel(), _u(c["biases_bf16_hex"], np.uint16))
            wb = oracle.affine_dequantize(wq, s, b, c["group_size"], c["bits"])
        assert np.array_equal(wb.ravel(), _u(c["w_bf16_hex"], np.uint16))
        y, a, _ = oracle.matmul_ref(x, wb, nthreads=1)
        assert np.array_equal(y.ravel(), np.array(c["y"]))
        assert np.array_equal(a.ravel(), np.array(c["a"]))
