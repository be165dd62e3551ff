"""quant_matmul_noalloc: the entry point for callers that cannot allocate device
memory (a host that owns every device byte through its own pool, or one that
cannot take an allocation's implicit synchronization on a first call).  It runs
the dequantize-then-GEMM pair with its bf16 staging buffer in the library's
fixed 32 MiB device array and must give the same result as quant_matmul.

This file is collected last on purpose: it shares the library's static scratch
and must pass both alone in a fresh process and after every other test.
"""
from __future__ import annotations

import numpy as np
import pytest

from _helpers import Problem, reference, assert_within_tolerance

ALIGNED = 256                       # fake, 16-byte aligned, never dereferenced
BQ_ERR_WORKSPACE = 7
BQ_ERR_UNSUPPORTED = 3


def test_noalloc_rejects_oversize_before_any_launch():
    import bit_quantized_gemm_quant_b200 as bq
    L = bq.lib()
    # 4096 x 4097 would need 2 elements more than fit -> K must keep its group; use N
    assert L.quant_matmul_noalloc(ALIGNED, ALIGNED, ALIGNED, None, ALIGNED, 64, 4097, 4096, 32, 4, 1, None) \
        == BQ_ERR_WORKSPACE
    assert L.quant_matmul_noalloc(ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 64, 8192, 4096, 64, 8, 1, None) \
        == BQ_ERR_WORKSPACE
    assert L.quant_matmul_noalloc(ALIGNED, ALIGNED, ALIGNED, None, ALIGNED, 64, 256, 512, 32, 4, 0, None) \
        == BQ_ERR_UNSUPPORTED
    assert L.quant_matmul_noalloc(None, None, None, None, None, 0, 256, 512, 32, 4, 1, None) == 0   # empty


@pytest.mark.gpu
def test_noalloc_matches_quant_matmul_two_calls_in_a_row():
    import torch
    import bit_quantized_gemm_quant_b200 as bq
    # two different problems back to back share the scratch: the second must not see the first's data
    cases = [("affine4", 1024, 2048, 160, 7), ("q4_0", 4096, 4096, 48, 8)]   # the second fills the whole array
    outs = []
    for fmt, N, K, M, seed in cases:
        p = Problem(fmt, N, K, seed=seed)
        wq, s, b = p.device()
        x = p.x(M).cuda()
        y_new = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        bq.quant_matmul_noalloc(x, wq, s, b, y_new, p.group_size, p.bits)
        y_old = bq.quant_matmul(x, wq, s, b, p.group_size, p.bits)
        torch.cuda.synchronize()
        rows = list(range(0, M, 7)) + [M - 1]
        y_ref, a_ref = reference(x, p.wb, rows=rows)
        assert_within_tolerance(y_new[rows], y_ref, a_ref, f"noalloc {fmt} vs oracle")
        # against the existing entry point, within the same tolerance
        assert_within_tolerance(y_new[rows], y_old[rows].double().cpu().numpy(), a_ref, f"noalloc {fmt} vs quant_matmul")
        outs.append((x, wq, s, b, p, y_new.clone()))
    # repeat the first problem after the second overwrote the scratch: same bits as before
    x, wq, s, b, p, y_first = outs[0]
    y_again = torch.empty_like(y_first)
    bq.quant_matmul_noalloc(x, wq, s, b, y_again, p.group_size, p.bits)
    torch.cuda.synchronize()
    assert torch.equal(y_again.view(torch.int16), y_first.view(torch.int16))
    assert bq.bq_device_status() == 0
