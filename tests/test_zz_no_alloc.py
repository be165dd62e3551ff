"""quant_matmul_noalloc: the entry point for callers that cannot allocate device
memory (a host that owns every device byte through its own pool, or one that
cannot take an allocation's implicit synchronization on a first call).  It takes
quant_matmul's own path with the library's fixed 32 MiB device array as its
scratch (the fused kernel's K-split partial sums, the unfused pair's bf16 copy
of W) and must give the same result as quant_matmul.

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
    # at 8192 tokens the path is the unfused pair, whose bf16 copy of W must fit the array:
    # 4097 x 4096 weights need 2 x 4096 bytes more than 32 MiB
    assert L.quant_matmul_noalloc(ALIGNED, ALIGNED, ALIGNED, None, ALIGNED, 8192, 4097, 4096, 32, 4, 1, None) \
        == BQ_ERR_WORKSPACE
    assert L.quant_matmul_noalloc(ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 8192, 8192, 4096, 64, 8, 1, None) \
        == BQ_ERR_WORKSPACE
    assert L.quant_matmul_noalloc(ALIGNED, ALIGNED, ALIGNED, None, ALIGNED, 64, 256, 512, 32, 4, 0, None) \
        == BQ_ERR_UNSUPPORTED
    assert L.quant_matmul_noalloc(None, None, None, None, None, 0, 256, 512, 32, 4, 1, None) == 0   # empty


@pytest.mark.gpu
def test_noalloc_matches_quant_matmul_two_calls_in_a_row():
    import torch
    import bit_quantized_gemm_quant_b200 as bq
    # problems back to back share the scratch: a later one must not see an earlier one's data.
    # decode (no scratch), fused with K split (partials in the array), the pair (W fills the array)
    cases = [("q4_0", 4096, 4096, 1, 6), ("affine4", 1024, 2048, 160, 7), ("q4_0", 12288, 4096, 48, 9),
             ("q4_0", 4096, 4096, 4096, 8)]
    probs = []
    for fmt, N, K, M, seed in cases:
        p = Problem(fmt, N, K, seed=seed)
        wq, s, b = p.device()
        probs.append((p, M, p.x(M).cuda(), wq, s, b, torch.empty(M, N, dtype=torch.bfloat16, device="cuda")))
    # first call on the device (loads the library's device code), then nothing may be allocated
    p, M, x, wq, s, b, y = probs[0]
    bq.quant_matmul_noalloc(x, wq, s, b, y, p.group_size, p.bits)
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    outs = []
    for p, M, x, wq, s, b, y in probs:
        bq.quant_matmul_noalloc(x, wq, s, b, y, p.group_size, p.bits)
        torch.cuda.synchronize()
        assert torch.cuda.mem_get_info()[0] == free_before, f"noalloc {p.fmt} M={M} allocated device memory"
        outs.append(y.clone())
    for (p, M, x, wq, s, b, y), y_new in zip(probs, outs):
        y_old = bq.quant_matmul(x, wq, s, b, p.group_size, p.bits)
        torch.cuda.synchronize()
        rows = sorted(set(list(range(0, M, max(1, M // 40))) + [M - 1]))
        y_ref, a_ref = reference(x, p.wb, rows=rows)
        assert_within_tolerance(y_new[rows], y_ref, a_ref, f"noalloc {p.fmt} M={M} vs oracle")
        # the same path as the existing entry point: the same bits
        assert torch.equal(y_new.view(torch.int16), y_old.view(torch.int16)), f"noalloc {p.fmt} M={M}"
    # repeat the first problems after later ones overwrote the scratch: same bits as before
    for (p, M, x, wq, s, b, y), y_first in list(zip(probs, outs))[:2]:
        y_again = torch.empty_like(y_first)
        bq.quant_matmul_noalloc(x, wq, s, b, y_again, p.group_size, p.bits)
        torch.cuda.synchronize()
        assert torch.equal(y_again.view(torch.int16), y_first.view(torch.int16))
    assert bq.bq_device_status() == 0
