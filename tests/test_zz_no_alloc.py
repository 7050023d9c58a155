"""bs_int_scaled_mm_noalloc through the C ABI: the wide kernel's stream-K split with the library's built-in
scratch gives int_scaled_mm's results, bit-exact as every INT8 result here is, on two calls in a row.

Every buffer is allocated before the first call; the calls themselves allocate nothing.  The file is named
to be collected last, and passes alone in a fresh process as well.
"""
from __future__ import annotations

import pytest
import torch

import int8_gemm_b200 as bs
import workloads as wl

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _split_tiles(M, N, K):
    """Tiles the stream-K rule splits for this shape on this device (the rule the entry point applies)."""
    prev = bs.set_stream_k(True)
    try:
        return bs.plan_for(bs.OP_INT_SCALED_MM, M, 1, N, K, torch.cuda.get_device_properties(0).multi_processor_count)
    finally:
        bs.set_stream_k(prev)


@pytest.mark.parametrize("M,N,K,splits", [(1024, 1024, 4096, True), (1000, 1800, 2080, True),
                                          (300, 1040, 8192, True), (4096, 4096, 4096, True),
                                          (256, 512, 1024, False)])
def test_noalloc_matches_int_scaled_mm_on_two_calls(M, N, K, splits, cuda_device):
    assert (_split_tiles(M, N, K)["sk_tiles"] > 0) == splits
    d = wl.int8_inputs(M, N, K, seed=4000 + M + N)
    A = d["A"].to(DEV)
    B = d["B_t"].to(DEV).t()
    s_a, s_b = d["s_a"].to(DEV).contiguous(), d["s_b"].to(DEV).contiguous()
    for out_dtype in (torch.int32, torch.float32, torch.bfloat16):
        ref = bs.int_scaled_mm(A, B, s_a, s_b, out_dtype=out_dtype)
        fill = -7 if out_dtype == torch.int32 else float("nan")
        outs = [torch.full((M, N), fill, dtype=out_dtype, device=DEV) for _ in range(2)]
        torch.cuda.synchronize()
        for o in outs:
            bs.bs_int_scaled_mm_noalloc(A, B, s_a, s_b, o)
        torch.cuda.synchronize()
        assert bs.device_error() == 0, "a wait of the split kernel timed out"
        for i, o in enumerate(outs):
            assert torch.equal(o, ref), f"call {i + 1}, {out_dtype}, {M}x{N}x{K}"


def test_noalloc_row_scale_only_and_no_scales(cuda_device):
    M, N, K = 1024, 1024, 4096
    d = wl.int8_inputs(M, N, K, seed=4100)
    A, B = d["A"].to(DEV), d["B_t"].to(DEV).t()
    s_a = d["s_a"].to(DEV).contiguous()
    for sa, sb in ((s_a, None), (None, None)):
        ref = bs.int_scaled_mm(A, B, sa, sb, out_dtype=torch.float32)
        out = torch.empty(M, N, dtype=torch.float32, device=DEV)
        for _ in range(2):
            out.fill_(float("nan"))
            bs.bs_int_scaled_mm_noalloc(A, B, sa, sb, out)
            assert torch.equal(out, ref)
