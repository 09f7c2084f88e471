"""The allocation-free decode-attention entry point.

Some callers cannot allocate device memory when they run the kernel (for
instance while recording a CUDA graph, or inside a runtime that owns a fixed
memory pool). bt_op_decode_attention_noalloc serves them from a fixed array
inside the library. This checks it through the C-ABI against the entry point
that takes caller scratch, on two calls in a row (the array keeps the first
call's contents), and that oversized problems are refused. This file is
collected last on purpose, so that a failure here leaves every other test run.
"""
import numpy as np
import pytest

from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu

BF16_TOL = 1e-2  # the bound the other bf16 attention tests use


@pytest.mark.parametrize("B,H,d,n,cap", [(4, 12, 64, 300, 544), (2, 16, 128, 700, 700)])
def test_noalloc_matches_scratch_entry_point_twice(B, H, d, n, cap):
    from hierarchical_global_local_b200 import native
    torch = gh.torch_mod()
    g = torch.Generator(device="cuda").manual_seed(B * 31 + n)
    q = torch.randn(B, H * d, device="cuda", generator=g).bfloat16()
    k = torch.randn(B, H, cap, d, device="cuda", generator=g).bfloat16()
    v = torch.randn(B, H, cap, d, device="cuda", generator=g).bfloat16()
    ref = native.decode_attention(q, k, v, n).float()
    for _ in range(2):
        got = native.decode_attention_noalloc(q, k, v, n).float()
        torch.cuda.synchronize()
        assert torch.allclose(got, ref, rtol=0, atol=BF16_TOL)
    # a different problem in between, then the first again
    q2 = torch.randn(B, H * d, device="cuda", generator=g).bfloat16()
    ref2 = native.decode_attention(q2, k, v, n // 2 + 1).float()
    got2 = native.decode_attention_noalloc(q2, k, v, n // 2 + 1).float()
    got3 = native.decode_attention_noalloc(q, k, v, n).float()
    torch.cuda.synchronize()
    assert torch.allclose(got2, ref2, rtol=0, atol=BF16_TOL)
    assert torch.allclose(got3, ref, rtol=0, atol=BF16_TOL)


def test_noalloc_refuses_oversized_problems():
    from hierarchical_global_local_b200 import native
    torch = gh.torch_mod()
    B, H, d, cap = 1024, 16, 64, 4   # 16384 pairs > 8192
    q = torch.zeros(B, H * d, device="cuda", dtype=torch.bfloat16)
    k = torch.zeros(B, H, cap, d, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(native.BtError) as ei:
        native.decode_attention_noalloc(q, k, k, 2)
    assert ei.value.code == native.BT_ECAPACITY
