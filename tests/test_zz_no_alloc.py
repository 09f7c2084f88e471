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


FP32_TOL = 1e-5  # fp32 inputs: the two entry points run the same kernel


@pytest.mark.parametrize("B,H,d,n,cap,dt", [(4, 12, 64, 300, 544, "bf16"), (2, 16, 128, 700, 700, "bf16"),
                                            (3, 8, 32, 129, 200, "bf16"), (2, 4, 64, 77, 96, "fp32")])
def test_noalloc_matches_scratch_entry_point_twice(B, H, d, n, cap, dt):
    from hierarchical_global_local_b200 import native
    torch = gh.torch_mod()
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    tol = BF16_TOL if dt == "bf16" else FP32_TOL
    g = torch.Generator(device="cuda").manual_seed(B * 31 + n)
    q = torch.randn(B, H * d, device="cuda", generator=g).to(tdt)
    k = torch.randn(B, H, cap, d, device="cuda", generator=g).to(tdt)
    v = torch.randn(B, H, cap, d, device="cuda", generator=g).to(tdt)
    ref = native.decode_attention(q, k, v, n).float()
    for _ in range(2):
        got = native.decode_attention_noalloc(q, k, v, n).float()
        torch.cuda.synchronize()
        assert torch.allclose(got, ref, rtol=0, atol=tol)
    # a different problem in between, then the first again
    q2 = torch.randn(B, H * d, device="cuda", generator=g).to(tdt)
    ref2 = native.decode_attention(q2, k, v, n // 2 + 1).float()
    got2 = native.decode_attention_noalloc(q2, k, v, n // 2 + 1).float()
    got3 = native.decode_attention_noalloc(q, k, v, n).float()
    torch.cuda.synchronize()
    assert torch.allclose(got2, ref2, rtol=0, atol=tol)
    assert torch.allclose(got3, ref, rtol=0, atol=tol)


def test_noalloc_largest_problem_and_no_device_allocation():
    """The largest problem inside the documented limits (B*H = 8192 pairs,
    d_head = 128) is served, and a call after the first one on the device
    leaves the device's free memory and torch's allocator unchanged."""
    from hierarchical_global_local_b200 import native
    torch = gh.torch_mod()
    B, H, d, n, cap = 512, 16, 128, 6, 8
    g = torch.Generator(device="cuda").manual_seed(5)
    q = torch.randn(B, H * d, device="cuda", generator=g).bfloat16()
    k = torch.randn(B, H, cap, d, device="cuda", generator=g).bfloat16()
    v = torch.randn(B, H, cap, d, device="cuda", generator=g).bfloat16()
    ref = native.decode_attention(q, k, v, n).float()
    out = torch.empty(B, H * d, device="cuda", dtype=torch.bfloat16)
    native.decode_attention_noalloc(q, k, v, n, out=out)   # first call on the device
    torch.cuda.synchronize()
    assert torch.allclose(out.float(), ref, rtol=0, atol=BF16_TOL)
    out.zero_()
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    native.decode_attention_noalloc(q, k, v, n, out=out)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 == free0
    assert torch.allclose(out.float(), ref, rtol=0, atol=BF16_TOL)


def test_noalloc_refuses_oversized_problems():
    from hierarchical_global_local_b200 import native
    torch = gh.torch_mod()
    B, H, d, cap = 1024, 16, 64, 4   # 16384 pairs > 8192
    q = torch.zeros(B, H * d, device="cuda", dtype=torch.bfloat16)
    k = torch.zeros(B, H, cap, d, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(native.BtError) as ei:
        native.decode_attention_noalloc(q, k, k, 2)
    assert ei.value.code == native.BT_ECAPACITY
