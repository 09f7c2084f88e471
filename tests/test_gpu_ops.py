"""Single-kernel parity through the op-level C-ABI (bt_ops.h) against the
oracle's primitives (fp64) on seeded inputs: split-K decode attention over
lengths that span several chunks with ragged tails, prefill attention, the
dense projection, LayerNorm and the embedder."""
import numpy as np
import pytest

import oracle.model as om
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu


def _t(a, dtype):
    torch = gh.torch_mod()
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to("cuda", dtype)


def _dtypes():
    torch = gh.torch_mod()
    return {"bf16": torch.bfloat16, "fp32": torch.float32}


@pytest.mark.parametrize("dt", ["bf16", "fp32"])
@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("n", [1, 5, 63, 64, 128, 129, 300, 543])
def test_decode_attention_matches_oracle(dt, d, n):
    from hierarchical_global_local_b200 import native
    torch = gh.torch_mod()
    tdt = _dtypes()[dt]
    g = np.random.default_rng(n * 7 + d)
    B, H, cap = 3, 2, 600
    q = g.standard_normal((B, H * d)).astype(np.float32)
    k = g.standard_normal((B, H, cap, d)).astype(np.float32)
    v = g.standard_normal((B, H, cap, d)).astype(np.float32)
    qt, kt, vt = _t(q, tdt), _t(k, tdt), _t(v, tdt)
    out = native.decode_attention(qt, kt, vt, n).float().cpu().numpy()
    # oracle on the values the device holds
    qr, kr, vr = (x.float().cpu().numpy().astype(np.float64) for x in (qt, kt, vt))
    ref = om.attend(qr.reshape(B, 1, H, d), kr[:, :, :n].transpose(0, 2, 1, 3),
                    vr[:, :, :n].transpose(0, 2, 1, 3), np.array([n - 1]),
                    np.arange(n)).reshape(B, H * d)
    tol = 1e-5 if dt == "fp32" else 1e-2
    assert np.abs(out - ref).max() <= tol * max(1.0, np.abs(ref).max())


def test_decode_attention_scratch_reusable_across_calls():
    from hierarchical_global_local_b200 import native
    torch = gh.torch_mod()
    g = np.random.default_rng(0)
    B, H, d, cap = 2, 3, 64, 700
    q = _t(g.standard_normal((B, H * d)), torch.bfloat16)
    k = _t(g.standard_normal((B, H, cap, d)), torch.bfloat16)
    v = _t(g.standard_normal((B, H, cap, d)), torch.bfloat16)
    scr = native.decode_attention_scratch(native.BT_BF16, B, H, d, cap)
    a = native.decode_attention(q, k, v, 650, scratch=scr)
    b = native.decode_attention(q, k, v, 650, scratch=scr)
    c = native.decode_attention(q, k, v, 200, scratch=scr)
    d2 = native.decode_attention(q, k, v, 200)
    assert torch.equal(a, b) and torch.equal(c, d2)


@pytest.mark.parametrize("dt", ["bf16", "fp32"])
@pytest.mark.parametrize("d,n", [(64, 1), (64, 37), (32, 16), (128, 70)])
def test_prefill_attention_matches_oracle(dt, d, n):
    from hierarchical_global_local_b200 import native
    tdt = _dtypes()[dt]
    g = np.random.default_rng(n + d)
    B, H, cap = 2, 2, n + 3
    q = g.standard_normal((B * n, H * d))
    k = g.standard_normal((B, H, cap, d))
    v = g.standard_normal((B, H, cap, d))
    qt, kt, vt = _t(q, tdt), _t(k, tdt), _t(v, tdt)
    out = native.prefill_attention(qt, kt, vt, n).float().cpu().numpy()
    qr, kr, vr = (x.float().cpu().numpy().astype(np.float64) for x in (qt, kt, vt))
    ref = om.attend(qr.reshape(B, n, H, d), kr[:, :, :n].transpose(0, 2, 1, 3),
                    vr[:, :, :n].transpose(0, 2, 1, 3), np.arange(n), np.arange(n))
    tol = 1e-5 if dt == "fp32" else 1e-2
    assert np.abs(out - ref.reshape(B * n, H * d)).max() <= tol * 4


@pytest.mark.parametrize("dt", ["bf16", "fp32"])
@pytest.mark.parametrize("M,N,K", [(1, 64, 64), (5, 200, 96), (64, 384, 128), (130, 257, 320)])
def test_linear_simt_matches_fp64(dt, M, N, K):
    from hierarchical_global_local_b200 import native
    tdt = _dtypes()[dt]
    g = np.random.default_rng(M + N + K)
    x, w, b = g.standard_normal((M, K)), g.standard_normal((N, K)), g.standard_normal(N)
    xt, wt = _t(x, tdt), _t(w, tdt)
    bt = _t(b, gh.torch_mod().float32)
    out = native.linear(xt, wt, bt, path=1).cpu().numpy()
    ref = xt.double().cpu().numpy() @ wt.double().cpu().numpy().T + b.astype(np.float32)
    assert np.abs(out - ref).max() <= 1e-3 * np.sqrt(K)


@pytest.mark.parametrize("dt", ["bf16", "fp32"])
def test_layernorm_matches_oracle(dt):
    from hierarchical_global_local_b200 import native
    torch = gh.torch_mod()
    g = np.random.default_rng(9)
    M, D = 37, 768
    h = g.standard_normal((M, D)) * 3 + 0.5
    ga, be = 1 + 0.1 * g.standard_normal(D), 0.1 * g.standard_normal(D)
    f32 = lambda a: _t(a, torch.float32)
    out = native.layernorm(f32(h), f32(ga), f32(be), 1e-5, _dtypes()[dt]).float().cpu().numpy()
    ref = om.layer_norm(h.astype(np.float32).astype(np.float64), ga.astype(np.float32),
                        be.astype(np.float32), 1e-5)
    tol = 2e-5 if dt == "fp32" else 2e-2
    assert np.abs(out - ref).max() <= tol * np.abs(ref).max()


@pytest.mark.parametrize("L", [1, 2, 4, 8])
def test_embedder_bitwise(L):
    from hierarchical_global_local_b200 import native
    torch = gh.torch_mod()
    g = np.random.default_rng(L)
    V, D, B, T = 101, 64, 3, 8 * L
    table = _t(g.standard_normal((V, D // L)), torch.bfloat16)
    toks = g.integers(0, V, size=(B, T)).astype(np.int32)
    h = native.embed_prompt(torch.from_numpy(toks).cuda(), table, L, D).cpu().numpy()
    ref = om.embed_blocks(toks, table.float().cpu().numpy(), L).reshape(-1, D)
    assert np.array_equal(h, ref)


def test_embedder_flags_bad_token():
    from hierarchical_global_local_b200 import native
    torch = gh.torch_mod()
    table = torch.zeros(10, 16, dtype=torch.float32, device="cuda")
    toks = torch.tensor([[1, 2, 99, 3]], dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    native.embed_prompt(toks, table, 4, 64, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & 1


@pytest.mark.parametrize("M,N,K", [(1, 128, 64), (2, 384, 128), (33, 768, 768), (64, 5376, 768),
                                   (64, 768, 3840), (100, 1000, 256), (256, 2048, 1024),
                                   (257, 768, 768), (1000, 2304, 768), (4096, 512, 192),
                                   (64, 50304, 768), (32, 4096, 512), (128, 9000, 1024)])
def test_linear_tensor_cores_match_fp64(M, N, K):
    """tcgen05 path (weights-as-A for M <= 256 with split K; activations-as-A
    above) against an fp64 product of the same bf16 operands."""
    from hierarchical_global_local_b200 import native
    torch = gh.torch_mod()
    g = np.random.default_rng(M * 3 + N + K)
    x, w, b = g.standard_normal((M, K)), g.standard_normal((N, K)), g.standard_normal(N)
    xt, wt = _t(x, torch.bfloat16), _t(w, torch.bfloat16)
    bt = _t(b, torch.float32)
    out = native.linear(xt, wt, bt, path=2).cpu().numpy()
    ref = xt.double().cpu().numpy() @ wt.double().cpu().numpy().T + b.astype(np.float32)
    err = np.abs(out - ref).max()
    assert err <= 1e-4 * np.sqrt(K) * 4, err
    # deterministic: a second call gives the same bits
    out2 = native.linear(xt, wt, bt, path=2).cpu().numpy()
    assert np.array_equal(out, out2)


@pytest.mark.parametrize("B,H,d,n,cap", [(64, 12, 64, 300, 544), (8, 16, 128, 2100, 2176),
                                         (256, 16, 64, 37, 544), (1, 1, 64, 1, 8),
                                         (100, 10, 64, 200, 208), (48, 12, 128, 77, 80)])
def test_decode_attention_bench_shapes(B, H, d, n, cap):
    """Decode attention at the workloads' shapes against the oracle's
    attention in fp64, in both partitions: whole (sequence, head) pairs per
    CTA (one, or an uneven two per CTA at 1,000 pairs) and stream-K (few
    pairs: pairs split across CTAs and merged)."""
    from hierarchical_global_local_b200 import native
    torch = gh.torch_mod()
    g = torch.Generator(device="cuda").manual_seed(B * 7 + n)
    q = torch.randn(B, H * d, device="cuda", generator=g).bfloat16()
    k = torch.randn(B, H, cap, d, device="cuda", generator=g).bfloat16()
    v = torch.randn(B, H, cap, d, device="cuda", generator=g).bfloat16()
    out = native.decode_attention(q, k, v, n).float().cpu().numpy()
    qr = q.double().cpu().numpy().reshape(B, 1, H, d)
    kr = k[:, :, :n].double().cpu().numpy().transpose(0, 2, 1, 3)
    vr = v[:, :, :n].double().cpu().numpy().transpose(0, 2, 1, 3)
    ref = om.attend(qr, kr, vr, np.array([n - 1]), np.arange(n)).reshape(B, H * d)
    assert np.abs(out - ref).max() <= 2e-2


@pytest.mark.parametrize("B,H,d,n,cap", [(2, 3, 64, 1, 8), (2, 2, 64, 37, 40), (1, 2, 64, 128, 128),
                                         (2, 2, 64, 300, 320), (1, 2, 128, 129, 136),
                                         (2, 1, 128, 513, 520)])
def test_prefill_attention_tensor_cores_matches_oracle(B, H, d, n, cap):
    """tcgen05 flash-attention prefill (query tiles of 128, causal and tail
    masking) against the oracle's causal attention in fp64."""
    from hierarchical_global_local_b200 import native
    torch = gh.torch_mod()
    g = torch.Generator(device="cuda").manual_seed(n * 13 + d)
    q = torch.randn(B * n, H * d, device="cuda", generator=g).bfloat16()
    k = torch.randn(B, H, cap, d, device="cuda", generator=g).bfloat16()
    v = torch.randn(B, H, cap, d, device="cuda", generator=g).bfloat16()
    # rows past n hold garbage in a real cache: make them huge to catch leaks
    k[:, :, n:] = 3e4
    v[:, :, n:] = float("nan")
    out = native.prefill_attention_tc(q, k, v, n).float().cpu().numpy()
    qr = q.double().cpu().numpy().reshape(B, n, H, d)
    kr = k[:, :, :n].double().cpu().numpy().transpose(0, 2, 1, 3)
    vr = v[:, :, :n].double().cpu().numpy().transpose(0, 2, 1, 3)
    ref = om.attend(qr, kr, vr, np.arange(n), np.arange(n)).reshape(B * n, H * d)
    assert np.isfinite(out).all()
    assert np.abs(out - ref).max() <= 3e-2
