"""Whole-model parity: CUDA path through the C-ABI vs the CPU oracle.

Tolerances: fp32 workloads, max |logit difference| <= 1e-4 at every
teacher-forced step; bf16 workloads, per-step relative L2 error of the
[B, V] logits <= 2e-2.
"""
import numpy as np
import pytest

import synth
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu

FP32_TOL = 1e-4
BF16_REL = 2e-2


def _run(shape, B, T, G, seed=3, rows=None, kind="uniform"):
    w = synth.make_weights(shape, seed=1000 + seed)
    toks = synth.make_tokens(batch=B, length=T + G, vocab=shape.vocab, kind=kind, seed=2000 + seed)
    model = gh.build_model(shape, w, max_batch=B, max_seq=T + G)
    gl, gn = gh.gpu_teacher_forced(model, toks, T, G)
    model.close()
    ol = gh.oracle_teacher_forced(shape, w, toks, T, G, rows=rows)
    if rows is not None:
        gl, gn = gl[:, rows], gn[:, rows]
    return gl, gn, ol


def test_tiny_fp32_workload_teacher_forced():
    wl = synth.WORKLOADS["tiny_fp32"]
    w = synth.make_weights(wl)
    toks = synth.make_tokens(wl)
    model = gh.build_model(wl.shape, w, wl.batch, wl.max_seq)
    gl, gn = gh.gpu_teacher_forced(model, toks, wl.prompt_len, wl.gen_len)
    model.close()
    ol = gh.oracle_teacher_forced(wl.shape, w, toks, wl.prompt_len, wl.gen_len)
    err = np.abs(gl - ol).max(axis=(1, 2))
    assert err.max() <= FP32_TOL, err
    # greedy ids are the argmax of the returned logits (lowest id on ties)
    assert np.array_equal(gn, gl.argmax(axis=-1))


@pytest.mark.parametrize("lb,P", [(4, 1), (2, 2), (8, 1)])
def test_small_bf16_block_transformer(lb, P):
    shape = synth.ModelShape(vocab=1000, d_model=256, n_heads=4, block_len=lb,
                             n_block_layers=2, n_token_layers=2, prefix_len=P)
    T = 12 * lb
    gl, gn, ol = _run(shape, B=3, T=T, G=3 * lb + 2)
    for s in range(gl.shape[0]):
        assert gh.rel_l2(gl[s], ol[s]) <= BF16_REL, (s, gh.rel_l2(gl[s], ol[s]))


@pytest.mark.parametrize("lb", [4, 8])
def test_small_bf16_layernorm_fused_in_gemm_epilogues(lb, monkeypatch):
    """The decode schedule that normalises in the residual GEMMs' epilogues
    (opt-in) gives the same logits as the oracle."""
    monkeypatch.setenv("BT_DECODE_LN", "fused")
    shape = synth.ModelShape(vocab=1000, d_model=256, n_heads=4, block_len=lb,
                             n_block_layers=2, n_token_layers=2, prefix_len=1)
    gl, gn, ol = _run(shape, B=3, T=8 * lb, G=3 * lb + 2, seed=5)
    for s in range(gl.shape[0]):
        assert gh.rel_l2(gl[s], ol[s]) <= BF16_REL, (s, gh.rel_l2(gl[s], ol[s]))


def test_small_bf16_vanilla_lb1():
    shape = synth.ModelShape(vocab=700, d_model=256, n_heads=2, block_len=1,
                             n_block_layers=3, n_token_layers=0, prefix_len=0,
                             use_token_decoder=False)
    gl, gn, ol = _run(shape, B=2, T=40, G=6)
    for s in range(gl.shape[0]):
        assert gh.rel_l2(gl[s], ol[s]) <= BF16_REL


def test_head_dim_128_bf16():
    shape = synth.ModelShape(vocab=500, d_model=512, n_heads=4, block_len=4,
                             n_block_layers=2, n_token_layers=1, prefix_len=1)
    gl, gn, ol = _run(shape, B=2, T=64, G=9)
    for s in range(gl.shape[0]):
        assert gh.rel_l2(gl[s], ol[s]) <= BF16_REL


def test_fp32_small_exact_tolerance_multi_prefix():
    shape = synth.ModelShape(vocab=300, d_model=128, n_heads=2, block_len=4,
                             n_block_layers=2, n_token_layers=2, prefix_len=3, dtype="fp32")
    gl, gn, ol = _run(shape, B=3, T=20, G=11)
    assert np.abs(gl - ol).max() <= FP32_TOL


def test_greedy_generation_feeds_own_argmax():
    shape = synth.ModelShape(vocab=300, d_model=128, n_heads=2, block_len=4,
                             n_block_layers=1, n_token_layers=1, prefix_len=1, dtype="fp32")
    torch = gh.torch_mod()
    w = synth.make_weights(shape, seed=77)
    B, T, G = 2, 16, 9
    toks = synth.make_tokens(batch=B, length=T, vocab=shape.vocab, seed=5)
    model = gh.build_model(shape, w, B, T + G)
    t = torch.from_numpy(toks).cuda()
    _, nxt = model.prefill(t)
    seq = [nxt.clone()]
    for _ in range(G - 1):
        _, nxt = model.decode(None)
        seq.append(nxt.clone())
    model.sync()
    gen = torch.stack(seq, 1).cpu().numpy()              # [B, G]
    model.close()
    full = np.concatenate([toks, gen], axis=1)
    ol = gh.oracle_teacher_forced(shape, w, full, T, G)  # oracle fed the same ids
    assert np.array_equal(ol.argmax(-1).T, gen)


def test_rows_are_independent_bitwise():
    shape = synth.ModelShape(vocab=512, d_model=256, n_heads=4, block_len=4,
                             n_block_layers=2, n_token_layers=2, prefix_len=1)
    w = synth.make_weights(shape, seed=11)
    B, T, G = 4, 32, 6
    toks = synth.make_tokens(batch=B, length=T + G, vocab=shape.vocab, seed=12)
    m = gh.build_model(shape, w, B, T + G)
    a, _ = gh.gpu_teacher_forced(m, toks, T, G)
    toks2 = toks.copy()
    toks2[2] = (toks2[2] + 17) % shape.vocab
    b, _ = gh.gpu_teacher_forced(m, toks2, T, G)
    m.close()
    assert np.array_equal(a[:, [0, 1, 3]], b[:, [0, 1, 3]])
    assert not np.array_equal(a[:, 2], b[:, 2])


def test_pythia160m_shape_sampled_rows():
    """Full-width Pythia-160M-scale model (V 50304, D 768, 6+6 layers) at a
    small batch and prompt; every step compared on all rows."""
    wl = synth.WORKLOADS["pythia160m_decode_heavy"]
    B, T, G = 3, 64, 10
    w = synth.make_weights(wl)
    toks = synth.make_tokens(wl, batch=B, length=T + G)
    m = gh.build_model(wl.shape, w, B, T + G)
    gl, _ = gh.gpu_teacher_forced(m, toks, T, G)
    m.close()
    ol = gh.oracle_teacher_forced(wl.shape, w, toks, T, G, dtype=np.float32)
    for s in range(G):
        assert gh.rel_l2(gl[s], ol[s]) <= BF16_REL, (s, gh.rel_l2(gl[s], ol[s]))


def test_fused_argmax_matches_returned_logits_bf16():
    """bf16 LM head: the greedy id computed in the GEMM epilogue equals the
    argmax of the logits the same call returns, at every step."""
    shape = synth.ModelShape(vocab=5000, d_model=256, n_heads=4, block_len=4,
                             n_block_layers=1, n_token_layers=1, prefix_len=1)
    w = synth.make_weights(shape, seed=21)
    B, T, G = 5, 24, 9
    toks = synth.make_tokens(batch=B, length=T + G, vocab=shape.vocab, seed=22)
    m = gh.build_model(shape, w, B, T + G)
    gl, gn = gh.gpu_teacher_forced(m, toks, T, G)
    m.close()
    assert np.array_equal(gn, gl.argmax(-1))


def _launches(model):
    from hierarchical_global_local_b200 import native
    return int(native.lib().bt_kernel_launches(model._h))


@pytest.mark.parametrize("lb,B,D,H,P,kind", [
    (4, 3, 256, 4, 1, "v2"), (8, 17, 256, 4, 1, "v2"), (2, 64, 256, 4, 1, "v2"),
    (4, 33, 512, 4, 2, "v2"),      # d_head 128, two prefix rows
    (8, 64, 256, 8, 1, "v2"),      # d_head 32, window of 8 rows
    (4, 5, 128, 4, 3, "v2"),       # one tile per GEMM row block, three prefix rows
    (4, 3, 256, 4, 1, "v1"), (8, 17, 256, 4, 1, "v1"),
    (2, 64, 1024, 16, 1, "v1")])    # too few CTAs left without items for GELU
def test_fused_token_step_matches_oracle_and_chain(lb, B, D, H, P, kind, monkeypatch):
    """The token-decoder half of a decode step as one persistent kernel (v1:
    grid barriers; v2: counter-synchronised, any prefix length): a token step is a
    single launch, its logits match the oracle, and they agree with the
    kernel-per-operation schedule on the same inputs."""
    monkeypatch.setenv("BT_DECODE_TOKEN_STEP", kind)
    shape = synth.ModelShape(vocab=3000, d_model=D, n_heads=H, block_len=lb,
                             n_block_layers=2, n_token_layers=3, prefix_len=P)
    T, G = 6 * lb, 3 * lb + 2
    w = synth.make_weights(shape, seed=31)
    toks = synth.make_tokens(batch=B, length=T + G, vocab=shape.vocab, seed=32)
    torch = gh.torch_mod()
    m = gh.build_model(shape, w, B, T + G)
    tok = torch.from_numpy(np.ascontiguousarray(toks)).cuda()
    m.prefill(tok[:, :T].contiguous())
    k0 = _launches(m)
    m.decode(tok[:, T].contiguous())  # position T: not the last of a block
    m.sync()
    assert _launches(m) - k0 == 1
    m.close()
    m = gh.build_model(shape, w, B, T + G)
    gl, gn = gh.gpu_teacher_forced(m, toks, T, G)
    m.close()
    monkeypatch.setenv("BT_DECODE_TOKEN_STEP", "chain")
    m = gh.build_model(shape, w, B, T + G)
    cl, cn = gh.gpu_teacher_forced(m, toks, T, G)
    m.close()
    ol = gh.oracle_teacher_forced(shape, w, toks, T, G)
    for s in range(G):
        assert gh.rel_l2(gl[s], ol[s]) <= BF16_REL, (s, gh.rel_l2(gl[s], ol[s]))
        assert gh.rel_l2(gl[s], cl[s]) <= 1e-2, (s, gh.rel_l2(gl[s], cl[s]))
    # greedy ids are the argmax of the returned logits (lowest id on ties)
    assert np.array_equal(gn, gl.argmax(axis=-1))


@pytest.mark.parametrize("lb,B,nbp", [(4, 5, 12), (8, 64, 12), (2, 33, 12), (2, 40, 70), (4, 64, 40)])
def test_fused_block_step_matches_oracle_and_chain(lb, B, nbp, monkeypatch):
    """A block step (block decoder with decode attention over the block cache,
    LN_b, the prefix projection, then the token decoder and the LM head) as
    one persistent kernel (opt-in): one launch per block step, logits match
    the oracle and agree with the kernel-per-operation block step. nbp prompt
    blocks: block caches of one unit of 32 entries and of several with a
    ragged last one, whose (sequence, head) runs are merged across warps."""
    monkeypatch.setenv("BT_DECODE_BLOCK_STEP", "fused")
    shape = synth.ModelShape(vocab=3000, d_model=256, n_heads=4, block_len=lb,
                             n_block_layers=3, n_token_layers=2, prefix_len=1)
    T, G = nbp * lb, 4 * lb + 3
    w = synth.make_weights(shape, seed=41)
    toks = synth.make_tokens(batch=B, length=T + G, vocab=shape.vocab, seed=42)
    torch = gh.torch_mod()
    m = gh.build_model(shape, w, B, T + G)
    tok = torch.from_numpy(np.ascontiguousarray(toks)).cuda()
    m.prefill(tok[:, :T].contiguous())
    for i in range(lb - 1):  # token steps up to the last position of the block
        m.decode(tok[:, T + i].contiguous())
    m.sync()
    k0 = _launches(m)
    m.decode(tok[:, T + lb - 1].contiguous())  # completes the block
    m.sync()
    assert _launches(m) - k0 == 1
    m.close()
    m = gh.build_model(shape, w, B, T + G)
    gl, gn = gh.gpu_teacher_forced(m, toks, T, G)
    m.close()
    monkeypatch.setenv("BT_DECODE_BLOCK_STEP", "chain")
    m = gh.build_model(shape, w, B, T + G)
    cl, cn = gh.gpu_teacher_forced(m, toks, T, G)
    m.close()
    ol = gh.oracle_teacher_forced(shape, w, toks, T, G)
    for s in range(G):
        assert gh.rel_l2(gl[s], ol[s]) <= BF16_REL, (s, gh.rel_l2(gl[s], ol[s]))
        assert gh.rel_l2(gl[s], cl[s]) <= 1e-2, (s, gh.rel_l2(gl[s], cl[s]))
    assert np.array_equal(gn, gl.argmax(axis=-1))


@pytest.mark.parametrize("lb,T,P", [(4, 49, 1), (4, 51, 1), (8, 61, 1), (2, 23, 2)])
def test_prompt_ending_inside_a_block_bf16(lb, T, P):
    """Prompt length not a multiple of L_B: the trailing tokens are prefilled
    into the token decoder after the prefix; every following step (token and
    block steps) matches the oracle."""
    shape = synth.ModelShape(vocab=1000, d_model=256, n_heads=4, block_len=lb,
                             n_block_layers=2, n_token_layers=2, prefix_len=P)
    gl, gn, ol = _run(shape, B=3, T=T, G=2 * lb + 3, seed=7)
    for s in range(gl.shape[0]):
        assert gh.rel_l2(gl[s], ol[s]) <= BF16_REL, (s, gh.rel_l2(gl[s], ol[s]))
    assert np.array_equal(gn, gl.argmax(axis=-1))


def test_prompt_ending_inside_a_block_fp32():
    """The fp32 workload shape with a prompt of 66 tokens (16 blocks + 2),
    max |logit difference| <= 1e-4 at every step."""
    wl = synth.WORKLOADS["tiny_fp32"]
    gl, gn, ol = _run(wl.shape, B=2, T=66, G=11, seed=8)
    err = np.abs(gl - ol).max(axis=(1, 2))
    assert err.max() <= FP32_TOL, err


def _ragged_run(shape, lengths, pad_id, G, seed):
    """Ragged batch through bt_prefill_ragged + teacher-forced decode calls;
    the oracle runs each sequence on its own."""
    from oracle.model import BlockTransformerOracle, ragged_generate_logits
    torch = gh.torch_mod()
    B = len(lengths)
    L = shape.block_len
    w = synth.make_weights(shape, seed=1000 + seed)
    stride = max(lengths) + G
    toks = synth.make_tokens(batch=B, length=stride, vocab=shape.vocab, seed=2000 + seed)
    padded = [n + ((L - n % L) % L if pad_id >= 0 else 0) for n in lengths]
    model = gh.build_model(shape, w, max_batch=B, max_seq=max(padded) + G)
    tok = torch.from_numpy(np.ascontiguousarray(toks)).cuda()
    logits = torch.empty(G, B, shape.vocab, dtype=torch.float32, device="cuda")
    nxt = torch.empty(G, B, dtype=torch.int32, device="cuda")
    model.prefill_ragged(tok, lengths, pad_id, logits=logits[0], next_tokens=nxt[0])
    for i in range(G - 1):
        feed = torch.tensor([int(toks[b, lengths[b] + i]) for b in range(B)], dtype=torch.int32,
                            device="cuda")
        model.decode(feed, logits=logits[i + 1], next_tokens=nxt[i + 1])
    model.sync()
    assert model.position == max(padded) + G - 1
    gl, gn = logits.cpu().numpy(), nxt.cpu().numpy()
    model.close()
    o = BlockTransformerOracle(shape, {n: w.values(n) for n in w.names()})
    ol = ragged_generate_logits(o, [toks[b, :lengths[b]] for b in range(B)],
                                [toks[b, lengths[b]:] for b in range(B)], G,
                                pad=pad_id >= 0, pad_id=max(pad_id, 0))
    return gl, gn, ol


@pytest.mark.parametrize("lb,pad_id,lengths", [
    (4, 0, [37, 50, 64, 41]),        # left padding to a block boundary
    (4, -1, [37, 41, 49, 53]),       # no padding, equal remainders (1)
    (8, 11, [29, 64, 9, 40, 17]),    # left padding, L_B 8
    (2, -1, [20, 34, 12]),           # no padding, aligned
])
def test_ragged_batch_matches_each_sequence_alone(lb, pad_id, lengths):
    """Sequences of different prompt lengths in one batch: every sequence's
    logits, at every step, match the oracle run on that sequence alone (its
    own number of blocks in the block decoder's cache)."""
    shape = synth.ModelShape(vocab=1000, d_model=256, n_heads=4, block_len=lb,
                             n_block_layers=2, n_token_layers=2, prefix_len=1)
    G = 2 * lb + 3
    gl, gn, ol = _ragged_run(shape, lengths, pad_id, G, seed=9)
    for b in range(len(lengths)):
        for s in range(G):
            e = gh.rel_l2(gl[s, b], ol[b][s])
            assert e <= BF16_REL, (b, s, e)
    assert np.array_equal(gn, gl.argmax(axis=-1))


def test_ragged_batch_fp32_and_vanilla():
    """fp32 (max |diff| <= 1e-4) ragged batch with padding, and the vanilla
    L_B = 1 model on a ragged batch."""
    wl = synth.WORKLOADS["tiny_fp32"]
    gl, _, ol = _ragged_run(wl.shape, [33, 64, 50], 5, 9, seed=10)
    for b in range(3):
        assert np.abs(gl[:, b] - ol[b]).max() <= FP32_TOL, b
    van = synth.ModelShape(vocab=800, d_model=256, n_heads=4, block_len=1, n_block_layers=3,
                           n_token_layers=0, prefix_len=0, use_token_decoder=False)
    gl, _, ol = _ragged_run(van, [21, 40, 33], -1, 6, seed=11)
    for b in range(3):
        for s in range(6):
            assert gh.rel_l2(gl[s, b], ol[b][s]) <= BF16_REL, (b, s)


def test_ragged_prefill_rejects_bad_lengths():
    from hierarchical_global_local_b200 import native
    torch = gh.torch_mod()
    shape = synth.ModelShape(vocab=500, d_model=256, n_heads=4, block_len=4,
                             n_block_layers=1, n_token_layers=1, prefix_len=1)
    w = synth.make_weights(shape, seed=3)
    m = gh.build_model(shape, w, 3, 80)
    tok = torch.zeros(3, 40, dtype=torch.int32, device="cuda")
    for lengths, pad in (([12, 13, 12], -1), ([0, 12, 12], 0), ([41, 12, 12], 0), ([12, 12, 12], 500)):
        with pytest.raises(native.BtError) as ei:
            m.prefill_ragged(tok, lengths, pad)
        assert ei.value.code == native.BT_EINVAL, (lengths, pad)
    m.close()


# ---- context-injection variants: summation (MEGABYTE-style) and a window of
# previous context embeddings, against the oracle's readings of them

@pytest.mark.parametrize("lb,T", [(4, 20), (4, 22), (2, 9), (8, 35)])
def test_fp32_summation_injection_exact_tolerance(lb, T):
    """Prompts ending on and inside a block (trailing tokens carry s_{j+1}),
    decode across several blocks."""
    shape = synth.ModelShape(vocab=300, d_model=128, n_heads=2, block_len=lb,
                             n_block_layers=2, n_token_layers=2, prefix_len=1, dtype="fp32",
                             injection="sum")
    gl, gn, ol = _run(shape, B=3, T=T, G=3 * lb + 3)
    assert np.abs(gl - ol).max() <= FP32_TOL


@pytest.mark.parametrize("w,P,T", [(2, 1, 20), (3, 1, 4), (3, 2, 10), (4, 1, 13)])
def test_fp32_context_window_exact_tolerance(w, P, T):
    """Windows longer than the prompt's blocks (zero context slots) and
    prompts ending inside a block; decode across several blocks so that the
    window moves on."""
    shape = synth.ModelShape(vocab=300, d_model=128, n_heads=2, block_len=4,
                             n_block_layers=2, n_token_layers=2, prefix_len=P, dtype="fp32",
                             context_window=w)
    gl, gn, ol = _run(shape, B=3, T=T, G=15)
    assert np.abs(gl - ol).max() <= FP32_TOL


@pytest.mark.parametrize("variant", [{"injection": "sum"}, {"context_window": 3}])
def test_bf16_context_variants(variant):
    shape = synth.ModelShape(vocab=1000, d_model=256, n_heads=4, block_len=4,
                             n_block_layers=2, n_token_layers=2, prefix_len=1, **variant)
    gl, gn, ol = _run(shape, B=3, T=26, G=14)
    for s in range(gl.shape[0]):
        assert gh.rel_l2(gl[s], ol[s]) <= BF16_REL, (s, gh.rel_l2(gl[s], ol[s]))


def test_context_window_refuses_ragged_batches():
    from hierarchical_global_local_b200 import native
    torch = gh.torch_mod()
    shape = synth.ModelShape(vocab=300, d_model=128, n_heads=2, block_len=4,
                             n_block_layers=1, n_token_layers=1, prefix_len=1, dtype="fp32",
                             context_window=2)
    model = gh.build_model(shape, synth.make_weights(shape, seed=3), 2, 32)
    toks = torch.zeros(2, 12, dtype=torch.int32, device="cuda")
    with pytest.raises(native.BtError) as e:
        model.prefill_ragged(toks, [12, 9])
    assert e.value.code == native.BT_ENOTSUP
    model.close()


# ---- grouped-query attention in the block decoder ---------------------------

@pytest.mark.parametrize("hk", [1, 2])
def test_fp32_gqa_block_decoder_exact_tolerance(hk):
    shape = synth.ModelShape(vocab=300, d_model=128, n_heads=4, block_len=4,
                             n_block_layers=2, n_token_layers=2, prefix_len=1, dtype="fp32",
                             n_kv_heads=hk)
    gl, gn, ol = _run(shape, B=3, T=22, G=14)
    assert np.abs(gl - ol).max() <= FP32_TOL


@pytest.mark.parametrize("H,hk", [(4, 1), (4, 2), (2, 1)])
def test_bf16_gqa_block_decoder(H, hk):
    """d_head 64 and 128: tensor-core prefill attention and the decode
    attention kernel read key/value head h / (H / H_kv)."""
    shape = synth.ModelShape(vocab=1000, d_model=256, n_heads=H, block_len=4,
                             n_block_layers=2, n_token_layers=2, prefix_len=1, n_kv_heads=hk)
    gl, gn, ol = _run(shape, B=3, T=64, G=14)
    for s in range(gl.shape[0]):
        assert gh.rel_l2(gl[s], ol[s]) <= BF16_REL, (s, gh.rel_l2(gl[s], ol[s]))
