"""Pins of the CPU oracle to things other than itself.

Each function returns a discrepancy (max abs difference, or a bool for the
bitwise invariants) between the oracle and an independent source:

* HF ``transformers`` GPTNeoX (an independent Pythia implementation) for the
  layer stack, the vanilla special case and the whole model assembled from
  two stacks;
* torch CPU functional ops for LayerNorm, GELU and attention;
* a complex-number statement of rotary embedding;
* brute-force loops for the embedder;
* closed forms (identity prefix projection, single-row token decoder);
* the locality/causality invariants of the method.

They take the oracle *module* as an argument so the mutation test can run
the same pins against a deliberately broken copy.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

import synth

SMALL = synth.ModelShape(vocab=97, d_model=64, n_heads=4, block_len=4,
                         n_block_layers=2, n_token_layers=2, prefix_len=2,
                         dtype="fp32")
VANILLA = synth.ModelShape(vocab=97, d_model=64, n_heads=4, block_len=1,
                           n_block_layers=3, n_token_layers=0, prefix_len=0,
                           use_token_decoder=False, dtype="fp32")


def params_of(shape, seed=7):
    w = synth.make_weights(shape, seed=seed)
    return {n: w.values(n) for n in w.names()}


def tokens_of(shape, B=2, S=24, seed=11):
    return synth.make_tokens(batch=B, length=S, vocab=shape.vocab, kind="uniform", seed=seed)


# --------------------------------------------------------------------------
# HF GPTNeoX stacks
# --------------------------------------------------------------------------

def _hf_model(shape, n_layers, vocab):
    from transformers import GPTNeoXConfig, GPTNeoXModel
    cfg = GPTNeoXConfig(
        vocab_size=vocab, hidden_size=shape.d_model, num_hidden_layers=n_layers,
        num_attention_heads=shape.n_heads, intermediate_size=4 * shape.d_model,
        hidden_act="gelu", max_position_embeddings=4096,
        rope_parameters={"rope_type": "default", "rope_theta": shape.rope_base,
                         "partial_rotary_factor": shape.rotary_pct},
        layer_norm_eps=shape.ln_eps, use_parallel_residual=True,
        attention_bias=True, hidden_dropout=0.0, attention_dropout=0.0,
        tie_word_embeddings=False)
    cfg._attn_implementation = "eager"
    return GPTNeoXModel(cfg).double().eval()


def _load_stack(model, shape, params, prefix, n_layers, fin_g, fin_b):
    D, H = shape.d_model, shape.n_heads
    d = D // H
    t = lambda a: torch.tensor(np.asarray(a, dtype=np.float64))
    with torch.no_grad():
        for l in range(n_layers):
            p = lambda n: params[f"{prefix}.{l}.{n}"]
            L = model.layers[l]
            L.input_layernorm.weight.copy_(t(p("ln1_g")))
            L.input_layernorm.bias.copy_(t(p("ln1_b")))
            L.post_attention_layernorm.weight.copy_(t(p("ln2_g")))
            L.post_attention_layernorm.bias.copy_(t(p("ln2_b")))
            # our rows: [q (H x d) | k | v]; HF rows: per head [q_h | k_h | v_h]
            w = np.asarray(p("w_qkv")).reshape(3, H, d, D).transpose(1, 0, 2, 3).reshape(3 * D, D)
            b = np.asarray(p("b_qkv")).reshape(3, H, d).transpose(1, 0, 2).reshape(3 * D)
            L.attention.query_key_value.weight.copy_(t(w))
            L.attention.query_key_value.bias.copy_(t(b))
            L.attention.dense.weight.copy_(t(p("w_o")))
            L.attention.dense.bias.copy_(t(p("b_o")))
            L.mlp.dense_h_to_4h.weight.copy_(t(p("w_1")))
            L.mlp.dense_h_to_4h.bias.copy_(t(p("b_1")))
            L.mlp.dense_4h_to_h.weight.copy_(t(p("w_2")))
            L.mlp.dense_4h_to_h.bias.copy_(t(p("b_2")))
        model.final_layer_norm.weight.copy_(t(params[fin_g]))
        model.final_layer_norm.bias.copy_(t(params[fin_b]))


def hf_stack_fn(shape, params, prefix, n_layers, fin_g, fin_b):
    """Return f(rows [B, n, D] float64) -> final-normed hidden [B, n, D]."""
    model = _hf_model(shape, n_layers, vocab=8)
    _load_stack(model, shape, params, prefix, n_layers, fin_g, fin_b)

    def f(rows):
        with torch.no_grad():
            x = torch.tensor(np.asarray(rows, dtype=np.float64))
            return model(inputs_embeds=x).last_hidden_state.numpy()
    return f


def pin_vanilla_vs_hf(om) -> float:
    """Invariant 3: L_B = 1 with no token decoder is a vanilla causal Pythia
    (HF GPTNeoXForCausalLM semantics: embed, stack, final norm, LM head)."""
    shape, params = VANILLA, params_of(VANILLA)
    toks = tokens_of(shape, S=19)
    ours = om.BlockTransformerOracle(shape, params).forward_full(toks)[:, 1:]
    f = hf_stack_fn(shape, params, "block", shape.n_block_layers, "lnf_b_g", "lnf_b_b")
    emb = params["blk_emb"][toks].astype(np.float64)
    ref = f(emb) @ params["w_lm"].astype(np.float64).T
    return float(np.abs(ours - ref).max())


def pin_block_model_vs_hf(om) -> float:
    """The full Block Transformer assembled from two HF stacks: block decoder
    over concatenated block embeddings, linear prefix, token decoder over
    [prefix; shifted block tokens], LM head on the token decoder's rows."""
    shape, params = SMALL, params_of(SMALL)
    S = 22   # 5 complete blocks + a partial one
    toks = tokens_of(shape, S=S)
    ours = om.BlockTransformerOracle(shape, params).forward_full(toks)
    fb = hf_stack_fn(shape, params, "block", shape.n_block_layers, "lnf_b_g", "lnf_b_b")
    ft = hf_stack_fn(shape, params, "token", shape.n_token_layers, "lnf_t_g", "lnf_t_b")
    B = toks.shape[0]
    L, P, D = shape.block_len, shape.prefix_len, shape.d_model
    n = S // L
    f64 = lambda n_: params[n_].astype(np.float64)
    err = 0.0
    for b in range(B):
        e = np.stack([np.concatenate([f64("blk_emb")[toks[b, i * L + j]] for j in range(L)])
                      for i in range(n)])
        c = fb(e[None])[0]
        for k in range(1, n + 1):
            pre = (f64("w_prefix") @ c[k - 1] + f64("b_prefix")).reshape(P, D)
            rows = [pre[i] for i in range(P)]
            rows += [f64("tok_emb")[toks[b, k * L + j]] for j in range(L - 1) if k * L + j < S]
            hid = ft(np.stack(rows)[None])[0]
            for j in range(L):
                t = k * L + j
                if t <= S and P - 1 + j < len(rows):
                    z = f64("w_lm") @ hid[P - 1 + j]
                    err = max(err, float(np.abs(ours[b, t] - z).max()))
    return err


# --------------------------------------------------------------------------
# primitive pins
# --------------------------------------------------------------------------

def pin_layer_norm(om) -> float:
    g = np.random.default_rng(1)
    x = g.standard_normal((5, 48)) * 3 + 1
    w, b = g.standard_normal(48), g.standard_normal(48)
    ref = torch.nn.functional.layer_norm(torch.tensor(x), (48,), torch.tensor(w),
                                         torch.tensor(b), eps=1e-5).numpy()
    return float(np.abs(om.layer_norm(x, w, b, 1e-5) - ref).max())


def pin_gelu(om) -> float:
    x = np.linspace(-6, 6, 1001)
    ref = torch.nn.functional.gelu(torch.tensor(x)).numpy()
    return float(np.abs(om.gelu(x) - ref).max())


def pin_attend(om) -> float:
    g = np.random.default_rng(2)
    q = g.standard_normal((2, 7, 3, 8))
    k = g.standard_normal((2, 7, 3, 8))
    v = g.standard_normal((2, 7, 3, 8))
    ours = om.attend(q, k, v, np.arange(7), np.arange(7))
    T = lambda a: torch.tensor(a).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(T(q), T(k), T(v), is_causal=True)
    return float(np.abs(ours - ref.permute(0, 2, 1, 3).numpy()).max())


def pin_rotary(om) -> float:
    """Rotary as complex multiplication: (x_i + i x_{i+r/2}) * exp(i pos w_i)."""
    g = np.random.default_rng(3)
    n, H, d, r, base = 9, 2, 16, 8, 10000.0
    x = g.standard_normal((1, n, H, d))
    pos = np.arange(n) * 3 + 1
    ours = om.rotary(x, pos, r, base)
    half = r // 2
    w = np.array([base ** (-(2.0 * i) / r) for i in range(half)])
    z = (x[..., :half] + 1j * x[..., half:r]) * np.exp(1j * pos[:, None, None] * w)
    ref = x.copy()
    ref[..., :half], ref[..., half:r] = z.real, z.imag
    return float(np.abs(ours - ref).max())


# --------------------------------------------------------------------------
# brute force / closed forms
# --------------------------------------------------------------------------

def pin_embedder_bruteforce(om) -> float:
    g = np.random.default_rng(4)
    V, L, De = 13, 4, 5
    table = g.standard_normal((V, De))
    toks = g.integers(0, V, size=(3, 12))
    ours = om.embed_blocks(toks, table, L)
    err = 0.0
    for b in range(3):
        for i in range(3):
            for j in range(L):
                for e in range(De):
                    err = max(err, abs(ours[b, i, j * De + e] - table[toks[b, i * L + j], e]))
    return float(err)


def pin_identity_prefix(om) -> float:
    """W_p = I, b_p = 0, P = 1 => the single prefix row equals c."""
    g = np.random.default_rng(5)
    c = g.standard_normal((3, 16))
    p = om.prefix_projection(c, np.eye(16), np.zeros(16), 1)
    return float(np.abs(p[:, 0] - c).max())


def pin_single_row_token_decoder(om) -> float:
    """L_B = 1, P = 1: the token decoder sees one row, so attention returns
    that row's value vector; the layer reduces to a closed form without
    softmax or rotary."""
    shape = synth.ModelShape(vocab=31, d_model=32, n_heads=2, block_len=1,
                             n_block_layers=1, n_token_layers=2, prefix_len=1,
                             dtype="fp32")
    params = params_of(shape, seed=9)
    toks = tokens_of(shape, S=6, seed=3)
    pred = om.BlockTransformerOracle(shape, params).forward_full(toks)
    P64 = {k: np.asarray(v, dtype=np.float64) for k, v in params.items()}
    D = shape.d_model

    def ln(x, g, b):
        mu = x.mean(-1, keepdims=True)
        return (x - mu) / np.sqrt(((x - mu) ** 2).mean(-1, keepdims=True) + 1e-5) * g + b

    def gel(x):
        return 0.5 * x * (1 + np.vectorize(math.erf)(x / math.sqrt(2)))

    # block decoder output from the oracle itself is taken as given: this
    # pin isolates the token decoder + prefix + head.
    o = om.BlockTransformerOracle(shape, params)
    e = om.embed_blocks(toks, o.g["blk_emb"], 1)
    from oracle.model import KVCache  # cache type only
    c = o.block_decoder(e, np.arange(e.shape[1]), [KVCache()])
    err = 0.0
    for t in range(1, toks.shape[1] + 1):
        h = c[:, t - 1] @ P64["w_prefix"].T + P64["b_prefix"]
        for l in range(2):
            p = lambda n: P64[f"token.{l}.{n}"]
            v = (ln(h, p("ln1_g"), p("ln1_b")) @ p("w_qkv").T + p("b_qkv"))[:, 2 * D:]
            m = ln(h, p("ln2_g"), p("ln2_b"))
            h = h + v @ p("w_o").T + p("b_o") + gel(m @ p("w_1").T + p("b_1")) @ p("w_2").T + p("b_2")
        z = ln(h, P64["lnf_t_g"], P64["lnf_t_b"]) @ P64["w_lm"].T
        err = max(err, float(np.abs(pred[:, t] - z).max()))
    return err


# --------------------------------------------------------------------------
# invariants
# --------------------------------------------------------------------------

def pin_incremental_equals_full(om, shape=SMALL, T=8, G=11) -> float:
    """Invariant 1: prefill + one-token decode steps reproduce the
    teacher-forced full-sequence logits at every generated position."""
    params = params_of(shape)
    toks = tokens_of(shape, S=T + G)
    o = om.BlockTransformerOracle(shape, params)
    full = o.forward_full(toks)
    inc = o.session().generate_logits(toks, T, G)
    return float(np.abs(inc - full[:, T:T + G].transpose(1, 0, 2)).max())


def pin_left_padding(om) -> bool:
    """Left padding: p = (-T) mod L_B pad ids in front, p = 0 for aligned
    prompts; prefill of the padded prompt equals the full pass over the
    padded sequence at the position after the prompt."""
    L = SMALL.block_len
    ok = True
    for T in range(1, 13):
        x = np.arange(100, 100 + T)
        y = om.left_pad(x, L, 7)
        p = (L - T % L) % L
        ok &= y.shape[0] == T + p and (y.shape[0] % L == 0)
        ok &= bool(np.all(y[:p] == 7)) and bool(np.array_equal(y[p:], x))
    params = params_of(SMALL)
    toks = tokens_of(SMALL, B=1, S=17)
    o = om.BlockTransformerOracle(SMALL, params)
    for T in (5, 7, 8):
        padded = om.left_pad(toks[0, :T], L, 3)
        seq = np.concatenate([padded, toks[0, T:]])[None]
        z = o.session().prefill(padded[None])
        full = o.forward_full(seq)
        ok &= float(np.abs(z - full[:, padded.shape[0]]).max()) < 1e-10
    return ok


def pin_ragged_vs_batched(om) -> float:
    """Ragged runs (one session per sequence) against the batched session:
    equal prompt lengths give the batched logits row for row."""
    params = params_of(SMALL)
    o = om.BlockTransformerOracle(SMALL, params)
    toks = tokens_of(SMALL, B=3, S=20)
    T, G = 9, 6
    batched = o.session().generate_logits(toks, T, G)           # [G, B, V]
    rag = om.ragged_generate_logits(o, [toks[b, :T] for b in range(3)],
                                    [toks[b, T:] for b in range(3)], G)
    return float(max(np.abs(rag[b] - batched[:, b]).max() for b in range(3)))


def pin_future_tokens_invisible(om) -> bool:
    """Invariant 2a: logits for x_t are bitwise unchanged when any x_t',
    t' >= t, is perturbed."""
    shape, params = SMALL, params_of(SMALL)
    toks = tokens_of(shape, S=20)
    o = om.BlockTransformerOracle(shape, params)
    base = o.forward_full(toks)
    ok = True
    for tp in (5, 8, 13, 19):
        x = toks.copy()
        x[:, tp] = (x[:, tp] + 1) % shape.vocab
        pert = o.forward_full(x)
        ok &= bool(np.array_equal(base[:, :tp + 1], pert[:, :tp + 1], equal_nan=True))
        ok &= not np.array_equal(base[:, tp + 1:], pert[:, tp + 1:])
    return ok


def pin_locality_without_block_layers(om) -> bool:
    """Invariant 2c: with no block-decoder layers, c_{k-1} = LN_b(e_{k-1}),
    so block k's logits depend only on blocks k-1 and k."""
    shape = synth.ModelShape(vocab=53, d_model=32, n_heads=2, block_len=4,
                             n_block_layers=0, n_token_layers=2, prefix_len=1,
                             dtype="fp32")
    params = params_of(shape, seed=5)
    toks = tokens_of(shape, S=24, seed=6)
    o = om.BlockTransformerOracle(shape, params)
    base = o.forward_full(toks)
    k = 4                                    # predicted block: positions 16..19
    ok = True
    for tp in range(0, 12):                  # blocks 0..2: invisible to block 4
        x = toks.copy()
        x[:, tp] = (x[:, tp] + 1) % shape.vocab
        ok &= bool(np.array_equal(o.forward_full(x)[:, 16:20], base[:, 16:20]))
    x = toks.copy()
    x[:, 13] = (x[:, 13] + 1) % shape.vocab  # block 3 feeds the prefix
    ok &= not np.array_equal(o.forward_full(x)[:, 16:20], base[:, 16:20])
    return ok


def pin_token_decoder_local(om) -> bool:
    """Invariant 2b: holding c_{k-1} fixed, block k's logits are bitwise
    unchanged when any token outside block k changes: run the token decoder
    of block k on the unperturbed c_{k-1} with tokens from a sequence that
    differs outside block k, and compare with the unperturbed logits."""
    shape, params = SMALL, params_of(SMALL)
    toks = tokens_of(shape, S=20)
    o = om.BlockTransformerOracle(shape, params)
    base = o.forward_full(toks)
    L, P = shape.block_len, shape.prefix_len
    e = om.embed_blocks(toks, o.g["blk_emb"], L)
    from oracle.model import KVCache
    c = o.block_decoder(e, np.arange(e.shape[1]), [KVCache() for _ in o.block_layers])
    k = 3
    x = toks.copy()
    x[:, :k * L] = (x[:, :k * L] + 5) % shape.vocab     # everything before block k
    x[:, (k + 1) * L:] = (x[:, (k + 1) * L:] + 7) % shape.vocab
    pre = om.prefix_projection(c[:, k - 1], o.g["w_prefix"], o.g["b_prefix"], P)
    rows = np.concatenate([pre, o.g["tok_emb"][x[:, k * L:k * L + L - 1]]], axis=1)
    z = o.token_decoder(rows, np.arange(P + L - 1), [KVCache() for _ in o.token_layers])
    return bool(np.allclose(z[:, P - 1:], base[:, k * L:(k + 1) * L], rtol=0, atol=1e-12))


def pin_batch_rows_independent(om) -> bool:
    shape, params = SMALL, params_of(SMALL)
    toks = tokens_of(shape, B=3, S=16)
    o = om.BlockTransformerOracle(shape, params)
    base = o.forward_full(toks)
    x = toks.copy()
    x[1] = (x[1] + 3) % shape.vocab
    pert = o.forward_full(x)
    return bool(np.allclose(base[[0, 2]], pert[[0, 2]], rtol=0, atol=1e-12, equal_nan=True))


# --------------------------------------------------------------------------
# context injection variants: summation (reading R9) and a window of previous
# context embeddings (reading R10)
# --------------------------------------------------------------------------

SUM = dataclasses.replace(SMALL, injection="sum", prefix_len=1)
WIN = dataclasses.replace(SMALL, context_window=3)


def pin_sum_injection_reduces_to_prefix(om) -> float:
    """Summation injection whose vectors s_1..s_{L_B-1} are zero (projection
    rows and bias beyond the first D) is the prefix model with P = 1 whose
    projection is the first D rows."""
    D = SUM.d_model
    ps = params_of(SUM)
    ps["w_prefix"] = ps["w_prefix"].copy()
    ps["b_prefix"] = ps["b_prefix"].copy()
    ps["w_prefix"][D:] = 0.0
    ps["b_prefix"][D:] = 0.0
    pp = dict(ps)
    pp["w_prefix"] = ps["w_prefix"][:D]
    pp["b_prefix"] = ps["b_prefix"][:D]
    toks = tokens_of(SUM, S=22)
    a = om.BlockTransformerOracle(SUM, ps).forward_full(toks)
    b = om.BlockTransformerOracle(dataclasses.replace(SUM, injection="prefix"), pp).forward_full(toks)
    return float(np.nanmax(np.abs(a - b)))


def pin_sum_injection_slot_reach(om) -> bool:
    """s_j is added to the input of in-block row j (row 0 holds s_0 alone):
    under the causal token decoder, changing slot j of the projection's
    bias changes exactly the predictions of in-block offsets j..L_B-1 of
    every block, and none before."""
    L, D = SUM.block_len, SUM.d_model
    ps = params_of(SUM)
    toks = tokens_of(SUM, S=20)
    base = om.BlockTransformerOracle(SUM, ps).forward_full(toks)
    ok = True
    for j in range(L):
        q = dict(ps)
        q["b_prefix"] = ps["b_prefix"].copy()
        q["b_prefix"][j * D:(j + 1) * D] += 0.5
        got = om.BlockTransformerOracle(SUM, q).forward_full(toks)
        for k in range(1, toks.shape[1] // L + 1):
            for jj in range(L):
                t = k * L + jj
                if t > toks.shape[1]:
                    continue
                changed = bool(np.any(np.abs(got[:, t] - base[:, t]) > 1e-9))
                ok &= changed == (jj >= j)
    return ok


def pin_window_assembly_bruteforce(om) -> float:
    """The token decoder of block k sees the projections of c_{k-w} ..
    c_{k-1}, oldest first, zero vectors before block 0, then the block's
    tokens: rebuild that input by hand from the block decoder's outputs
    (projection written out as a loop over the P output rows) and compare
    with the full pass."""
    w, P, L, D = WIN.context_window, WIN.prefix_len, WIN.block_len, WIN.d_model
    ps = params_of(WIN)
    toks = tokens_of(WIN, S=21)
    o = om.BlockTransformerOracle(WIN, ps)
    full = o.forward_full(toks)
    B, S = toks.shape
    n = S // L
    e = om.embed_blocks(toks, o.g["blk_emb"], L)
    c = o.block_decoder(e, np.arange(n), o._fresh(o.block_layers))
    W, bias = o.g["w_prefix"], o.g["b_prefix"]
    worst = 0.0
    for k in range(1, n + 1):
        rows = []
        for i in range(k - w, k):
            ci = c[:, i] if i >= 0 else np.zeros((B, D))
            for r in range(P):
                rows.append(ci @ W[r * D:(r + 1) * D].T + bias[r * D:(r + 1) * D])
        for j in range(L - 1):
            t = k * L + j
            rows.append(o.g["tok_emb"][toks[:, min(t, S - 1)]])
        u = np.stack(rows, axis=1)
        z = o.token_decoder(u, np.arange(u.shape[1]), o._fresh(o.token_layers))
        for j in range(L):
            t = k * L + j  # predicted from the tokens before it: defined for t <= S
            if t <= S:
                worst = max(worst, float(np.abs(z[:, w * P - 1 + j] - full[:, t]).max()))
    return worst


# --------------------------------------------------------------------------
# grouped-query attention in the block decoder (reading R11)
# --------------------------------------------------------------------------

GQA = dataclasses.replace(SMALL, n_kv_heads=2)


def pin_gqa_equals_mha_with_shared_kv_rows(om) -> float:
    """GQA with H_kv heads is multi-head attention whose query head h uses
    copies of key/value head h // (H / H_kv): duplicate those projection
    rows (a loop over the H query heads) into an MHA model and compare the
    full pass."""
    H, hk, D = GQA.n_heads, GQA.n_kv_heads, GQA.d_model
    d, g = D // H, H // GQA.n_kv_heads
    pg = params_of(GQA)
    pm = dict(pg)
    for l in range(GQA.n_block_layers):
        w, b = pg[f"block.{l}.w_qkv"], pg[f"block.{l}.b_qkv"]
        wk, wv = w[D:D + hk * d], w[D + hk * d:D + 2 * hk * d]
        bk, bv = b[D:D + hk * d], b[D + hk * d:D + 2 * hk * d]
        rk, rv, ck, cv = [], [], [], []
        for h in range(H):
            j = h // g
            rk.append(wk[j * d:(j + 1) * d])
            rv.append(wv[j * d:(j + 1) * d])
            ck.append(bk[j * d:(j + 1) * d])
            cv.append(bv[j * d:(j + 1) * d])
        pm[f"block.{l}.w_qkv"] = np.concatenate([w[:D]] + rk + rv, axis=0)
        pm[f"block.{l}.b_qkv"] = np.concatenate([b[:D]] + ck + cv, axis=0)
    toks = tokens_of(GQA, S=22)
    a = om.BlockTransformerOracle(GQA, pg).forward_full(toks)
    m = om.BlockTransformerOracle(dataclasses.replace(GQA, n_kv_heads=0), pm).forward_full(toks)
    return float(np.nanmax(np.abs(a - m)))
