"""CPU oracle of the Block Transformer's global-to-local inference path.

TEST INFRASTRUCTURE ONLY. This module is the slow, plain reference that the
CUDA path is checked against. Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import it; the product path never does.

Sources. The method is the Block Transformer (arXiv 2406.02657) as described
on the explainer page "Block Transformer: Global-to-Local Language Modeling
for Fast Inference" (cited below as [BT] with its section numbers; "orig."
names the original paper's section that the page paraphrases). The page
describes the model in prose; this file restates it in numpy, fp64 by
default, batch rows vectorised, no blocking or fusion.

Readings where the page is silent (each listed again in the design notes):
  R1  The token decoder of block k sees P prefix rows followed by the first
      L_B - 1 tokens of block k (teacher forcing "shifted by one",
      [BT] §3.4 "The Block Decoder", training task step 4); row P-1+j
      predicts token j of block k.
  R2  Concatenation order: token j of a block fills dims [j*D/L_B, (j+1)*D/L_B).
  R3  A final LayerNorm follows each decoder stack (Pythia's final norm):
      LN_b before the prefix projection (and before the LM head in vanilla
      mode), LN_t before the LM head.
  R4  Proj is one linear layer with bias, reshaped row-major: p_k is
      dims [(k-1)D, kD) of W_p c + b_p.
  R5  Positions: block decoder uses the block index; token decoder uses
      0..P+L_B-2 (prefix first), restarting every block.
  R6  Pythia layer: parallel residual, LayerNorm (eps 1e-5, biased
      variance), rotary on the first 25% of each head's dims (rotate-half
      pairing i <-> i + r/2, inv_freq_i = base^(-2i/r), base 10000),
      exact-erf GELU, 4x MLP, scores scaled by 1/sqrt(d_head), untied LM
      head without bias, no embedding norm.
  R7  Inference left padding adds p = (-T) mod L_B pad tokens before the
      prompt (at most L_B - 1, so that the prompt ends on a block boundary);
      the pad id is the caller's choice.
  R8  A prompt whose length is not a multiple of L_B without padding: its
      trailing T mod L_B tokens form the incomplete current block and enter
      the token decoder (the model's own definition of those positions).
  R9  Summation injection ([BT] §3.4 "The Token Decoder", alternatives to
      prefix tokens: MEGABYTE-style sum): Proj maps c to L_B vectors
      s_0..s_{L_B-1} (W_s [L_B*D, D] + b_s, row-major as in R4); the token
      decoder's input rows are s_0 (the position that predicts the block's
      first token, where no token of the block is known yet) and
      s_j + E(x_{j-1}) for j = 1..L_B-1, at positions 0..L_B-1.
  R10 Window of previous context embeddings ([BT] §6 "Limitations",
      App. B.3 direction): the prefix holds Proj(c) of the last w context
      embeddings c_{i-w+1} .. c_i, oldest first, each through the same
      projection (w*P rows); context embeddings before the first block are
      zero vectors (their rows are b_p). w = 1 is the base model.
  R11 Grouped-query attention in the block decoder ([BT] §3.4 "The Block
      Decoder": standard attention, so multi-query / grouped-query
      attention applies; §6 and App. D.2): H_kv key/value heads, query head
      h reads key/value head floor(h / (H / H_kv)) (consecutive groups);
      W_qkv rows are q (H d_head) | k (H_kv d_head) | v (H_kv d_head), the
      cache holds H_kv heads. The token decoder keeps H_kv = H.

Pins (tests/test_oracle_*.py): HF GPTNeoX (an independent Pythia
implementation) for the layer stack and the vanilla special case;
torch CPU functional ops for LayerNorm / GELU / attention; brute-force
embedder and prefix; the closed-form single-row token decoder; the
locality/causality invariants; incremental decode equal to full-sequence
recomputation.
"""
from __future__ import annotations

import math
from typing import Dict, List, Mapping, Optional, Tuple

import numpy as np
from scipy.special import erf

__all__ = [
    "layer_norm", "gelu", "rotary", "attend", "pythia_layer", "embed_blocks",
    "prefix_projection", "left_pad", "BlockTransformerOracle", "ragged_generate_logits",
]


# --------------------------------------------------------------------------
# primitives of the Pythia layer ([BT] §5 "Experimental setup", base model:
# Pythia via GPT-NeoX; shape details per reading R6)
# --------------------------------------------------------------------------

def layer_norm(x: np.ndarray, g: np.ndarray, b: np.ndarray, eps: float) -> np.ndarray:
    """LayerNorm over the last axis with biased variance."""
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * g + b


def gelu(x: np.ndarray) -> np.ndarray:
    """Exact GELU: x * Phi(x), Phi the standard normal CDF."""
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def rotary(x: np.ndarray, pos: np.ndarray, r: int, base: float) -> np.ndarray:
    """Partial rotary embedding on the first r dims of each head.

    x: [..., n, H, d]; pos: [n] integer positions. Pair i with i + r/2
    (rotate-half form), angle pos * base^(-2i/r), i < r/2.
    """
    if r == 0:
        return x
    half = r // 2
    i = np.arange(half, dtype=np.float64)
    inv_freq = base ** (-2.0 * i / r)
    ang = pos.astype(np.float64)[:, None] * inv_freq[None, :]          # [n, half]
    cos = np.cos(ang)[:, None, :].astype(x.dtype)                     # [n, 1, half]
    sin = np.sin(ang)[:, None, :].astype(x.dtype)
    x1 = x[..., :half]
    x2 = x[..., half:r]
    out = x.copy()
    out[..., :half] = x1 * cos - x2 * sin
    out[..., half:r] = x2 * cos + x1 * sin
    return out


def attend(q: np.ndarray, k: np.ndarray, v: np.ndarray,
           q_pos: np.ndarray, k_pos: np.ndarray) -> np.ndarray:
    """Causal softmax attention by position: key j is visible to query i iff
    k_pos[j] <= q_pos[i]. Masked keys are excluded from the max and the sum.

    q: [B, nq, H, d]; k, v: [B, nk, H, d] -> [B, nq, H, d].
    """
    d = q.shape[-1]
    s = np.einsum("bqhd,bkhd->bhqk", q, k) / math.sqrt(d)
    visible = k_pos[None, :] <= q_pos[:, None]                         # [nq, nk]
    s = np.where(visible[None, None], s, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    p = np.where(visible[None, None], np.exp(s - m), 0.0)
    p = p / p.sum(axis=-1, keepdims=True)
    return np.einsum("bhqk,bkhd->bqhd", p, v)


class KVCache:
    """Per-layer key/value history [B, n, H, d] (appended in position order)."""

    def __init__(self):
        self.k: Optional[np.ndarray] = None
        self.v: Optional[np.ndarray] = None
        self.pos: Optional[np.ndarray] = None

    def append(self, k, v, pos):
        if self.k is None:
            self.k, self.v, self.pos = k, v, pos.copy()
        else:
            self.k = np.concatenate([self.k, k], axis=1)
            self.v = np.concatenate([self.v, v], axis=1)
            self.pos = np.concatenate([self.pos, pos])

    def __len__(self):
        return 0 if self.k is None else self.k.shape[1]


def pythia_layer(h: np.ndarray, p: Mapping[str, np.ndarray], pos: np.ndarray,
                 cache: KVCache, n_heads: int, rotary_dims: int,
                 eps: float, rope_base: float, n_kv_heads: Optional[int] = None) -> np.ndarray:
    """One Pythia layer with parallel attention + MLP residual ([BT] §3.4,
    "The Block Decoder": standard causal self-attention and feed-forward
    layers; reading R6 for the Pythia form).

    h: [B, n, D] residual rows at positions ``pos`` (new rows); their keys and
    values are appended to ``cache`` and every new row attends causally over
    the cache. n_kv_heads < n_heads: grouped-query attention (reading R11).
    """
    B, n, D = h.shape
    d = D // n_heads
    hk = n_heads if not n_kv_heads else n_kv_heads
    Dk = hk * d
    a = layer_norm(h, p["ln1_g"], p["ln1_b"], eps)
    m = layer_norm(h, p["ln2_g"], p["ln2_b"], eps)
    qkv = a @ p["w_qkv"].T + p["b_qkv"]                               # [B, n, D + 2 Dk]
    q = qkv[..., :D].reshape(B, n, n_heads, d)
    k = qkv[..., D:D + Dk].reshape(B, n, hk, d)
    v = qkv[..., D + Dk:D + 2 * Dk].reshape(B, n, hk, d)
    q = rotary(q, pos, rotary_dims, rope_base)
    k = rotary(k, pos, rotary_dims, rope_base)
    cache.append(k, v, pos)
    g = n_heads // hk                                                  # query heads per K/V head
    kk = np.repeat(cache.k, g, axis=2)
    vv = np.repeat(cache.v, g, axis=2)
    att = attend(q, kk, vv, pos, cache.pos).reshape(B, n, D)
    mlp = gelu(m @ p["w_1"].T + p["b_1"]) @ p["w_2"].T + p["b_2"]
    return h + (att @ p["w_o"].T + p["b_o"]) + mlp


# --------------------------------------------------------------------------
# embedder and prefix projection
# --------------------------------------------------------------------------

def embed_blocks(tokens: np.ndarray, table: np.ndarray, block_len: int) -> np.ndarray:
    """Lookup-and-concatenate embedder ([BT] §3.4 "The Embedder" [orig. §2.2]).

    tokens: [B, n*L_B] -> [B, n, D]; token j of block i fills dims
    [j*D/L_B, (j+1)*D/L_B) (reading R2).
    """
    B, S = tokens.shape
    n = S // block_len
    rows = table[tokens[:, :n * block_len]]                          # [B, n*L_B, D/L_B]
    return rows.reshape(B, n, block_len * table.shape[1])


def prefix_projection(c: np.ndarray, w: np.ndarray, b: np.ndarray, P: int) -> np.ndarray:
    """p_1..p_P = Proj(c_i), Proj a linear map R^D -> R^{P x D}
    ([BT] §3.4 "The Token Decoder", prefix mechanism [orig. §2.4]; R4).

    c: [..., D] -> [..., P, D].
    """
    D = c.shape[-1]
    out = c @ w.T + b
    return out.reshape(*c.shape[:-1], P, D)


def left_pad(tokens: np.ndarray, block_len: int, pad_id: int) -> np.ndarray:
    """Inference left padding ([BT] §3.4 "The Embedder", prompts whose length
    is not a multiple of L_B [orig. §2.2, App. H]): the first block is padded
    on the left with pad tokens so that the prompt ends on a block boundary.

    tokens: [T] -> [T + p], p = (-T) mod L_B in [0, L_B - 1] (reading R7).
    """
    tokens = np.asarray(tokens)
    p = (-tokens.shape[0]) % block_len
    return np.concatenate([np.full(p, pad_id, dtype=tokens.dtype), tokens])


# --------------------------------------------------------------------------
# the model
# --------------------------------------------------------------------------

class BlockTransformerOracle:
    """Block Transformer forward passes on the host.

    ``params`` maps the parameter names of ``synth.param_names`` to arrays
    (row-major [out, in] matrices). ``shape`` carries the model hyper-
    parameters (vocab, d_model, n_heads, block_len, n_block_layers,
    n_token_layers, prefix_len, rotary_dims, use_token_decoder, ln_eps,
    rope_base).
    """

    def __init__(self, shape, params: Mapping[str, np.ndarray],
                 dtype=np.float64):
        self.s = shape
        self.dtype = dtype
        self.sum_injection = getattr(shape, "injection", "prefix") == "sum"
        self.window = int(getattr(shape, "context_window", 1))
        assert self.window >= 1 and not (self.sum_injection and self.window > 1)
        get = (lambda n: np.asarray(params[n], dtype=dtype))
        gl = ["blk_emb", "lnf_b_g", "lnf_b_b", "w_lm"]
        if shape.use_token_decoder:
            gl += ["w_prefix", "b_prefix", "tok_emb", "lnf_t_g", "lnf_t_b"]
        self.g = {n: get(n) for n in gl}
        lnames = ["ln1_g", "ln1_b", "ln2_g", "ln2_b", "w_qkv", "b_qkv",
                  "w_o", "b_o", "w_1", "b_1", "w_2", "b_2"]
        self.block_layers = [{n: get(f"block.{l}.{n}") for n in lnames}
                             for l in range(shape.n_block_layers)]
        n_t = shape.n_token_layers if shape.use_token_decoder else 0
        self.token_layers = [{n: get(f"token.{l}.{n}") for n in lnames}
                             for l in range(n_t)]

    # ---- stacks -----------------------------------------------------------
    def _stack(self, h, layers, pos, caches, n_kv_heads=None):
        s = self.s
        for lw, cache in zip(layers, caches):
            h = pythia_layer(h, lw, pos, cache, s.n_heads, s.rotary_dims,
                             s.ln_eps, s.rope_base, n_kv_heads)
        return h

    def block_decoder(self, e: np.ndarray, pos: np.ndarray,
                      caches: List[KVCache]) -> np.ndarray:
        """Causal transformer over block embeddings ([BT] §3.4 "The Block
        Decoder" [orig. §2.3]); returns the context embeddings
        c = LN_b(h) (reading R3)."""
        h = self._stack(e, self.block_layers, pos, caches, getattr(self.s, "n_kv_heads", 0) or None)
        return layer_norm(h, self.g["lnf_b_g"], self.g["lnf_b_b"], self.s.ln_eps)

    def token_decoder(self, u: np.ndarray, pos: np.ndarray,
                      caches: List[KVCache]) -> np.ndarray:
        """Causal transformer over [prefix rows; current block's tokens], no
        access outside the block ([BT] §3.2 item 3, §3.4 "The Token
        Decoder" [orig. §2.4]). Returns logits of every row (R3)."""
        h = self._stack(u, self.token_layers, pos, caches)
        z = layer_norm(h, self.g["lnf_t_g"], self.g["lnf_t_b"], self.s.ln_eps)
        return z @ self.g["w_lm"].T

    def _fresh(self, layers) -> List[KVCache]:
        return [KVCache() for _ in layers]

    # ---- context injection (R4, R9, R10) ---------------------------------
    @property
    def n_ctx_rows(self) -> int:
        """Rows in front of a block's tokens in the token decoder: w * P
        projected prefix rows, or the one row s_0 of summation injection."""
        return 1 if self.sum_injection else self.window * self.s.prefix_len

    def context_input(self, c_win: np.ndarray) -> Tuple[np.ndarray, Optional[np.ndarray]]:
        """c_win: [B, w, D] the window's context embeddings, oldest first.
        Returns the context rows [B, n_ctx_rows, D] and, in summation
        injection, the vectors added to the token rows 1..L_B-1
        ([B, L_B - 1, D], else None)."""
        B, w, D = c_win.shape
        if self.sum_injection:
            sv = prefix_projection(c_win[:, -1], self.g["w_prefix"], self.g["b_prefix"], self.s.block_len)
            return sv[:, :1], sv[:, 1:]
        rows = prefix_projection(c_win, self.g["w_prefix"], self.g["b_prefix"], self.s.prefix_len)
        return rows.reshape(B, w * self.s.prefix_len, D), None

    def token_rows(self, tok: np.ndarray, j: np.ndarray, add: Optional[np.ndarray]) -> np.ndarray:
        """Input rows of tokens tok [B, r] at in-block offsets j [r] (token
        j of the block is the input of row n_ctx + j): E(x), plus s_{j+1} in
        summation injection."""
        rows = self.g["tok_emb"][tok]
        if add is not None:
            rows = rows + add[:, j]
        return rows

    # ---- full-sequence, teacher-forced layout ----------------------------
    def forward_full(self, tokens: np.ndarray) -> np.ndarray:
        """Teacher-forced logits for every predictable position.

        tokens: [B, S] int. Returns pred [B, S+1, V] where pred[:, t]
        predicts token t; rows t < L_B (t < 1 in vanilla mode) are NaN.
        Training layout of [BT] §3.4 "The Block Decoder" (autoregressive
        training task, steps 1-4).
        """
        s = self.s
        dt = self.dtype
        tokens = np.asarray(tokens)
        B, S = tokens.shape
        L = s.block_len
        n = S // L
        V = s.vocab
        pred = np.full((B, S + 1, V), np.nan, dtype=dt)
        e = embed_blocks(tokens, self.g["blk_emb"], L)                 # [B, n, D]
        c = self.block_decoder(e, np.arange(n), self._fresh(self.block_layers))
        if not s.use_token_decoder:
            # vanilla special case (L_B = 1): next-token logits from c_t
            assert L == 1
            pred[:, 1:n + 1] = c @ self.g["w_lm"].T
            return pred
        P = self.n_ctx_rows
        D = s.d_model
        w = self.window
        # block k (1..n) is predicted from c_{k-w} .. c_{k-1} (zeros before
        # block 0, R10)
        c_pad = np.concatenate([np.zeros((B, w - 1, D), dtype=dt), c], axis=1)
        nrows = P + L - 1
        u = np.zeros((B, n, nrows, D), dtype=dt)
        for k in range(1, n + 1):
            rows, add = self.context_input(c_pad[:, k - 1:k - 1 + w])
            u[:, k - 1, :P] = rows
            for j in range(L - 1):
                t = k * L + j
                if t < S:
                    u[:, k - 1, P + j] = self.token_rows(tokens[:, t:t + 1], np.array([j]), add)[:, 0]
        # rows whose input token is unknown (t >= S) only feed later rows of
        # the same block; their logits are never used.
        uu = u.reshape(B * n, nrows, D)
        zz = self.token_decoder(uu, np.arange(nrows), self._fresh(self.token_layers))
        zz = zz.reshape(B, n, nrows, V)
        for k in range(1, n + 1):
            for j in range(L):
                t = k * L + j
                if t <= S:
                    pred[:, t] = zz[:, k - 1, P - 1 + j]
        return pred

    # ---- incremental: prefill + decode steps ----------------------------
    def session(self) -> "OracleSession":
        return OracleSession(self)


class OracleSession:
    """Prefill then one token per decode call, with explicit KV caches
    ([BT] §2 "prefill vs. decode"; §3.4 cost analysis: the block decoder
    runs once per L_B tokens, the token decoder only for the current block)."""

    def __init__(self, model: BlockTransformerOracle):
        self.m = model
        self.s = model.s
        self.t = 0
        self.block_caches: List[KVCache] = []
        self.token_caches: List[KVCache] = []
        self.cur_block: Optional[np.ndarray] = None   # [B, L_B] tokens of the open block
        self.c_win: Optional[np.ndarray] = None       # [B, w, D] last w context embeddings
        self.add: Optional[np.ndarray] = None         # summation injection: s_1..s_{L_B-1}

    def _token_rows(self, rows: np.ndarray, pos: np.ndarray) -> np.ndarray:
        return self.m.token_decoder(rows, pos, self.token_caches)

    def _push_context(self, c: np.ndarray) -> None:
        """c [B, D] becomes the newest context embedding of the window."""
        if self.c_win is None:
            B, D = c.shape
            self.c_win = np.zeros((B, self.m.window, D), dtype=self.m.dtype)
        self.c_win = np.concatenate([self.c_win[:, 1:], c[:, None]], axis=1)

    def _start_block(self, trailing: Optional[np.ndarray] = None) -> np.ndarray:
        """New token-decoder block: reset local KV, feed the context rows of
        the window and the tokens of the block already known (``trailing``
        [B, r], r < L_B, at local positions n_ctx..n_ctx+r-1); return logits
        of the last row fed, which predict token r of the block."""
        m = self.m
        self.token_caches = m._fresh(m.token_layers)
        rows, self.add = m.context_input(self.c_win)
        if trailing is not None and trailing.shape[1] > 0:
            r = trailing.shape[1]
            rows = np.concatenate([rows, m.token_rows(trailing, np.arange(r), self.add)], axis=1)
        z = self._token_rows(rows, np.arange(rows.shape[1]))
        return z[:, -1]

    def prefill(self, tokens: np.ndarray) -> np.ndarray:
        """Process the prompt; return logits predicting token T.

        Only the most recent block enters the token decoder: its prefix comes
        from c_{n-1}; earlier blocks never do ([BT] §3.4 token-decoder cost
        analysis, "prefill computation near zero" [orig. §2.4]). The block
        decoder runs over the n = floor(T / L_B) complete blocks; when T is
        not a multiple of L_B the r = T - n L_B trailing tokens are the first
        tokens of the current block and enter the token decoder after the
        prefix (reading R8), exactly as if they had been fed by r decode
        calls."""
        s, m = self.s, self.m
        tokens = np.asarray(tokens)
        B, T = tokens.shape
        L = s.block_len
        assert T >= L
        n = T // L
        r = T - n * L
        self.block_caches = m._fresh(m.block_layers)
        e = embed_blocks(tokens[:, :n * L], m.g["blk_emb"], L)
        c_all = m.block_decoder(e, np.arange(n), self.block_caches)       # c_0 .. c_{n-1}
        c = c_all[:, -1]
        self.c_win = None
        for i in range(max(0, n - m.window), n):
            self._push_context(c_all[:, i])
        self.t = T
        self.cur_block = np.zeros((B, L), dtype=np.int64)
        self.cur_block[:, :r] = tokens[:, n * L:]
        if not s.use_token_decoder:
            return c @ m.g["w_lm"].T
        return self._start_block(tokens[:, n * L:])

    def decode(self, tok: np.ndarray) -> np.ndarray:
        """Feed token x_t (t = tokens seen so far); return logits for x_{t+1}.

        If x_t completes block k = t // L_B, the block decoder appends e_k to
        its cache (position k) and a new token-decoder block starts from c_k;
        otherwise the token decoder appends one row at local position
        n_ctx_rows + (t mod L_B)."""
        s, m = self.s, self.m
        tok = np.asarray(tok)
        L = s.block_len
        t = self.t
        j = t % L
        self.cur_block[:, j] = tok
        self.t = t + 1
        if j == L - 1:
            k = t // L
            e = embed_blocks(self.cur_block, m.g["blk_emb"], L)          # [B, 1, D]
            c = m.block_decoder(e, np.array([k]), self.block_caches)[:, 0]
            if not s.use_token_decoder:
                return c @ m.g["w_lm"].T
            self._push_context(c)
            return self._start_block()
        row = m.token_rows(tok[:, None], np.array([j]), self.add)
        z = self._token_rows(row, np.array([m.n_ctx_rows + j]))
        return z[:, 0]

    def generate_logits(self, tokens: np.ndarray, prompt_len: int,
                        steps: int) -> np.ndarray:
        """Teacher-forced run: prefill tokens[:, :T], then feed tokens
        T..T+steps-2. Returns [steps, B, V]: logits for x_T .. x_{T+steps-1}."""
        out = [self.prefill(tokens[:, :prompt_len])]
        for i in range(steps - 1):
            out.append(self.decode(tokens[:, prompt_len + i]))
        return np.stack(out)


def ragged_generate_logits(model: BlockTransformerOracle, prompts, continuations, steps: int,
                           pad: bool = False, pad_id: int = 0) -> List[np.ndarray]:
    """Teacher-forced runs of sequences with different prompt lengths, each
    on its own (rows of a batch are independent: [BT] §3.2, every sequence
    has its own block and token decoders' state).

    prompts[b]: [T_b] token ids; continuations[b]: the tokens fed after the
    prompt (at least steps - 1). pad = True left-pads every prompt to a
    block boundary first (``left_pad``). Returns, per sequence, the logits
    [steps, V] predicting the token after the prompt and after each fed
    token.
    """
    out = []
    for pr, cont in zip(prompts, continuations):
        pr = np.asarray(pr)
        if pad:
            pr = left_pad(pr, model.s.block_len, pad_id)
        seq = np.concatenate([pr, np.asarray(cont)[:steps - 1]])[None, :]
        out.append(model.session().generate_logits(seq, pr.shape[0], steps)[:, 0])
    return out
