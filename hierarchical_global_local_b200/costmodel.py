"""Algorithmic bytes and FLOPs of Block Transformer inference.

The three cost buckets (compute, parameter reads, KV-cache reads) and their
scaling follow "Block Transformer: Global-to-Local Language Modeling for Fast
Inference" (explainer page, §3.4 "The Inference Cost Model and Bottleneck
Decomposition" [orig. §2.1, App. E]): the block decoder reads its
parameters once per L_B tokens and a KV cache L_B times shorter (KV I/O
falls by L_B^2); the token decoder reads its parameters every token and a
local KV cache of at most P + L_B - 1 rows.

"Algorithmic" bytes count what the method must move at least once per step:
every parameter the step uses, every KV row it attends over or appends, the
embedding rows it gathers and the logits it stores (if any). Intermediate
activations are excluded: a fused implementation need not write them.
Pure host arithmetic; no device code.
"""
from __future__ import annotations

import dataclasses
from typing import Optional


def kv_bytes_per_token(n_layers: int, d_model: int, bytes_per_elem: int = 2) -> int:
    """Keys and values of one token across all layers: 2 * N * D * bytes."""
    return 2 * n_layers * d_model * bytes_per_elem


def total_kv_reads(seq_len: int) -> int:
    """Decode steps 1..L read 1, 2, ..., L cached states: L(L+1)/2."""
    return seq_len * (seq_len + 1) // 2


def block_decoder_kv_io_ratio(seq_len: int, block_len: int) -> float:
    """Vanilla KV reads over block-decoder KV reads while decoding seq_len
    tokens with the same depth: L(L+1)/2 token-sized states against
    n(n+1)/2 block states, n = L / L_B (states are the same width D), which
    tends to L_B^2."""
    n = seq_len // block_len
    return total_kv_reads(seq_len) / total_kv_reads(n)


def token_decoder_kv_reduction(seq_len: int, block_len: int) -> float:
    """R = L / L_B: a token attends over <= L_B local rows instead of L."""
    return seq_len / block_len


@dataclasses.dataclass(frozen=True)
class Shape:
    vocab: int
    d_model: int
    n_heads: int
    block_len: int
    n_block_layers: int
    n_token_layers: int
    prefix_len: int
    use_token_decoder: bool = True
    bytes_per_elem: int = 2

    @classmethod
    def of(cls, s) -> "Shape":
        return cls(s.vocab, s.d_model, s.n_heads, s.block_len, s.n_block_layers,
                   s.n_token_layers if s.use_token_decoder else 0,
                   s.prefix_len if s.use_token_decoder else 0,
                   s.use_token_decoder, 4 if s.dtype == "fp32" else 2)


def layer_params(D: int) -> int:
    """Pythia layer: W_qkv 3D^2, W_o D^2, W_1 4D^2, W_2 4D^2; biases 9D; LN 4D."""
    return 12 * D * D + 13 * D


@dataclasses.dataclass
class Cost:
    bytes: float = 0.0
    flops: float = 0.0

    def __iadd__(self, o: "Cost") -> "Cost":
        self.bytes += o.bytes
        self.flops += o.flops
        return self

    def time(self, hbm_gbs: float, tflops: float) -> float:
        return max(self.bytes / (hbm_gbs * 1e9), self.flops / (tflops * 1e12))


def _head(s: Shape, B: int, store_logits: bool) -> Cost:
    eb, D, V = s.bytes_per_elem, s.d_model, s.vocab
    by = (V * D + 2 * D) * eb + (B * V * 4 if store_logits else 0)
    return Cost(by, 2.0 * B * V * D)


def _layers(s: Shape, n_layers: int, rows: int, kv_rows_read: int,
            kv_rows_written: int, attn_pairs: int) -> Cost:
    """n_layers Pythia layers over ``rows`` new rows (all sequences), reading
    ``kv_rows_read`` and appending ``kv_rows_written`` KV rows per layer;
    attn_pairs = (query, key) pairs per head per layer (all sequences)."""
    eb, D, H = s.bytes_per_elem, s.d_model, s.n_heads
    d = D // H
    by = n_layers * (layer_params(D) * eb
                     + (kv_rows_read + kv_rows_written) * 2 * D * eb)
    fl = n_layers * (2.0 * rows * 12 * D * D + 4.0 * H * d * attn_pairs)
    return Cost(by, fl)


def token_step(s: Shape, B: int, j: int, store_logits: bool = False) -> Cost:
    """Decode call that feeds the token at local index j < L_B - 1 of its
    block: one token-decoder row at local position P + j attends over
    P + j + 1 rows, then the LM head."""
    eb, D = s.bytes_per_elem, s.d_model
    rows = s.prefix_len + j + 1
    c = Cost(B * D * eb, 0.0)                                   # E_tok gather
    c += _layers(s, s.n_token_layers, B, B * (rows - 1), B, B * rows)
    c += _head(s, B, store_logits)
    return c


def block_step(s: Shape, B: int, k: int, store_logits: bool = False) -> Cost:
    """Decode call that completes block k: embed it, one block-decoder row
    at block position k attends over k + 1 cached entries; then the prefix
    projection and the token decoder over P prefix rows (or, vanilla, the
    LM head on the block decoder's output)."""
    eb, D, P = s.bytes_per_elem, s.d_model, s.prefix_len
    c = Cost(B * D * eb, 0.0)                                   # E_blk gathers
    c += _layers(s, s.n_block_layers, B, B * k, B, B * (k + 1))
    c += Cost(2 * D * eb, 0.0)                                  # LN_b
    if s.use_token_decoder:
        c += Cost((P * D * D + P * D) * eb, 2.0 * B * P * D * D)
        c += _layers(s, s.n_token_layers, B * P, 0, B * P, B * P * (P + 1) // 2)
    c += _head(s, B, store_logits)
    return c


def prefill(s: Shape, B: int, T: int, store_logits: bool = False) -> Cost:
    eb, D, P = s.bytes_per_elem, s.d_model, s.prefix_len
    n = T // s.block_len
    c = Cost(B * T * 4 + B * n * D * eb, 0.0)                   # tokens + E_blk rows
    c += _layers(s, s.n_block_layers, B * n, 0, B * n, B * n * (n + 1) // 2)
    c += Cost(2 * D * eb, 0.0)
    if s.use_token_decoder:
        c += Cost((P * D * D + P * D) * eb, 2.0 * B * P * D * D)
        c += _layers(s, s.n_token_layers, B * P, 0, B * P, B * P * (P + 1) // 2)
    c += _head(s, B, store_logits)
    return c


def decode_step(s: Shape, B: int, t: int, store_logits: bool = False) -> Cost:
    """Cost of the decode call that feeds token position t."""
    L = s.block_len
    if t % L == L - 1:
        return block_step(s, B, t // L, store_logits)
    return token_step(s, B, t % L, store_logits)


@dataclasses.dataclass
class GenerateCost:
    prefill: Cost
    decode: Cost
    n_block_steps: int
    n_token_steps: int

    def roofline_seconds(self, hbm_gbs: float, tflops: float) -> float:
        return (self.prefill.time(hbm_gbs, tflops)
                + self.decode.time(hbm_gbs, tflops))


def generate(s: Shape, B: int, T: int, G: int, store_logits: bool = False,
             per_step_roofline: Optional[tuple] = None) -> GenerateCost:
    """Prefill (predicts x_T) then G - 1 decode calls feeding x_T..x_{T+G-2}.

    The decode bucket sums bytes and FLOPs over steps; each step is HBM-bound
    at these shapes, so summing bytes is the same as summing per-step
    roofline times (asserted when ``per_step_roofline`` = (GB/s, TF/s)).
    """
    pre = prefill(s, B, T, store_logits)
    dec = Cost()
    nb = nt = 0
    per_step = 0.0
    for t in range(T, T + G - 1):
        c = decode_step(s, B, t, store_logits)
        if t % s.block_len == s.block_len - 1:
            nb += 1
        else:
            nt += 1
        if per_step_roofline:
            per_step += c.time(*per_step_roofline)
        dec += c
    g = GenerateCost(pre, dec, nb, nt)
    if per_step_roofline:
        g.decode_roofline_per_step = per_step
    return g


def decode_attention_bytes(B: int, H: int, n: int, d: int, bytes_per_elem: int = 2) -> int:
    """Block-decoder decode attention, one launch: read n keys and n values
    per (b, h) plus q, write o (the unit of the kernel's roofline)."""
    return B * H * (2 * n * d * bytes_per_elem + 2 * d * bytes_per_elem)
