"""Put a model's parameters on the GPU and build it through the C-ABI binding.

Parameters come as numpy arrays holding the exact bytes the device should
hold: bf16 as their uint16 bit patterns, fp32 as float32 (for instance the
synthetic weights of the seeded input generators). Names follow
``native.BlockTransformer``: globals ``blk_emb, lnf_b_g, ...`` and per layer
``block.{l}.*`` / ``token.{l}.*``.
"""
from __future__ import annotations

from typing import Mapping

import numpy as np

from . import native


def upload(params) -> dict:
    """name -> CUDA tensor with the exact bytes of each parameter. ``params``
    is a mapping name -> numpy array, or an object with ``names()`` and
    ``device_bytes(name)``."""
    import torch
    if hasattr(params, "device_bytes"):
        items = [(n, params.device_bytes(n)) for n in params.names()]
    else:
        items = list(params.items())
    out = {}
    for n, a in items:
        if a.dtype == np.uint16:
            t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16).copy()).view(torch.bfloat16)
        else:
            t = torch.from_numpy(np.ascontiguousarray(a))
        out[n] = t.cuda()
    return out


def model_config(shape, max_batch: int, max_seq: int) -> native.ModelConfig:
    """C-ABI configuration of a model shape (any object with the fields
    vocab, d_model, n_heads, block_len, n_block_layers, n_token_layers,
    prefix_len, rotary_dims, use_token_decoder, dtype, ln_eps, rope_base)."""
    return native.ModelConfig(
        vocab=shape.vocab, d_model=shape.d_model, n_heads=shape.n_heads,
        block_len=shape.block_len, n_block_layers=shape.n_block_layers,
        n_token_layers=shape.n_token_layers if shape.use_token_decoder else 0,
        prefix_len=shape.prefix_len if shape.use_token_decoder else 1,
        rotary_dims=shape.rotary_dims, use_token_decoder=shape.use_token_decoder,
        max_batch=max_batch, max_seq=max_seq, dtype=shape.dtype, ln_eps=shape.ln_eps,
        rope_base=shape.rope_base, injection=getattr(shape, "injection", "prefix"),
        context_window=getattr(shape, "context_window", 1), n_kv_heads=getattr(shape, "n_kv_heads", 0))


def build_model(shape, params, max_batch: int, max_seq: int) -> native.BlockTransformer:
    """A model on the current CUDA device with room for max_batch sequences
    of max_seq tokens (prompt + generated)."""
    return native.BlockTransformer(model_config(shape, max_batch, max_seq), upload(params))


def teacher_forced_logits(model: native.BlockTransformer, tokens: np.ndarray, T: int, G: int):
    """Prefill tokens[:, :T], then feed tokens T .. T+G-2 one decode call at a
    time; returns the logits of every call [G, B, V] (fp32 numpy) and the
    greedy ids [G, B]."""
    import torch
    B = tokens.shape[0]
    V = model.cfg.vocab
    tok = torch.from_numpy(np.ascontiguousarray(tokens)).cuda()
    logits = torch.empty(G, B, V, dtype=torch.float32, device="cuda")
    nxt = torch.empty(G, B, dtype=torch.int32, device="cuda")
    model.prefill(tok[:, :T].contiguous(), logits=logits[0], next_tokens=nxt[0])
    for i in range(G - 1):
        model.decode(tok[:, T + i].contiguous(), logits=logits[i + 1], next_tokens=nxt[i + 1])
    model.sync()
    return logits.cpu().numpy(), nxt.cpu().numpy()


# ---- memory planning: the maximum-throughput methodology --------------------
# The method's throughput comparisons use, for every model, the largest batch
# that fits in device memory (FlexGen's "maximum throughput" setting), and
# report the memory one sequence costs. A model's device footprint is exactly
# its workspace (bt_workspace_bytes: repacked weights, block and local KV
# caches, activation buffers and scratch, all sized from the configuration);
# the caller's original weight buffers are no longer read once bt_create's
# copy has run. So both numbers follow from the workspace formula alone.

def workspace_bytes(shape, max_batch: int, max_seq: int) -> int:
    """Device bytes of a model with room for max_batch sequences of max_seq
    tokens (0 if the configuration is invalid, for instance too large)."""
    try:
        return native.workspace_bytes(model_config(shape, max_batch, max_seq))
    except native.BtError:
        return 0


def memory_per_sample(shape, max_seq: int) -> float:
    """Bytes each additional sequence of max_seq tokens adds to the model's
    footprint: the slope of the workspace in the batch capacity between 32
    and 64 sequences (block and local KV caches, per-row activation buffers,
    logits; a few scratch buffers follow the launch plan, so the slope
    varies by under 1 % elsewhere)."""
    lo, hi = 32, 64
    a, b = workspace_bytes(shape, lo, max_seq), workspace_bytes(shape, hi, max_seq)
    if a == 0 or b == 0:
        raise ValueError("invalid configuration")
    return (b - a) / (hi - lo)


def max_batch_by_memory(shape, max_seq: int, budget_bytes: int, limit: int = 1 << 20) -> int:
    """The largest batch capacity B <= limit whose workspace fits in
    budget_bytes (0 if not even one sequence fits). The workspace grows with
    B, so a doubling search followed by bisection finds it."""
    def fits(b: int) -> bool:
        n = workspace_bytes(shape, b, max_seq)
        return 0 < n <= budget_bytes
    if not fits(1):
        return 0
    lo, hi = 1, 2
    while hi <= limit and fits(hi):
        lo, hi = hi, hi * 2
    hi = min(hi, limit + 1)
    while hi - lo > 1:  # fits(lo), not fits(hi) (or hi past the limit)
        mid = (lo + hi) // 2
        if fits(mid):
            lo = mid
        else:
            hi = mid
    return lo
