"""Helpers shared by the GPU tests: upload synthetic weights, build a model
through the C-ABI binding, run the oracle on the same inputs."""
from __future__ import annotations

import numpy as np

import synth


def torch_mod():
    import torch
    return torch


def upload(weights: synth.Weights):
    """name -> CUDA tensor holding the exact device bytes (bf16 or fp32)."""
    torch = torch_mod()
    out = {}
    for n in weights.names():
        a = weights.device_bytes(n)
        if a.dtype == np.uint16:
            t = torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16)
        else:
            t = torch.from_numpy(np.ascontiguousarray(a))
        out[n] = t.cuda()
    return out


def model_config(shape: synth.ModelShape, max_batch: int, max_seq: int):
    from hierarchical_global_local_b200 import native
    return native.ModelConfig(
        vocab=shape.vocab, d_model=shape.d_model, n_heads=shape.n_heads,
        block_len=shape.block_len, n_block_layers=shape.n_block_layers,
        n_token_layers=shape.n_token_layers if shape.use_token_decoder else 0,
        prefix_len=shape.prefix_len if shape.use_token_decoder else 1,
        rotary_dims=shape.rotary_dims, use_token_decoder=shape.use_token_decoder,
        max_batch=max_batch, max_seq=max_seq, dtype=shape.dtype, ln_eps=shape.ln_eps,
        rope_base=shape.rope_base)


def build_model(shape, weights, max_batch, max_seq):
    from hierarchical_global_local_b200 import native
    return native.BlockTransformer(model_config(shape, max_batch, max_seq), upload(weights))


def gpu_teacher_forced(model, tokens: np.ndarray, T: int, G: int):
    """Prefill tokens[:, :T] then feed T..T+G-2; returns logits [G, B, V]
    (fp32 numpy) and next-token ids [G, B]."""
    torch = torch_mod()
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


def oracle_teacher_forced(shape, weights: synth.Weights, tokens, T, G, rows=None,
                          dtype=np.float64):
    from oracle.model import BlockTransformerOracle
    params = {n: weights.values(n) for n in weights.names()}
    o = BlockTransformerOracle(shape, params, dtype=dtype)
    tk = tokens if rows is None else tokens[rows]
    return o.session().generate_logits(tk, T, G)


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))
