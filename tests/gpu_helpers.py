"""Helpers shared by the GPU tests: upload synthetic weights, build a model
through the C-ABI binding, run the oracle on the same inputs."""
from __future__ import annotations

import numpy as np

import synth
from hierarchical_global_local_b200 import loader


def torch_mod():
    import torch
    return torch


def upload(weights: synth.Weights):
    """name -> CUDA tensor holding the exact device bytes (bf16 or fp32)."""
    return loader.upload(weights)


def model_config(shape: synth.ModelShape, max_batch: int, max_seq: int):
    return loader.model_config(shape, max_batch, max_seq)


def build_model(shape, weights, max_batch, max_seq):
    return loader.build_model(shape, weights, max_batch, max_seq)


def gpu_teacher_forced(model, tokens: np.ndarray, T: int, G: int):
    """Prefill tokens[:, :T] then feed T..T+G-2; returns logits [G, B, V]
    (fp32 numpy) and next-token ids [G, B]."""
    return loader.teacher_forced_logits(model, tokens, T, G)


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
