"""Seeded synthetic inputs shared by the oracle and the CUDA path.

This module holds workload descriptions (model shapes and run lengths) and
deterministic generators for random-init weights and token streams. It holds
none of the model's arithmetic: nothing here normalises, projects, attends or
predicts. Both the CPU oracle and the GPU tests/bench draw their inputs from
here, so the two sides see bit-identical weights and token ids.

Recipe (Block Transformer, arXiv 2406.02657, as described on the explainer
page "Block Transformer: Global-to-Local Language Modeling for Fast
Inference"):

* Weights: every matrix and every bias ~ N(0, 0.02); LayerNorm gain
  1 + N(0, 0.02) and shift N(0, 0.02), so that a dropped gain or bias changes
  the result. Drawn in fp32 with numpy PCG64, one independent stream per
  tensor (SeedSequence(seed, spawn_key=(tensor_index,))), seed = 1000 + the
  workload family index.
* bf16 workloads round every parameter to bf16 (round to nearest even) here,
  once; the oracle consumes those rounded values, the GPU the bf16 bits.
* Tokens: seed = 2000 + family index. "uniform" draws ids in [0, V);
  "zipf" draws rank r in 1..V with P(r) proportional to r**-1.1 by inverse
  CDF over the finite support (id = r - 1).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Iterator, List, Optional, Tuple

import numpy as np

__all__ = [
    "ModelShape", "Workload", "WORKLOADS", "workload", "layer_param_shapes",
    "global_param_shapes", "param_names", "make_weights", "make_tokens",
    "round_to_bf16_bits", "bf16_bits_to_f32", "Weights",
]


@dataclasses.dataclass(frozen=True)
class ModelShape:
    vocab: int
    d_model: int
    n_heads: int
    block_len: int          # L_B
    n_block_layers: int     # N_b
    n_token_layers: int     # N_t
    prefix_len: int = 1     # P
    rotary_pct: float = 0.25
    use_token_decoder: bool = True
    dtype: str = "bf16"     # "fp32" or "bf16": storage/compute type of the path
    ln_eps: float = 1e-5
    rope_base: float = 10000.0
    # how the context embedding reaches the token decoder: "prefix" (P
    # projected rows in front of the block's tokens) or "sum" (L_B projected
    # vectors added to the token decoder's input rows, MEGABYTE-style)
    injection: str = "prefix"
    context_window: int = 1  # w: the last w context embeddings feed the prefix
    n_kv_heads: int = 0      # block decoder's key/value heads (0: n_heads; < n_heads: GQA)

    @property
    def proj_rows(self) -> int:
        """Rows of D outputs of the context projection: P, or L_B in "sum"
        injection."""
        return self.block_len if self.injection == "sum" else self.prefix_len

    @property
    def d_head(self) -> int:
        return self.d_model // self.n_heads

    @property
    def rotary_dims(self) -> int:
        return int(self.d_head * self.rotary_pct)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    family: int             # seeds: weights 1000+family, tokens 2000+family
    shape: ModelShape
    batch: int
    prompt_len: int
    gen_len: int
    tokens: str             # "uniform" | "zipf"

    @property
    def max_seq(self) -> int:
        return self.prompt_len + self.gen_len

    @property
    def weight_seed(self) -> int:
        return 1000 + self.family

    @property
    def token_seed(self) -> int:
        return 2000 + self.family


_V = 50304


def _sweep(lb: int) -> Workload:
    if lb == 1:   # vanilla: block decoder over single tokens, no token decoder
        shape = ModelShape(_V, 1024, 16, 1, 24, 0, prefix_len=0,
                           use_token_decoder=False)
    else:
        shape = ModelShape(_V, 1024, 16, lb, 12, 12, prefix_len=1)
    return Workload(f"lb_sweep_L{lb}", 3, shape, 128, 2048, 512, "zipf")


WORKLOADS: Dict[str, Workload] = {w.name: w for w in [
    # Tiny Block Transformer, fp32 (parity at 1e-4 max abs).
    Workload("tiny_fp32", 0,
             ModelShape(512, 128, 4, 4, 2, 2, prefix_len=1, dtype="fp32"),
             2, 64, 16, "uniform"),
    # Pythia-160M-scale Block Transformer, bf16.
    Workload("pythia160m_prefill_heavy", 1,
             ModelShape(_V, 768, 12, 4, 6, 6, prefix_len=1), 64, 2048, 128, "zipf"),
    Workload("pythia160m_decode_heavy", 1,
             ModelShape(_V, 768, 12, 4, 6, 6, prefix_len=1), 64, 128, 2048, "zipf"),
    # Pythia-410M-scale Block Transformer, bf16, decode-heavy.
    Workload("pythia410m_decode_heavy", 2,
             ModelShape(_V, 1024, 16, 4, 12, 12, prefix_len=1), 256, 128, 2048, "zipf"),
    # L_B sweep at d_model 1024 (L_B = 1 is the vanilla 24-layer baseline).
    *[_sweep(lb) for lb in (1, 2, 4, 8)],
    # Long-context Block Transformer, d_model 2048, d_head 128, bf16.
    Workload("long_context", 4,
             ModelShape(_V, 2048, 16, 4, 12, 12, prefix_len=1), 32, 8192, 512, "uniform"),
]}


def workload(name: str, **overrides) -> Workload:
    """Return a named workload, optionally with batch/prompt/gen overridden."""
    w = WORKLOADS[name]
    return dataclasses.replace(w, **overrides) if overrides else w


# --------------------------------------------------------------------------
# parameter inventory (names, shapes; row-major [out, in] for matrices)
# --------------------------------------------------------------------------

def layer_param_shapes(s: ModelShape, block: bool = False) -> List[Tuple[str, Tuple[int, ...]]]:
    """Parameters of one layer; block = True: a block-decoder layer, whose
    q|k|v rows carry n_kv_heads key/value heads."""
    D = s.d_model
    hk = (s.n_kv_heads or s.n_heads) if block else s.n_heads
    Nq = D + 2 * hk * s.d_head
    return [
        ("ln1_g", (D,)), ("ln1_b", (D,)), ("ln2_g", (D,)), ("ln2_b", (D,)),
        ("w_qkv", (Nq, D)), ("b_qkv", (Nq,)),
        ("w_o", (D, D)), ("b_o", (D,)),
        ("w_1", (4 * D, D)), ("b_1", (4 * D,)),
        ("w_2", (D, 4 * D)), ("b_2", (D,)),
    ]


def global_param_shapes(s: ModelShape) -> List[Tuple[str, Tuple[int, ...]]]:
    D, V, P = s.d_model, s.vocab, s.proj_rows
    out = [("blk_emb", (V, D // s.block_len)),
           ("lnf_b_g", (D,)), ("lnf_b_b", (D,))]
    if s.use_token_decoder:
        out += [("w_prefix", (P * D, D)), ("b_prefix", (P * D,)),
                ("tok_emb", (V, D)), ("lnf_t_g", (D,)), ("lnf_t_b", (D,))]
    out += [("w_lm", (V, D))]
    return out


def param_names(s: ModelShape) -> List[Tuple[str, Tuple[int, ...]]]:
    """Flat, ordered inventory: globals then block layers then token layers."""
    names = list(global_param_shapes(s))
    for l in range(s.n_block_layers):
        names += [(f"block.{l}.{n}", sh) for n, sh in layer_param_shapes(s, block=True)]
    n_t = s.n_token_layers if s.use_token_decoder else 0
    for l in range(n_t):
        names += [(f"token.{l}.{n}", sh) for n, sh in layer_param_shapes(s)]
    return names


# --------------------------------------------------------------------------
# bf16 rounding (data preparation, not model arithmetic)
# --------------------------------------------------------------------------

def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------------------
# weights
# --------------------------------------------------------------------------

class Weights:
    """Named parameter tensors.

    ``values(name)`` is the exact parameter value as fp32 (already rounded to
    bf16 for bf16 shapes). ``device_bytes(name)`` is what a device copy holds:
    uint16 bf16 bits, or the fp32 array itself.
    """

    def __init__(self, shape: ModelShape, seed: int,
                 only: Optional[List[str]] = None):
        self.shape = shape
        self.seed = seed
        self._inv = param_names(shape)
        self._index = {n: i for i, (n, _) in enumerate(self._inv)}
        self._shapes = dict(self._inv)
        self._f32: Dict[str, np.ndarray] = {}
        self._bits: Dict[str, np.ndarray] = {}
        for n in (only if only is not None else [n for n, _ in self._inv]):
            self._materialise(n)

    def names(self) -> List[str]:
        return [n for n, _ in self._inv]

    def _draw(self, name: str) -> np.ndarray:
        ss = np.random.SeedSequence(self.seed, spawn_key=(self._index[name],))
        g = np.random.Generator(np.random.PCG64(ss))
        x = g.standard_normal(self._shapes[name], dtype=np.float32)
        x *= np.float32(0.02)
        base = name.rsplit(".", 1)[-1]
        if base.endswith("_g") and base.startswith(("ln", "lnf")):
            x += np.float32(1.0)
        return x

    def _materialise(self, name: str) -> None:
        x = self._draw(name)
        if self.shape.dtype == "bf16":
            bits = round_to_bf16_bits(x)
            self._bits[name] = bits
            self._f32[name] = bf16_bits_to_f32(bits)
        else:
            self._f32[name] = x

    def values(self, name: str) -> np.ndarray:
        if name not in self._f32:
            self._materialise(name)
        return self._f32[name]

    def device_bytes(self, name: str) -> np.ndarray:
        if self.shape.dtype == "bf16":
            if name not in self._bits:
                self._materialise(name)
            return self._bits[name]
        return self.values(name)

    def __getitem__(self, name: str) -> np.ndarray:
        return self.values(name)

    def replace(self, name: str, value: np.ndarray) -> None:
        """Overwrite a parameter (tests use this for special cases)."""
        v = np.asarray(value, dtype=np.float32).reshape(self._shapes[name])
        if self.shape.dtype == "bf16":
            self._bits[name] = round_to_bf16_bits(v)
            self._f32[name] = bf16_bits_to_f32(self._bits[name])
        else:
            self._f32[name] = v.copy()


def make_weights(w: Workload | ModelShape, seed: Optional[int] = None,
                 only: Optional[List[str]] = None) -> Weights:
    if isinstance(w, Workload):
        return Weights(w.shape, w.weight_seed if seed is None else seed, only)
    return Weights(w, 1000 if seed is None else seed, only)


# --------------------------------------------------------------------------
# tokens
# --------------------------------------------------------------------------

def _zipf_cdf(vocab: int, a: float) -> np.ndarray:
    r = np.arange(1, vocab + 1, dtype=np.float64)
    p = r ** (-a)
    c = np.cumsum(p)
    return c / c[-1]


def make_tokens(w: Workload | None = None, *, batch: Optional[int] = None,
                length: Optional[int] = None, vocab: Optional[int] = None,
                kind: Optional[str] = None, seed: Optional[int] = None,
                zipf_a: float = 1.1) -> np.ndarray:
    """Token stream [batch, length] int32 (prompt followed by continuation)."""
    if w is not None:
        batch = w.batch if batch is None else batch
        length = w.max_seq if length is None else length
        vocab = w.shape.vocab if vocab is None else vocab
        kind = w.tokens if kind is None else kind
        seed = w.token_seed if seed is None else seed
    assert batch is not None and length is not None and vocab is not None
    g = np.random.Generator(np.random.PCG64(2000 if seed is None else seed))
    if kind == "zipf":
        u = g.random((batch, length))
        ids = np.searchsorted(_zipf_cdf(vocab, zipf_a), u, side="right")
        ids = np.minimum(ids, vocab - 1)
    else:
        ids = g.integers(0, vocab, size=(batch, length))
    return ids.astype(np.int32)


def iter_workloads() -> Iterator[Workload]:
    return iter(WORKLOADS.values())
