"""ctypes binding of the C-ABI in include/bt.h and include/bt_ops.h.

Argument marshalling only: every step of the inference path runs in the
native library's CUDA kernels. torch is used for device memory (weights,
workspace, inputs, outputs) and for the current CUDA stream. If the native
library is missing this module raises; there is no fallback.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Mapping, Optional, Tuple

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "lib", "libbt_b200.so")

BT_OK, BT_EINVAL, BT_EWORKSPACE, BT_ECAPACITY, BT_ESTATE, BT_ECUDA, BT_EDEVICE, BT_ENOTSUP = \
    0, -1, -2, -3, -4, -5, -6, -7
BT_FP32, BT_BF16 = 0, 1

c_void_p, c_int, c_int32, c_size_t, c_float = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int32,
                                               ctypes.c_size_t, ctypes.c_float)


class BtError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        msg = f"{what}: {code} ({_strerror(code)})"
        if code == BT_ECUDA:
            msg += f": {lib().bt_last_cuda_error().decode()}"
        super().__init__(msg)


class BtConfig(ctypes.Structure):
    _fields_ = [(n, c_int32) for n in (
        "vocab", "d_model", "n_heads", "block_len", "n_block_layers", "n_token_layers",
        "prefix_len", "rotary_dims", "use_token_decoder", "max_batch", "max_seq", "dtype")] + \
        [("ln_eps", c_float), ("rope_base", c_float),
         ("context_injection", c_int32), ("context_window", c_int32), ("n_kv_heads", c_int32)]


LAYER_FIELDS = ("ln1_g", "ln1_b", "ln2_g", "ln2_b", "w_qkv", "b_qkv", "w_o", "b_o",
                "w_1", "b_1", "w_2", "b_2")
GLOBAL_FIELDS = ("blk_emb", "lnf_b_g", "lnf_b_b", "w_prefix", "b_prefix", "tok_emb",
                 "lnf_t_g", "lnf_t_b", "w_lm")


class BtLayerWeights(ctypes.Structure):
    _fields_ = [(n + "_dev", c_void_p) for n in LAYER_FIELDS]


class BtWeights(ctypes.Structure):
    _fields_ = [(n + "_dev", c_void_p) for n in GLOBAL_FIELDS] + [
        ("block_layers", ctypes.POINTER(BtLayerWeights)),
        ("token_layers", ctypes.POINTER(BtLayerWeights))]


_LIB = None


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"native library not found at {LIB_PATH}; build it with "
                "`python -m hierarchical_global_local_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        sig = {
            "bt_workspace_bytes": (c_size_t, [ctypes.POINTER(BtConfig)]),
            "bt_create": (c_int, [ctypes.POINTER(BtConfig), ctypes.POINTER(BtWeights), c_void_p,
                                  c_size_t, c_void_p, ctypes.POINTER(c_void_p)]),
            "bt_prefill": (c_int, [c_void_p, c_void_p, c_int32, c_int32, c_void_p, c_void_p]),
            "bt_prefill_ragged": (c_int, [c_void_p, c_void_p, c_int32, ctypes.POINTER(c_int32), c_int32,
                                          c_int32, c_void_p, c_void_p]),
            "bt_decode_step": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p]),
            "bt_sync": (c_int, [c_void_p]),
            "bt_position": (c_int, [c_void_p]),
            "bt_destroy": (c_int, [c_void_p]),
            "bt_strerror": (ctypes.c_char_p, [c_int]),
            "bt_last_cuda_error": (ctypes.c_char_p, []),
            "bt_kernel_launches": (ctypes.c_int64, [c_void_p]),
            "bt_profile_begin": (c_int, [c_void_p, c_int32]),
            "bt_profile_end": (c_int, [c_void_p, c_void_p, c_int32, c_void_p]),
            "bt_op_decode_attention_scratch_bytes": (c_size_t, [c_int] * 5),
            "bt_op_decode_attention": (c_int, [c_int, c_void_p, c_int, c_void_p, c_void_p, c_int,
                                               c_int, c_int, c_int, c_int, c_void_p, c_int,
                                               c_void_p, c_size_t, c_void_p]),
            "bt_op_decode_attention_noalloc": (c_int, [c_int, c_void_p, c_int, c_void_p, c_void_p,
                                                       c_int, c_int, c_int, c_int, c_int,
                                                       c_void_p, c_int, c_void_p]),
            "bt_op_prefill_attention": (c_int, [c_int, c_void_p, c_int, c_void_p, c_void_p, c_int,
                                                c_int, c_int, c_int, c_int, c_void_p, c_int,
                                                c_void_p]),
            "bt_op_prefill_attention_tc": (c_int, [c_void_p, c_int, c_void_p, c_void_p, c_int, c_int,
                                                   c_int, c_int, c_int, c_int, c_void_p, c_int,
                                                   c_void_p]),
            "bt_op_linear_scratch_bytes": (c_size_t, [c_int, c_int]),
            "bt_op_linear": (c_int, [c_int, c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_int,
                                     c_int, c_int, c_int, c_int, c_void_p, c_size_t, c_void_p]),
            "bt_op_layernorm": (c_int, [c_int, c_void_p, c_int, c_int, c_void_p, c_void_p,
                                        c_float, c_void_p, c_void_p]),
            "bt_op_embed_prompt": (c_int, [c_int, c_void_p, c_int, c_int, c_int, c_void_p, c_int,
                                           c_int, c_void_p, c_void_p, c_void_p]),
            "bt_op_grid_barrier_selftest": (c_int, [c_int, c_int, ctypes.c_longlong, c_void_p, c_void_p,
                                                    c_void_p, c_void_p]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _LIB = L
    return _LIB


def exported_symbols():
    """Names of the entry points the binding expects the library to export."""
    return [
        "bt_workspace_bytes", "bt_create", "bt_prefill", "bt_prefill_ragged", "bt_decode_step", "bt_sync",
        "bt_position", "bt_destroy", "bt_strerror", "bt_last_cuda_error",
        "bt_kernel_launches", "bt_profile_begin", "bt_profile_end",
        "bt_op_decode_attention_scratch_bytes", "bt_op_decode_attention",
        "bt_op_decode_attention_noalloc",
        "bt_op_prefill_attention", "bt_op_prefill_attention_tc",
        "bt_op_linear_scratch_bytes", "bt_op_linear",
        "bt_op_layernorm", "bt_op_embed_prompt", "bt_op_grid_barrier_selftest"]


def _strerror(code: int) -> str:
    try:
        return lib().bt_strerror(code).decode()
    except Exception:
        return "?"


def _check(code: int, what: str) -> None:
    if code != BT_OK:
        raise BtError(code, what)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream() -> int:
    import torch
    return torch.cuda.current_stream().cuda_stream


# --------------------------------------------------------------------------
# model
# --------------------------------------------------------------------------

@dataclasses.dataclass
class ModelConfig:
    vocab: int
    d_model: int
    n_heads: int
    block_len: int
    n_block_layers: int
    n_token_layers: int
    prefix_len: int
    rotary_dims: int
    use_token_decoder: bool
    max_batch: int
    max_seq: int
    dtype: str = "bf16"       # "bf16" | "fp32"
    ln_eps: float = 1e-5
    rope_base: float = 10000.0
    injection: str = "prefix"  # "prefix" | "sum"
    context_window: int = 1
    n_kv_heads: int = 0        # block decoder (0: n_heads)

    def c(self) -> BtConfig:
        return BtConfig(self.vocab, self.d_model, self.n_heads, self.block_len,
                        self.n_block_layers, self.n_token_layers, self.prefix_len,
                        self.rotary_dims, 1 if self.use_token_decoder else 0, self.max_batch,
                        self.max_seq, BT_BF16 if self.dtype == "bf16" else BT_FP32,
                        self.ln_eps, self.rope_base, 1 if self.injection == "sum" else 0,
                        self.context_window, self.n_kv_heads)


def workspace_bytes(cfg: ModelConfig) -> int:
    c = cfg.c()
    n = lib().bt_workspace_bytes(ctypes.byref(c))
    if n == 0:
        raise BtError(BT_EINVAL, "bt_workspace_bytes")
    return n


class BlockTransformer:
    """A Block Transformer on the current CUDA device.

    ``weights`` maps parameter names to CUDA tensors in the config dtype:
    globals ``blk_emb, lnf_b_g, lnf_b_b, w_prefix, b_prefix, tok_emb, lnf_t_g,
    lnf_t_b, w_lm`` and per layer ``block.{l}.{ln1_g, ..., b_2}`` /
    ``token.{l}.{...}`` (layouts in include/bt.h). The weights are copied into
    the model's workspace on creation. All work runs on the CUDA stream that
    is current when the model is created.
    """

    def __init__(self, cfg: ModelConfig, weights: Mapping[str, "object"]):
        import torch
        self.cfg = cfg
        self._c = cfg.c()
        nbytes = workspace_bytes(cfg)
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        L = lambda prefix, n: (BtLayerWeights * max(n, 1))(*[
            BtLayerWeights(*[_ptr(weights[f"{prefix}.{l}.{f}"]) for f in LAYER_FIELDS])
            for l in range(n)])
        n_t = cfg.n_token_layers if cfg.use_token_decoder else 0
        self._blk_layers = L("block", cfg.n_block_layers)
        self._tok_layers = L("token", n_t)
        g = [(_ptr(weights[f]) if f in weights else None) for f in GLOBAL_FIELDS]
        self._w = BtWeights(*g, ctypes.cast(self._blk_layers, ctypes.POINTER(BtLayerWeights)),
                            ctypes.cast(self._tok_layers, ctypes.POINTER(BtLayerWeights)))
        self._stream = _stream()
        h = c_void_p()
        _check(lib().bt_create(ctypes.byref(self._c), ctypes.byref(self._w),
                               self.workspace.data_ptr(), nbytes, self._stream, ctypes.byref(h)),
               "bt_create")
        self._h = h
        self._keep = weights      # weights must outlive the creation copy
        self.sync()
        self._keep = None
        self.batch = 0

    def prefill(self, tokens, logits=None, next_tokens=None) -> Tuple[object, object]:
        """tokens: int32 CUDA [B, T]. Returns (logits [B, V] fp32 or None,
        next_tokens [B] int32)."""
        import torch
        B, T = tokens.shape
        assert tokens.dtype == torch.int32 and tokens.is_contiguous()
        if next_tokens is None:
            next_tokens = torch.empty(B, dtype=torch.int32, device="cuda")
        _check(lib().bt_prefill(self._h, tokens.data_ptr(), B, T, _ptr(logits),
                                _ptr(next_tokens)), "bt_prefill")
        self.batch = B
        return logits, next_tokens

    def prefill_ragged(self, tokens, lengths, pad_id: int = -1, logits=None,
                       next_tokens=None) -> Tuple[object, object]:
        """tokens: int32 CUDA [B, row_stride], sequence b's prompt in the first
        lengths[b] entries of its row; pad_id >= 0 left-pads every prompt to a
        block boundary (see bt_prefill_ragged)."""
        import torch
        B, stride = tokens.shape
        assert tokens.dtype == torch.int32 and tokens.is_contiguous() and len(lengths) == B
        if next_tokens is None:
            next_tokens = torch.empty(B, dtype=torch.int32, device="cuda")
        lens = (c_int32 * B)(*[int(x) for x in lengths])
        _check(lib().bt_prefill_ragged(self._h, tokens.data_ptr(), stride, lens, B, int(pad_id),
                                       _ptr(logits), _ptr(next_tokens)), "bt_prefill_ragged")
        self.batch = B
        return logits, next_tokens

    def decode(self, tokens=None, logits=None, next_tokens=None):
        """Feed one token per sequence (int32 CUDA [B], or None for greedy)."""
        import torch
        if next_tokens is None:
            next_tokens = torch.empty(self.batch, dtype=torch.int32, device="cuda")
        _check(lib().bt_decode_step(self._h, _ptr(tokens), _ptr(logits), _ptr(next_tokens)),
               "bt_decode_step")
        return logits, next_tokens

    def sync(self) -> None:
        _check(lib().bt_sync(self._h), "bt_sync")

    @property
    def position(self) -> int:
        return lib().bt_position(self._h)

    def close(self) -> None:
        if getattr(self, "_h", None):
            lib().bt_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# --------------------------------------------------------------------------
# single-kernel entry points
# --------------------------------------------------------------------------

def _dt(t) -> int:
    import torch
    return BT_BF16 if t.dtype == torch.bfloat16 else BT_FP32


def decode_attention_scratch(dtype: int, B: int, H: int, d: int, cap: int):
    import torch
    n = lib().bt_op_decode_attention_scratch_bytes(dtype, B, H, d, cap)
    return torch.zeros(n, dtype=torch.uint8, device="cuda")


def decode_attention(q, k, v, n: int, out=None, scratch=None):
    """q [B, H*d]; k, v [B, H, cap, d]; attends over entries 0..n-1."""
    import torch
    B, H, cap, d = k.shape
    if out is None:
        out = torch.empty(B, H * d, dtype=q.dtype, device="cuda")
    if scratch is None:
        scratch = decode_attention_scratch(_dt(q), B, H, d, cap)
    _check(lib().bt_op_decode_attention(_dt(q), q.data_ptr(), q.stride(0), k.data_ptr(),
                                        v.data_ptr(), B, H, d, cap, n, out.data_ptr(),
                                        out.stride(0), scratch.data_ptr(), scratch.numel(),
                                        _stream()), "bt_op_decode_attention")
    return out


def decode_attention_noalloc(q, k, v, n: int, out=None):
    """Decode attention through the entry point that takes no scratch and
    allocates nothing (fixed array inside the library; see bt_ops.h)."""
    import torch
    B, H, cap, d = k.shape
    if out is None:
        out = torch.empty(B, H * d, dtype=q.dtype, device="cuda")
    _check(lib().bt_op_decode_attention_noalloc(_dt(q), q.data_ptr(), q.stride(0), k.data_ptr(),
                                                v.data_ptr(), B, H, d, cap, n, out.data_ptr(),
                                                out.stride(0), _stream()),
           "bt_op_decode_attention_noalloc")
    return out


def prefill_attention(q, k, v, n: int, out=None):
    """q [B*n, H*d] (rows b*n + i); k, v [B, H, cap, d]; causal over 0..n-1."""
    import torch
    B, H, cap, d = k.shape
    if out is None:
        out = torch.empty(B * n, H * d, dtype=q.dtype, device="cuda")
    _check(lib().bt_op_prefill_attention(_dt(q), q.data_ptr(), q.stride(0), k.data_ptr(),
                                         v.data_ptr(), B, H, d, cap, n, out.data_ptr(),
                                         out.stride(0), _stream()), "bt_op_prefill_attention")
    return out


def prefill_attention_tc(q, k, v, n: int, out=None):
    """Tensor-core prefill attention; builds V^T [B*H][d][vt_ld] from v."""
    import torch
    B, H, cap, d = k.shape
    vt_ld = (cap + 63) // 64 * 64
    vt = torch.zeros(B * H * d, vt_ld, dtype=v.dtype, device="cuda")
    vt[:, :cap] = v.permute(0, 1, 3, 2).reshape(B * H * d, cap)
    if out is None:
        out = torch.empty(B * n, H * d, dtype=q.dtype, device="cuda")
    _check(lib().bt_op_prefill_attention_tc(q.data_ptr(), q.stride(0), k.data_ptr(), vt.data_ptr(),
                                            vt_ld, B, H, d, cap, n, out.data_ptr(), out.stride(0),
                                            _stream()), "bt_op_prefill_attention_tc")
    return out


def linear(x, w, bias=None, path: int = 0, out=None, scratch=None):
    """out = x w^T (+ bias) in fp32; x [M, K], w [N, K] (same dtype)."""
    import torch
    M, K = x.shape
    N = w.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.float32, device="cuda")
    if scratch is None:
        scratch = torch.zeros(lib().bt_op_linear_scratch_bytes(M, N), dtype=torch.uint8,
                              device="cuda")
    _check(lib().bt_op_linear(_dt(x), x.data_ptr(), x.stride(0), w.data_ptr(), _ptr(bias),
                              out.data_ptr(), out.stride(0), M, N, K, path, scratch.data_ptr(),
                              scratch.numel(), _stream()), "bt_op_linear")
    return out


def layernorm(h, g, b, eps: float, dtype):
    import torch
    M, D = h.shape
    out = torch.empty(M, D, dtype=dtype, device="cuda")
    _check(lib().bt_op_layernorm(_dt(out), h.data_ptr(), M, D, g.data_ptr(), b.data_ptr(), eps,
                                 out.data_ptr(), _stream()), "bt_op_layernorm")
    return out


def embed_prompt(tokens, table, L: int, D: int, status=None):
    import torch
    B, T = tokens.shape
    V = table.shape[0]
    h = torch.empty(B * (T // L), D, dtype=torch.float32, device="cuda")
    _check(lib().bt_op_embed_prompt(_dt(table), tokens.data_ptr(), B, T, L, table.data_ptr(), V, D,
                                    h.data_ptr(), _ptr(status), _stream()), "bt_op_embed_prompt")
    return h


def grid_barrier_selftest(rounds: int, withhold_cta: int = -1, wait_cycles: int = 2_000_000_000):
    """Run the bounded grid-barrier self-test; returns (status word, barriers
    passed summed over CTAs, the three barrier words) after synchronising."""
    import torch
    words = torch.zeros(3, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    passed = torch.zeros(1, dtype=torch.int32, device="cuda")
    _check(lib().bt_op_grid_barrier_selftest(rounds, withhold_cta, wait_cycles, words.data_ptr(),
                                             status.data_ptr(), passed.data_ptr(), _stream()),
           "bt_op_grid_barrier_selftest")
    torch.cuda.synchronize()
    return int(status.item()), int(passed.item()), [int(x) for x in words.tolist()]
