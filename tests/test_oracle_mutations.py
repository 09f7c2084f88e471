"""Planted mistakes: each plausible bug in the oracle must fail at least one pin.

Mistakes are planted in the CPU oracle only (monkeypatched module globals).
"""
import math

import numpy as np
import pytest

import oracle.model as om
from tests import oracle_pins as pins

TOL = 1e-6

# originals, captured before any test patches the module
ORIG = {n: getattr(om, n) for n in ("rotary", "layer_norm", "gelu", "attend",
                                    "embed_blocks", "prefix_projection",
                                    "pythia_layer")}


def _first_failing_pin(mod):
    """Name of the first pin the module fails, or None. Exceptions propagate:
    a mutation that merely crashes does not count as caught."""
    checks = [
        ("layer_norm", lambda: pins.pin_layer_norm(mod) < TOL),
        ("gelu", lambda: pins.pin_gelu(mod) < TOL),
        ("attend", lambda: pins.pin_attend(mod) < TOL),
        ("rotary", lambda: pins.pin_rotary(mod) < TOL),
        ("embedder", lambda: pins.pin_embedder_bruteforce(mod) == 0.0),
        ("identity_prefix", lambda: pins.pin_identity_prefix(mod) < TOL),
        ("single_row", lambda: pins.pin_single_row_token_decoder(mod) < TOL),
        ("future_invisible", lambda: pins.pin_future_tokens_invisible(mod)),
        ("locality_nb0", lambda: pins.pin_locality_without_block_layers(mod)),
        ("incremental", lambda: pins.pin_incremental_equals_full(mod) < TOL),
        ("incremental_partial", lambda: pins.pin_incremental_equals_full(mod, T=10, G=7) < TOL),
        ("hf_vanilla", lambda: pins.pin_vanilla_vs_hf(mod) < TOL),
        ("hf_block_model", lambda: pins.pin_block_model_vs_hf(mod) < TOL),
        ("sum_reduces_to_prefix", lambda: pins.pin_sum_injection_reduces_to_prefix(mod) < TOL),
        ("sum_slot_reach", lambda: pins.pin_sum_injection_slot_reach(mod)),
        ("window_assembly", lambda: pins.pin_window_assembly_bruteforce(mod) < TOL),
        ("incremental_sum", lambda: pins.pin_incremental_equals_full(mod, shape=pins.SUM, T=6, G=9) < TOL),
        ("incremental_window", lambda: pins.pin_incremental_equals_full(mod, shape=pins.WIN, T=6, G=9) < TOL),
        ("gqa_vs_mha", lambda: pins.pin_gqa_equals_mha_with_shared_kv_rows(mod) < TOL),
        ("incremental_gqa", lambda: pins.pin_incremental_equals_full(mod, shape=pins.GQA, T=6, G=9) < TOL),
    ]
    for name, c in checks:
        if not c():
            return name
    return None


def _rotary_wrong_sign(x, pos, r, base):
    return ORIG["rotary"](x, -pos, r, base)


def _rotary_wrong_freq(x, pos, r, base):
    # exponent over the head dim instead of the rotary dims
    return ORIG["rotary"](x, pos, r, base ** 2)


def _ln_unbiased(x, g, b, eps):
    mu = x.mean(-1, keepdims=True)
    var = ((x - mu) ** 2).sum(-1, keepdims=True) / (x.shape[-1] - 1)
    return (x - mu) / np.sqrt(var + eps) * g + b


def _gelu_tanh(x):
    return 0.5 * x * (1 + np.tanh(math.sqrt(2 / math.pi) * (x + 0.044715 * x ** 3)))


def _attend_no_mask(q, k, v, q_pos, k_pos):
    return ORIG["attend"](q, k, v, np.full_like(q_pos, 10 ** 9), k_pos)


def _attend_scale_d(q, k, v, q_pos, k_pos):
    return ORIG["attend"](q / math.sqrt(q.shape[-1]), k, v, q_pos, k_pos)


def _embed_reversed(tokens, table, L):
    return ORIG["embed_blocks"](tokens[:, ::-1].copy(), table, L)[:, ::-1]


def _embed_reversed_within_block(tokens, table, L):
    B, S = tokens.shape
    n = S // L
    t = tokens[:, :n * L].reshape(B, n, L)[:, :, ::-1].reshape(B, n * L)
    return ORIG["embed_blocks"](t, table, L)


def _prefix_colmajor(c, w, b, P):
    D = c.shape[-1]
    out = c @ w.T + b
    return np.swapaxes(out.reshape(*c.shape[:-1], D, P), -1, -2)


def _layer_drop_bias_o(h, p, pos, cache, H, r, eps, base, hk=None):
    p2 = dict(p)
    p2["b_o"] = np.zeros_like(p["b_o"])
    return ORIG["pythia_layer"](h, p2, pos, cache, H, r, eps, base, hk)


def _layer_serial_residual(h, p, pos, cache, H, r, eps, base, hk=None):
    # GPT-2 style sequential residual instead of Pythia's parallel form
    p_att = dict(p)
    for n in ("w_1", "b_1", "w_2", "b_2"):
        p_att[n] = np.zeros_like(p[n])
    h1 = ORIG["pythia_layer"](h, p_att, pos, cache, H, r, eps, base, hk)
    m = ORIG["layer_norm"](h1, p["ln2_g"], p["ln2_b"], eps)
    return h1 + ORIG["gelu"](m @ p["w_1"].T + p["b_1"]) @ p["w_2"].T + p["b_2"]


_ORIG_START = om.OracleSession._start_block


def _start_block_trailing_shifted(self, trailing=None):
    # trailing prompt tokens one local position too far
    if trailing is None or trailing.shape[1] == 0:
        return _ORIG_START(self, trailing)
    m = self.m
    self.token_caches = m._fresh(m.token_layers)
    pre, add = m.context_input(self.c_win)
    self.add = add
    rows = np.concatenate([pre, m.token_rows(trailing, np.arange(trailing.shape[1]), add)], axis=1)
    P = pre.shape[1]
    pos = np.concatenate([np.arange(P), P + 1 + np.arange(trailing.shape[1])])
    return self._token_rows(rows, pos)[:, -1]


def _start_block_trailing_dropped(self, trailing=None):
    return _ORIG_START(self, None)


SESSION_MUTATIONS = {
    "trailing_shifted": _start_block_trailing_shifted,
    "trailing_dropped": _start_block_trailing_dropped,
}


def _layer_gqa_interleaved(h, p, pos, cache, H, r, eps, base, hk=None):
    # query head h reads key/value head h % H_kv instead of h // (H / H_kv)
    if not hk or hk == H:
        return ORIG["pythia_layer"](h, p, pos, cache, H, r, eps, base, hk)
    B, n, D = h.shape
    d = D // H
    Dk = hk * d
    a = ORIG["layer_norm"](h, p["ln1_g"], p["ln1_b"], eps)
    m = ORIG["layer_norm"](h, p["ln2_g"], p["ln2_b"], eps)
    qkv = a @ p["w_qkv"].T + p["b_qkv"]
    q = ORIG["rotary"](qkv[..., :D].reshape(B, n, H, d), pos, r, base)
    k = ORIG["rotary"](qkv[..., D:D + Dk].reshape(B, n, hk, d), pos, r, base)
    v = qkv[..., D + Dk:].reshape(B, n, hk, d)
    cache.append(k, v, pos)
    kk = np.tile(cache.k, (1, 1, H // hk, 1))
    vv = np.tile(cache.v, (1, 1, H // hk, 1))
    att = ORIG["attend"](q, kk, vv, pos, cache.pos).reshape(B, n, D)
    mlp = ORIG["gelu"](m @ p["w_1"].T + p["b_1"]) @ p["w_2"].T + p["b_2"]
    return h + (att @ p["w_o"].T + p["b_o"]) + mlp


MUTATIONS = {
    "gqa_interleaved": ("pythia_layer", _layer_gqa_interleaved),
    "rotary_sign": ("rotary", _rotary_wrong_sign),
    "rotary_freq": ("rotary", _rotary_wrong_freq),
    "ln_unbiased": ("layer_norm", _ln_unbiased),
    "gelu_tanh": ("gelu", _gelu_tanh),
    "attend_no_mask": ("attend", _attend_no_mask),
    "attend_scale_d": ("attend", _attend_scale_d),
    "embed_reversed": ("embed_blocks", _embed_reversed_within_block),
    "prefix_colmajor": ("prefix_projection", _prefix_colmajor),
    "drop_b_o": ("pythia_layer", _layer_drop_bias_o),
    "serial_residual": ("pythia_layer", _layer_serial_residual),
}


# context injection variants (readings R9, R10): planted on the model class
_ORIG_CTX = om.BlockTransformerOracle.context_input
_ORIG_ROWS = om.BlockTransformerOracle.token_rows


def _ctx_window_newest_first(self, c_win):
    return _ORIG_CTX(self, c_win[:, ::-1])


def _ctx_window_clamped(self, c_win):
    # history before block 0 repeats the oldest known embedding instead of zeros
    c = c_win.copy()
    nz = np.abs(c).sum(axis=-1) > 0
    for b in range(c.shape[0]):
        idx = np.flatnonzero(nz[b])
        if idx.size:
            c[b, :idx[0]] = c[b, idx[0]]
    return _ORIG_CTX(self, c)


def _ctx_sum_slots_shifted(self, c_win):
    rows, add = _ORIG_CTX(self, c_win)
    if add is None:
        return rows, add
    # s_j added one row early: token rows get s_{j+2}, the last gets s_1
    return rows, np.roll(add, -1, axis=1)


def _rows_sum_own_slot(self, tok, j, add):
    # token j of the block gets s_j instead of s_{j+1}
    rows = self.g["tok_emb"][tok]
    if add is not None:
        full = np.concatenate([np.zeros_like(add[:, :1]), add], axis=1)
        rows = rows + full[:, j]
    return rows


MODEL_MUTATIONS = {
    "window_newest_first": ("context_input", _ctx_window_newest_first),
    "window_clamped_history": ("context_input", _ctx_window_clamped),
    "sum_slots_shifted": ("context_input", _ctx_sum_slots_shifted),
    "sum_own_slot": ("token_rows", _rows_sum_own_slot),
}


@pytest.mark.parametrize("mutation", sorted(MODEL_MUTATIONS))
def test_planted_injection_mistake_is_caught(mutation, monkeypatch):
    name, fn = MODEL_MUTATIONS[mutation]
    monkeypatch.setattr(om.BlockTransformerOracle, name, fn)
    caught_by = _first_failing_pin(om)
    print(f"{mutation}: caught by {caught_by}")
    assert caught_by is not None, f"no pin caught the planted mistake {mutation}"


def test_unmutated_oracle_passes_every_pin():
    assert _first_failing_pin(om) is None


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_planted_mistake_is_caught(mutation, monkeypatch):
    name, fn = MUTATIONS[mutation]
    monkeypatch.setattr(om, name, fn)
    caught_by = _first_failing_pin(om)
    print(f"{mutation}: caught by {caught_by}")
    assert caught_by is not None, f"no pin caught the planted mistake {mutation}"


@pytest.mark.parametrize("mutation", sorted(SESSION_MUTATIONS))
def test_planted_prefill_mistake_is_caught(mutation, monkeypatch):
    monkeypatch.setattr(om.OracleSession, "_start_block", SESSION_MUTATIONS[mutation])
    caught_by = _first_failing_pin(om)
    print(f"{mutation}: caught by {caught_by}")
    assert caught_by is not None, f"no pin caught the planted mistake {mutation}"
