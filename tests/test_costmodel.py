"""Bytes/FLOPs model against the page's worked numbers (no GPU)."""
import json
import os

import pytest

from hierarchical_global_local_b200 import costmodel as cm
import synth

G = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                "cost_model_worked_examples.json")))


def test_llama7b_worked_example():
    g = G["llama7b"]
    assert 2 * g["n_params"] == g["flops_per_token"]
    assert g["n_params"] * g["bytes_per_elem"] == g["param_bytes"]
    per_tok = cm.kv_bytes_per_token(g["n_layers"], g["d_model"], g["bytes_per_elem"])
    assert per_tok == g["kv_bytes_per_token"]
    assert per_tok * g["seq_len"] * g["batch"] == g["kv_total_gib"] * 2 ** 30


def test_total_kv_reads():
    assert cm.total_kv_reads(G["kv_reads_sum"]["L"]) == G["kv_reads_sum"]["value"]
    assert sum(range(1, 101)) == cm.total_kv_reads(100)


def test_token_decoder_reduction():
    t = G["token_decoder_reduction"]
    assert cm.token_decoder_kv_reduction(t["L"], t["block_len"]) == t["R"]


def test_block_decoder_kv_io_falls_by_block_len_squared():
    t = G["block_decoder_kv_io"]
    r = cm.block_decoder_kv_io_ratio(t["L"], t["block_len"])
    assert abs(r / t["ratio_limit"] - 1) < 0.01
    for lb in (2, 8):
        assert abs(cm.block_decoder_kv_io_ratio(4096, lb) / lb ** 2 - 1) < 0.01


def test_block_step_kv_bytes_match_cache_size():
    s = cm.Shape.of(synth.WORKLOADS["pythia160m_decode_heavy"].shape)
    a = cm.block_step(s, 64, 100)
    b = cm.block_step(s, 64, 101)
    # one more cached entry per (sequence, layer): 2 * D * 2 bytes each
    assert b.bytes - a.bytes == 64 * 6 * 2 * 768 * 2


def test_generate_schedule_counts():
    s = cm.Shape.of(synth.WORKLOADS["pythia160m_decode_heavy"].shape)
    g = cm.generate(s, 64, 128, 2048)
    assert g.n_block_steps + g.n_token_steps == 2047
    # fed positions 128..2174; a block completes when t % 4 == 3: 131, ..., 2171
    assert g.n_block_steps == 511


def test_decode_heavy_is_bandwidth_bound_prefill_heavy_prefill_is_compute_bound():
    s = cm.Shape.of(synth.WORKLOADS["pythia160m_decode_heavy"].shape)
    bw, tf = 6539.5, 1624.7
    g = cm.generate(s, 64, 128, 2048, per_step_roofline=(bw, tf))
    assert g.decode.bytes / (bw * 1e9) > g.decode.flops / (tf * 1e12)
    p = cm.prefill(s, 64, 2048)
    assert p.flops / (tf * 1e12) > p.bytes / (bw * 1e9)


def test_vanilla_has_no_token_decoder_cost():
    s = cm.Shape.of(synth.WORKLOADS["lb_sweep_L1"].shape)
    c = cm.decode_step(s, 128, 2048)
    assert s.n_token_layers == 0 and s.prefix_len == 0
    assert c.bytes > 0
