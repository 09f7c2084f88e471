"""The CPU oracle against independent sources (no GPU)."""
import pytest

import oracle.model as om
from tests import oracle_pins as pins

# fp64 oracle vs fp64 references: agreement to rounding
TIGHT = 1e-10
# HF GPTNeoX builds its rotary cos/sin tables in fp32 even in a float64
# model, so agreement there is ~1e-8 relative; a real mistake (sign, index,
# dropped term) shows up at 1e-3 or more.
HF_TOL = 1e-6


def test_layer_norm_matches_torch():
    assert pins.pin_layer_norm(om) < TIGHT


def test_gelu_matches_torch_exact_erf():
    assert pins.pin_gelu(om) < TIGHT


def test_attention_matches_torch_sdpa_causal():
    assert pins.pin_attend(om) < TIGHT


def test_rotary_matches_complex_rotation():
    assert pins.pin_rotary(om) < TIGHT


def test_embedder_matches_brute_force():
    assert pins.pin_embedder_bruteforce(om) == 0.0


def test_identity_prefix_projection():
    assert pins.pin_identity_prefix(om) < TIGHT


def test_vanilla_special_case_equals_hf_gptneox():
    """Invariant 3: L_B = 1, no token decoder == vanilla Pythia (HF)."""
    assert pins.pin_vanilla_vs_hf(om) < HF_TOL


def test_block_transformer_equals_model_assembled_from_hf_stacks():
    assert pins.pin_block_model_vs_hf(om) < HF_TOL


def test_single_row_token_decoder_closed_form():
    assert pins.pin_single_row_token_decoder(om) < 1e-9


@pytest.mark.parametrize("variant", ["small", "vanilla", "P1_L2"])
def test_incremental_equals_full_sequence(variant):
    """Invariant 1."""
    import synth
    shape = {"small": pins.SMALL, "vanilla": pins.VANILLA,
             "P1_L2": synth.ModelShape(vocab=41, d_model=32, n_heads=2, block_len=2,
                                       n_block_layers=1, n_token_layers=3,
                                       prefix_len=1, dtype="fp32")}[variant]
    assert pins.pin_incremental_equals_full(om, shape) < 1e-10


@pytest.mark.parametrize("T", [5, 6, 7, 9, 10, 11])
def test_incremental_equals_full_sequence_partial_block_prompt(T):
    """Invariant 1 for prompts that end inside a block: the trailing tokens
    prefilled into the token decoder give the full pass's logits."""
    assert pins.pin_incremental_equals_full(om, pins.SMALL, T=T, G=9) < 1e-10


def test_left_padding():
    """Left padding adds (-T) mod L_B pad tokens (none for aligned prompts),
    and a padded prompt is run as the aligned sequence it becomes."""
    assert pins.pin_left_padding(om)


def test_ragged_batch_equals_batched_rows():
    """The per-sequence runs of a ragged batch agree with the batched session
    on every row when the rows' prompt lengths are equal, and each row of a
    ragged batch equals its own single-sequence run."""
    assert pins.pin_ragged_vs_batched(om) < 1e-12


def test_future_tokens_do_not_change_past_logits():
    """Invariant 2a."""
    assert pins.pin_future_tokens_invisible(om)


def test_token_decoder_sees_only_its_block_given_context():
    """Invariant 2b."""
    assert pins.pin_token_decoder_local(om)


def test_literal_locality_without_block_layers():
    """Invariant 2c."""
    assert pins.pin_locality_without_block_layers(om)


def test_batch_rows_are_independent():
    assert pins.pin_batch_rows_independent(om)


# ---- context injection variants (readings R9, R10) ------------------------

def test_sum_injection_reduces_to_prefix_model():
    assert pins.pin_sum_injection_reduces_to_prefix(om) < 1e-10


def test_sum_injection_slot_j_reaches_rows_from_j():
    assert pins.pin_sum_injection_slot_reach(om)


def test_window_of_context_embeddings_matches_hand_assembly():
    assert pins.pin_window_assembly_bruteforce(om) < 1e-10


@pytest.mark.parametrize("shape_name", ["SUM", "WIN"])
@pytest.mark.parametrize("T", [4, 6, 8, 13])
def test_injection_variants_incremental_equals_full(shape_name, T):
    """Invariant 1 for both variants, prompts shorter than the window (T = 4:
    one block, two zero context slots) and ending inside a block."""
    assert pins.pin_incremental_equals_full(om, shape=getattr(pins, shape_name), T=T, G=11) < 1e-10


# ---- grouped-query attention in the block decoder (reading R11) ------------

def test_gqa_equals_mha_with_shared_key_value_rows():
    assert pins.pin_gqa_equals_mha_with_shared_kv_rows(om) < 1e-10


@pytest.mark.parametrize("T", [8, 10])
def test_gqa_incremental_equals_full(T):
    assert pins.pin_incremental_equals_full(om, shape=pins.GQA, T=T, G=11) < 1e-10
