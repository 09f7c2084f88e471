"""Memory planning of the maximum-throughput methodology (host logic only).

The method's throughput comparisons run every model at the largest batch
its memory allows and report memory per sample (Block Transformer explainer
page, §5 "Evaluation Methodology", and Appendix J batch-size sensitivity).
``loader.max_batch_by_memory`` and ``loader.memory_per_sample`` derive both
from the library's workspace formula (``bt_workspace_bytes``), which is a
pure host function: these tests need no GPU.
"""
import pytest

import synth
from hierarchical_global_local_b200 import loader, native

pytestmark = pytest.mark.filterwarnings("ignore")


@pytest.fixture(scope="module")
def lib():
    try:
        return native.lib()
    except Exception as e:  # pragma: no cover - the library is built by build()
        pytest.skip(f"native library unavailable: {e}")


def _wl(name):
    return synth.WORKLOADS[name]


def test_max_batch_is_the_inverse_of_the_workspace(lib):
    """With a budget of exactly ws(B), the planner returns B; one byte less
    returns B - 1 (the workspace grows strictly with the batch)."""
    w = _wl("pythia160m_decode_heavy")
    for B in (1, 7, 100, 333):
        ws = loader.workspace_bytes(w.shape, B, w.max_seq)
        assert loader.max_batch_by_memory(w.shape, w.max_seq, ws) == B
        assert loader.max_batch_by_memory(w.shape, w.max_seq, ws - 1) == B - 1


def test_nothing_fits_below_one_sequence(lib):
    w = _wl("pythia160m_decode_heavy")
    ws1 = loader.workspace_bytes(w.shape, 1, w.max_seq)
    assert loader.max_batch_by_memory(w.shape, w.max_seq, ws1 - 1) == 0
    assert loader.max_batch_by_memory(w.shape, w.max_seq, 0) == 0


def test_max_batch_monotone_in_budget_and_limit(lib):
    w = _wl("pythia410m_decode_heavy")
    prev = 0
    for gb in (1, 2, 5, 10, 20, 40):
        b = loader.max_batch_by_memory(w.shape, w.max_seq, int(gb * 1e9))
        assert b >= prev
        prev = b
    assert loader.max_batch_by_memory(w.shape, w.max_seq, int(40e9), limit=17) == 17


def test_memory_per_sample_is_the_workspace_slope(lib):
    """ws(B + k) - ws(B) = k * memory_per_sample: exactly over the span the
    slope is taken on (32 -> 64 sequences), and within 1 % elsewhere (a few
    scratch buffers are sized per launch plan, not strictly per row)."""
    w = _wl("pythia160m_prefill_heavy")
    mps = loader.memory_per_sample(w.shape, w.max_seq)
    assert mps > 0
    d = loader.workspace_bytes(w.shape, 64, w.max_seq) - loader.workspace_bytes(w.shape, 32, w.max_seq)
    assert d == 32 * mps
    for B, k in ((1, 1), (10, 90), (200, 300)):
        d = loader.workspace_bytes(w.shape, B + k, w.max_seq) - loader.workspace_bytes(w.shape, B, w.max_seq)
        assert abs(d - k * mps) <= 0.01 * k * mps


def test_block_transformer_needs_less_memory_per_sample_than_vanilla(lib):
    """At equal width and depth the block decoder's KV cache is L_B-fold
    shorter and the token decoder's is bounded by P + L_B - 1 rows: the
    vanilla L_B = 1 model (24 layers of full-length KV) needs several times
    the memory per sample of L_B = 4 (12 block layers at a quarter of the
    length: 8x less KV, diluted by per-row activation buffers), and memory
    per sample falls with L_B."""
    mps = {lb: loader.memory_per_sample(_wl(f"lb_sweep_L{lb}").shape, _wl(f"lb_sweep_L{lb}").max_seq)
           for lb in (1, 2, 4, 8)}
    assert mps[1] > mps[2] > mps[4] > mps[8]
    assert 4.0 < mps[1] / mps[4] < 8.0


def test_every_benchmark_workload_is_supported(lib):
    for name, w in synth.WORKLOADS.items():
        assert loader.workspace_bytes(w.shape, w.batch, w.max_seq) > 0, name


def test_configurations_past_32_bit_buffers_are_refused(lib):
    """Kernels index within one buffer in 32 bits: a batch whose prefill
    activation rows times 5 d_model (the widest per-row buffer) reach 2^31
    elements is not supported, and the planner stops below it whatever the
    budget."""
    w = _wl("pythia160m_decode_heavy")
    n_cap = -(-w.max_seq // w.shape.block_len)
    b_edge = (2 ** 31 - 1) // (n_cap * 5 * w.shape.d_model)
    assert loader.workspace_bytes(w.shape, b_edge, w.max_seq) > 0
    assert loader.workspace_bytes(w.shape, b_edge + 1, w.max_seq) == 0
    with pytest.raises(native.BtError):
        native.workspace_bytes(loader.model_config(w.shape, b_edge + 1, w.max_seq))
    assert loader.max_batch_by_memory(w.shape, w.max_seq, 10 ** 15) == b_edge
