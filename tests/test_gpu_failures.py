"""Failure detection through the C-ABI, with failures made on the host:
calls in the wrong state, capacity overruns and out-of-range token ids fed
by the caller. None of these faults, traps or hangs the GPU: the library
returns an error code, or a kernel clamps the bad id, sets a bit of the
status word and finishes, and bt_sync reports BT_EDEVICE once.
"""
import numpy as np
import pytest

import synth
from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu

SHAPE = synth.ModelShape(vocab=700, d_model=256, n_heads=4, block_len=4,
                         n_block_layers=2, n_token_layers=2, prefix_len=1)


def _model(B=2, max_seq=40):
    w = synth.make_weights(SHAPE, seed=51)
    return gh.build_model(SHAPE, w, B, max_seq), w


def test_decode_before_prefill_is_a_state_error():
    from hierarchical_global_local_b200 import native
    m, _ = _model()
    with pytest.raises(native.BtError) as ei:
        m.decode(None)
    assert ei.value.code == native.BT_ESTATE
    assert m.position == native.BT_ESTATE
    m.close()


def test_capacity_errors():
    from hierarchical_global_local_b200 import native
    torch = gh.torch_mod()
    m, _ = _model(B=2, max_seq=20)
    tok = torch.zeros(3, 16, dtype=torch.int32, device="cuda")
    with pytest.raises(native.BtError) as ei:          # batch above max_batch
        m.prefill(tok)
    assert ei.value.code == native.BT_ECAPACITY
    with pytest.raises(native.BtError) as ei:          # prompt reaches max_seq
        m.prefill(torch.zeros(2, 20, dtype=torch.int32, device="cuda"))
    assert ei.value.code == native.BT_ECAPACITY
    m.prefill(tok[:2].contiguous())
    for _ in range(4):                                  # positions 16 .. 19
        m.decode(None)
    assert m.position == 20
    with pytest.raises(native.BtError) as ei:          # position 20 would exceed max_seq
        m.decode(None)
    assert ei.value.code == native.BT_ECAPACITY
    m.sync()
    m.close()


@pytest.mark.parametrize("where", ["prefill", "decode_token_step", "decode_block_step"])
def test_out_of_range_token_is_reported_once_and_the_model_recovers(where):
    """A token id >= V is clamped on the device and flagged; bt_sync returns
    BT_EDEVICE once, and the next prefill of valid ids gives the same logits
    as a fresh model."""
    from hierarchical_global_local_b200 import native
    torch = gh.torch_mod()
    B, T = 2, 16
    m, w = _model(B, 40)
    toks = synth.make_tokens(batch=B, length=T + 8, vocab=SHAPE.vocab, seed=52)
    good = torch.from_numpy(np.ascontiguousarray(toks)).cuda()
    bad = good.clone()
    if where == "prefill":
        bad[1, 5] = SHAPE.vocab + 3
        m.prefill(bad[:, :T].contiguous())
    else:
        m.prefill(good[:, :T].contiguous())
        m.sync()
        steps = 1 if where == "decode_token_step" else 4   # the 4th feed completes a block
        for i in range(steps):
            feed = good[:, T + i].contiguous()
            if i == steps - 1:
                feed = feed.clone()
                feed[0] = -7
            m.decode(feed)
    with pytest.raises(native.BtError) as ei:
        m.sync()
    assert ei.value.code == native.BT_EDEVICE
    m.sync()                                            # reported once, then clear
    # recovery: a new session on the same model matches a fresh model
    lg = torch.empty(B, SHAPE.vocab, device="cuda")
    m.prefill(good[:, :T].contiguous(), logits=lg)
    m.decode(good[:, T].contiguous(), logits=lg)
    m.sync()
    m.close()
    f, _ = _model(B, 40)
    lf = torch.empty(B, SHAPE.vocab, device="cuda")
    f.prefill(good[:, :T].contiguous(), logits=lf)
    f.decode(good[:, T].contiguous(), logits=lf)
    f.sync()
    f.close()
    assert torch.equal(lg, lf)


def test_grid_barrier_passes_every_round():
    """The bounded grid barrier of the persistent decode kernel: 200 rounds
    with every CTA arriving pass with a clean status and leave the counters
    ready for the next launch."""
    from hierarchical_global_local_b200 import native
    torch = gh.torch_mod()
    G = torch.cuda.get_device_properties(0).multi_processor_count
    st, passed, words = native.grid_barrier_selftest(200)
    assert st == 0 and passed == 200 * G and words == [0, 0, 0]


def test_grid_barrier_wait_runs_out_without_a_fault():
    """One CTA withholds its arrival: every wait runs out after ~1e5 cycles,
    the kernel returns with ST_WAIT_TIMEOUT in the status word and the abort
    word set, and the context stays usable (a clean run follows)."""
    import time
    from hierarchical_global_local_b200 import native
    torch = gh.torch_mod()
    G = torch.cuda.get_device_properties(0).multi_processor_count
    t0 = time.perf_counter()
    st, passed, words = native.grid_barrier_selftest(50, withhold_cta=G // 2, wait_cycles=100_000)
    assert time.perf_counter() - t0 < 10.0
    assert st & 2, st                        # ST_WAIT_TIMEOUT
    assert passed == 0
    assert words[2] == 1 and words[0] == 0 and words[1] == 0
    st, passed, words = native.grid_barrier_selftest(100)
    assert st == 0 and passed == 100 * G


def test_model_runs_with_a_short_wait_bound(monkeypatch):
    """BT_WAIT_CYCLES sets the bound of every wait inside the persistent
    decode kernel; a bound far below a second (1e6 cycles) is still far
    above any barrier of a healthy step, so logits are unchanged."""
    torch = gh.torch_mod()
    B, T = 2, 16
    toks = synth.make_tokens(batch=B, length=T + 6, vocab=SHAPE.vocab, seed=53)
    good = torch.from_numpy(np.ascontiguousarray(toks)).cuda()
    out = []
    for bound in (None, "1000000"):
        if bound:
            monkeypatch.setenv("BT_WAIT_CYCLES", bound)
        m, _ = _model(B, 40)
        lg = torch.empty(6, B, SHAPE.vocab, device="cuda")
        m.prefill(good[:, :T].contiguous(), logits=lg[0])
        for i in range(5):
            m.decode(good[:, T + i].contiguous(), logits=lg[i + 1])
        m.sync()
        m.close()
        out.append(lg)
    assert torch.equal(out[0], out[1])
