"""The C-ABI library loads and exports every entry point declared in
include/*.h; host-side validation works without a GPU (no compute calls)."""
import ctypes
import os
import re

import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for h in ("bt.h", "bt_ops.h"):
        src = open(os.path.join(ROOT, "include", h)).read()
        names += re.findall(r"^BT_API[^(]*?\b(bt_\w+)\(", src, flags=re.M)
    return names


@pytest.fixture(scope="module")
def native():
    from hierarchical_global_local_b200 import build, native
    build.build()
    return native


def test_every_declared_symbol_is_exported(native):
    L = native.lib()
    declared = _declared()
    assert len(declared) >= 16
    missing = [n for n in declared if not hasattr(L, n)]
    assert not missing, missing
    assert sorted(declared) == sorted(native.exported_symbols())


def test_workspace_bytes_valid_and_invalid(native):
    wl = synth.WORKLOADS["pythia160m_decode_heavy"]
    from tests.gpu_helpers import model_config
    cfg = model_config(wl.shape, wl.batch, wl.max_seq)
    n = native.workspace_bytes(cfg)
    # at least the repacked weights and both KV caches
    D, V = 768, 50304
    weights = 12 * 12 * D * D * 2 + 2 * V * D * 2 + V * (D // 4) * 2
    kv = 2 * 6 * 64 * D * ((wl.max_seq + 3) // 4) * 2
    assert n >= weights + kv
    bad = model_config(wl.shape, wl.batch, wl.max_seq)
    bad.n_heads = 7                 # D % H != 0
    with pytest.raises(native.BtError):
        native.workspace_bytes(bad)
    bad2 = model_config(wl.shape, wl.batch, wl.max_seq)
    bad2.use_token_decoder = False  # vanilla requires L_B = 1
    with pytest.raises(native.BtError):
        native.workspace_bytes(bad2)


def test_create_rejects_null_arguments_without_touching_the_gpu(native):
    L = native.lib()
    c = native.ModelConfig(512, 128, 4, 4, 2, 2, 1, 8, True, 2, 80, "fp32").c()
    h = ctypes.c_void_p()
    assert L.bt_create(ctypes.byref(c), None, None, 0, None, ctypes.byref(h)) == native.BT_EINVAL
    w = native.BtWeights()
    assert L.bt_create(ctypes.byref(c), ctypes.byref(w), None, 0, None,
                       ctypes.byref(h)) == native.BT_EWORKSPACE
    assert L.bt_decode_step(None, None, None, None) == native.BT_EINVAL
    assert L.bt_prefill(None, None, 1, 4, None, None) == native.BT_EINVAL


def test_strerror_names_every_code(native):
    L = native.lib()
    for code in range(0, -8, -1):
        s = L.bt_strerror(code).decode()
        assert s and s != "unknown status"


def test_workspace_bytes_deterministic_and_monotone(native):
    """The workspace size is a pure function of the configuration (no device
    query) and grows with the batch and sequence capacity."""
    from tests.gpu_helpers import model_config
    wl = synth.WORKLOADS["pythia160m_decode_heavy"]
    base = native.workspace_bytes(model_config(wl.shape, wl.batch, wl.max_seq))
    assert base == native.workspace_bytes(model_config(wl.shape, wl.batch, wl.max_seq))
    assert native.workspace_bytes(model_config(wl.shape, wl.batch + 1, wl.max_seq)) > base
    assert native.workspace_bytes(model_config(wl.shape, wl.batch, wl.max_seq + 4 * 64)) > base
    assert native.workspace_bytes(model_config(wl.shape, 1, wl.max_seq)) < base
