"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point the header declares, and rejects bad arguments before it
touches a device."""
import ctypes
import os
import re

import pytest

from vla_flow_matching_denoise_b200 import binding, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            src = open(os.path.join(inc, f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"\b(fm_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def test_header_declares_the_binding_exports():
    assert set(_declared()) == set(binding.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_status_strings_and_version(lib):
    assert lib.fm_abi_version() == 1
    assert lib.fm_status_string(0) == b"FM_OK"
    assert lib.fm_status_string(5) == b"FM_ERR_TIMEOUT"


def test_null_handles_are_safe(lib):
    assert lib.fm_expert_destroy(None) == 0
    assert lib.fm_trace_bytes(None) == 0
    assert lib.fm_sync(None, None) == 1
    assert lib.fm_denoise(None, None, 1, 10, None, None) == 1
    assert lib.fm_set_prefix_varlen(None, None, None, 1, None, 0, None) == 1
    assert lib.fm_quantize_act_e4m3(None, None, 1, 256, None, None, None) == 1
    assert lib.fm_set_prefix_builder(None, None, 64) == 1
    assert lib.fm_build_prefix(None, None, 1, 1, None) == 1
    assert lib.fm_get_prefix_kv(None, 0, 0, None, None) == 1
    assert lib.fm_get_nvfp4_weights(None, 0, 4, None, None, None) == 1
    assert lib.fm_get_fp8_weights(None, 0, 0, None, None) == 1


def _cfg(**kw):
    c = binding.make_config(synth.WORKLOADS["tiny"])
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("field,value,status", [
    ("d_model", 100, 1),          # not a multiple of 64
    ("head_dim", 96, 6),          # unsupported head width
    ("n_q_heads", 3, 1),          # not a multiple of n_kv_heads
    ("chunk_len", 64, 6),         # more than one 50-row tile
    ("max_steps", 65, 1),         # modulation rows per tile
    ("rms_eps", 0.0, 1),
    ("wtype", 7, 1),
    ("max_batch", 0, 1),
])
def test_create_rejects_bad_config_before_touching_the_device(lib, field, value, status):
    cfg = _cfg(**{field: value})
    h = ctypes.c_void_p()
    w = binding.FmWeights()
    st = lib.fm_expert_create(ctypes.byref(cfg), ctypes.byref(w), 0, ctypes.byref(h))
    assert st == status, lib.fm_last_error(None)
    assert not h.value
    assert lib.fm_last_error(None)


@pytest.mark.parametrize("field,value", [("d_ff", 1088), ("n_q_heads", 2), ("d_model", 192)])
def test_create_rejects_w8a8_shapes_before_touching_the_device(lib, field, value):
    # the W8A8 path quantises o and u per row in blocks of 256 columns and
    # runs on the batched kernels (d a multiple of 256)
    cfg = _cfg(wtype=binding.FM_W_W8A8_E4M3, **{field: value})
    if field == "n_q_heads":
        cfg.n_kv_heads = 1
    h = ctypes.c_void_p()
    w = binding.FmWeights()
    st = lib.fm_expert_create(ctypes.byref(cfg), ctypes.byref(w), 0, ctypes.byref(h))
    assert st == 6, lib.fm_last_error(None)
    assert not h.value
    assert b"W8A8" in lib.fm_last_error(None)


def test_create_rejects_null_weights(lib):
    cfg = _cfg()
    h = ctypes.c_void_p()
    assert lib.fm_expert_create(ctypes.byref(cfg), None, 0, ctypes.byref(h)) == 1
    assert lib.fm_expert_create(ctypes.byref(cfg), ctypes.byref(binding.FmWeights()), 0,
                                ctypes.byref(h)) == 1


def test_binding_raises_when_library_missing(tmp_path):
    with pytest.raises(FileNotFoundError):
        binding._lib = None
        try:
            binding.load(str(tmp_path / "nope.so"))
        finally:
            binding._lib = None
