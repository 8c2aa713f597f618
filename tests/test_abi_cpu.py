"""CPU-side checks of the boundary: the library loads, exports every entry
point declared in include/*.h, and rejects invalid arguments on the host
before touching a device."""
import ctypes
import glob
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for hdr in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(hdr).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(onela_\w+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_decode_entry_points():
    names = declared_symbols()
    for n in ("onela_create", "onela_set_prompt_state", "onela_prefill", "onela_decode_step",
              "onela_reset", "onela_status", "onela_destroy", "onela_fold", "onela_read_root_state",
              "onela_read_fold_depth"):
        assert n in names


def test_library_exports_every_declared_symbol():
    import linear_attention_beam_shared_b200 as L
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (onela_\w+)", out))
    missing = [n for n in declared_symbols() if n not in exported]
    assert not missing, f"declared but not exported: {missing}"
    lib = ctypes.CDLL(L.LIB_PATH)
    for n in declared_symbols():
        assert getattr(lib, n) is not None


def test_error_strings():
    import linear_attention_beam_shared_b200 as L
    for code in range(0, 9):
        assert L.error_string(code) != "unknown error"
    assert L.error_string(99) == "unknown error"


@pytest.mark.parametrize("field,value", [
    ("R", 0), ("H", 0), ("d_k", 0), ("d_k", 257), ("d_v", 300), ("W_max", 0), ("T_max", 0),
    ("T_max", 65), ("s0_dtype", 7), ("qkv_dtype", -1), ("kernel", 9), ("s0_split", 1),
    ("device", -1),
])
def test_create_rejects_bad_config_on_the_host(field, value):
    import linear_attention_beam_shared_b200 as L
    cfg = L._lib.onela_config(1, 2, 64, 64, 8, 3, 0, 1, 0, 0, 0)
    setattr(cfg, field, value)
    out = ctypes.c_void_p()
    assert L._lib.lib.onela_create(ctypes.byref(cfg), ctypes.byref(out)) == L.ONELA_ERR_ARG
    assert out.value is None


def test_null_arguments_are_rejected():
    import linear_attention_beam_shared_b200 as L
    lib = L._lib.lib
    assert lib.onela_create(None, None) == L.ONELA_ERR_ARG
    assert lib.onela_set_prompt_state(None, None, None) == L.ONELA_ERR_ARG
    assert lib.onela_decode_step(None, 1, 1, *([None] * 9)) == L.ONELA_ERR_ARG
    assert lib.onela_reset(None, None) == L.ONELA_ERR_ARG
    assert lib.onela_status(None, None) == L.ONELA_ERR_ARG
    assert lib.onela_destroy(None) == L.ONELA_ERR_ARG
    assert lib.onela_read_records(None, 1, None, None, None, None) == L.ONELA_ERR_ARG
    assert lib.onela_read_ancestry(None, 1, None, None) == L.ONELA_ERR_ARG
    assert lib.onela_prefill(None, 4, None, None, None, None, None) == L.ONELA_ERR_ARG
    assert lib.onela_read_prompt_state(None, None, None) == L.ONELA_ERR_ARG
    assert lib.onela_fold(None, 3, None) == L.ONELA_ERR_ARG
    assert lib.onela_read_root_state(None, None, None) == L.ONELA_ERR_ARG
    assert lib.onela_read_fold_depth(None, None, None) == L.ONELA_ERR_ARG
    assert lib.onela_set_prefill_segments(None, 0) == L.ONELA_ERR_ARG
    assert lib.onela_set_wait_policy(None, 10**9, 0) == L.ONELA_ERR_ARG
    assert lib.onela_steps_done(None) == -1
    assert lib.onela_select_beams(1, 4, 4, 2, *([None] * 6), 0, 0, None) == L.ONELA_ERR_ARG


def test_select_rejects_bad_sizes_on_the_host():
    import linear_attention_beam_shared_b200 as L
    lib = L._lib.lib
    p = ctypes.c_void_p(16)  # never dereferenced: the checks come first
    args = (p, p, p, p, p, p)
    assert lib.onela_select_beams(1, 4, 4, 2049, *args, 1 << 30, 0, None) == L.ONELA_ERR_ARG  # W > 2048
    assert lib.onela_select_beams(1, 2, 2, 5, *args, 1 << 30, 0, None) == L.ONELA_ERR_ARG     # W > W_prev C
    assert lib.onela_select_beams(0, 4, 4, 2, *args, 1 << 30, 0, None) == L.ONELA_ERR_ARG     # R = 0
    need = lib.onela_select_scratch_bytes(2, 256, 256, 256)
    assert need == 2 * 2 * 16 * 256 * 8
    assert lib.onela_select_beams(2, 256, 256, 256, *args, need - 1, 0, None) == L.ONELA_ERR_SCRATCH


def test_binding_refuses_cpu_tensors():
    import torch
    import linear_attention_beam_shared_b200 as L
    with pytest.raises(ValueError):
        L._lib._ptr(torch.zeros(3), "x")
