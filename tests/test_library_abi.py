"""The C-ABI library builds, loads and exports every function its header declares.

CPU only: no compute call is made (there is no GPU here)."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(re.findall(r"\b(e0_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


def test_header_declares_the_boundary_calls():
    names = declared_functions()
    for required in ("e0_create", "e0_destroy", "e0_register_model", "e0_moe_layer_forward",
                     "e0_prerouter_predict", "e0_stream_register", "e0_stage_experts",
                     "e0_moe_stack_decode", "e0_get_stats", "e0_sync_status", "e0_last_error"):
        assert required in names


def test_library_builds_loads_and_exports_every_declared_symbol():
    from int4_expert_streaming_prerouter_b200 import build
    path = build.build()
    lib = ctypes.CDLL(path)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    # the binding's signature table covers the header
    import int4_expert_streaming_prerouter_b200 as e0
    assert set(declared_functions()) <= set(e0._SIGS)
    lib.e0_last_error.restype = ctypes.c_char_p
    assert isinstance(lib.e0_last_error(), bytes)   # the thread's last message (earlier tests may have set one)


def test_create_rejects_unsupported_dims_without_touching_a_gpu():
    import int4_expert_streaming_prerouter_b200 as e0
    L = e0.lib()
    bad = e0.make_dims(100, 16, 128, 4, 8)          # d not a multiple of 256
    h = ctypes.c_void_p()
    assert L.e0_create(ctypes.byref(bad), 1, 1, ctypes.byref(h)) == -1
    assert b"unsupported dims" in L.e0_last_error()
    assert L.e0_create(None, 1, 1, ctypes.byref(h)) == -1
    assert L.e0_moe_layer_forward(None, 0, None, 1, None, None, None, None, None, None) == -1
    assert L.e0_sync_status(None) == -1
    assert L.e0_moe_stack_decode_host(None, None, 1, 0, None, None, 0, 0, None) == -1
    assert L.e0_host_io_wait(None, None) == -1
