"""The C-ABI library loads and exports every function include/muonh.h declares (no GPU)."""
import ctypes
import os
import re

import pytest

import pretraining_optimizer_b200 as P
from pretraining_optimizer_b200 import muonh as B

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "muonh.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(muonh_[a-z_]+)\s*\(", text)))


def test_header_declares_the_binding_surface():
    assert set(declared_functions()) == set(P.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(P.library_path())
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_struct_layouts_match_the_header():
    assert ctypes.sizeof(B.MatrixDesc) == 80
    assert ctypes.sizeof(B.Config) == 8
    assert ctypes.sizeof(B.Stats) == 24
    assert B.MatrixDesc.radius.offset == 40 and B.MatrixDesc.ns_c.offset == 64
    assert B.MatrixDesc.update_rule.offset == 68 and B.MatrixDesc.update_scale.offset == 76


def test_status_strings_and_argument_checks_without_a_gpu():
    lib = P.library()
    assert lib.muonh_status_string(0) == b"ok"
    assert lib.muonh_status_string(2) == b"misaligned pointer or stride"
    ctx = ctypes.c_void_p()
    # NULL descriptor list is rejected before any CUDA call
    st = lib.muonh_init(ctypes.byref(ctx), None, 0, None, None)
    assert st == 1 and ctx.value is None
    assert b"n <= 0" in lib.muonh_last_error()
    # a misaligned weight pointer is rejected before any CUDA call
    d = (B.MatrixDesc * 1)()
    d[0] = B.MatrixDesc(0x1004, 0x2000, 4, 8, 8, 0.0, 0.95, 1, 5, 3.4445, -4.775, 2.0315)
    cfg = B.Config(0, 1e-7)
    assert lib.muonh_init(ctypes.byref(ctx), d, 1, ctypes.byref(cfg), None) == 2
    d[0] = B.MatrixDesc(0x1000, 0x2000, 4, 8, 6, 0.0, 0.95, 1, 5, 3.4445, -4.775, 2.0315)
    assert lib.muonh_init(ctypes.byref(ctx), d, 1, ctypes.byref(cfg), None) == 1   # ld < cols
    d[0] = B.MatrixDesc(0x1000, 0x2000, 4, 8, 8, 0.0, 0.95, 1, 65, 3.4445, -4.775, 2.0315)
    assert lib.muonh_init(ctypes.byref(ctx), d, 1, ctypes.byref(cfg), None) == 1   # ns_steps > 64
    cfg_bad = B.Config(7, 1e-7)
    d[0] = B.MatrixDesc(0x1000, 0x2000, 4, 8, 8, 0.0, 0.95, 1, 5, 3.4445, -4.775, 2.0315)
    assert lib.muonh_init(ctypes.byref(ctx), d, 1, ctypes.byref(cfg_bad), None) == 1
    assert lib.muonh_step(None, None, None, None, None) == 1
