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
    assert ctypes.sizeof(B.Config) == 16 and B.Config.groups.offset == 8 and B.Config.ns_form.offset == 12
    assert ctypes.sizeof(B.Stats) == 24
    # muonh_step_args: a device pointer and an fp32 lr, padded to 16 bytes (the kernels' own table layout)
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    assert re.search(r"typedef struct \{\s*const float\* grad;\s*float lr;\s*float pad_;\s*\} muonh_step_args;", text)
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
    assert lib.muonh_init(ctypes.byref(ctx), d, 1, ctypes.byref(B.Config(0, 1e-7, 4)), None) == 1   # groups
    assert b"groups" in lib.muonh_last_error()
    assert lib.muonh_init(ctypes.byref(ctx), d, 1, ctypes.byref(B.Config(0, 1e-7, 0, 3)), None) == 1   # ns_form
    assert b"ns_form" in lib.muonh_last_error()
    assert lib.muonh_step(None, None, None, None, None) == 1
    assert lib.muonh_step_device(None, None, None, None) == 1


def _desc(**kw):
    base = dict(w=0x1000, m=0x2000, rows=4, cols=8, ld=8, radius=0.0, beta=0.95, nesterov=1, ns_steps=5,
                ns_a=3.4445, ns_b=-4.775, ns_c=2.0315, update_rule=0, weight_decay=0.0, update_scale=1.0)
    base.update(kw)
    d = (B.MatrixDesc * 1)()
    d[0] = B.MatrixDesc(*[base[f] for f, _ in B.MatrixDesc._fields_])
    return d


@pytest.mark.parametrize("kw,status", [
    (dict(rows=0), 1), (dict(cols=0), 1),                      # empty matrices
    (dict(rows=1 << 21), 1),                                   # beyond the largest dimension
    (dict(rows=16640, cols=16640, ld=16640), 6),               # Newton-Schulz side above 16384: unsupported
    (dict(update_rule=3), 1),                                  # unknown update rule
    (dict(update_rule=1, update_scale=0.0), 1),                # ordinary Muon needs a positive scale
    (dict(beta=float("nan")), 1),                              # non-finite momentum
])
def test_descriptor_edge_cases_without_a_gpu(kw, status):
    """Every descriptor check runs before the first CUDA call."""
    lib = P.library()
    ctx = ctypes.c_void_p()
    cfg = B.Config(0, 1e-7)
    assert lib.muonh_init(ctypes.byref(ctx), _desc(**kw), 1, ctypes.byref(cfg), None) == status
    assert ctx.value is None and lib.muonh_last_error()


def test_auxiliary_argument_checks_without_a_gpu():
    lib = P.library()
    ptrs = (ctypes.c_void_p * 17)(*([0x1000] * 17))
    assert lib.muonh_average(0x1000, 0, ptrs, 0, 0, 16, None) == 1       # k = 0
    assert lib.muonh_average(0x1000, 0, ptrs, 0, 17, 16, None) == 1      # k above 16
    assert lib.muonh_average(0x1000, 5, ptrs, 0, 2, 16, None) == 1       # unknown dtype
    assert lib.muonh_average(0x1000, 0, ptrs, 0, 2, -1, None) == 1       # negative count
    assert lib.muonh_average(0x1004, 0, ptrs, 0, 2, 16, None) == 2       # misaligned output
    assert lib.muonh_average(None, 0, ptrs, 0, 2, 0, None) == 0          # empty: nothing to do
    cfg = B.AdamWConfig(1e-3, 0.9, 0.95, 1e-8, 0.1)
    t = (B.AdamWTensor * 1)(B.AdamWTensor(0x1000, 0x2000, 0x3000, 0x4000, 8))
    assert lib.muonh_adamw_step(t, 1, ctypes.byref(cfg), 0, None) == 1   # step counts from 1
    bad = B.AdamWConfig(1e-3, 1.0, 0.95, 1e-8, 0.1)
    assert lib.muonh_adamw_step(t, 1, ctypes.byref(bad), 1, None) == 1   # beta1 must be < 1
    t[0] = B.AdamWTensor(0x1002, 0x2000, 0x3000, 0x4000, 8)
    assert lib.muonh_adamw_step(t, 1, ctypes.byref(cfg), 1, None) == 2   # not 4-byte aligned
    assert lib.muonh_adamw_step(t, 0, ctypes.byref(cfg), 1, None) == 0   # no tensors
    x = ctypes.c_void_p(0x5000)
    assert lib.muonh_momentum_norm_noalloc(0x1000, 0x2000, 0, 8, 8, 0.95, 1, x, None) == 1   # empty
    assert lib.muonh_momentum_norm_noalloc(0x1008, 0x2000, 4, 8, 8, 0.95, 1, x, None) == 2  # misaligned


def test_wait_probe_argument_check_without_a_gpu():
    lib = P.library()
    assert lib.muonh_check_wait_timeout(0.0, None) == 1
    assert lib.muonh_check_wait_timeout(11.0, None) == 1


def test_binding_rejects_cpu_tensors():
    """No CPU fallback: host tensors are refused before anything runs."""
    import torch
    from pretraining_optimizer_b200 import MuonH, adamw_step, average
    w = torch.zeros(8, 16)
    with pytest.raises(TypeError):
        MuonH([w])
    with pytest.raises(TypeError):
        average([w.flatten(), w.flatten()])
    with pytest.raises(TypeError):
        adamw_step([w], [w.clone()], [w.clone()], [w.clone()], 1, 1e-3)


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    """Without libmuonh.so the binding raises instead of falling back."""
    from pretraining_optimizer_b200 import muonh as M
    monkeypatch.setattr(M, "_LIB", None)
    monkeypatch.setattr(M, "library_path", lambda: str(tmp_path / "libmuonh.so"))
    with pytest.raises(RuntimeError, match="missing"):
        M.library()
