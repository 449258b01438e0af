"""ctypes binding of libmuonh.so: argument marshalling only.

Every step of the optimizer runs in the library's CUDA kernels; PyTorch is
used for device memory (the caller's weight, momentum and gradient tensors)
and streams.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, Structure, c_char_p, c_float, c_int32, c_int64, c_size_t, c_uint32, c_void_p

QUINTIC = (3.4445, -4.7750, 2.0315)
NS_FP16, NS_BF16, NS_FP32 = 0, 1, 2
_PREC = {"fp16": NS_FP16, "bf16": NS_BF16, "fp32": NS_FP32}
RULE_HYPERBALL, RULE_DECOUPLED_WD, RULE_ELR_ALIGNED = 0, 1, 2
_RULE = {"hyperball": RULE_HYPERBALL, "decoupled_wd": RULE_DECOUPLED_WD, "elr_aligned": RULE_ELR_ALIGNED}
FLAG_NONFINITE_INPUT = 1
FLAG_ZERO_UPDATE = 2
FLAG_NONFINITE_UPDATE = 4
FLAG_DEGENERATE = 8
FLAG_TIMEOUT = 16

EXPORTED_SYMBOLS = (
    "muonh_init", "muonh_step", "muonh_step_device", "muonh_get_stats", "muonh_get_update", "muonh_get_radius",
    "muonh_export_state", "muonh_import_state", "muonh_device_status", "muonh_last_launch_count",
    "muonh_enable_timing", "muonh_phase_times", "muonh_phase_flops", "muonh_momentum_norm_noalloc",
    "muonh_average",
    "muonh_adamw_step", "muonh_check_wait_timeout", "muonh_destroy", "muonh_status_string", "muonh_last_error",
)
DTYPE_F32, DTYPE_BF16 = 0, 1
AVERAGE_MAX_INPUTS = 16
ADAMW_MAX_TENSORS = 32
PHASES = ("momentum_norm", "finalize_input", "write_x", "ns_gram", "ns_square", "ns_apply",
          "update_dots", "finalize_update", "project", "finalize_step", "ns_product")
NS_FORMS = {"auto": 0, "y": 1, "gram": 2}


class MatrixDesc(Structure):
    _fields_ = [("w", c_void_p), ("m", c_void_p), ("rows", c_int64), ("cols", c_int64),
                ("ld", c_int64), ("radius", c_float), ("beta", c_float), ("nesterov", c_int32),
                ("ns_steps", c_int32), ("ns_a", c_float), ("ns_b", c_float), ("ns_c", c_float),
                ("update_rule", c_int32), ("weight_decay", c_float), ("update_scale", c_float)]


class Config(Structure):
    _fields_ = [("ns_precision", c_int32), ("eps", c_float), ("groups", c_int32), ("ns_form", c_int32)]


class Stats(Structure):
    _fields_ = [("elr", c_float), ("pre_norm", c_float), ("post_norm", c_float),
                ("update_norm", c_float), ("input_norm", c_float), ("flags", c_uint32)]


class AdamWTensor(Structure):
    _fields_ = [("p", c_void_p), ("m", c_void_p), ("v", c_void_p), ("g", c_void_p), ("count", c_int64)]


class AdamWConfig(Structure):
    _fields_ = [("lr", c_float), ("beta1", c_float), ("beta2", c_float), ("eps", c_float),
                ("weight_decay", c_float)]


class MuonHError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"muonh status {status}: {message}")
        self.status = status


def library_path() -> str:
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmuonh.so")


_LIB = None


def library() -> ctypes.CDLL:
    """Load libmuonh.so (raises if it has not been built)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m pretraining_optimizer_b200.build`")
    lib = ctypes.CDLL(path)
    lib.muonh_init.argtypes = [POINTER(c_void_p), POINTER(MatrixDesc), c_int32, POINTER(Config), c_void_p]
    lib.muonh_step.argtypes = [c_void_p, POINTER(c_float), POINTER(c_void_p), c_void_p, c_void_p]
    lib.muonh_step_device.argtypes = [c_void_p, c_void_p, c_void_p, c_void_p]
    lib.muonh_get_stats.argtypes = [c_void_p, POINTER(Stats)]
    lib.muonh_get_update.argtypes = [c_void_p, c_int32, c_void_p, c_int64, c_void_p]
    lib.muonh_get_radius.argtypes = [c_void_p, POINTER(c_float)]
    lib.muonh_export_state.argtypes = [c_void_p, c_void_p, POINTER(c_size_t)]
    lib.muonh_import_state.argtypes = [c_void_p, c_void_p, c_size_t]
    lib.muonh_device_status.argtypes = [c_void_p]
    lib.muonh_last_launch_count.argtypes = [c_void_p]
    lib.muonh_last_launch_count.restype = c_int32
    lib.muonh_enable_timing.argtypes = [c_void_p, c_int32]
    lib.muonh_phase_times.argtypes = [c_void_p, POINTER(c_float), POINTER(c_int64)]
    lib.muonh_phase_flops.argtypes = [c_void_p, POINTER(ctypes.c_double)]
    lib.muonh_momentum_norm_noalloc.argtypes = [c_void_p, c_void_p, c_int64, c_int64, c_int64, c_float,
                                                c_int32, c_void_p, c_void_p]
    lib.muonh_average.argtypes = [c_void_p, c_int32, POINTER(c_void_p), c_int32, c_int32, c_int64, c_void_p]
    lib.muonh_adamw_step.argtypes = [POINTER(AdamWTensor), c_int32, POINTER(AdamWConfig), c_int64, c_void_p]
    lib.muonh_check_wait_timeout.argtypes = [ctypes.c_double, c_void_p]
    lib.muonh_destroy.argtypes = [c_void_p]
    lib.muonh_destroy.restype = None
    lib.muonh_status_string.argtypes = [c_int32]
    lib.muonh_status_string.restype = c_char_p
    lib.muonh_last_error.argtypes = []
    lib.muonh_last_error.restype = c_char_p
    for name in ("muonh_init", "muonh_step", "muonh_step_device", "muonh_get_stats", "muonh_get_update", "muonh_get_radius",
                 "muonh_export_state", "muonh_import_state", "muonh_device_status",
                 "muonh_enable_timing", "muonh_phase_times", "muonh_phase_flops", "muonh_momentum_norm_noalloc",
                 "muonh_average", "muonh_adamw_step", "muonh_check_wait_timeout"):
        getattr(lib, name).restype = c_int32
    _LIB = lib
    return lib


def _check(status: int) -> None:
    if status != 0:
        lib = library()
        msg = lib.muonh_last_error().decode() or lib.muonh_status_string(status).decode()
        raise MuonHError(status, msg)


def _stream_handle(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _matrix_view(t, what: str):
    import torch
    if not isinstance(t, torch.Tensor) or t.dtype != torch.float32 or not t.is_cuda or t.dim() != 2:
        raise TypeError(f"{what} must be a 2-D fp32 CUDA tensor")
    if t.stride(1) != 1:
        raise ValueError(f"{what} must have unit column stride")
    return t.data_ptr(), t.shape[0], t.shape[1], max(t.stride(0), t.shape[1])


def momentum_norm_noalloc(m, g, beta=0.95, nesterov=True, x_norm=None, stream=None):
    """Allocation-free momentum stage for one matrix (no context, no device
    allocation inside the library): m <- beta m + g in place; returns the
    device fp64 tensor holding ||X||_F of the Newton-Schulz input."""
    import torch
    mp, rows, cols, ld = _matrix_view(m, "m")
    gp, gr, gc, gld = _matrix_view(g, "g")
    if (gr, gc, gld) != (rows, cols, ld):
        raise ValueError("g must match m in shape and stride")
    if x_norm is None:
        x_norm = torch.empty((), dtype=torch.float64, device=m.device)
    _check(library().muonh_momentum_norm_noalloc(mp, gp, rows, cols, ld, float(beta), int(bool(nesterov)),
                                                 x_norm.data_ptr(), _stream_handle(stream)))
    return x_norm


def check_wait_timeout(seconds: float = 0.2, stream=None) -> int:
    """Run the bounded-wait failure probe (see muonh_check_wait_timeout);
    returns its status: 5 (MUONH_ERR_TIMEOUT) when the wait gave up as designed."""
    return int(library().muonh_check_wait_timeout(float(seconds), _stream_handle(stream)))


def _flat_view(t, what: str, dtypes):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype not in dtypes or not t.is_contiguous():
        raise TypeError(f"{what} must be a contiguous CUDA tensor of dtype {', '.join(map(str, dtypes))}")
    return t.data_ptr(), t.numel()


def average(checkpoints, out=None, stream=None):
    """Equal average of k <= 16 same-shape fp32 or bf16 CUDA tensors,
    (c_0 + ... + c_{k-1}) / k summed in fp32.  `out` (default: a new tensor
    of the inputs' dtype) may be fp32 or bf16 and may be checkpoints[0]."""
    import torch
    dtypes = (torch.float32, torch.bfloat16)
    checkpoints = list(checkpoints)
    if not 1 <= len(checkpoints) <= AVERAGE_MAX_INPUTS:
        raise ValueError(f"between 1 and {AVERAGE_MAX_INPUTS} checkpoints")
    ptrs, count = [], None
    for i, c in enumerate(checkpoints):
        ptr, n = _flat_view(c, f"checkpoints[{i}]", dtypes)
        if c.dtype != checkpoints[0].dtype or c.shape != checkpoints[0].shape or c.device != checkpoints[0].device:
            raise ValueError("checkpoints must share dtype, shape and device")
        ptrs.append(ptr)
        count = n
    if out is None:
        out = torch.empty_like(checkpoints[0])
    optr, on = _flat_view(out, "out", dtypes)
    if on != count:
        raise ValueError("out must have as many elements as each checkpoint")
    code = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16}
    arr = (c_void_p * len(ptrs))(*ptrs)
    _check(library().muonh_average(optr, code[out.dtype], arr, code[checkpoints[0].dtype], len(ptrs), count,
                                   _stream_handle(stream)))
    return out


def adamw_step(params, exp_avgs, exp_avg_sqs, grads, step, lr, beta1=0.9, beta2=0.95, eps=1e-8,
               weight_decay=0.1, stream=None):
    """One AdamW step (1-based `step`) over lists of fp32 CUDA tensors,
    updated in place: params, first moments, second moments; grads read."""
    import torch
    lists = (list(params), list(exp_avgs), list(exp_avg_sqs), list(grads))
    n = len(lists[0])
    if any(len(x) != n for x in lists):
        raise ValueError("params, exp_avgs, exp_avg_sqs and grads must have equal lengths")
    ts = (AdamWTensor * max(n, 1))()
    for i in range(n):
        views = [_flat_view(x[i], f"tensor {i}", (torch.float32,)) for x in lists]
        if len({v[1] for v in views}) != 1:
            raise ValueError(f"tensor {i}: p, m, v and g differ in size")
        ts[i] = AdamWTensor(views[0][0], views[1][0], views[2][0], views[3][0], views[0][1])
    cfg = AdamWConfig(lr, beta1, beta2, eps, weight_decay)
    _check(library().muonh_adamw_step(ts, n, ctypes.byref(cfg), int(step), _stream_handle(stream)))


class MuonH:
    """MuonH over a list of fp32 CUDA weight matrices (updated in place).

    lr passed to step() is the effective LR eta^H of each matrix
    (the caller applies the hyperball multiplier and the schedule).
    beta, nesterov, ns_steps, ns_coeffs, update_rule, weight_decay and
    update_scale take one value for every matrix or a per-matrix sequence.
    groups=1 keeps every kernel of the step on the caller's stream (no
    overlap of elementwise and Newton-Schulz work); 0 lets the library split
    a large set into two overlapping groups; 2 or 3 asks for that many.  ns_form picks the evaluation
    of the Newton-Schulz iteration: "auto" (Gram-space runs where they save
    FLOPs), "y" (Y-space for every matrix) or "gram" (Gram-space wherever
    the fp16 path can run it)."""

    def __init__(self, weights, momenta=None, *, beta=0.95, nesterov=True, ns_steps=5,
                 ns_coeffs=QUINTIC, eps=1e-7, ns_precision="fp16", radii=None, stream=None,
                 update_rule="hyperball", weight_decay=0.0, update_scale=1.0, groups=0, ns_form="auto"):
        import torch
        self._lib = library()
        self.weights = list(weights)
        n = len(self.weights)
        if momenta is None:
            momenta = [torch.zeros_like(w) for w in self.weights]
        self.momenta = list(momenta)
        if len(self.momenta) != n:
            raise ValueError("one momentum tensor per weight")
        prec = _PREC[ns_precision] if isinstance(ns_precision, str) else int(ns_precision)
        descs = (MatrixDesc * n)()
        self.shapes = []
        for i, (w, m) in enumerate(zip(self.weights, self.momenta)):
            wp, rows, cols, ld = _matrix_view(w, f"weights[{i}]")
            mp, mr, mc, mld = _matrix_view(m, f"momenta[{i}]")
            if (mr, mc, mld) != (rows, cols, ld):
                raise ValueError(f"momenta[{i}] must match weights[{i}] in shape and stride")
            R = 0.0 if radii is None else float(radii[i])
            a, b, c = ns_coeffs if not isinstance(ns_coeffs[0], (tuple, list)) else ns_coeffs[i]
            steps = ns_steps if isinstance(ns_steps, int) else ns_steps[i]
            bt = beta if isinstance(beta, (int, float)) else beta[i]
            rule = update_rule if isinstance(update_rule, (str, int)) else update_rule[i]
            rule = _RULE[rule] if isinstance(rule, str) else int(rule)
            wd = weight_decay if isinstance(weight_decay, (int, float)) else weight_decay[i]
            us = update_scale if isinstance(update_scale, (int, float)) else update_scale[i]
            nv = nesterov if isinstance(nesterov, (bool, int)) else nesterov[i]
            descs[i] = MatrixDesc(wp, mp, rows, cols, ld, R, bt, int(bool(nv)), steps, a, b, c,
                                  rule, wd, us)
            self.shapes.append((rows, cols, ld))
        form = NS_FORMS[ns_form] if isinstance(ns_form, str) else int(ns_form)
        cfg = Config(prec, eps, int(groups), form)
        ctx = c_void_p()
        _check(self._lib.muonh_init(ctypes.byref(ctx), descs, n, ctypes.byref(cfg), _stream_handle(stream)))
        self._ctx = ctx
        self.n = n
        self._lr = (c_float * n)()
        self._g = (c_void_p * n)()

    # ---------------------------------------------------------------- step
    def step(self, grads, lr, stats=None, stream=None) -> None:
        """grads: list of fp32 CUDA tensors shaped like the weights; lr: float or
        per-matrix sequence; stats: None or a CUDA tensor of >= 24*n bytes."""
        n = self.n
        if len(grads) != n:
            raise ValueError("one gradient per weight")
        if isinstance(lr, (int, float)):
            for i in range(n):
                self._lr[i] = lr
        else:
            for i in range(n):
                self._lr[i] = lr[i]
        for i, g in enumerate(grads):
            gp, r, c, ld = _matrix_view(g, f"grads[{i}]")
            if (r, c, ld) != self.shapes[i]:
                raise ValueError(f"grads[{i}] must match weights[{i}] in shape and stride")
            self._g[i] = gp
        sp = None
        if stats is not None:
            if not stats.is_cuda or stats.numel() * stats.element_size() < 24 * n:
                raise ValueError("stats must be a CUDA tensor of at least 24*n bytes")
            sp = stats.data_ptr()
        _check(self._lib.muonh_step(self._ctx, self._lr, self._g, sp, _stream_handle(stream)))

    def step_args(self, grads, lr):
        """A CUDA tensor holding the device argument table of muonh_step_device
        (one 16-byte record per matrix: gradient pointer, lr) for these
        gradients and lr (float or per-matrix sequence).  Its lr fields are
        also reachable as `args.view(torch.float32)[2::4]`, so a captured
        graph can be given a new schedule value in place."""
        import torch
        n = self.n
        if len(grads) != n:
            raise ValueError("one gradient per weight")
        rec = torch.zeros((n, 2), dtype=torch.int64)
        lrs = torch.empty(n, dtype=torch.float32)
        for i, g in enumerate(grads):
            gp, r, c, ld = _matrix_view(g, f"grads[{i}]")
            if (r, c, ld) != self.shapes[i]:
                raise ValueError(f"grads[{i}] must match weights[{i}] in shape and stride")
            if gp % 16:
                raise ValueError(f"grads[{i}] must be 16-byte aligned")
            rec[i, 0] = gp
            lrs[i] = lr if isinstance(lr, (int, float)) else lr[i]
        rec.view(torch.float32)[:, 2] = lrs
        return rec.to(self.weights[0].device)

    def step_device(self, args, stats=None, stream=None) -> None:
        """One step reading its arguments from the device table `args` (see
        step_args); enqueues kernels only, so it can be captured in a CUDA graph."""
        if not args.is_cuda or args.numel() * args.element_size() < 16 * self.n:
            raise ValueError("args must be a CUDA tensor of at least 16*n bytes")
        sp = None
        if stats is not None:
            if not stats.is_cuda or stats.numel() * stats.element_size() < 24 * self.n:
                raise ValueError("stats must be a CUDA tensor of at least 24*n bytes")
            sp = stats.data_ptr()
        _check(self._lib.muonh_step_device(self._ctx, args.data_ptr(), sp, _stream_handle(stream)))

    def step_raw(self, grad_ptrs, lr_values, stats_ptr=None, stream_handle=0) -> None:
        """Lowest-overhead step: pointers and values already marshalled."""
        _check(self._lib.muonh_step(self._ctx, lr_values, grad_ptrs, stats_ptr, stream_handle))

    # ---------------------------------------------------------- inspection
    def stats(self) -> list[dict]:
        out = (Stats * self.n)()
        _check(self._lib.muonh_get_stats(self._ctx, out))
        return [dict(elr=s.elr, pre_norm=s.pre_norm, post_norm=s.post_norm, update_norm=s.update_norm,
                     input_norm=s.input_norm, flags=s.flags) for s in out]

    def update(self, i: int, stream=None):
        """Matrix i's Newton-Schulz output O of the last step (fp32, W's shape)."""
        import torch
        rows, cols, _ = self.shapes[i]
        dst = torch.empty((rows, cols), dtype=torch.float32, device=self.weights[i].device)
        _check(self._lib.muonh_get_update(self._ctx, i, dst.data_ptr(), cols, _stream_handle(stream)))
        return dst

    def radii(self) -> list[float]:
        out = (c_float * self.n)()
        _check(self._lib.muonh_get_radius(self._ctx, out))
        return list(out)

    def last_launch_count(self) -> int:
        return int(self._lib.muonh_last_launch_count(self._ctx))

    def enable_timing(self, enable: bool = True) -> None:
        _check(self._lib.muonh_enable_timing(self._ctx, int(bool(enable))))

    def phase_flops(self) -> dict:
        """{phase: tensor-core FLOPs its launches executed in the last step}."""
        out = (ctypes.c_double * len(PHASES))()
        _check(self._lib.muonh_phase_flops(self._ctx, out))
        return {name: float(out[i]) for i, name in enumerate(PHASES)}

    def phase_times(self) -> dict:
        """{phase: (total ms, launches)} recorded since the previous call."""
        ms = (c_float * len(PHASES))()
        cnt = (c_int64 * len(PHASES))()
        _check(self._lib.muonh_phase_times(self._ctx, ms, cnt))
        return {name: (float(ms[i]), int(cnt[i])) for i, name in enumerate(PHASES)}

    def device_status(self) -> None:
        _check(self._lib.muonh_device_status(self._ctx))

    def export_state(self) -> bytes:
        size = c_size_t(0)
        _check(self._lib.muonh_export_state(self._ctx, None, ctypes.byref(size)))
        buf = ctypes.create_string_buffer(size.value)
        _check(self._lib.muonh_export_state(self._ctx, buf, ctypes.byref(size)))
        return buf.raw[: size.value]

    def import_state(self, blob: bytes) -> None:
        buf = ctypes.create_string_buffer(blob, len(blob))
        _check(self._lib.muonh_import_state(self._ctx, buf, len(blob)))

    def close(self) -> None:
        if getattr(self, "_ctx", None):
            self._lib.muonh_destroy(self._ctx)
            self._ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
