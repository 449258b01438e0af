"""MuonH optimizer step for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library libmuonh.so (include/muonh.h) built
from csrc/ by `python -m pretraining_optimizer_b200.build`; this package only
marshals arguments to it.  There is no fallback: importing `MuonH` without the
built library raises.
"""
from .muonh import (  # noqa: F401
    MuonH, MuonHError, QUINTIC, NS_FP16, NS_BF16, NS_FP32,
    FLAG_NONFINITE_INPUT, FLAG_ZERO_UPDATE, FLAG_NONFINITE_UPDATE, FLAG_DEGENERATE,
    FLAG_TIMEOUT, PHASES, library, library_path, EXPORTED_SYMBOLS, momentum_norm_noalloc,
    average, adamw_step, check_wait_timeout,
)
