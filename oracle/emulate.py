"""16-bit storage emulation of the Newton-Schulz iteration (test infrastructure only).

The iteration of oracle.muonh.newton_schulz (quintic Muon update, the Muon
internals the Puro-2B report leaves open; see that module) restated with
the storage points of a tensor-core implementation whose operands are kept
in a 16-bit format and whose products accumulate exactly enough (fp32
accumulation of 16-bit operands; here fp64) that the storage roundings
dominate:

    Y_0 = r(X / (||X||_F + eps))
    repeat:  A = r(Y Y^T);   B' = r(a I + b A + c A A);   Y = r(B' Y)

with r() rounding to nearest even in the chosen format.  An fp16 operand is
stored times a power of two that keeps its largest entry near the top of
the fp16 range (a power of two changes no relative rounding error); bf16
needs no scaling.  The emulation cannot reproduce a kernel bit for bit (the
tensor cores sum in their own order), but it predicts the size of the
error that storing the operands in 16 bits must cause, which the tests use
to pin the precision of each operand format.
"""
from __future__ import annotations

import numpy as np

from .muonh import QUINTIC


def round_fp16(x):
    """RNE to fp16 after scaling the array by a power of two into range."""
    x = np.asarray(x, dtype=np.float64)
    amax = float(np.max(np.abs(x))) if x.size else 0.0
    if amax == 0.0 or not np.isfinite(amax):
        return x.astype(np.float16).astype(np.float64)
    e = int(np.floor(np.log2(32768.0 / amax)))
    s = np.ldexp(1.0, e)
    return (x * s).astype(np.float16).astype(np.float64) / s


def round_bf16(x):
    """RNE to bfloat16 (the upper 16 bits of an fp32), via fp32."""
    f = np.asarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


ROUND = {"fp16": round_fp16, "bf16": round_bf16, "fp64": lambda x: np.asarray(x, dtype=np.float64)}


def newton_schulz_stored(X, steps=5, coeffs=QUINTIC, eps=1e-7, storage="fp16"):
    """Newton-Schulz with every stored operand rounded to `storage`
    ("fp16", "bf16" or "fp64" = no rounding).  Returns O as fp64."""
    r = ROUND[storage]
    a, b, c = coeffs
    X = np.asarray(X, dtype=np.float64)
    tall = X.shape[0] > X.shape[1]
    Y = X.T if tall else X
    Y = r(Y / (np.linalg.norm(Y) + eps))
    eye = np.eye(Y.shape[0])
    for _ in range(steps):
        A = r(Y @ Y.T)
        Bp = r(a * eye + b * A + c * (A @ A))
        Y = r(Bp @ Y)
    return Y.T.copy() if tall else Y
