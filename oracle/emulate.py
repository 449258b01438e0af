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


def mirror_upper_tiles(P, tile=256):
    """A symmetric product as a kernel that computes only the tiles on and
    above the diagonal stores it: every block below the diagonal is the
    transpose of its mirror block."""
    out = np.array(P, dtype=np.float64, copy=True)
    n = out.shape[0]
    for i in range(0, n, tile):
        for j in range(0, i, tile):
            out[i:i + tile, j:j + tile] = out[j:j + tile, i:i + tile].T
    return out


def round_off_diagonal(B, r):
    """B stored through r() except its diagonal, which is kept exactly (the
    rounding residual of each diagonal entry carried separately in fp32 and
    added back in the product that uses B)."""
    out = r(B)
    np.fill_diagonal(out, np.diag(np.asarray(B, dtype=np.float64)))
    return out


def newton_schulz_stored(X, steps=5, coeffs=QUINTIC, eps=1e-7, storage="fp16", exact_diagonal=False):
    """Newton-Schulz with every stored operand rounded to `storage`
    ("fp16", "bf16" or "fp64" = no rounding).  exact_diagonal=True keeps the
    diagonal of B' = a I + b A + c A A unrounded (round_off_diagonal): once
    the iterate's singular values approach 1, A is close to I and B' to
    p(1) I, so B' is dominated by its diagonal, whose rounding is the
    largest single error of a bf16 B'.  Returns O as fp64."""
    r = ROUND[storage]
    a, b, c = coeffs
    X = np.asarray(X, dtype=np.float64)
    tall = X.shape[0] > X.shape[1]
    Y = X.T if tall else X
    Y = r(Y / (np.linalg.norm(Y) + eps))
    eye = np.eye(Y.shape[0])
    for _ in range(steps):
        A = r(Y @ Y.T)
        Bp = a * eye + b * A + c * (A @ A)
        Bp = round_off_diagonal(Bp, r) if exact_diagonal else r(Bp)
        Y = r(Bp @ Y)
    return Y.T.copy() if tall else Y


def newton_schulz_gram_stored(X, groups=(3, 2), coeffs=QUINTIC, eps=1e-7, storage="fp16", tile=256):
    """The same quintic iteration restated in Gram space, with restarts.

    With A_k = Y_k Y_k^T and p(A) = a I + b A + c A A, one iteration is
    Y_{k+1} = p(A_k) Y_k, so A_{k+1} = p(A_k) A_k p(A_k) = A_k p(A_k)^2 (the
    factors are polynomials in one symmetric matrix and commute), and g
    iterations in a row apply Q = p(A_{k+g-1}) ... p(A_k) to Y_k once.  Each
    entry of `groups` is such a run of iterations, entered from a fresh Gram
    matrix of the current Y (a restart) and left through Y <- r(Q Y); the
    entries sum to the step count.  groups = (1,)*steps is the Y-space form
    of newton_schulz_stored.  In exact arithmetic every grouping gives the
    same O; they differ only in where the 16-bit storage rounds (r(), as in
    newton_schulz_stored), and every r x r product here is symmetric, so it
    is stored through mirror_upper_tiles.  Returns O as fp64."""
    r = ROUND[storage]
    a, b, c = coeffs
    if any(g < 1 for g in groups):
        raise ValueError("groups must be positive run lengths")
    X = np.asarray(X, dtype=np.float64)
    tall = X.shape[0] > X.shape[1]
    Y = X.T if tall else X
    Y = r(Y / (np.linalg.norm(Y) + eps))
    eye = np.eye(Y.shape[0])

    def sym(P):
        return r(mirror_upper_tiles(P, tile))

    for g in groups:
        A = sym(Y @ Y.T)
        Q = None
        for j in range(g):
            Bp = sym(a * eye + b * A + c * (A @ A))
            Q = Bp if Q is None else sym(Bp @ Q)
            if j + 1 < g:
                A = sym(sym(A @ Bp) @ Bp)
        Y = r(Q @ Y)
    return Y.T.copy() if tall else Y
