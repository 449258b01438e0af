"""MuonH step, restated step by step in plain NumPy (test infrastructure only).

Sources (Puro-2B report):
  * arXiv HTML, Sec. 3.3 "Hyperball Optimization", Eq. (1): for each wrapped
    matrix the radius is fixed at R = ||W_0||_F, the Muon update is
    normalised, u_hat = u/||u||_F, then W~ = W - eta R u_hat and
    W_{t+1} = R W~/||W~||_F.
  * Sec. 3.3.1, Eq. (4) and the paragraph after it: the effective LR is the
    displacement norm over the weight norm, eta ||u||/||W||; under Eq. (1) the
    displacement eta R u_hat has norm eta R while ||W|| = R, so it equals eta.
  * Reading notes, Sec. 2.5: the same Eq. (1), restated with eta^H.
The pages name the Muon update u but do not define its internals (reading
notes, Sec. 2.5: Muon yields an update of the weight's shape).  Its
internals -- heavy-ball momentum with a Nesterov look-ahead, Frobenius
normalisation, and a quintic Newton-Schulz iteration with coefficients
(3.4445, -4.7750, 2.0315) -- are the common Muon formulation, and every
one of them is a per-matrix parameter of both the oracle and the library.

Every function computes in `dtype` (float64 unless asked otherwise) with
NumPy's matmul as the only library primitive.
"""
from __future__ import annotations

import numpy as np

QUINTIC = (3.4445, -4.7750, 2.0315)

RULE_HYPERBALL = 0          # Eq. (1): MuonH
RULE_DECOUPLED_WD = 1       # Eq. (3): ordinary Muon with decoupled weight decay
RULE_ELR_ALIGNED = 2        # Eq. (5): ordinary Muon, scalar LR set online to a prescribed ELR

FLAG_NONFINITE_INPUT = 1    # the Newton-Schulz input X has a NaN/Inf entry
FLAG_ZERO_UPDATE = 2        # ||X||_F == 0 or ||O||_F == 0: no displacement
FLAG_NONFINITE_UPDATE = 4   # X finite but the orthogonalised O is not
FLAG_DEGENERATE = 8         # ||W~||_F == 0: projection undefined, W kept


def momentum_update(M, G, beta, nesterov=True, dtype=np.float64):
    """Heavy-ball momentum in sum form, M_t = beta M_{t-1} + G_t.

    The Newton-Schulz input is the Nesterov look-ahead X = G_t + beta M_t,
    or X = M_t without Nesterov.  (The lerp form M = beta M + (1-beta) G gives
    X scaled by (1-beta); the scale cancels in the Frobenius normalisation
    that follows, so the update direction is the same.)
    Returns (M_t, X)."""
    M = np.asarray(M, dtype=dtype)
    G = np.asarray(G, dtype=dtype)
    M_new = beta * M + G
    X = G + beta * M_new if nesterov else M_new.copy()
    return M_new, X


def newton_schulz(X, steps=5, coeffs=QUINTIC, eps=1e-7, dtype=np.float64):
    """Quintic Newton-Schulz orthogonalisation of X (the Muon update).

    The iteration runs on the wide orientation (rows <= cols); a tall X is
    transposed first and the result transposed back, which in exact
    arithmetic gives the same matrix.  Steps:
        Y_0 = X / (||X||_F + eps)
        repeat `steps` times:  A = Y Y^T;  B = b A + c A A;  Y = a Y + B Y
    Returns O, same shape as X."""
    a, b, c = coeffs
    X = np.asarray(X, dtype=dtype)
    tall = X.shape[0] > X.shape[1]
    Y = X.T if tall else X
    Y = Y / (np.linalg.norm(Y) + eps)
    for _ in range(steps):
        A = Y @ Y.T
        B = b * A + c * (A @ A)
        Y = a * Y + B @ Y
    return Y.T.copy() if tall else Y


def radius(W0, dtype=np.float64):
    """R = ||W_0||_F (Sec. 3.3, fixed once per matrix)."""
    return float(np.linalg.norm(np.asarray(W0, dtype=dtype)))


def hyperball_update(W, O, lr, R, dtype=np.float64):
    """Eq. (1): u_hat = O/||O||_F; W~ = W - lr R u_hat; W_{t+1} = R W~/||W~||_F.

    Returns (W_{t+1}, stats).  stats: elr = ||lr R u_hat||_F / ||W_t||_F,
    pre_norm = ||W_t||_F, post_norm = ||W_{t+1}||_F, update_norm = ||O||_F,
    flags.  A zero update (||O|| = 0) skips the displacement and only
    re-projects; a non-finite O or a zero W~ leaves W unchanged."""
    W = np.asarray(W, dtype=dtype)
    O = np.asarray(O, dtype=dtype)
    w_norm = float(np.linalg.norm(W))
    o_norm = float(np.linalg.norm(O))
    flags = 0
    if not np.isfinite(o_norm):
        flags |= FLAG_NONFINITE_UPDATE
        return W.copy(), dict(elr=0.0, pre_norm=w_norm, post_norm=w_norm,
                              update_norm=o_norm, flags=flags)
    if o_norm == 0.0:
        flags |= FLAG_ZERO_UPDATE
        W_tilde = W
        elr = 0.0
    else:
        displacement = (lr * R / o_norm) * O
        W_tilde = W - displacement
        elr = float(np.linalg.norm(displacement)) / w_norm
    wt_norm = float(np.linalg.norm(W_tilde))
    if wt_norm == 0.0:
        flags |= FLAG_DEGENERATE
        return W.copy(), dict(elr=0.0, pre_norm=w_norm, post_norm=w_norm,
                              update_norm=o_norm, flags=flags)
    W_new = (R / wt_norm) * W_tilde
    return W_new, dict(elr=elr, pre_norm=w_norm,
                       post_norm=float(np.linalg.norm(W_new)),
                       update_norm=o_norm, flags=flags)


def muon_update(W, O, lr, weight_decay=0.0, update_scale=1.0, rule=RULE_DECOUPLED_WD,
                dtype=np.float64):
    """Ordinary Muon on one matrix, with the update u = update_scale * O.

    Eq. (3) (report Sec. 3.3.1): W_{t+1} = (1 - lambda eta) W_t - eta u_t with
    eta = lr; its effective LR, Eq. (4), is eta ||u||_F / ||W_t||_F.
    Eq. (5): the scalar LR is set online, eta = rho ||W_t||_F / ||u_t||_F with
    rho = lr the prescribed effective LR, so Eq. (4) gives exactly rho; W is
    not projected.  A zero update leaves W unchanged.
    Returns (W_{t+1}, stats) with the fields of hyperball_update plus eta."""
    W = np.asarray(W, dtype=dtype)
    O = np.asarray(O, dtype=dtype)
    u = update_scale * O
    w_norm = float(np.linalg.norm(W))
    u_norm = float(np.linalg.norm(u))
    o_norm = float(np.linalg.norm(O))
    if not np.isfinite(u_norm):
        return W.copy(), dict(elr=0.0, pre_norm=w_norm, post_norm=w_norm, update_norm=o_norm,
                              flags=FLAG_NONFINITE_UPDATE, eta=0.0)
    if u_norm == 0.0:
        return W.copy(), dict(elr=0.0, pre_norm=w_norm, post_norm=w_norm, update_norm=o_norm,
                              flags=FLAG_ZERO_UPDATE, eta=0.0)
    eta = lr if rule == RULE_DECOUPLED_WD else lr * w_norm / u_norm
    W_new = (1.0 - weight_decay * eta) * W - eta * u
    return W_new, dict(elr=eta * u_norm / w_norm, pre_norm=w_norm,
                       post_norm=float(np.linalg.norm(W_new)), update_norm=o_norm, flags=0,
                       eta=eta)


def muonh_step(W, M, G, lr, R, beta=0.95, nesterov=True, ns_steps=5,
               coeffs=QUINTIC, eps=1e-7, dtype=np.float64, ns_dtype=None,
               rule=RULE_HYPERBALL, weight_decay=0.0, update_scale=1.0):
    """One step for one matrix: momentum, Newton-Schulz, then Eq. (1)
    (rule RULE_HYPERBALL, MuonH) or ordinary Muon by Eq. (3) / Eq. (5).

    Returns (W_{t+1}, M_t, O, stats) where stats also carries
    input_norm = ||X||_F.  A non-finite X leaves W unchanged (M follows the
    plain arithmetic) and sets FLAG_NONFINITE_INPUT.  `ns_dtype` (default:
    `dtype`) sets the precision of the Newton-Schulz products alone, so a
    large matrix can run its O(r^2 c) matmuls in fp32 while every norm and
    the projection stay in `dtype`."""
    M_new, X = momentum_update(M, G, beta, nesterov, dtype)
    x_norm = float(np.linalg.norm(X))
    if not np.isfinite(x_norm):
        W = np.asarray(W, dtype=dtype)
        w_norm = float(np.linalg.norm(W))
        return W.copy(), M_new, None, dict(
            elr=0.0, pre_norm=w_norm, post_norm=w_norm, update_norm=0.0,
            input_norm=x_norm, flags=FLAG_NONFINITE_INPUT)
    O = newton_schulz(X, ns_steps, coeffs, eps, ns_dtype or dtype).astype(dtype)
    if rule == RULE_HYPERBALL:
        W_new, st = hyperball_update(W, O, lr, R, dtype)
    else:
        W_new, st = muon_update(W, O, lr, weight_decay, update_scale, rule, dtype)
    if x_norm == 0.0:
        st["flags"] |= FLAG_ZERO_UPDATE
    st["input_norm"] = x_norm
    return W_new, M_new, O, st


def run_steps(W0_list, grad_fn, lrs, beta=0.95, nesterov=True, ns_steps=5,
              coeffs=QUINTIC, eps=1e-7, dtype=np.float64, R_list=None,
              keep_updates=False):
    """Run len(lrs) MuonH steps over a list of matrices.

    grad_fn(step, i) returns the gradient of matrix i at step `step`;
    lrs[t] is either one float or a per-matrix list.  Momentum starts at 0.
    Returns dict(W=list, M=list, R=list, stats=[per step list of per-matrix
    dicts], O=[last step's updates] if keep_updates)."""
    W = [np.asarray(w, dtype=dtype) for w in W0_list]
    M = [np.zeros_like(w) for w in W]
    R = list(R_list) if R_list is not None else [radius(w, dtype) for w in W]
    all_stats, last_O = [], None
    for t, lr_t in enumerate(lrs):
        step_stats, last_O = [], []
        for i in range(len(W)):
            lr = lr_t[i] if isinstance(lr_t, (list, tuple)) else lr_t
            W[i], M[i], O, st = muonh_step(W[i], M[i], grad_fn(t, i), lr, R[i],
                                           beta, nesterov, ns_steps, coeffs, eps, dtype)
            step_stats.append(st)
            if keep_updates:
                last_O.append(O)
        all_stats.append(step_stats)
    out = dict(W=W, M=M, R=R, stats=all_stats)
    if keep_updates:
        out["O"] = last_O
    return out
