"""Pins for the CPU oracle (no GPU).  Each test ties an oracle function to a
fact fixed by the report or by the mathematics, not to a retyped copy of it."""
import os

import numpy as np
import pytest

import oracle
import synth
from oracle import QUINTIC

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed=0):
    return np.random.default_rng(seed).standard_normal(shape)


def _scalar_iterate(sig, coeffs, steps):
    """Singular-value picture: Y -> aY + (bYY^T + c(YY^T)^2)Y maps each
    singular value s of Y to a s + b s^3 + c s^5 and keeps the vectors."""
    a, b, c = coeffs
    for _ in range(steps):
        sig = a * sig + b * sig ** 3 + c * sig ** 5
    return sig


@pytest.mark.parametrize("shape", [(8, 16), (16, 8), (32, 64), (64, 128), (1, 5), (5, 1), (24, 24)])
@pytest.mark.parametrize("steps", [1, 2, 5])
def test_newton_schulz_equals_polynomial_on_singular_values(shape, steps):
    X = _rand(shape, seed=shape[0] * 1000 + shape[1])
    eps = 1e-7
    O = oracle.newton_schulz(X, steps, QUINTIC, eps)
    U, s, Vt = np.linalg.svd(X / (np.linalg.norm(X) + eps), full_matrices=False)
    expect = (U * _scalar_iterate(s, QUINTIC, steps)) @ Vt
    assert O.shape == X.shape
    assert np.linalg.norm(O - expect) <= 1e-10 * np.linalg.norm(expect)


def test_newton_schulz_output_band():
    """Tuned quintic, 5 steps: singular values of O lie in the image of the
    scalar map over the input band (grid-evaluated here)."""
    X = _rand((96, 200), seed=3)
    O = oracle.newton_schulz(X, 5, QUINTIC, 1e-7)
    s_in = np.linalg.svd(X / np.linalg.norm(X), compute_uv=False)
    s_out = np.linalg.svd(O, compute_uv=False)
    grid = np.linspace(s_in.min(), s_in.max(), 200001)
    img = _scalar_iterate(grid, QUINTIC, 5)
    assert s_out.min() >= img.min() - 1e-9 and s_out.max() <= img.max() + 1e-9
    # the tuned map keeps every value of a well-spread spectrum near 1
    assert 0.6 < s_out.min() and s_out.max() < 1.25


@pytest.mark.parametrize("coeffs", [(1.5, -0.5, 0.0), (15 / 8, -10 / 8, 3 / 8)])
def test_newton_schulz_converges_to_polar_factor(coeffs):
    rng = np.random.default_rng(7)
    U, _ = np.linalg.qr(rng.standard_normal((40, 40)))
    V, _ = np.linalg.qr(rng.standard_normal((90, 40)))
    s = np.geomspace(1.0, 0.1, 40)                       # condition number 10
    X = (U * s) @ V.T
    polar = U @ V.T
    errs = [np.linalg.norm(oracle.newton_schulz(X, k, coeffs, 0.0) - polar) / np.linalg.norm(polar)
            for k in range(0, 41, 5)]
    assert all(e1 <= e0 + 1e-14 for e0, e1 in zip(errs, errs[1:]))
    assert errs[-1] < 1e-10


def test_tuned_quintic_does_not_converge():
    """The tuned coefficients trade convergence for speed: p(1) != 1."""
    assert abs(_scalar_iterate(np.array([1.0]), QUINTIC, 1)[0] - 0.701) < 1e-3


def test_newton_schulz_transpose_and_scale():
    X = _rand((20, 50), seed=11)
    O = oracle.newton_schulz(X, 5, QUINTIC, 0.0)
    Ot = oracle.newton_schulz(X.T.copy(), 5, QUINTIC, 0.0)
    assert np.allclose(Ot, O.T, rtol=0, atol=1e-12)
    O3 = oracle.newton_schulz(1e-3 * X, 5, QUINTIC, 0.0)
    assert np.allclose(O3, O, rtol=0, atol=1e-12)


def _golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            lhs, rhs = line.split("|")
            rows.append(([float(v) for v in lhs.split()], [float(v) for v in rhs.split()]))
    return rows


def test_hyperball_hand_solved_cases():
    rows = _golden_rows("hyperball_two_element.txt")
    assert len(rows) == 3
    for (w0, w1, o0, o1, lr, R), (n0, n1, elr) in rows:
        W_new, st = oracle.hyperball_update(np.array([[w0, w1]]), np.array([[o0, o1]]), lr, R)
        assert np.allclose(W_new, [[n0, n1]], rtol=0, atol=1e-14)
        assert abs(st["elr"] - elr) < 1e-15


def test_radius_hand_solved_cases():
    """R = ||W_0||_F (Sec. 3.3, Eq. (1)) on hand-solved matrices, two of which
    have a spectral norm different from the Frobenius norm."""
    rows = _golden_rows("radius_hand_solved.txt")
    assert len(rows) == 5
    for lhs, (R,) in rows:
        r, c = int(lhs[0]), int(lhs[1])
        W = np.array(lhs[2:], dtype=np.float64).reshape(r, c)
        assert abs(oracle.radius(W) - R) <= 1e-15 * max(1.0, R), (W, oracle.radius(W), R)
        # float32 input is read in fp64: the same R for exactly representable entries
        assert abs(oracle.radius(W.astype(np.float32)) - R) <= 1e-15 * max(1.0, R)


def test_run_steps_carries_momentum_and_fixes_the_radius():
    """run_steps over three steps: the radius is ||W_0||_F of each matrix
    (hand-known here) and the momentum buffer carries across steps,
    M_k = sum_j beta^(k-j) G_j, with the reported input norm
    ||G_k + beta M_k||_F at every step."""
    beta = 0.95
    shapes = [(4, 9), (9, 4)]
    W0 = [np.full(shapes[0], 0.5), np.full(shapes[1], -0.25)]   # ||.||_F = 0.5*6 = 3, 0.25*6 = 1.5
    Gs = {(t, i): _rand(shapes[i], seed=300 + 10 * t + i) * 1e-3 for t in range(3) for i in range(2)}
    out = oracle.run_steps(W0, lambda t, i: Gs[(t, i)], [0.01, 0.02, 0.005], beta=beta)
    assert out["R"] == [3.0, 1.5]
    for i in range(2):
        for k in range(3):
            geo = sum(beta ** (k - j) * Gs[(j, i)] for j in range(k + 1))
            x_norm = np.linalg.norm(Gs[(k, i)] + beta * geo)
            assert abs(out["stats"][k][i]["input_norm"] - x_norm) <= 1e-13 * x_norm, (i, k)
        geo = sum(beta ** (2 - j) * Gs[(j, i)] for j in range(3))
        assert np.allclose(out["M"][i], geo, rtol=0, atol=1e-16)
        assert abs(np.linalg.norm(out["W"][i]) - out["R"][i]) <= 1e-13 * out["R"][i]


def test_hyperball_invariants():
    """||W_{t+1}|| = R and effective LR = lr (Sec. 3.3.1)."""
    rng = np.random.default_rng(5)
    for lr in (0.0, 1e-4, 0.012, 0.3):
        W = rng.standard_normal((30, 70))
        R = np.linalg.norm(W)
        O = rng.standard_normal((30, 70))
        W_new, st = oracle.hyperball_update(W, O, lr, R)
        assert abs(np.linalg.norm(W_new) - R) <= 1e-13 * R
        assert abs(st["elr"] - lr) <= 1e-14
        assert abs(st["post_norm"] - R) <= 1e-13 * R
        # the update is scale-free: O and 7 O give the same step
        W7, _ = oracle.hyperball_update(W, 7.0 * O, lr, R)
        assert np.allclose(W7, W_new, rtol=0, atol=1e-14)


def test_momentum_geometric_sum():
    """After k steps from M=0: M_k = sum_j beta^(k-j) G_j; X = G_k + beta M_k."""
    beta = 0.95
    Gs = [_rand((6, 9), seed=100 + j) for j in range(5)]
    M = np.zeros((6, 9))
    for k, G in enumerate(Gs):
        M, X = oracle.momentum_update(M, G, beta, nesterov=True)
        geo = sum(beta ** (k - j) * Gs[j] for j in range(k + 1))
        assert np.allclose(M, geo, rtol=0, atol=1e-13)
        assert np.allclose(X, Gs[k] + beta * geo, rtol=0, atol=1e-13)
    _, Xp = oracle.momentum_update(np.zeros((6, 9)), Gs[0], 0.0, nesterov=True)
    assert np.array_equal(Xp, Gs[0])
    M2, X2 = oracle.momentum_update(M, Gs[0], beta, nesterov=False)
    assert np.array_equal(X2, M2)


def test_lerp_momentum_gives_the_same_direction():
    beta = 0.9
    G1, G2 = _rand((8, 12), 1), _rand((8, 12), 2)
    _, Xs = oracle.momentum_update(oracle.momentum_update(np.zeros((8, 12)), G1, beta)[0], G2, beta)
    Ml = (1 - beta) * G1                                   # lerp form, one step
    Ml = beta * Ml + (1 - beta) * G2
    Xl = (1 - beta) * G2 + beta * Ml
    assert np.allclose(Xl, (1 - beta) * Xs, rtol=0, atol=1e-14)
    assert np.allclose(oracle.newton_schulz(Xl, 5, QUINTIC, 0.0),
                       oracle.newton_schulz(Xs, 5, QUINTIC, 0.0), rtol=0, atol=1e-12)


def test_step_edge_cases():
    W = _rand((4, 6), 9)
    R = np.linalg.norm(W)
    Z = np.zeros((4, 6))
    # zero gradient and zero momentum: no displacement, re-projection only
    W1, M1, O, st = oracle.muonh_step(W, Z, Z, 0.01, R)
    assert st["flags"] & oracle.FLAG_ZERO_UPDATE and st["elr"] == 0.0
    assert np.allclose(W1, W, rtol=0, atol=1e-15)
    # non-finite gradient: W kept, flag raised
    G = _rand((4, 6), 10)
    G[1, 2] = np.nan
    W2, M2, O2, st2 = oracle.muonh_step(W, Z, G, 0.01, R)
    assert st2["flags"] & oracle.FLAG_NONFINITE_INPUT and np.array_equal(W2, W)
    # lr = 0 re-projects onto the same sphere
    W3, _, _, st3 = oracle.muonh_step(W, Z, _rand((4, 6), 12), 0.0, R)
    assert st3["elr"] == 0.0 and np.allclose(W3, W, rtol=0, atol=1e-14)


def test_multi_step_norm_stays_on_sphere():
    shapes = [(16, 40), (40, 16)]
    W0 = [_rand(s, 20 + i) * 0.02 for i, s in enumerate(shapes)]
    out = oracle.run_steps(W0, lambda t, i: _rand(shapes[i], 1000 * t + i) * 1e-3, [0.01] * 6)
    for i in range(2):
        assert abs(np.linalg.norm(out["W"][i]) - out["R"][i]) <= 1e-12 * out["R"][i]
        for st in out["stats"]:
            assert abs(st[i]["elr"] - 0.01) < 1e-12


def test_ordinary_muon_rules_hand_solved():
    """Eq. (3) and Eq. (5) of Sec. 3.3.1 on hand-solved cases."""
    rows = _golden_rows("muon_rules_two_element.txt")
    assert len(rows) == 3
    for (rule, lr, lam, s), (n0, n1, elr, eta) in rows:
        W_new, st = oracle.muon_update(np.array([[3.0, 4.0]]), np.array([[0.0, 2.0]]), lr, lam, s, int(rule))
        assert np.allclose(W_new, [[n0, n1]], rtol=0, atol=1e-14)
        assert abs(st["elr"] - elr) < 1e-15 and abs(st["eta"] - eta) < 1e-15


def test_elr_aligned_rule_hits_the_prescribed_elr():
    """Eq. (5): the induced effective LR (Eq. (4)) equals rho for any update
    scale, and the step direction is the Eq. (3) direction at that eta."""
    rng = np.random.default_rng(9)
    for scale in (1.0, 0.2, 37.0):
        W = 0.02 * rng.standard_normal((24, 60))
        G = 1e-3 * rng.standard_normal((24, 60))
        W1, _, O, st = oracle.muonh_step(W, np.zeros_like(W), G, 0.015, 0.0, rule=oracle.RULE_ELR_ALIGNED,
                                         weight_decay=0.1, update_scale=scale)
        assert abs(st["elr"] - 0.015) < 1e-14
        W3, st3 = oracle.muon_update(W, O, st["eta"], 0.1, scale, oracle.RULE_DECOUPLED_WD)
        assert np.allclose(W1, W3, rtol=0, atol=1e-15)
        # no projection: the norm drifts from ||W_0||
        assert abs(np.linalg.norm(W1) - np.linalg.norm(W)) > 1e-6


# ---------------------------------------------------------------- 16-bit storage emulation
def test_storage_emulation_without_rounding_is_the_oracle():
    from oracle import emulate
    X = synth.gaussian_gradient(0, 0, 64, 160)
    assert np.allclose(emulate.newton_schulz_stored(X, storage="fp64"), oracle.newton_schulz(X), rtol=0, atol=1e-13)


def test_round_helpers_match_their_formats():
    """fp16: the library cast after an exact power-of-two scaling; bf16: the
    top 16 bits of fp32, rounded to nearest even (ties checked by hand)."""
    from oracle import emulate
    x = np.random.default_rng(0).standard_normal(1000) * 1e-4
    r = emulate.round_fp16(x)
    assert np.all(np.abs(r - x) <= 2.0 ** -11 * np.abs(x) + 1e-300)
    # 1 + 2^-8 is a bf16 tie between 1 and 1 + 2^-7: even mantissa wins (1.0);
    # 1 + 3 * 2^-8 ties between 1 + 2^-7 and 1 + 2^-6: 1 + 2^-6 is even
    ties = emulate.round_bf16(np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -9)]))
    assert list(ties) == [1.0, 1 + 2.0 ** -6, -1.0]


@pytest.mark.parametrize("storage,lo,hi", [("fp16", 4e-4, 2e-3), ("bf16", 3e-3, 1.6e-2)])
def test_storage_error_of_each_operand_format(storage, lo, hi):
    """5 tuned quintic steps on a 256 x 512 Gaussian input: storing the
    operands in fp16 (10+1 significand bits) costs ~1e-3 relative error,
    bf16 (7+1 bits) about 8x more; the 1e-2 gate admits fp16 with margin."""
    from oracle import emulate
    X = synth.gaussian_gradient(0, 0, 256, 512)
    ref = oracle.newton_schulz(X)
    O = emulate.newton_schulz_stored(X, storage=storage)
    err = np.linalg.norm(O - ref) / np.linalg.norm(ref)
    assert lo <= err <= hi, err


def test_round_off_diagonal_keeps_only_the_diagonal():
    from oracle import emulate
    B = np.array([[3.4257, 1.0 + 2.0 ** -9, 0.3], [1.0 + 2.0 ** -9, 0.7001, -2.5e-3], [0.3, -2.5e-3, 1.1]])
    out = emulate.round_off_diagonal(B, emulate.round_bf16)
    assert np.array_equal(np.diag(out), np.diag(B))
    off = ~np.eye(3, dtype=bool)
    assert np.array_equal(out[off], emulate.round_bf16(B)[off])
    assert out[0, 1] == 1.0                      # a bf16 tie rounded to even off the diagonal


def test_exact_diagonal_emulation():
    """Without rounding the exact-diagonal emulation is the oracle; with bf16
    storage, keeping B's diagonal exact removes its largest rounding error:
    on inputs whose iterate is small (r = 70) the error drops below the bf16
    storage error of the plain form by a fifth or more."""
    from oracle import emulate
    X = synth.gaussian_gradient(0, 1, 70, 130).astype(np.float64)
    ref = oracle.newton_schulz(X)
    assert np.allclose(emulate.newton_schulz_stored(X, storage="fp64", exact_diagonal=True), ref, rtol=0, atol=1e-13)
    plain = np.linalg.norm(emulate.newton_schulz_stored(X, storage="bf16") - ref) / np.linalg.norm(ref)
    diag = np.linalg.norm(emulate.newton_schulz_stored(X, storage="bf16", exact_diagonal=True) - ref) / np.linalg.norm(ref)
    assert diag <= 0.8 * plain and diag <= 1e-2, (diag, plain)


def test_newton_schulz_is_orthogonally_equivariant():
    """NS(U X V^T) = U NS(X) V^T for orthogonal U, V: the iteration acts on
    singular values only (a max-norm or element-wise scaling would break this)."""
    rng = np.random.default_rng(11)
    X = rng.standard_normal((24, 40))
    U, _ = np.linalg.qr(rng.standard_normal((24, 24)))
    V, _ = np.linalg.qr(rng.standard_normal((40, 40)))
    lhs = oracle.newton_schulz(U @ X @ V.T)
    rhs = U @ oracle.newton_schulz(X) @ V.T
    assert np.allclose(lhs, rhs, rtol=0, atol=1e-12)


def test_newton_schulz_ignores_the_input_scale():
    """The input is Frobenius-normalised first, so a positive scale of X
    changes nothing beyond the eps guard."""
    X = _rand((32, 48), seed=4)
    assert np.allclose(oracle.newton_schulz(3.7 * X, eps=0.0), oracle.newton_schulz(X, eps=0.0), rtol=0, atol=1e-12)


@pytest.mark.parametrize("groups", [(5,), (3, 2), (2, 2, 1), (1, 4)])
def test_gram_space_form_without_rounding_is_the_oracle(groups):
    """A_{k+1} = A_k p(A_k)^2 and one Q = prod p(A_k) per run of iterations
    reproduce the Y-space iteration exactly (up to fp64 rounding)."""
    from oracle import emulate
    for X in (_rand((256, 512), seed=5), _rand((640, 384), seed=6),
              synth.ill_conditioned_gradient(1, 0, 256, 512).astype(np.float64)):
        O = emulate.newton_schulz_gram_stored(X, groups, storage="fp64")
        assert np.linalg.norm(O - oracle.newton_schulz(X)) <= 1e-10 * np.linalg.norm(O)


@pytest.mark.parametrize("storage", ["fp16", "bf16"])
def test_gram_space_form_with_unit_runs_is_the_y_space_emulation(storage):
    from oracle import emulate
    X = _rand((256, 512), seed=7)
    assert np.array_equal(emulate.newton_schulz_gram_stored(X, (1,) * 5, storage=storage),
                          emulate.newton_schulz_stored(X, storage=storage))


def test_gram_space_form_needs_restarts_in_fp16():
    """Stored in fp16, runs of three and two iterations stay inside the 1e-2
    bar and within 2x of the Y-space form's storage error, while one run of
    five loses an ill-conditioned input: Q's entries span up to a^5
    (p(0) = a) and fp16 keeps 11 bits of them."""
    from oracle import emulate
    gauss = synth.gaussian_gradient(0, 0, 256, 512).astype(np.float64)
    ill = synth.ill_conditioned_gradient(1, 0, 256, 512).astype(np.float64)
    for X in (gauss, ill):
        ref = oracle.newton_schulz(X)
        err = np.linalg.norm(emulate.newton_schulz_gram_stored(X, (3, 2)) - ref) / np.linalg.norm(ref)
        err_y = np.linalg.norm(emulate.newton_schulz_stored(X) - ref) / np.linalg.norm(ref)
        assert err <= 1e-2 and err <= 2 * err_y
    ref = oracle.newton_schulz(ill)
    err5 = np.linalg.norm(emulate.newton_schulz_gram_stored(ill, (5,)) - ref) / np.linalg.norm(ref)
    assert err5 > 1e-1
