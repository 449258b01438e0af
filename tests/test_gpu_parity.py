"""CUDA path vs the fp64 oracle on the same seeded inputs (B200 only)."""
import numpy as np
import pytest

import oracle
import synth
from parity_helpers import (FP16_NS_TOL, FP32_NS_TOL, NORM_TOL, W_TOL_10, rel_fro, run_gpu,
                            run_oracle, tile_rel_fro_max)

pytestmark = pytest.mark.gpu


def _single():
    wl = synth.workload("single_256x512")
    W0 = [wl.weight(0)]
    return wl, W0


@pytest.mark.parametrize("prec,ns_tol,w_tol", [("fp16", FP16_NS_TOL, W_TOL_10),
                                               ("bf16", FP16_NS_TOL, W_TOL_10),
                                               ("fp32", FP32_NS_TOL, 1e-5)])
def test_single_matrix_ten_steps(prec, ns_tol, w_tol):
    """256 x 512, 10 steps, lr 0.01, beta 0.95 Nesterov, tuned quintic x 5.
    Both 16-bit operand types are held to the same gates: 1e-2 on O against
    fp64 and 1e-3 R on W after the 10 steps."""
    wl, W0 = _single()
    keep = (0, 4, 9)
    g = run_gpu(W0, wl.grad, wl.lrs, prec=prec, keep_updates=keep)
    o = run_oracle(W0, wl.grad, wl.lrs, keep_updates=keep)
    R = o["R"][0]
    assert abs(g["R"][0] - R) <= NORM_TOL * R
    for t in keep:
        assert rel_fro(g["O"][t][0], o["O"][t][0]) <= ns_tol, (t, rel_fro(g["O"][t][0], o["O"][t][0]))
        if prec != "bf16":
            # block by block (32 blocks of 64 x 64): no localised error hides in the average
            worst = tile_rel_fro_max(g["O"][t][0], o["O"][t][0], tile=64)
            assert worst <= ns_tol, (t, worst)
    for t in range(len(wl.lrs)):
        gs, os_ = g["stats"][t][0], o["stats"][t][0]
        assert gs["flags"] == 0
        assert abs(gs["elr"] - os_["elr"]) <= NORM_TOL * os_["elr"]
        assert abs(gs["post_norm"] - R) <= NORM_TOL * R
        assert abs(gs["pre_norm"] - os_["pre_norm"]) <= NORM_TOL * R
        assert abs(gs["input_norm"] - os_["input_norm"]) <= NORM_TOL * os_["input_norm"]
        assert abs(gs["update_norm"] - os_["update_norm"]) <= ns_tol * os_["update_norm"]
    assert np.linalg.norm(g["W"][0] - o["W"][0]) / R <= w_tol
    assert rel_fro(g["M"][0], o["M"][0]) <= 1e-6


@pytest.mark.parametrize("coeffs,tol", [((1.0, 0.0, 0.0), 2e-3),    # O = X0: K1 path only
                                        ((0.0, 1.0, 0.0), 4e-3),    # O = (X X^T) X: GRAM + APPLY
                                        ((0.0, 0.0, 1.0), 6e-3),    # O = (X X^T)^2 X: SQUARE
                                        ((3.4445, -4.7750, 2.0315), 5e-3)])
@pytest.mark.parametrize("shape", [(256, 512), (512, 256), (384, 1000), (1000, 300)])
def test_one_iteration_isolates_each_gemm(coeffs, tol, shape):
    W0 = [synth.initial_weight(0, *shape)]
    grad = lambda t, i: synth.gaussian_gradient(t, i, *shape)
    g = run_gpu(W0, grad, [0.01], ns_steps=1, coeffs=coeffs, keep_updates=(0,))
    o = run_oracle(W0, grad, [0.01], ns_steps=1, coeffs=coeffs, keep_updates=(0,))
    assert rel_fro(g["O"][0][0], o["O"][0][0]) <= tol


@pytest.mark.parametrize("prec", ["fp16", "fp32"])
def test_mixed_shapes_grouped_in_one_context(prec):
    """Several shape classes, tall and wide, ragged sizes, a strided view,
    odd column counts (scalar path), a 1 x n and an n x 1 matrix."""
    shapes = [(256, 512), (512, 256), (256, 512), (1000, 300), (130, 70), (1, 300), (300, 1),
              (96, 301), (640, 384)]
    strides = [None, None, 520, None, None, None, None, None, 400]
    W0 = [synth.initial_weight(i, *s) for i, s in enumerate(shapes)]
    grad = lambda t, i: synth.gaussian_gradient(t, i, *shapes[i])
    lrs = [[0.01 + 0.001 * i for i in range(len(shapes))]] * 3
    tol = FP16_NS_TOL if prec == "fp16" else FP32_NS_TOL
    g = run_gpu(W0, grad, lrs, prec=prec, keep_updates=(2,), strides=strides)
    o = run_oracle(W0, grad, lrs, keep_updates=(2,))
    for i, s in enumerate(shapes):
        assert rel_fro(g["O"][2][i], o["O"][2][i]) <= tol, (i, s, rel_fro(g["O"][2][i], o["O"][2][i]))
        worst = tile_rel_fro_max(g["O"][2][i], o["O"][2][i], tile=64)
        assert worst <= tol, (i, s, worst)
        R = o["R"][i]
        assert abs(g["stats"][2][i]["post_norm"] - R) <= NORM_TOL * R, (i, s)
        assert abs(g["stats"][2][i]["elr"] - o["stats"][2][i]["elr"]) <= NORM_TOL * o["stats"][2][i]["elr"]
        assert np.linalg.norm(g["W"][i] - o["W"][i]) / R <= (1e-3 if prec == "fp16" else 1e-5), (i, s)


@pytest.mark.parametrize("shape", [(2048, 6144), (6144, 2048)])
def test_fp32_mode_at_qwen3_inner_dimension(shape):
    """FP32 mode on the Qwen3-1.7B MLP shapes, where the Gram products sum over
    K = 6144 and the square and apply products over K = 2048: two steps, every
    quantity within 1e-5 of the fp64 oracle (O also block by block)."""
    W0 = [synth.initial_weight(4, *shape)]
    grad = lambda t, i: synth.gaussian_gradient(t, 4, *shape)
    lrs = [0.008, 0.00784]
    g = run_gpu(W0, grad, lrs, prec="fp32", keep_updates=(0, 1))
    o = run_oracle(W0, grad, lrs, keep_updates=(0, 1))
    R = o["R"][0]
    assert abs(g["R"][0] - R) <= NORM_TOL * R
    for t in range(2):
        assert rel_fro(g["O"][t][0], o["O"][t][0]) <= FP32_NS_TOL, (t, rel_fro(g["O"][t][0], o["O"][t][0]))
        worst = tile_rel_fro_max(g["O"][t][0], o["O"][t][0], tile=256)
        assert worst <= FP32_NS_TOL, (t, worst)
        gs, os_ = g["stats"][t][0], o["stats"][t][0]
        assert gs["flags"] == 0
        for key in ("elr", "pre_norm", "post_norm", "input_norm", "update_norm"):
            assert abs(gs[key] - os_[key]) <= NORM_TOL * abs(os_[key]), (t, key, gs[key], os_[key])
    assert np.linalg.norm(g["W"][0] - o["W"][0]) / R <= 1e-5
    assert rel_fro(g["M"][0], o["M"][0]) <= 1e-6


def test_per_matrix_nesterov_and_beta():
    """The look-ahead and beta are per-matrix descriptor fields: one context
    holds a Nesterov matrix and a plain heavy-ball one with another beta."""
    shapes = [(256, 512), (512, 256)]
    W0 = [synth.initial_weight(i, *s) for i, s in enumerate(shapes)]
    grad = lambda t, i: synth.gaussian_gradient(t, i, *shapes[i])
    import torch
    from pretraining_optimizer_b200 import MuonH
    dev = torch.device("cuda:0")
    W = [torch.from_numpy(w).to(dev) for w in W0]
    M = [torch.zeros_like(w) for w in W]
    opt = MuonH(W, M, beta=[0.95, 0.9], nesterov=[True, False])
    for t in range(3):
        opt.step([torch.from_numpy(grad(t, i)).to(dev) for i in range(2)], 0.01)
    O = [opt.update(i).cpu().numpy() for i in range(2)]
    st = opt.stats()
    opt.close()
    for i, (bt, nv) in enumerate([(0.95, True), (0.9, False)]):
        o = run_oracle([W0[i]], lambda t, _: grad(t, i), [0.01] * 3, beta=bt, nesterov=nv, keep_updates=(2,))
        assert rel_fro(O[i], o["O"][2][0]) <= FP16_NS_TOL, i
        assert rel_fro(M[i].cpu().numpy(), o["M"][0]) <= 1e-6, i
        assert abs(st[i]["input_norm"] - o["stats"][2][0]["input_norm"]) <= NORM_TOL * o["stats"][2][0]["input_norm"]
        assert np.linalg.norm(W[i].cpu().numpy() - o["W"][0]) / o["R"][0] <= 1e-4, i


@pytest.mark.parametrize("prec,form,margin", [("fp16", "y", 5e-3), ("fp16", "gram", 5e-3), ("bf16", "y", 1e-2)])
def test_output_spectrum_lies_in_the_band_of_the_quintic(prec, form, margin):
    """The iteration maps each singular value s of the normalised input to
    p^5(s), p(s) = a s + b s^3 + c s^5: the singular values of the GPU's O
    lie in the image of p^5 over the input's singular values (evaluated on a
    fine grid), up to a 16-bit margin."""
    shape = (192, 448)
    W0 = [synth.initial_weight(0, *shape)]
    grad = lambda t, i: synth.gaussian_gradient(t, 0, *shape)
    g = run_gpu(W0, grad, [0.01], prec=prec, keep_updates=(0,), ns_form=form)
    _, X = oracle.momentum_update(np.zeros(shape), grad(0, 0), 0.95, True)
    s_in = np.linalg.svd(X / np.linalg.norm(X), compute_uv=False)
    grid = np.linspace(s_in.min(), s_in.max(), 100001)
    a, b, c = oracle.QUINTIC
    img = grid
    for _ in range(5):
        img = a * img + b * img ** 3 + c * img ** 5
    s_out = np.linalg.svd(g["O"][0][0].astype(np.float64), compute_uv=False)
    assert s_out.min() >= img.min() - margin and s_out.max() <= img.max() + margin, (s_out.min(), s_out.max(),
                                                                                     img.min(), img.max())
    assert 0.6 < s_out.min() and s_out.max() < 1.25


def test_edge_cases_zero_nan_and_zero_lr():
    shapes = [(128, 256)] * 4
    W0 = [synth.initial_weight(i, *s) for i, s in enumerate(shapes)]

    def grad(t, i):
        gr = synth.gaussian_gradient(t, i, *shapes[i])
        if i == 0:
            return np.zeros_like(gr)            # zero gradient, zero momentum
        if i == 1:
            gr[3, 7] = np.nan                   # non-finite gradient
        return gr

    lrs = [[0.01, 0.01, 0.0, 0.02]]
    g = run_gpu(W0, grad, lrs, keep_updates=(0,))
    o = run_oracle(W0, grad, lrs)
    st = g["stats"][0]
    assert st[0]["flags"] & oracle.FLAG_ZERO_UPDATE and st[0]["elr"] == 0.0
    assert np.allclose(g["W"][0], W0[0], rtol=1e-6, atol=1e-7)
    assert st[1]["flags"] & oracle.FLAG_NONFINITE_INPUT
    assert np.array_equal(g["W"][1], W0[1])
    assert st[2]["flags"] == 0 and st[2]["elr"] == 0.0
    assert np.allclose(g["W"][2], o["W"][2], rtol=0, atol=1e-6)
    assert st[3]["flags"] == 0 and abs(st[3]["elr"] - 0.02) <= NORM_TOL * 0.02


def test_zero_newton_schulz_steps_uses_the_normalised_input():
    """ns_steps = 0: O = X/(||X|| + eps) (fp16 storage), mixed with a matrix that iterates."""
    shapes = [(256, 512), (512, 256)]
    W0 = [synth.initial_weight(i, *s) for i, s in enumerate(shapes)]
    grad = lambda t, i: synth.gaussian_gradient(t, i, *shapes[i])
    for steps in (0, 1):
        g = run_gpu(W0, grad, [0.01, 0.01], ns_steps=steps, keep_updates=(1,))
        o = run_oracle(W0, grad, [0.01, 0.01], ns_steps=steps, keep_updates=(1,))
        for i in range(2):
            assert rel_fro(g["O"][1][i], o["O"][1][i]) <= (1e-3 if steps == 0 else 4e-3)
            assert abs(g["stats"][1][i]["post_norm"] - o["R"][i]) <= NORM_TOL * o["R"][i]
            assert np.linalg.norm(g["W"][i] - o["W"][i]) / o["R"][i] <= 1e-4


def test_convergent_coefficients_reach_the_polar_factor():
    """With (15/8, -10/8, 3/8) the iteration converges to U V^T (fp32 NS mode, 30 steps)."""
    rng = np.random.default_rng(3)
    U, _ = np.linalg.qr(rng.standard_normal((128, 128)))
    V, _ = np.linalg.qr(rng.standard_normal((384, 128)))
    G = ((U * np.geomspace(1.0, 0.05, 128)) @ V.T).astype(np.float32)
    W0 = [synth.initial_weight(0, 128, 384)]
    g = run_gpu(W0, lambda t, i: G, [0.01], prec="fp32", ns_steps=30,
                coeffs=(15 / 8, -10 / 8, 3 / 8), keep_updates=(0,), beta=0.0)
    polar = U @ V.T
    assert rel_fro(g["O"][0][0], polar) <= 1e-5


def test_bitwise_deterministic():
    wl, W0 = _single()
    a = run_gpu(W0, wl.grad, wl.lrs[:3], keep_updates=(2,))
    b = run_gpu(W0, wl.grad, wl.lrs[:3], keep_updates=(2,))
    assert np.array_equal(a["W"][0], b["W"][0]) and np.array_equal(a["O"][2][0], b["O"][2][0])


@pytest.mark.parametrize("ns_form", ["auto", "gram"])
def test_checkpoint_resume_is_bitwise(ns_form):
    """10 straight steps == 5 steps, export/import into a new context, 5 steps
    (in the Y-space form and, forced, in the Gram-space form)."""
    import torch
    from pretraining_optimizer_b200 import MuonH
    wl, W0 = _single()
    grads = [[torch.from_numpy(wl.grad(t, 0)).cuda()] for t in range(10)]
    W = [torch.from_numpy(W0[0]).cuda()]
    opt = MuonH(W, ns_form=ns_form)
    for t in range(10):
        opt.step(grads[t], wl.lrs[t])
    straight = W[0].cpu().numpy()
    opt.close()
    W2 = [torch.from_numpy(W0[0]).cuda()]
    M2 = [torch.zeros_like(W2[0])]
    opt = MuonH(W2, M2, ns_form=ns_form)
    for t in range(5):
        opt.step(grads[t], wl.lrs[t])
    blob = opt.export_state()
    w_ck, m_ck = W2[0].clone(), M2[0].clone()
    opt.close()
    opt = MuonH([w_ck], [m_ck], radii=[1.0], ns_form=ns_form)   # radius replaced by the imported state
    opt.import_state(blob)
    for t in range(5, 10):
        opt.step(grads[t], wl.lrs[t])
    torch.cuda.synchronize()
    assert np.array_equal(w_ck.cpu().numpy(), straight)
    opt.close()


@pytest.mark.parametrize("prec,ns_tol,w_tol", [("fp16", FP16_NS_TOL, 2e-4), ("fp32", FP32_NS_TOL, 2e-6)])
@pytest.mark.parametrize("rule", ["decoupled_wd", "elr_aligned"])
def test_ordinary_muon_rules(rule, prec, ns_tol, w_tol):
    """Eq. (3) (eta = lr) and Eq. (5) (eta = lr ||W||/||u||) through the same
    kernels: a wide and a tall matrix, 5 steps, weight decay 0.1, u = 0.2 O."""
    shapes = [(256, 512), (640, 384)]
    W0 = [synth.initial_weight(i, *s) for i, s in enumerate(shapes)]
    grad = lambda t, i: synth.gaussian_gradient(t, i, *shapes[i])
    lrs = [0.02, 0.015, 0.01, 0.01, 0.005]
    kw = dict(rule=rule, weight_decay=0.1, update_scale=0.2)
    g = run_gpu(W0, grad, lrs, prec=prec, keep_updates=(4,), **kw)
    o = run_oracle(W0, grad, lrs, keep_updates=(4,), **kw)
    for i in range(len(shapes)):
        assert rel_fro(g["O"][4][i], o["O"][4][i]) <= ns_tol
        for t, lr in enumerate(lrs):
            gs, os_ = g["stats"][t][i], o["stats"][t][i]
            assert gs["flags"] == 0
            assert abs(gs["pre_norm"] - os_["pre_norm"]) <= NORM_TOL * os_["pre_norm"], (t, i)
            assert abs(gs["post_norm"] - os_["post_norm"]) <= w_tol * os_["post_norm"], (t, i)
            if rule == "elr_aligned":
                assert abs(gs["elr"] - lr) <= NORM_TOL * lr, (t, i, gs["elr"])     # Eq. (4) = rho
            else:
                assert abs(gs["elr"] - os_["elr"]) <= ns_tol * os_["elr"], (t, i)
        # no projection: the norm moves, unlike MuonH
        assert abs(g["stats"][4][i]["post_norm"] - o["R"][i]) > 1e-3 * o["R"][i]
        assert np.linalg.norm(g["W"][i] - o["W"][i]) / np.linalg.norm(o["W"][i]) <= w_tol, i


def test_phase_timing_does_not_disturb_the_step():
    """Timing on for two steps, read the per-phase times, then keep stepping
    with a new gradient buffer: the results match an untimed context bit for bit."""
    import torch
    from pretraining_optimizer_b200 import MuonH
    dev = torch.device("cuda:0")
    shapes = [(256, 512), (640, 384)]
    W0 = [synth.initial_weight(i, *s) for i, s in enumerate(shapes)]
    runs = []
    for timed in (False, True):
        W = [torch.from_numpy(w).to(dev) for w in W0]
        opt = MuonH(W)
        for t in range(4):
            if timed:
                opt.enable_timing(t < 2)
            G = [torch.from_numpy(synth.gaussian_gradient(t, i, *s)).to(dev) for i, s in enumerate(shapes)]
            opt.step(G, 0.01)
            if timed and t == 1:
                ph = opt.phase_times()
                for name in ("momentum_norm", "ns_gram", "ns_square", "ns_apply", "project", "finalize_step"):
                    # 5 Newton-Schulz iterations a step; the elementwise phases may take
                    # one launch per kind of tile (wide, tall) each step
                    ok = ph[name][1] == 10 if name.startswith("ns_") else ph[name][1] in (2, 4)
                    assert ok and ph[name][0] > 0, (name, ph[name])
        torch.cuda.synchronize()
        opt.device_status()
        runs.append([w.cpu().numpy() for w in W])
        opt.close()
    for a, b in zip(*runs):
        assert np.array_equal(a, b)


@pytest.mark.parametrize("prec,ns_tol,w_tol", [("fp16", FP16_NS_TOL, 1e-3), ("bf16", FP16_NS_TOL, 1e-3)])
def test_two_group_schedule_with_general_path_matrices(prec, ns_tol, w_tol):
    """A set large enough for the two-group schedule (a 4096 x 4096 matrix
    forms group 0) whose second group holds matrices of the general path (odd
    column count) and of the warp-tiled path (strided view, tall): the small
    matrices match the oracle, the large one keeps its invariants."""
    shapes = [(4096, 4096), (130, 70), (640, 384), (1000, 300)]
    strides = [None, None, 400, None]
    W0 = [synth.initial_weight(i, *s) for i, s in enumerate(shapes)]
    grad = lambda t, i: synth.gaussian_gradient(t, i, *shapes[i])
    lrs = [0.01, 0.02, 0.015]
    g = run_gpu(W0, grad, lrs, prec=prec, keep_updates=(2,), strides=strides)
    o = run_oracle(W0[1:], lambda t, i: grad(t, i + 1), lrs, keep_updates=(2,))
    for i in range(1, len(shapes)):
        R = o["R"][i - 1]
        assert rel_fro(g["O"][2][i], o["O"][2][i - 1]) <= ns_tol, (i, rel_fro(g["O"][2][i], o["O"][2][i - 1]))
        assert np.linalg.norm(g["W"][i] - o["W"][i - 1]) / R <= w_tol, i
        for t in range(len(lrs)):
            assert abs(g["stats"][t][i]["post_norm"] - R) <= NORM_TOL * R, (t, i)
    R0 = g["R"][0]
    for t, lr in enumerate(lrs):
        st = g["stats"][t][0]
        assert st["flags"] == 0 and abs(st["post_norm"] - R0) <= NORM_TOL * R0 and abs(st["elr"] - lr) <= NORM_TOL * lr


def test_grouping_gives_the_same_bits():
    """groups=1 runs every kernel on the caller's stream, one after another;
    two and three groups overlap elementwise and GEMM work: a set large
    enough for the overlap gives the same W, M and stats bit for bit
    (fixed partial-sum slots, fixed order) whatever the grouping."""
    import torch
    from pretraining_optimizer_b200 import MuonH
    dev = torch.device("cuda:0")
    shapes = [(4096, 4096), (640, 384), (1000, 300), (1024, 2048)]
    W0 = [synth.initial_weight(i, *s) for i, s in enumerate(shapes)]
    runs = []
    for groups in (0, 1, 3):
        W = [torch.from_numpy(w).to(dev) for w in W0]
        M = [torch.zeros_like(w) for w in W]
        opt = MuonH(W, M, groups=groups)
        for t in range(3):
            opt.step([torch.from_numpy(synth.gaussian_gradient(t, i, *s)).to(dev) for i, s in enumerate(shapes)],
                     0.01)
        launches = opt.last_launch_count()
        st = opt.stats()
        opt.close()
        runs.append(([w.cpu().numpy() for w in W], [m.cpu().numpy() for m in M], st, launches))
    (Wa, Ma, sa, la), (Wb, Mb, sb, lb), (Wc, Mc, sc, lc) = runs
    assert lc > la > lb     # three, two and one groups really ran
    for W_, M_, s_ in ((Wb, Mb, sb), (Wc, Mc, sc)):
        for i in range(len(shapes)):
            assert np.array_equal(Wa[i], W_[i]) and np.array_equal(Ma[i], M_[i]), i
            assert sa[i] == s_[i], i


@pytest.mark.parametrize("prec", ["fp16", "bf16"])
@pytest.mark.parametrize("shape", [(256, 512), (1000, 300), (130, 70)])
def test_error_matches_the_storage_emulation(prec, shape):
    """The kernel stores Y, A and B' in 16 bits and accumulates in fp32: its
    NS error against fp64 matches the oracle's 16-bit storage emulation (the
    same roundings, in another summation order) to within 25 %."""
    from oracle import emulate
    W0 = [synth.initial_weight(0, *shape)]
    grad = lambda t, i: synth.gaussian_gradient(t, i, *shape)
    g = run_gpu(W0, grad, [0.01], prec=prec, keep_updates=(0,))
    M, X = oracle.momentum_update(np.zeros(shape), grad(0, 0), 0.95, True)
    ref = oracle.newton_schulz(X)
    # bf16 operands: the kernel keeps B's diagonal exact (its rounding residual in fp32)
    emu = rel_fro(emulate.newton_schulz_stored(X, storage=prec, exact_diagonal=prec == "bf16"), ref)
    err = rel_fro(g["O"][0][0], ref)
    assert 0.8 * emu <= err <= 1.25 * emu, (err, emu)


def test_bounded_wait_gives_up_and_the_gpu_stays_usable():
    """Failure path without a fault: a wait that can never complete gives up
    after its limit and reports MUONH_ERR_TIMEOUT; the GPU then runs a
    normal step that matches the oracle."""
    import time
    from pretraining_optimizer_b200 import check_wait_timeout
    t0 = time.perf_counter()
    st = check_wait_timeout(0.3)
    dt = time.perf_counter() - t0
    assert st == 5, st
    assert 0.25 <= dt <= 5.0, dt
    wl, W0 = _single()
    g = run_gpu(W0, wl.grad, wl.lrs[:1], keep_updates=(0,))
    o = run_oracle(W0, wl.grad, wl.lrs[:1], keep_updates=(0,))
    assert rel_fro(g["O"][0][0], o["O"][0][0]) <= FP16_NS_TOL
