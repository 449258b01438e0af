"""The Gram-space evaluation of the Newton-Schulz iteration on the CUDA path
(B200 only): runs of up to three iterations carried on r x r matrices
(A_{k+1} = A_k p(A_k)^2, Y <- Q Y once per run), checked against the fp64
oracle's Y-space iteration, which it equals in exact arithmetic, and against
the oracle's fp16 storage emulation of the same form."""
import numpy as np
import pytest

import oracle
import synth
from parity_helpers import FP16_NS_TOL, NORM_TOL, W_TOL_10, rel_fro, run_gpu, run_oracle, tile_rel_fro_max

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("form", ["gram", "y"])
def test_gram_form_matches_the_oracle(form):
    """Wide, tall, ragged and square matrices, every one in the Gram form when
    asked for (and in the Y-space form as the control), 10 steps."""
    shapes = [(256, 768), (768, 256), (300, 1000), (512, 512), (130, 70), (256, 512)]
    strides = [None, None, None, None, None, 520]
    W0 = [synth.initial_weight(i, *s) for i, s in enumerate(shapes)]
    grad = lambda t, i: synth.gaussian_gradient(t, i, *shapes[i])
    lrs = [0.01] * 10
    keep = (0, 9)
    g = run_gpu(W0, grad, lrs, keep_updates=keep, strides=strides, ns_form=form)
    o = run_oracle(W0, grad, lrs, keep_updates=keep)
    for i, s in enumerate(shapes):
        R = o["R"][i]
        for t in keep:
            err = rel_fro(g["O"][t][i], o["O"][t][i])
            assert err <= FP16_NS_TOL, (form, i, s, t, err)
            worst = tile_rel_fro_max(g["O"][t][i], o["O"][t][i], tile=64)
            assert worst <= FP16_NS_TOL, (form, i, s, t, worst)
        for t in range(len(lrs)):
            gs, os_ = g["stats"][t][i], o["stats"][t][i]
            assert gs["flags"] == 0
            assert abs(gs["post_norm"] - R) <= NORM_TOL * R
            assert abs(gs["elr"] - os_["elr"]) <= NORM_TOL * os_["elr"]
            assert abs(gs["input_norm"] - os_["input_norm"]) <= NORM_TOL * os_["input_norm"]
        assert np.linalg.norm(g["W"][i] - o["W"][i]) / R <= W_TOL_10, (form, i, s)


@pytest.mark.parametrize("shape", [(256, 768), (640, 256), (512, 2048)])
def test_gram_form_error_matches_its_storage_emulation(shape):
    """The kernels store Y, A, T = A P, P = p(A) and Q in fp16 and accumulate
    in fp32: the NS error against fp64 matches the oracle's fp16 emulation of
    the Gram-space form, runs (3, 2), within 25 %."""
    from oracle import emulate
    W0 = [synth.initial_weight(0, *shape)]
    grad = lambda t, i: synth.gaussian_gradient(t, i, *shape)
    g = run_gpu(W0, grad, [0.01], keep_updates=(0,), ns_form="gram")
    _, X = oracle.momentum_update(np.zeros(shape), grad(0, 0), 0.95, True)
    ref = oracle.newton_schulz(X)
    emu = rel_fro(emulate.newton_schulz_gram_stored(X, (3, 2), storage="fp16"), ref)
    err = rel_fro(g["O"][0][0], ref)
    assert 0.8 * emu <= err <= 1.25 * emu, (err, emu)


@pytest.mark.parametrize("gradient", ["gaussian", "ill_conditioned"])
def test_gram_form_at_the_qwen3_mlp_shapes(gradient):
    """2048 x 6144 (down) and 6144 x 2048 (gate, up) take the Gram form by
    default: two steps against the fp64 oracle, and the first step's error
    against the fp16 emulation of the form."""
    from oracle import emulate
    shapes = [(2048, 6144), (6144, 2048)]
    W0 = [synth.initial_weight(6 - 2 * i, *s) for i, s in enumerate(shapes)]

    def grad(t, i):
        if gradient == "gaussian":
            return synth.gaussian_gradient(t, 6 - 2 * i, *shapes[i])
        return synth.ill_conditioned_gradient(t, 6 - 2 * i, *shapes[i])

    lrs = [0.008, 0.00784]
    g = run_gpu(W0, grad, lrs, keep_updates=(0, 1))
    assert g["flops"]["ns_product"] > 0          # the default form here is the Gram form
    o = run_oracle(W0, grad, lrs, keep_updates=(0, 1))
    for i in range(2):
        R = o["R"][i]
        for t in range(2):
            err = rel_fro(g["O"][t][i], o["O"][t][i])
            assert err <= FP16_NS_TOL, (i, t, err)
            assert tile_rel_fro_max(g["O"][t][i], o["O"][t][i], tile=256) <= FP16_NS_TOL, (i, t)
            assert abs(g["stats"][t][i]["post_norm"] - R) <= NORM_TOL * R
            assert abs(g["stats"][t][i]["elr"] - lrs[t]) <= NORM_TOL * lrs[t]
        assert np.linalg.norm(g["W"][i] - o["W"][i]) / R <= 1e-4, i
    _, X = oracle.momentum_update(np.zeros(shapes[0]), grad(0, 0), 0.95, True)
    ref = oracle.newton_schulz(X)
    emu = rel_fro(emulate.newton_schulz_gram_stored(X, (3, 2), storage="fp16"), ref)
    err = rel_fro(g["O"][0][0], ref)
    assert 0.8 * emu <= err <= 1.25 * emu, (err, emu)


def _upper(r_pad):
    b = r_pad // 256
    return b * (b + 1) // 2


def test_executed_flops_of_each_form():
    """The tensor-core FLOPs the library reports per phase equal the tile
    counts of each form: Y-space per iteration Y Y^T and B' on the upper
    256 x 256 tiles, B' Y on all; Gram-space per run of g one Y Y^T, g
    squares and 4 g - 3 - g other products on the upper tiles, one Q Y."""
    shapes = [(512, 1536), (256, 512)]
    W0 = [synth.initial_weight(i, *s) for i, s in enumerate(shapes)]
    grad = lambda t, i: synth.gaussian_gradient(t, i, *shapes[i])
    tile = 2 * 256 * 256
    flops = {}
    for form in ("y", "gram"):
        flops[form] = run_gpu(W0, grad, [0.01], ns_form=form)["flops"]
    y = flops["y"]
    exp_gram = exp_sq = exp_apply = 0
    for r, c in shapes:
        exp_gram += 5 * _upper(r) * tile * c
        exp_sq += 5 * _upper(r) * tile * r
        exp_apply += 5 * (r // 256) * (c // 256) * tile * r
    assert (y["ns_gram"], y["ns_square"], y["ns_apply"], y["ns_product"]) == (exp_gram, exp_sq, exp_apply, 0)
    gf = flops["gram"]
    exp_gram = exp_sq = exp_apply = exp_prod = 0
    for r, c in shapes:
        for g in (3, 2):
            exp_gram += _upper(r) * tile * c
            exp_sq += g * _upper(r) * tile * r
            exp_prod += (3 * g - 3) * _upper(r) * tile * r
            exp_apply += (r // 256) * (c // 256) * tile * r
    assert (gf["ns_gram"], gf["ns_square"], gf["ns_apply"], gf["ns_product"]) == (exp_gram, exp_sq, exp_apply,
                                                                                   exp_prod)


def test_automatic_form_choice():
    """The automatic choice takes the Gram-space form where it saves FLOPs,
    c >= 2r with r >= 1024 (here 1024 x 2048 and its tall transpose), and the
    Y-space form for a square class and for r < 1024: the per-phase FLOPs
    are the sum of each matrix's own form."""
    shapes = [(1024, 2048), (2048, 2048), (512, 1536), (2048, 1024)]
    W0 = [synth.initial_weight(i, *s) for i, s in enumerate(shapes)]
    grad = lambda t, i: synth.gaussian_gradient(t, i, *shapes[i])
    f = run_gpu(W0, grad, [0.01])["flops"]
    tile = 2 * 256 * 256
    exp = {"ns_gram": 0, "ns_square": 0, "ns_apply": 0, "ns_product": 0}
    for rows, cols in shapes:
        r, c = min(rows, cols), max(rows, cols)
        if r >= 1024 and c >= 2 * r:
            for g in (3, 2):
                exp["ns_gram"] += _upper(r) * tile * c
                exp["ns_square"] += g * _upper(r) * tile * r
                exp["ns_product"] += (3 * g - 3) * _upper(r) * tile * r
                exp["ns_apply"] += (r // 256) * (c // 256) * tile * r
        else:
            exp["ns_gram"] += 5 * _upper(r) * tile * c
            exp["ns_square"] += 5 * _upper(r) * tile * r
            exp["ns_apply"] += 5 * (r // 256) * (c // 256) * tile * r
    assert {k: f[k] for k in exp} == exp


@pytest.mark.parametrize("ns_steps", [1, 2, 3, 4, 6, 7])
def test_gram_form_run_lengths(ns_steps):
    """Other step counts split into other runs ((1), (2), (3), (2, 2),
    (3, 3), (3, 2, 2)); each matches the oracle, and the run structure
    shows in the executed FLOPs: one Y Y^T and one Q Y per run."""
    shape = (256, 768)
    W0 = [synth.initial_weight(0, *shape)]
    grad = lambda t, i: synth.gaussian_gradient(t, 0, *shape)
    g = run_gpu(W0, grad, [0.01, 0.01], ns_steps=ns_steps, keep_updates=(1,), ns_form="gram")
    o = run_oracle(W0, grad, [0.01, 0.01], ns_steps=ns_steps, keep_updates=(1,))
    assert rel_fro(g["O"][1][0], o["O"][1][0]) <= FP16_NS_TOL, (ns_steps, rel_fro(g["O"][1][0], o["O"][1][0]))
    assert np.linalg.norm(g["W"][0] - o["W"][0]) / o["R"][0] <= 1e-4
    runs = -(-ns_steps // 3)
    tile = 2 * 256 * 256
    assert g["flops"]["ns_gram"] == runs * tile * 768            # one upper tile, K = 768
    assert g["flops"]["ns_apply"] == runs * 3 * tile * 256       # three tiles, K = 256
    assert g["flops"]["ns_square"] == ns_steps * tile * 256


def test_gram_form_beside_y_space_matrices_of_the_same_class():
    """Matrices with fewer Newton-Schulz steps than the context's largest
    stay in the Y-space form, in the same shape class as Gram-form ones."""
    shapes = [(256, 768)] * 3
    W0 = [synth.initial_weight(i, *s) for i, s in enumerate(shapes)]
    grad = lambda t, i: synth.gaussian_gradient(t, i, *shapes[i])
    steps = [5, 3, 5]
    g = run_gpu(W0, grad, [0.01] * 3, ns_steps=steps, keep_updates=(2,), ns_form="gram")
    for i in range(3):
        o = run_oracle([W0[i]], lambda t, _: grad(t, i), [0.01] * 3, ns_steps=steps[i], keep_updates=(2,))
        assert rel_fro(g["O"][2][i], o["O"][2][0]) <= FP16_NS_TOL, i
        assert np.linalg.norm(g["W"][i] - o["W"][0]) / o["R"][0] <= 1e-4, i


def test_gram_form_with_the_convergent_quintic():
    """(15/8, -10/8, 3/8) has other bounds on the stored Q (its p(0) is 15/8)
    and converges: 9 steps in the Gram form reach the oracle's output."""
    coeffs = (15 / 8, -10 / 8, 3 / 8)
    shape = (256, 768)
    W0 = [synth.initial_weight(0, *shape)]
    grad = lambda t, i: synth.gaussian_gradient(t, 0, *shape)
    g = run_gpu(W0, grad, [0.01], ns_steps=9, coeffs=coeffs, keep_updates=(0,), ns_form="gram")
    o = run_oracle(W0, grad, [0.01], ns_steps=9, coeffs=coeffs, keep_updates=(0,))
    assert rel_fro(g["O"][0][0], o["O"][0][0]) <= FP16_NS_TOL


@pytest.mark.parametrize("rule", ["decoupled_wd", "elr_aligned"])
def test_ordinary_muon_rules_on_the_gram_form(rule):
    """Eq. (3) and Eq. (5) read O from the buffer the last Gram-space run
    wrote: wide and tall matrices, 4 steps, weight decay 0.1, u = 0.2 O."""
    shapes = [(256, 768), (768, 256)]
    W0 = [synth.initial_weight(i, *s) for i, s in enumerate(shapes)]
    grad = lambda t, i: synth.gaussian_gradient(t, i, *shapes[i])
    lrs = [0.02, 0.015, 0.01, 0.005]
    kw = dict(rule=rule, weight_decay=0.1, update_scale=0.2)
    g = run_gpu(W0, grad, lrs, keep_updates=(3,), ns_form="gram", **kw)
    o = run_oracle(W0, grad, lrs, keep_updates=(3,), **kw)
    for i in range(2):
        assert rel_fro(g["O"][3][i], o["O"][3][i]) <= FP16_NS_TOL, i
        assert np.linalg.norm(g["W"][i] - o["W"][i]) / np.linalg.norm(o["W"][i]) <= 2e-4, i
        for t, lr in enumerate(lrs):
            gs, os_ = g["stats"][t][i], o["stats"][t][i]
            assert gs["flags"] == 0
            if rule == "elr_aligned":
                assert abs(gs["elr"] - lr) <= NORM_TOL * lr, (t, i)
            else:
                assert abs(gs["elr"] - os_["elr"]) <= FP16_NS_TOL * os_["elr"], (t, i)


def test_groups_split_by_form_give_the_same_bits():
    """A set whose matrix groups hold both forms: with two groups the first
    group's momentum pass and the last group's projection run in two parts
    (Y-space matrices, then Gram-space ones) around the Gram-space and
    Y-space GEMMs; with three groups the end groups hold one form each and
    are not split; one group runs everything in sequence.  W, M and the
    stats agree bit for bit, and the split schedule launches more kernels."""
    import torch
    from pretraining_optimizer_b200 import MuonH
    dev = torch.device("cuda:0")
    # NS work: the three 2048 x 6144 (Gram-space) matrices dominate, so two
    # groups end after the second of them and each holds both forms
    shapes = [(2048, 6144), (1024, 1024), (6144, 2048), (512, 768), (2048, 6144), (1024, 2048)]
    W0 = [synth.initial_weight(i, *s) for i, s in enumerate(shapes)]
    runs = []
    for groups in (1, 2, 3):
        W = [torch.from_numpy(w).to(dev) for w in W0]
        M = [torch.zeros_like(w) for w in W]
        opt = MuonH(W, M, groups=groups)
        for t in range(2):
            opt.step([torch.from_numpy(synth.gaussian_gradient(t, i, *s)).to(dev) for i, s in enumerate(shapes)],
                     [0.01, 0.02, 0.01, 0.015, 0.01, 0.02])
        launches = opt.last_launch_count()
        st = opt.stats()
        opt.device_status()
        opt.close()
        runs.append(([w.cpu().numpy() for w in W], [m.cpu().numpy() for m in M], st, launches))
    (W1, M1, s1, l1), (W2, M2, s2, l2), (W3, M3, s3, l3) = runs
    assert l2 > l1 and l3 > l1
    for W_, M_, s_ in ((W2, M2, s2), (W3, M3, s3)):
        for i in range(len(shapes)):
            assert np.array_equal(W1[i], W_[i]) and np.array_equal(M1[i], M_[i]), i
            assert s1[i] == s_[i], i
    # and the result is the method's: the Gram-space matrices against the oracle
    for i in (0, 2, 4):
        R = oracle.radius(W0[i])
        w, m = W0[i].astype(np.float64), np.zeros(shapes[i])
        for t, lr in enumerate([0.01, 0.01]):
            w, m, _, _ = oracle.muonh_step(w, m, synth.gaussian_gradient(t, i, *shapes[i]), lr, R)
        assert rel_fro(W1[i], w) <= W_TOL_10, i
