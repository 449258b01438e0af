"""Full-size workloads on the CUDA path, checked against the fp64 oracle on
sampled matrices (B200 only).

Every matrix of the set runs through the same muonh_step launches bench.py
times.  Sampled matrices take their inputs from `synth` (bit-identical to the
oracle's); the others get device-drawn inputs of the same distribution.  The
oracle follows the sampled matrices from step 0 for a few steps; at later
steps it restarts from the GPU's own (W, M) snapshot and checks that single
step ("one by one").  The closed-form invariants of Eq. (1), ||W|| = R and
elr = lr, are checked on every matrix at every step."""
import numpy as np
import pytest

import oracle
import synth
from parity_helpers import FP16_NS_TOL, NORM_TOL, W_TOL_10, rel_fro, tile_rel_fro_max

pytestmark = pytest.mark.gpu


def _device_gradient(kind, t, shape, gen, dev):
    import torch
    m, n = shape
    if kind == "gaussian":
        return torch.randn(shape, generator=gen, device=dev) * synth.GRAD_STD
    a = torch.randn((m, 8), generator=gen, device=dev)
    b = torch.randn((n, 8), generator=gen, device=dev)
    low = a @ b.T
    low *= 0.1 / torch.linalg.norm(low)
    if t % 10 == 9:
        chi2 = torch._standard_gamma(torch.full(shape, 1.5, device=dev)) * 2.0
        noise = 1e-3 * torch.randn(shape, generator=gen, device=dev) / torch.sqrt(chi2 / 3.0)
    else:
        noise = 1e-5 * torch.randn(shape, generator=gen, device=dev)
    return low + noise


class FullRun:
    """The whole matrix set on the GPU; synth inputs for `sample`."""

    def __init__(self, wl, sample, seed=7):
        import torch
        from pretraining_optimizer_b200 import MuonH
        self.torch = torch
        self.wl = wl
        self.sample = set(sample)
        self.dev = torch.device("cuda:0")
        self.gen = torch.Generator(device=self.dev)
        self.gen.manual_seed(seed)
        self.shapes = [(m.rows, m.cols) for m in wl.matrices]
        self.W, self.M = [], []
        for i, s in enumerate(self.shapes):
            if i in self.sample:
                w = torch.from_numpy(wl.weight(i)).to(self.dev)
            else:
                w = torch.randn(s, generator=self.gen, device=self.dev) * synth.W0_STD
            self.W.append(w)
            self.M.append(torch.zeros_like(w))
        self.G = [torch.empty_like(w) for w in self.W]
        self.opt = MuonH(self.W, self.M, beta=wl.beta, nesterov=wl.nesterov, ns_steps=wl.ns_steps,
                         ns_coeffs=wl.ns_coeffs)
        self.R = self.opt.radii()
        self.t = 0

    def step(self):
        torch = self.torch
        for i, s in enumerate(self.shapes):
            if i in self.sample:
                self.G[i].copy_(torch.from_numpy(self.wl.grad(self.t, i)))
            else:
                self.G[i].copy_(_device_gradient(self.wl.gradient, self.t, s, self.gen, self.dev))
        lr = self.wl.lrs[self.t]
        self.opt.step(self.G, lr)
        stats = self.opt.stats()
        for i, st in enumerate(stats):
            R = self.R[i]
            assert st["flags"] == 0, (self.t, i, st)
            assert np.isfinite(st["post_norm"]) and abs(st["post_norm"] - R) <= NORM_TOL * R, (self.t, i, st)
            if lr > 0:
                assert abs(st["elr"] - lr) <= NORM_TOL * lr, (self.t, i, st["elr"], lr)
        self.t += 1
        return stats

    def host(self, i):
        return (self.W[i].cpu().numpy().astype(np.float64), self.M[i].cpu().numpy().astype(np.float64))

    def close(self):
        self.opt.device_status()
        self.opt.close()


def _oracle_from_start(wl, sample, steps):
    W = {i: wl.weight(i).astype(np.float64) for i in sample}
    M = {i: np.zeros_like(W[i]) for i in sample}
    R = {i: oracle.radius(wl.weight(i)) for i in sample}
    out = {}
    for t in range(steps):
        for i in sample:
            W[i], M[i], O, st = oracle.muonh_step(W[i], M[i], wl.grad(t, i), wl.lrs[t], R[i], wl.beta,
                                                  wl.nesterov, wl.ns_steps, wl.ns_coeffs)
            if t == steps - 1:
                out[i] = (W[i], O, st)
    return out, R


def _one_step_check(run, wl, sample, t_check):
    """Snapshot (W, M) of the sampled matrices before step t_check, run that
    step on the GPU and compare with the oracle started from the snapshot."""
    snap = {i: run.host(i) for i in sample}
    assert run.t == t_check
    stats = run.step()
    for i in sample:
        W, M = snap[i]
        Wn, _, O, st = oracle.muonh_step(W, M, wl.grad(t_check, i), wl.lrs[t_check], run.R[i], wl.beta,
                                        wl.nesterov, wl.ns_steps, wl.ns_coeffs)
        O_gpu = run.opt.update(i).cpu().numpy()
        assert rel_fro(O_gpu, O) <= FP16_NS_TOL, (t_check, i, rel_fro(O_gpu, O))
        worst = tile_rel_fro_max(O_gpu, O, tile=256)
        assert worst <= FP16_NS_TOL, (t_check, i, worst)
        assert np.linalg.norm(run.W[i].cpu().numpy() - Wn) / run.R[i] <= 1e-4, (t_check, i)
        assert abs(stats[i]["update_norm"] - st["update_norm"]) <= FP16_NS_TOL * st["update_norm"]
        assert abs(stats[i]["input_norm"] - st["input_norm"]) <= NORM_TOL * st["input_norm"]


def _check_sampled_against_oracle(run, wl, sample, steps):
    ref, R = _oracle_from_start(wl, sample, steps)
    for i in sample:
        W_ref, O_ref, st = ref[i]
        O_gpu = run.opt.update(i).cpu().numpy()
        assert rel_fro(O_gpu, O_ref) <= FP16_NS_TOL, (i, rel_fro(O_gpu, O_ref))
        # every 256 x 256 block of O, the output tile of the Newton-Schulz GEMMs
        worst = tile_rel_fro_max(O_gpu, O_ref, tile=256)
        assert worst <= FP16_NS_TOL, (i, worst)
        assert np.linalg.norm(run.W[i].cpu().numpy() - W_ref) / R[i] <= W_TOL_10, i


def test_qwen3_1p7b_set_50_steps():
    """196 matrices, 1.409e9 parameters, 50 steps of linear decay from 0.008."""
    wl = synth.workload("qwen3_1.7b")
    sample = list(range(7))                       # layer 0: every shape and orientation
    run = FullRun(wl, sample)
    for _ in range(10):
        run.step()
    _check_sampled_against_oracle(run, wl, sample, 10)
    while run.t < 49:
        run.step()
    _one_step_check(run, wl, [1, 4, 6], 49)     # k_proj, gate_proj (tall), down_proj
    run.close()


def test_qwen3_0p6b_set_wsd_20_steps():
    """196 matrices, 4.40e8 parameters, 20 WSD steps (2 warmup, 10 stable,
    8 decay to 0, peak 0.012); the oracle follows layer 0 for all 20 steps."""
    wl = synth.workload("qwen3_0.6b")
    sample = list(range(7))
    run = FullRun(wl, sample)
    for _ in range(20):
        run.step()
    _check_sampled_against_oracle(run, wl, sample, 20)
    run.close()


def test_qwen3_1p7b_ill_conditioned_100_steps():
    """Rank-8 gradients plus small noise, Student-t(3) noise every 10th step:
    every matrix stays finite and on its sphere for 100 steps; sampled steps
    (including heavy-tailed ones) match the oracle one by one."""
    wl = synth.workload("qwen3_1.7b_illcond")
    sample = [1, 6]
    run = FullRun(wl, sample)
    for t_check in (9, 59, 99):
        while run.t < t_check:
            run.step()
        _one_step_check(run, wl, sample, t_check)
    for w in run.W:
        assert bool(run.torch.isfinite(w).all())
    run.close()


@pytest.mark.parametrize("shape", synth.SWEEP_SHAPES)
def test_shape_sweep_one_step(shape):
    """Two matrices of each sweep shape in one context; the first checked
    against the oracle (its Newton-Schulz products in fp32 for 8192 x 8192,
    norms and projection in fp64)."""
    import torch
    from pretraining_optimizer_b200 import MuonH
    dev = torch.device("cuda:0")
    W0 = [synth.initial_weight(i, *shape) for i in range(2)]
    G = [synth.gaussian_gradient(0, i, *shape) for i in range(2)]
    W = [torch.from_numpy(w).to(dev) for w in W0]
    opt = MuonH(W)
    opt.step([torch.from_numpy(g).to(dev) for g in G], 0.01)
    O = opt.update(0).cpu().numpy()
    st = opt.stats()
    opt.close()
    ns_dtype = np.float32 if shape[0] * shape[1] > 4096 * 4096 else np.float64
    R = oracle.radius(W0[0])
    W_ref, _, O_ref, _ = oracle.muonh_step(W0[0], np.zeros_like(W0[0]), G[0], 0.01, R, ns_dtype=ns_dtype)
    assert rel_fro(O, O_ref) <= FP16_NS_TOL
    assert np.linalg.norm(W[0].cpu().numpy() - W_ref) / R <= 1e-4
    for i in range(2):
        assert abs(st[i]["post_norm"] - oracle.radius(W0[i])) <= NORM_TOL * oracle.radius(W0[i])
