"""The allocation-free momentum entry point (B200 only).

Callers that cannot allocate device memory -- code running while a stream is
captured in the global mode, programs whose device memory belongs to a
framework allocator or a fixed arena, loops that must not take the driver's
allocation locks -- use muonh_momentum_norm_noalloc, whose scratch is an
array compiled into the library.  Over two calls in a row it must give the
fp64 oracle's momentum buffer and Newton-Schulz input norm, and agree with
what muonh_step does to the same buffer.  This file is collected last, so a
stop at the first failure has run every other test."""
import numpy as np
import pytest

import oracle
import synth
from parity_helpers import NORM_TOL, rel_fro

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape", [(256, 512), (768, 256), (96, 301)])
@pytest.mark.parametrize("nesterov", [True, False])
def test_noalloc_momentum_matches_the_oracle_and_the_step_on_two_calls(shape, nesterov):
    import torch
    from pretraining_optimizer_b200 import MuonH, momentum_norm_noalloc
    dev = torch.device("cuda:0")
    beta = 0.95
    W = torch.from_numpy(synth.initial_weight(0, *shape)).to(dev)
    M_step = torch.zeros_like(W)
    opt = MuonH([W], [M_step], beta=beta, nesterov=nesterov)
    M = torch.zeros_like(W)
    M_ref = np.zeros(shape)
    x_norm = torch.empty((), dtype=torch.float64, device=dev)
    for t in range(2):
        g = synth.gaussian_gradient(t, 0, *shape)
        G = torch.from_numpy(g).to(dev)
        opt.step([G], 0.01)
        momentum_norm_noalloc(M, G, beta=beta, nesterov=nesterov, x_norm=x_norm)
        torch.cuda.synchronize()
        # the oracle, fp64: M_t = beta M_{t-1} + G_t and ||X||_F
        M_ref, X_ref = oracle.momentum_update(M_ref, g, beta, nesterov)
        ref_norm = float(np.linalg.norm(X_ref))
        got = float(x_norm.item())
        assert rel_fro(M.cpu().numpy(), M_ref) <= 1e-6, (t, rel_fro(M.cpu().numpy(), M_ref))
        assert abs(got - ref_norm) <= NORM_TOL * ref_norm, (t, got, ref_norm)
        # the context-based step on the same inputs
        step_norm = opt.stats()[0]["input_norm"]
        assert rel_fro(M.cpu().numpy(), M_step.cpu().numpy()) <= 1e-6, t
        assert abs(got - step_norm) <= NORM_TOL * step_norm, (t, got, step_norm)
    opt.close()


def test_noalloc_rejects_matrices_beyond_its_scratch():
    import torch
    m = torch.zeros((16, 16), device="cuda:0")
    # a 65,537-tile shape described through a strided view of a small buffer is
    # rejected before any kernel runs (rows x 512 columns, 8 rows per tile)
    big_rows = 8 * 65537
    from pretraining_optimizer_b200 import muonh as B
    st = B.library().muonh_momentum_norm_noalloc(m.data_ptr(), m.data_ptr(), big_rows, 512, 512, 0.95, 1,
                                                 m.data_ptr(), None)
    assert st == 6
    assert b"too large" in B.library().muonh_last_error()
    assert np.count_nonzero(m.cpu().numpy()) == 0
