"""The allocation-free momentum entry point against muonh_step (B200 only).

Callers that cannot allocate device memory (stream capture in global mode,
framework-owned or fixed-arena device memory, allocation-lock-free loops)
use muonh_momentum_norm_noalloc, whose scratch is compiled into the library.
Over two calls in a row it must reproduce what muonh_step does to the
momentum buffer and the input norm it reports."""
import numpy as np
import pytest

import synth
from parity_helpers import NORM_TOL

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape", [(256, 512), (768, 256), (96, 301)])
def test_noalloc_momentum_matches_the_step_on_two_calls(shape):
    import torch
    from pretraining_optimizer_b200 import MuonH, momentum_norm_noalloc
    dev = torch.device("cuda:0")
    W = torch.from_numpy(synth.initial_weight(0, *shape)).to(dev)
    M_ref = torch.zeros_like(W)
    opt = MuonH([W], [M_ref])
    M = torch.zeros_like(W)
    x_norm = torch.empty((), dtype=torch.float64, device=dev)
    for t in range(2):
        G = torch.from_numpy(synth.gaussian_gradient(t, 0, *shape)).to(dev)
        opt.step([G], 0.01)
        momentum_norm_noalloc(M, G, beta=0.95, nesterov=True, x_norm=x_norm)
        torch.cuda.synchronize()
        ref_norm = opt.stats()[0]["input_norm"]
        assert np.array_equal(M.cpu().numpy(), M_ref.cpu().numpy()), t
        assert abs(float(x_norm.item()) - ref_norm) <= NORM_TOL * ref_norm, (t, float(x_norm.item()), ref_norm)
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
