"""muonh_step_device: the step with its per-matrix arguments (gradient
pointer, lr) in device memory, captured in a CUDA graph and replayed with
new gradients and learning rates, gives the same bits as muonh_step with
host arguments (B200 only)."""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


def _grads(t, shapes, dev):
    import torch
    return [torch.from_numpy(synth.gaussian_gradient(t, i, *s)).to(dev) for i, s in enumerate(shapes)]


@pytest.mark.parametrize("shapes", [
    # two matrix groups (internal GEMM stream), the Gram-space form, general-path matrices
    [(4096, 4096), (2048, 6144), (640, 384), (130, 70)],
    # one group on the caller's stream
    [(256, 512), (512, 256), (96, 301)],
])
def test_captured_step_replays_the_host_argument_step(shapes):
    import torch
    from pretraining_optimizer_b200 import MuonH
    dev = torch.device("cuda:0")
    W0 = [synth.initial_weight(i, *s) for i, s in enumerate(shapes)]
    lrs = [0.01, 0.008, 0.012, 0.0]

    W_ref = [torch.from_numpy(w).to(dev) for w in W0]
    M_ref = [torch.zeros_like(w) for w in W_ref]
    opt = MuonH(W_ref, M_ref)
    stats_ref = []
    for t, lr in enumerate(lrs):
        opt.step(_grads(t, shapes, dev), lr)
        stats_ref.append(opt.stats())
    torch.cuda.synchronize()
    opt.close()

    W = [torch.from_numpy(w).to(dev) for w in W0]
    M = [torch.zeros_like(w) for w in W]
    opt = MuonH(W, M)
    G = [torch.empty_like(w) for w in W]          # the gradient buffers the graph reads
    args = opt.step_args(G, lrs[0])
    lr_field = args.view(torch.float32)[:, 2]     # each 16-byte record: pointer, lr, padding
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        opt.step_device(args)
    for t, lr in enumerate(lrs):
        for g, src in zip(G, _grads(t, shapes, dev)):
            g.copy_(src)
        lr_field.fill_(lr)
        graph.replay()
        torch.cuda.synchronize()
        assert opt.stats() == stats_ref[t], t
    for i in range(len(shapes)):
        assert np.array_equal(W[i].cpu().numpy(), W_ref[i].cpu().numpy()), i
        assert np.array_equal(M[i].cpu().numpy(), M_ref[i].cpu().numpy()), i
    del graph
    opt.device_status()
    opt.close()


def test_device_arguments_without_capture_match_host_arguments():
    """Called directly, muonh_step_device is the host-argument step too."""
    import torch
    from pretraining_optimizer_b200 import MuonH
    dev = torch.device("cuda:0")
    shapes = [(256, 768), (768, 256)]
    W0 = [synth.initial_weight(i, *s) for i, s in enumerate(shapes)]
    runs = []
    for device_args in (False, True):
        W = [torch.from_numpy(w).to(dev) for w in W0]
        opt = MuonH(W)
        for t, lr in enumerate([0.01, 0.02]):
            G = _grads(t, shapes, dev)
            if device_args:
                opt.step_device(opt.step_args(G, [lr, 0.5 * lr]))
            else:
                opt.step(G, [lr, 0.5 * lr])
        torch.cuda.synchronize()
        runs.append([w.cpu().numpy() for w in W])
        opt.close()
    for a, b in zip(*runs):
        assert np.array_equal(a, b)
