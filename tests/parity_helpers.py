"""Shared pieces of the GPU parity tests: run the CUDA path and the oracle on
the same seeded inputs and compare."""
import numpy as np

import oracle

FP16_NS_TOL = 1e-2      # relative Frobenius error of O vs fp64 (16-bit NS, fp16 or bf16 operands)
FP32_NS_TOL = 1e-5      # relative Frobenius error of O vs fp64 (fp32 NS mode)
NORM_TOL = 1e-5         # weight norms and effective LR, relative
W_TOL_10 = 1e-3         # ||W_gpu - W_ref||_F / R after 10 steps (16-bit NS)


def rel_fro(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (nb if nb > 0 else 1.0)


def tile_rel_fro_max(a, b, tile=128):
    """Largest relative Frobenius error over the tile x tile blocks of a
    against b (ragged edge blocks included): a localised mistake, such as one
    wrong output tile of a GEMM, shows here although the whole-matrix error
    averages it away."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    worst = 0.0
    for i in range(0, b.shape[0], tile):
        for j in range(0, b.shape[1], tile):
            worst = max(worst, rel_fro(a[i:i + tile, j:j + tile], b[i:i + tile, j:j + tile]))
    return worst


def run_gpu(W0, grad_fn, lrs, *, prec="fp16", ns_steps=5, coeffs=oracle.QUINTIC, beta=0.95,
            nesterov=True, eps=1e-7, keep_updates=(), radii=None, strides=None, rule="hyperball",
            weight_decay=0.0, update_scale=1.0, ns_form="auto"):
    """Run len(lrs) steps through the C-ABI; returns W, M (numpy fp32), per-step stats,
    and {step: [O_i]} for the steps listed in keep_updates."""
    import torch
    from pretraining_optimizer_b200 import MuonH
    dev = torch.device("cuda:0")

    def place(a, i):
        t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
        if strides is not None and strides[i] is not None:
            big = torch.zeros((a.shape[0], strides[i]), dtype=torch.float32, device=dev)
            big[:, : a.shape[1]] = t.to(dev)
            return big[:, : a.shape[1]]
        return t.to(dev)

    W = [place(w, i) for i, w in enumerate(W0)]
    M = [place(np.zeros_like(w), i) for i, w in enumerate(W0)]
    opt = MuonH(W, M, beta=beta, nesterov=nesterov, ns_steps=ns_steps, ns_coeffs=coeffs, eps=eps,
                ns_precision=prec, radii=radii, update_rule=rule, weight_decay=weight_decay,
                update_scale=update_scale, ns_form=ns_form)
    stats, updates = [], {}
    for t, lr in enumerate(lrs):
        G = [place(grad_fn(t, i), i) for i in range(len(W0))]
        opt.step(G, lr)
        stats.append(opt.stats())
        if t in keep_updates:
            updates[t] = [opt.update(i).cpu().numpy() for i in range(len(W0))]
    torch.cuda.synchronize()
    opt.device_status()
    out = dict(W=[w.cpu().numpy() for w in W], M=[m.cpu().numpy() for m in M], stats=stats,
               O=updates, R=opt.radii(), launches=opt.last_launch_count(), flops=opt.phase_flops())
    opt.close()
    return out


def run_oracle(W0, grad_fn, lrs, *, ns_steps=5, coeffs=oracle.QUINTIC, beta=0.95, nesterov=True,
               eps=1e-7, keep_updates=(), R_list=None, rule="hyperball", weight_decay=0.0,
               update_scale=1.0):
    rule_id = {"hyperball": oracle.RULE_HYPERBALL, "decoupled_wd": oracle.RULE_DECOUPLED_WD,
               "elr_aligned": oracle.RULE_ELR_ALIGNED}[rule]
    W = [np.asarray(w, dtype=np.float64) for w in W0]
    M = [np.zeros_like(w) for w in W]
    R = list(R_list) if R_list is not None else [oracle.radius(w) for w in W]
    stats, updates = [], {}
    for t, lr in enumerate(lrs):
        st_t, O_t = [], []
        for i in range(len(W)):
            lri = lr[i] if isinstance(lr, (list, tuple)) else lr
            W[i], M[i], O, st = oracle.muonh_step(W[i], M[i], grad_fn(t, i), lri, R[i], beta, nesterov,
                                                  ns_steps, coeffs, eps, rule=rule_id,
                                                  weight_decay=weight_decay, update_scale=update_scale)
            st_t.append(st)
            O_t.append(O)
        stats.append(st_t)
        if t in keep_updates:
            updates[t] = O_t
    return dict(W=W, M=M, stats=stats, O=updates, R=R)
