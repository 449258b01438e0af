"""Checkpoint averaging and the AdamW group on the CUDA path vs the oracle (B200 only)."""
import numpy as np
import pytest

from oracle import aux
import synth

pytestmark = pytest.mark.gpu


def _dev():
    import torch
    return torch.device("cuda:0")


def _bf16_round(x):
    """Round-to-nearest-even of fp64 values to bf16, returned as fp64."""
    import torch
    return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.bfloat16).to(torch.float64).numpy()


@pytest.mark.parametrize("in_dtype,out_dtype", [("f32", "f32"), ("bf16", "f32"), ("bf16", "bf16"), ("f32", "bf16")])
@pytest.mark.parametrize("k,count", [(6, 1_000_003), (1, 4099), (16, 12_345), (2, 3), (6, 0)])
def test_average_matches_the_oracle(in_dtype, out_dtype, k, count):
    """Six checkpoints as in the release recipe, plus k = 1, the maximum k = 16
    and ragged counts (vector body + scalar tail, a 3-element input, empty)."""
    import torch
    from pretraining_optimizer_b200 import average
    rng = np.random.default_rng(count + k)
    host = [rng.standard_normal(count) * 0.02 for _ in range(k)]
    tdt = torch.float32 if in_dtype == "f32" else torch.bfloat16
    dev = [torch.from_numpy(h).to(_dev(), tdt) for h in host]
    as_stored = [d.to(torch.float64).cpu().numpy() for d in dev]
    out = average(dev, out=torch.empty(count, device=_dev(), dtype=torch.float32 if out_dtype == "f32" else torch.bfloat16))
    got = out.to(torch.float64).cpu().numpy()
    ref = aux.checkpoint_average(as_stored)
    # k - 1 fp32 adds of partial sums below k max|x| and one divide by k: each
    # rounding costs at most 2^-24 max|x| after the division
    f32_bound = (k + 1) * 2.0 ** -24 * np.max(np.abs(as_stored), axis=0, initial=0.0)
    if out_dtype == "f32":
        assert np.all(np.abs(got - ref) <= f32_bound + 1e-30)
    else:
        # the fp32 result rounded once more to bf16: equal to the bf16 rounding of the
        # exact mean except where the exact mean is within fp32 error of a bf16 tie
        exact = _bf16_round(ref)
        mismatch = got != exact
        assert mismatch.mean() <= 1e-3 if count > 1000 else not mismatch.any()
        assert np.all(np.abs(got - ref) <= 2.0 ** -8 * (np.abs(ref) + f32_bound) + f32_bound + 1e-30)


def test_average_in_place_and_dyadic_exact():
    """out aliasing the first input; dyadic values average exactly."""
    import torch
    from pretraining_optimizer_b200 import average
    base = np.array([1.0, -2.0, 0.5, 3.0, 0.25, -0.125, 8.0], dtype=np.float32)
    dev = [torch.from_numpy(base * (i + 1)).to(_dev()) for i in range(6)]
    average(dev, out=dev[0])
    assert np.array_equal(dev[0].cpu().numpy(), base * 3.5)


def test_average_rejects_bad_arguments():
    import torch
    from pretraining_optimizer_b200 import MuonHError, average
    x = torch.zeros(64, device=_dev())
    with pytest.raises(ValueError):
        average([x] * 17)
    with pytest.raises(MuonHError) as e:
        average([x[1:], x[1:]], out=torch.zeros(63, device=_dev()))
    assert e.value.status == 2


def _adamw_case(sizes, offsets, steps, wd, seed=3):
    import torch
    from pretraining_optimizer_b200 import adamw_step
    rng = np.random.default_rng(seed)
    p0 = [rng.standard_normal(n) * 0.02 for n in sizes]
    grads = [[rng.standard_normal(n) * 10.0 ** rng.integers(-6, -1) for n in sizes] for _ in range(steps)]
    bufs = []
    for n, off in zip(sizes, offsets):
        # each tensor a view at `off` elements into a larger buffer (misaligned for off % 4 != 0)
        store = [torch.zeros(n + off, device=_dev()) for _ in range(4)]
        bufs.append([s[off:] for s in store])
    for (p, m, v, g), h in zip(bufs, p0):
        p.copy_(torch.from_numpy(h))
    P = [h.astype(np.float32).astype(np.float64) for h in p0]
    M = [np.zeros(n) for n in sizes]
    V = [np.zeros(n) for n in sizes]
    lrs = [3e-3, 2e-3, 1e-3, 1e-3, 5e-4][:steps]
    for t in range(steps):
        for (p, m, v, g), gh in zip(bufs, grads[t]):
            g.copy_(torch.from_numpy(gh))
        adamw_step([b[0] for b in bufs], [b[1] for b in bufs], [b[2] for b in bufs], [b[3] for b in bufs],
                   t + 1, lrs[t], 0.9, 0.95, 1e-8, wd)
        for i in range(len(sizes)):
            gh = grads[t][i].astype(np.float32).astype(np.float64)
            P[i], M[i], V[i] = aux.adamw_step(P[i], M[i], V[i], gh, t + 1, lrs[t], 0.9, 0.95, 1e-8, wd)
    return [[x.cpu().numpy().astype(np.float64) for x in b[:3]] for b in bufs], P, M, V, lrs


@pytest.mark.parametrize("wd", [0.0, 0.1])
def test_adamw_matches_the_oracle(wd):
    """40 tensors (two launches), aligned and misaligned views, ragged sizes,
    an empty tensor, a chunk-sized one and a multi-chunk embedding-like one;
    5 steps.  fp32 kernel vs fp64 oracle: each step moves p by at most lr,
    so the p error stays a small multiple of fp32 rounding of |p| + lr."""
    sizes = [1, 3, 4096, 4097, 0, 2048 * 151] + [128 + 37 * i for i in range(34)]
    offsets = [0, 1, 0, 2, 0, 0] + [(i % 3) * 4 + (i % 2) for i in range(34)]
    got, P, M, V, lrs = _adamw_case(sizes, offsets, 5, wd)
    for i in range(len(sizes)):
        gp, gm, gv = got[i]
        assert np.all(np.abs(gp - P[i]) <= 1e-6 * np.abs(P[i]) + 1e-6 * sum(lrs)), i
        # m = b1 m + (1 - b1) g can cancel: its error is relative to the tensor's scale
        assert np.all(np.abs(gm - M[i]) <= 1e-6 * np.max(np.abs(M[i]), initial=0.0) + 1e-30), i
        assert np.all(np.abs(gv - V[i]) <= 1e-6 * np.abs(V[i]) + 1e-37), i


def test_adamw_rejects_bad_arguments():
    import torch
    from pretraining_optimizer_b200 import MuonHError, adamw_step
    x = torch.zeros(8, device=_dev())
    with pytest.raises(MuonHError):
        adamw_step([x], [x.clone()], [x.clone()], [x.clone()], 0, 1e-3)          # step must be >= 1
    with pytest.raises(MuonHError):
        adamw_step([x], [x.clone()], [x.clone()], [x.clone()], 1, 1e-3, beta1=1.0)
