"""LR schedule helpers against the values the report prints (no GPU)."""
import os

import pytest

from pretraining_optimizer_b200 import schedules as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "schedule_worked_values.txt")


def _rows():
    out = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        lhs, val, tol, _cite = [x.strip() for x in line.split("|")]
        fn, *args = lhs.split()
        out.append((fn, [float(a) for a in args], float(val), float(tol)))
    return out


def _eval(fn, args):
    if fn == "phase1_base_lr":
        return S.phase1_base_lr(args[0])
    if fn == "hyperball_phase1":
        return S.hyperball_lr(S.phase1_base_lr(args[0]))
    if fn == "phase2_base_lr":
        return S.phase2_base_lr(args[0], args[1])
    if fn == "production_no_cma":
        return S.production_base_lr(int(args[0]), cma_from=None)
    if fn == "production":
        return S.production_base_lr(int(args[0]))
    if fn == "hyperball_production":
        return S.hyperball_lr(S.production_base_lr(int(args[0])))
    if fn == "cosine":
        return S.cosine_lr(int(args[0]), int(args[1]))
    raise KeyError(fn)


@pytest.mark.parametrize("row", _rows(), ids=lambda r: f"{r[0]}{r[1]}")
def test_printed_worked_values(row):
    fn, args, val, tol = row
    got = _eval(fn, args)
    assert abs(got - val) <= tol * abs(val), (fn, args, got, val)


def test_phase1_shape():
    assert S.phase1_base_lr(0) == 0.0
    assert S.phase1_base_lr(500) == pytest.approx(2.5e-3)
    # the power decay is continuous at the end of warm-up and tends to 5e-4
    assert S.phase1_base_lr(1000 + 1e-9) == pytest.approx(5e-3)
    assert 5e-4 < S.phase1_base_lr(10 ** 9) < 5.2e-4


def test_wsd_matches_the_workload_schedule():
    import synth
    lrs = [S.wsd_lr(k, 20, 0.012, 2, 8 / 20) for k in range(20)]
    assert lrs == pytest.approx(synth.wsd_lr())


def test_production_schedule_is_continuous_and_decaying():
    """Eq. (10) hands over to Eq. (11) at the Phase-1 endpoint with no jump
    beyond the report's rounding of eta0 (1.04e-3), both decay afterwards,
    and the CMA continuation holds its constant."""
    k1 = S.PHASE1_TOKENS / S.TOKENS_PER_STEP
    before = S.production_base_lr(int(k1), cma_from=None)
    after = S.production_base_lr(int(k1) + 1, cma_from=None)
    assert abs(after - before) <= 0.005 * before
    ks = list(range(1001, 300000, 997))
    lrs = [S.production_base_lr(k, cma_from=None) for k in ks]
    assert all(b <= a + 1e-15 for a, b in zip(lrs, lrs[1:]))
    assert all(S.production_base_lr(k) == S.CMA_BASE_LR for k in (218000, 250000, 400000))


def test_hyperball_lr_scales_the_base_lr():
    """Sec. 3.3.1: the Hyperball LR is m times the base LR (m = 10 in production)."""
    assert S.hyperball_lr(1e-3) == pytest.approx(1e-2)
    assert S.hyperball_lr(1e-3, m=2) == pytest.approx(2e-3)
