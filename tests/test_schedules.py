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
