"""Learning-rate schedules of the Puro-2B recipe (host side).

The MuonH step takes each matrix's effective LR eta^H directly; these helpers
produce it.  Sources (Puro-2B report, arXiv HTML):
  * App. C, Eq. (10): Phase-1 base LR, 1,000 warm-up steps then an
    inverse-square-root power decay with an asymptotic floor of 5e-4.
  * App. C, Eq. (11): Phase-2 base LR, linear in the Phase-2 samples s from
    eta0 ~= 1.04e-3 to eta_min = 1e-5 over a sample budget S.
  * Sec. 3.3.1: eta^H = m eta^base with m = 10 in production (m = 2 in the
    App. D ladder, m = 3 in the App. F WSD sweeps).
  * Sec. 3.3.2: warmup-stable-decay with a linear decay, as in the sweeps.
  * Sec. 3.4: the CMA continuation holds the base LR at its step-218,000
    value, 4.08e-5 (eta^H = 4.08e-4).
  * Sec. 3.5: supervised fine-tuning uses a cosine decay of the base LR from
    1e-5 to 1e-7.
"""
from __future__ import annotations

import math

TOKENS_PER_STEP = 1536 * 4096          # global batch 1,536 sequences of 4,096 tokens (App. C)
SAMPLES_PER_STEP = 1536
PHASE1_TOKENS = 438.84e9               # Table 7
PHASE2_HORIZONS_TOKENS = (60.1e9, 120.1e9, 240.2e9, 480.5e9, 960.9e9)   # App. C, Fig. 13(a)
CMA_BASE_LR = 4.08e-5                  # Sec. 3.4
PRODUCTION_MULTIPLIER = 10.0           # Sec. 3.3.1


def phase1_base_lr(k: float) -> float:
    """Eq. (10): 5e-3 k/1000 for 0 <= k <= 1000, else
    5e-4 + 4.5e-3 (1 + (k - 1000)/1000)^(-1/2)."""
    if k < 0:
        raise ValueError("step must be >= 0")
    if k <= 1000:
        return 5e-3 * k / 1000.0
    return 5e-4 + 4.5e-3 * (1.0 + (k - 1000.0) / 1000.0) ** -0.5


def phase2_base_lr(s: float, S: float, eta0: float = 1.04e-3, eta_min: float = 1e-5) -> float:
    """Eq. (11): eta0 + (eta_min - eta0) s / S for 0 <= s <= S (s, S in samples)."""
    if not 0 <= s <= S:
        raise ValueError("need 0 <= s <= S")
    return eta0 + (eta_min - eta0) * s / S


def hyperball_lr(base_lr: float, m: float = PRODUCTION_MULTIPLIER) -> float:
    """Sec. 3.3.1: the Hyperball weight LR (= the effective LR of a MuonH
    matrix) is m times the base LR."""
    return m * base_lr


def wsd_lr(k: int, total: int, peak: float, warmup: int, decay_ratio: float) -> float:
    """Warmup-stable-decay, 0-based step k of `total`: linear warm-up
    peak (k+1)/warmup, constant `peak`, then over the last decay_ratio*total
    steps a linear decay peak (total-1-k)/decay that reaches 0 on the last step."""
    decay = int(round(decay_ratio * total))
    if k < warmup:
        return peak * (k + 1) / warmup
    start = total - decay
    if k < start:
        return peak
    return peak * max(0.0, (total - 1 - k) / decay) if decay > 0 else 0.0


def cosine_lr(k: int, total: int, lr_max: float = 1e-5, lr_min: float = 1e-7) -> float:
    """Sec. 3.5: cosine decay from lr_max to lr_min over `total` steps."""
    t = min(max(k, 0), total) / total
    return lr_min + 0.5 * (lr_max - lr_min) * (1.0 + math.cos(math.pi * t))


def production_base_lr(step: int, phase2_horizon_tokens: float = PHASE2_HORIZONS_TOKENS[-1],
                       cma_from: int | None = 218_000) -> float:
    """Base LR of the production run at a global optimizer step: Eq. (10)
    through Phase 1, Eq. (11) from the Phase-1 endpoint, and the CMA
    constant from step `cma_from` on (None: no continuation)."""
    k1 = PHASE1_TOKENS / TOKENS_PER_STEP
    if cma_from is not None and step >= cma_from:
        return CMA_BASE_LR
    if step <= k1:
        return phase1_base_lr(step)
    S = phase2_horizon_tokens / 4096.0
    s = min((step - k1) * SAMPLES_PER_STEP, S)
    return phase2_base_lr(s, S)
