"""CPU oracle for the MuonH optimizer step -- TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously correct NumPy restatement (fp64 by default) of one
MuonH step, written from the Puro-2B report (arXiv HTML, Sec. 3.3 "Hyperball
Optimization", Eq. (1) and Eqs. (3)-(5); reading notes Sec. 2.5).  It shares
no code with the CUDA path and imports nothing from it.  Only tests/,
__graft_entry__.smoke() and the CPU-baseline leg of bench.py may import it;
the product path never calls it.

Pins (tests/test_oracle.py, run with -m "not gpu") tie every function to
something other than itself: the singular-value form of the Newton-Schulz
polynomial checked with a library SVD, convergence to the polar factor with
a convergent coefficient set, the closed-form hyperball invariants
(||W_{t+1}||_F = R, effective LR = lr), hand-solved two-element examples
and hand-solved radii R = ||W_0||_F, and the geometric-sum form of the
momentum buffer, also carried across the steps of run_steps.  oracle.aux (checkpoint
averaging, AdamW) and oracle.emulate (16-bit storage emulation of the
iteration) are pinned in tests/test_oracle_aux.py and tests/test_oracle.py.
"""
from .muonh import (  # noqa: F401
    QUINTIC, FLAG_NONFINITE_INPUT, FLAG_ZERO_UPDATE, FLAG_NONFINITE_UPDATE,
    FLAG_DEGENERATE, RULE_HYPERBALL, RULE_DECOUPLED_WD, RULE_ELR_ALIGNED,
    momentum_update, newton_schulz, hyperball_update, muon_update,
    radius, muonh_step, run_steps,
)
