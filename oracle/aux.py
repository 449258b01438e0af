"""Oracle restatements of the two auxiliary operations (test infrastructure only).

* Checkpoint averaging (Puro-2B report, Sec. 3.4 and the CMA paragraph of
  the reading notes Sec. 2.7): the released parameters are the equal
  average of six checkpoints, theta_bar = (1/k) sum_i theta_i, parameters
  only (no optimizer state).
* AdamW for the parameter group outside MuonH (Table 8: embeddings,
  normalisation layers, LM head and other parameters, weight decay 0.1, the
  base LR; Adam betas (0.9, 0.95) in App. E).  The pages use AdamW without
  restating it; this is its standard definition with decoupled weight decay
  and bias-corrected moments:
      p <- p (1 - lr wd);  m <- b1 m + (1-b1) g;  v <- b2 v + (1-b2) g^2
      p <- p - lr (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps)
"""
from __future__ import annotations

import numpy as np


def checkpoint_average(thetas, dtype=np.float64):
    """(1/k) sum_i theta_i in `dtype`."""
    acc = np.zeros_like(np.asarray(thetas[0], dtype=dtype))
    for t in thetas:
        acc = acc + np.asarray(t, dtype=dtype)
    return acc / len(thetas)


def adamw_step(p, m, v, g, t, lr, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, dtype=np.float64):
    """One AdamW step at 1-based step t.  Returns (p, m, v)."""
    p = np.asarray(p, dtype=dtype) * (1.0 - lr * weight_decay)
    g = np.asarray(g, dtype=dtype)
    m = beta1 * np.asarray(m, dtype=dtype) + (1.0 - beta1) * g
    v = beta2 * np.asarray(v, dtype=dtype) + (1.0 - beta2) * g * g
    m_hat = m / (1.0 - beta1 ** t)
    v_hat = v / (1.0 - beta2 ** t)
    p = p - lr * m_hat / (np.sqrt(v_hat) + eps)
    return p, m, v
