"""The oracle pins must catch plausible mistakes: each case below plants one
in a copy of the oracle (on the CPU, never in the CUDA path) and expects the
pin tests to fail against it."""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = {
    "dropped A^2 term": ("B = b * A + c * (A @ A)", "B = b * A"),
    "b and c swapped": ("B = b * A + c * (A @ A)", "B = c * A + b * (A @ A)"),
    "O not normalised": ("displacement = (lr * R / o_norm) * O", "displacement = (lr * R) * O"),
    "wrong sign of B Y": ("Y = a * Y + B @ Y", "Y = a * Y - B @ Y"),
    "scaled Gram": ("A = Y @ Y.T", "A = 1.0001 * (Y @ Y.T)"),
    "transposed Gram (Y^T Y on square inputs)": ("A = Y @ Y.T", "A = Y.T @ Y if Y.shape[0] == Y.shape[1] else Y @ Y.T"),
    "product order B Y -> Y B (square inputs)": ("Y = a * Y + B @ Y",
                                                 "Y = a * Y + (Y @ B if Y.shape[0] == Y.shape[1] else B @ Y)"),
    "||W|| used for R": ("displacement = (lr * R / o_norm) * O", "displacement = (lr * w_norm / o_norm) * O"),
    "projection onto ||W||": ("W_new = (R / wt_norm) * W_tilde", "W_new = (R / w_norm) * W_tilde"),
    "lerp momentum": ("M_new = beta * M + G", "M_new = beta * M + (1 - beta) * G"),
    "stale Nesterov term": ("X = G + beta * M_new if nesterov", "X = G + beta * M if nesterov"),
    "max-norm input scaling": ("Y = Y / (np.linalg.norm(Y) + eps)", "Y = Y / (np.abs(Y).max() + eps)"),
    "ELR over R": ("elr = float(np.linalg.norm(displacement)) / w_norm",
                   "elr = float(np.linalg.norm(displacement)) / R"),
    "Eq. (5) without the update scale": ("else lr * w_norm / u_norm", "else lr * w_norm / o_norm"),
    "Eq. (3) without weight decay": ("W_new = (1.0 - weight_decay * eta) * W - eta * u", "W_new = W - eta * u"),
    "spectral norm for R": ("return float(np.linalg.norm(np.asarray(W0, dtype=dtype)))",
                            "return float(np.linalg.norm(np.asarray(W0, dtype=dtype), 2))"),
    "squared norm for R": ("return float(np.linalg.norm(np.asarray(W0, dtype=dtype)))",
                           "return float(np.linalg.norm(np.asarray(W0, dtype=dtype)) ** 2)"),
    "momentum reset every step in run_steps": ("W[i], M[i], O, st = muonh_step(W[i], M[i], grad_fn(t, i)",
                                               "W[i], M[i], O, st = muonh_step(W[i], 0 * M[i], grad_fn(t, i)"),
}

# mistakes in the auxiliary oracles: (file, pin tests, old, new)
AUX_MUTATIONS = {
    "AdamW without bias correction": ("aux.py", "tests/test_oracle_aux.py",
                                      "m_hat = m / (1.0 - beta1 ** t)", "m_hat = m"),
    "AdamW without weight decay": ("aux.py", "tests/test_oracle_aux.py",
                                   "p = np.asarray(p, dtype=dtype) * (1.0 - lr * weight_decay)",
                                   "p = np.asarray(p, dtype=dtype)"),
    "average over k - 1": ("aux.py", "tests/test_oracle_aux.py",
                           "return acc / len(thetas)", "return acc / max(1, len(thetas) - 1)"),
    "bf16 rounding by truncation": ("emulate.py", "tests/test_oracle.py",
                                    "u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000", "u = u & 0xFFFF0000"),
    "Gram update with one factor of p(A)": ("emulate.py", "tests/test_oracle.py",
                                            "A = sym(sym(A @ Bp) @ Bp)", "A = sym(A @ Bp)"),
    "Q kept from the last iteration only": ("emulate.py", "tests/test_oracle.py",
                                            "Q = Bp if Q is None else sym(Bp @ Q)", "Q = Bp"),
    "diagonal rounded anyway": ("emulate.py", "tests/test_oracle.py",
                                "    np.fill_diagonal(out, np.diag(np.asarray(B, dtype=np.float64)))\n", ""),
    "lower tiles left unwritten": ("emulate.py", "tests/test_oracle.py",
                                   "out[i:i + tile, j:j + tile] = out[j:j + tile, i:i + tile].T",
                                   "out[i:i + tile, j:j + tile] = 0.0"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTATIONS[name]
    for d in ("oracle", "synth", "tests"):
        shutil.copytree(os.path.join(ROOT, d), tmp_path / d, ignore=shutil.ignore_patterns("__pycache__"))
    shutil.copy(os.path.join(ROOT, "pytest.ini"), tmp_path / "pytest.ini")
    src = tmp_path / "oracle" / "muonh.py"
    text = src.read_text()
    assert old in text, "the oracle changed: update this mutation"
    src.write_text(text.replace(old, new))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "tests/test_oracle.py", "-m", "not gpu",
                        "-p", "no:cacheprovider"], cwd=tmp_path, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0, f"pins did not catch: {name}"


@pytest.mark.parametrize("name", sorted(AUX_MUTATIONS))
def test_aux_pins_catch_planted_mistake(name, tmp_path):
    fname, tests, old, new = AUX_MUTATIONS[name]
    for d in ("oracle", "synth", "tests", "pretraining_optimizer_b200"):
        shutil.copytree(os.path.join(ROOT, d), tmp_path / d,
                        ignore=shutil.ignore_patterns("__pycache__", "*.so", "csrc"))
    shutil.copy(os.path.join(ROOT, "pytest.ini"), tmp_path / "pytest.ini")
    src = tmp_path / "oracle" / fname
    text = src.read_text()
    assert old in text, "the oracle changed: update this mutation"
    src.write_text(text.replace(old, new))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", tests, "-m", "not gpu",
                        "-p", "no:cacheprovider"], cwd=tmp_path, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0, f"pins did not catch: {name}"


@pytest.mark.parametrize("tests", ["tests/test_oracle.py", "tests/test_oracle_aux.py"])
def test_harness_passes_without_a_mistake(tests, tmp_path):
    """Control: the copied tree passes its pins when nothing is planted, so a
    failure above comes from the planted mistake, not from the copy."""
    for d in ("oracle", "synth", "tests", "pretraining_optimizer_b200"):
        shutil.copytree(os.path.join(ROOT, d), tmp_path / d,
                        ignore=shutil.ignore_patterns("__pycache__", "*.so", "csrc"))
    shutil.copy(os.path.join(ROOT, "pytest.ini"), tmp_path / "pytest.ini")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", tests, "-m", "not gpu",
                        "-p", "no:cacheprovider"], cwd=tmp_path, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout[-2000:]
