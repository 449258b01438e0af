"""Seeded synthetic inputs for the MuonH optimizer step.

This package is the only code shared by the CUDA path's tests and benchmark
and by the CPU oracle.  It holds no optimizer arithmetic: it only names the
matrix-shape sets, draws the initial weights and the gradients from seeded
generators, and lists the per-step learning rates of each workload.

Shapes follow the Qwen3 architecture table of the Puro-2B report
(Appendix D, Table 10: d_model, d_ff, 16 query heads, 8 KV heads,
head dimension 128, 28 layers).  Every weight is stored PyTorch-style as
[out_features, in_features], row-major, fp32.

Seeds: stream (0, i) draws W0 of matrix i, stream (1, t, i) draws the
gradient of matrix i at step t (0-based).  NumPy's SeedSequence/PCG64 is
used, so the bytes are identical on every machine.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

W0_STD = 0.02
GRAD_STD = 1e-3
SEED_W0 = 0
SEED_GRAD = 1

_PROJ_ORDER = ("q_proj", "k_proj", "v_proj", "o_proj", "gate_proj", "up_proj", "down_proj")


@dataclass(frozen=True)
class MatrixSpec:
    name: str
    rows: int
    cols: int

    @property
    def size(self) -> int:
        return self.rows * self.cols


def qwen3_layer_shapes(d_model: int, d_ff: int, n_q: int = 16, n_kv: int = 8,
                       d_head: int = 128) -> list[tuple[str, int, int]]:
    """The seven hidden matrices of one Qwen3 decoder layer, [out, in]."""
    q = n_q * d_head
    kv = n_kv * d_head
    return [
        ("q_proj", q, d_model),
        ("k_proj", kv, d_model),
        ("v_proj", kv, d_model),
        ("o_proj", d_model, q),
        ("gate_proj", d_ff, d_model),
        ("up_proj", d_ff, d_model),
        ("down_proj", d_model, d_ff),
    ]


def qwen3_matrix_set(d_model: int, d_ff: int, layers: int = 28) -> list[MatrixSpec]:
    out = []
    for layer in range(layers):
        for name, r, c in qwen3_layer_shapes(d_model, d_ff):
            out.append(MatrixSpec(f"layers.{layer}.{name}", r, c))
    return out


def qwen3_0p6b() -> list[MatrixSpec]:
    """Qwen3-0.6B hidden-matrix set: 196 matrices, 440,401,920 parameters."""
    return qwen3_matrix_set(1024, 3072)


def qwen3_1p7b() -> list[MatrixSpec]:
    """Qwen3-1.7B hidden-matrix set (embedding/LM head excluded):
    196 matrices, 1,409,286,144 parameters."""
    return qwen3_matrix_set(2048, 6144)


QWEN3_VOCAB = 151936


def qwen3_adamw_group(d_model: int, layers: int = 28, vocab: int = QWEN3_VOCAB,
                      d_head: int = 128) -> list[tuple[str, int]]:
    """The parameters outside the matrix set, which AdamW trains: the input
    embedding and the (untied) LM head, vocab x d_model each; per layer the
    two RMSNorm weights (d_model) and the q/k norms (d_head); the final norm.
    For Qwen3-1.7B with untied head: 622,453,760 elements, which with the
    matrix set makes the ~2.03e9 parameters of the model."""
    out = [("embed_tokens", vocab * d_model), ("lm_head", vocab * d_model)]
    for layer in range(layers):
        out += [(f"layers.{layer}.input_layernorm", d_model), (f"layers.{layer}.post_attention_layernorm", d_model),
                (f"layers.{layer}.q_norm", d_head), (f"layers.{layer}.k_norm", d_head)]
    out.append(("norm", d_model))
    return out


def single_256x512() -> list[MatrixSpec]:
    return [MatrixSpec("w", 256, 512)]


SWEEP_SHAPES = [(512, 512), (1024, 4096), (2048, 2048), (4096, 4096),
                (8192, 2048), (2048, 8192), (8192, 8192)]


def sweep_set(rows: int, cols: int, batch: int) -> list[MatrixSpec]:
    return [MatrixSpec(f"sweep.{rows}x{cols}.{i}", rows, cols) for i in range(batch)]


def sweep_batch_size(rows: int, cols: int, bytes_per_elem: int = 4,
                     min_bytes: int = 1 << 30) -> int:
    """Smallest batch whose weights hold at least `min_bytes`."""
    return max(1, math.ceil(min_bytes / (rows * cols * bytes_per_elem)))


# ---------------------------------------------------------------- generators

def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def initial_weight(i: int, rows: int, cols: int, std: float = W0_STD) -> np.ndarray:
    """W0 of matrix i: i.i.d. N(0, std^2), fp32."""
    w = _rng(SEED_W0, i).standard_normal((rows, cols), dtype=np.float32)
    w *= np.float32(std)
    return w


def gaussian_gradient(step: int, i: int, rows: int, cols: int,
                      std: float = GRAD_STD) -> np.ndarray:
    """Gradient of matrix i at step `step`: i.i.d. N(0, std^2), fp32."""
    g = _rng(SEED_GRAD, step, i).standard_normal((rows, cols), dtype=np.float32)
    g *= np.float32(std)
    return g


def ill_conditioned_gradient(step: int, i: int, rows: int, cols: int,
                             rank: int = 8, frob: float = 0.1,
                             noise_std: float = 1e-5, heavy_every: int = 10,
                             heavy_scale: float = 1e-3, nu: float = 3.0) -> np.ndarray:
    """Rank-`rank` product A B^T (A, B ~ N(0,1)) scaled to Frobenius norm
    `frob`, plus i.i.d. N(0, noise_std^2) noise.  On every `heavy_every`-th
    step (0-based step % heavy_every == heavy_every - 1) the noise is replaced
    by heavy_scale * Student-t(nu) entries."""
    rng = _rng(SEED_GRAD, step, i)
    a = rng.standard_normal((rows, rank))
    b = rng.standard_normal((cols, rank))
    lowrank = a @ b.T
    lowrank *= frob / np.linalg.norm(lowrank)
    if step % heavy_every == heavy_every - 1:
        noise = heavy_scale * rng.standard_t(nu, size=(rows, cols))
    else:
        noise = noise_std * rng.standard_normal((rows, cols))
    return (lowrank + noise).astype(np.float32)


# ------------------------------------------------------ learning-rate inputs

def constant_lr(steps: int, lr: float = 0.01) -> list[float]:
    return [lr] * steps


def wsd_lr(peak: float = 0.012, warmup: int = 2, stable: int = 10, decay: int = 8) -> list[float]:
    """Warmup-stable-decay with linear warmup and linear decay to 0.

    0-based step k: warmup peak*(k+1)/warmup, then `stable` steps at peak,
    then peak*(warmup+stable+decay-1-k)/decay, ending at 0."""
    out = []
    for k in range(warmup):
        out.append(peak * (k + 1) / warmup)
    out += [peak] * stable
    last = warmup + stable + decay - 1
    for k in range(warmup + stable, warmup + stable + decay):
        out.append(peak * (last - k) / decay)
    return out


def linear_decay_lr(steps: int, peak: float = 0.008) -> list[float]:
    """peak * (1 - k/steps), k = 0..steps-1."""
    return [peak * (1.0 - k / steps) for k in range(steps)]


# ------------------------------------------------------------ named workloads

@dataclass(frozen=True)
class Workload:
    name: str
    matrices: list
    lrs: list
    gradient: str = "gaussian"       # or "ill_conditioned"
    beta: float = 0.95
    nesterov: bool = True
    ns_steps: int = 5
    ns_coeffs: tuple = (3.4445, -4.7750, 2.0315)

    def grad(self, step: int, i: int) -> np.ndarray:
        m = self.matrices[i]
        if self.gradient == "ill_conditioned":
            return ill_conditioned_gradient(step, i, m.rows, m.cols)
        return gaussian_gradient(step, i, m.rows, m.cols)

    def weight(self, i: int) -> np.ndarray:
        m = self.matrices[i]
        return initial_weight(i, m.rows, m.cols)


def workload(name: str) -> Workload:
    """Named workloads; "<set>:L" keeps the first L layers of a Qwen3 set;
    "sweep_<rows>x<cols>" is one shape of the roofline sweep, batched to at
    least 1 GiB of fp32 weights, at a constant lr of 0.01."""
    if ":" in name:
        base, layers = name.split(":")
        wl = workload(base)
        keep = 7 * int(layers)
        return Workload(name, wl.matrices[:keep], wl.lrs, wl.gradient, wl.beta, wl.nesterov,
                        wl.ns_steps, wl.ns_coeffs)
    if name == "single_256x512":
        return Workload(name, single_256x512(), constant_lr(10, 0.01))
    if name == "qwen3_0.6b":
        return Workload(name, qwen3_0p6b(), wsd_lr())
    if name == "qwen3_1.7b":
        return Workload(name, qwen3_1p7b(), linear_decay_lr(50))
    if name == "qwen3_1.7b_illcond":
        return Workload(name, qwen3_1p7b(), linear_decay_lr(100), gradient="ill_conditioned")
    if name.startswith("sweep_"):
        rows, cols = parse_sweep_name(name)
        return Workload(name, sweep_set(rows, cols, sweep_batch_size(rows, cols)), constant_lr(10, 0.01))
    raise KeyError(name)


def parse_sweep_name(name: str) -> tuple[int, int]:
    """"sweep_<rows>x<cols>" -> (rows, cols), for a shape of SWEEP_SHAPES."""
    try:
        rows, cols = (int(v) for v in name[len("sweep_"):].split("x"))
    except ValueError:
        raise KeyError(name) from None
    if (rows, cols) not in SWEEP_SHAPES:
        raise KeyError(name)
    return rows, cols
