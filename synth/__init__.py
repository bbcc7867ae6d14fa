"""Seeded synthetic inputs for the AutoRound tuning path and the W4A16 kernels.

This module only draws random numbers and stores them; it holds none of the
quantization arithmetic.  Both the CPU oracle (``oracle/``) and the CUDA path
(``post_weight_quantization_autoround_b200``) take their inputs from here, so
the two sides always see the same bytes.

Distributions follow the workloads the AutoRound pages and the build's
configuration list describe: Llama-shaped linear layers with weights
~N(0, 0.02) in which 0.1 % of the entries are scaled by 20 (outliers), and
calibration activations ~N(0, 1) in which 8 input channels are scaled by 50
(activation outlier channels).  Trained weights and calibration text are not
available, so these stand in for them.

Every tensor draws from its own child stream of one ``numpy.random.SeedSequence``
(PCG64), in a fixed order, so adding a tensor never changes the others.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np

__all__ = [
    "to_bf16_bits",
    "bf16_bits_to_f32",
    "make_linear",
    "make_mlp",
    "make_decoder",
    "make_activations",
    "Workload",
    "WORKLOADS",
]

# Fixed child-stream slots of the SeedSequence.  Never reorder.
_S_W, _S_W_OUT, _S_X, _S_X_OUT, _S_ACT, _S_MLP_G, _S_MLP_U, _S_MLP_D, _S_STATE = range(9)
_N_STREAMS = 12


def _streams(seed: int):
    return [np.random.Generator(np.random.PCG64(s)) for s in np.random.SeedSequence(seed).spawn(_N_STREAMS)]


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Store float32 values as bfloat16 bit patterns (round to nearest, ties to even).

    Storage step of the generator: the workloads are specified as bf16 tensors.
    Inputs here are always finite.
    """
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    return ((b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def _weights(rng_v, rng_o, n_out: int, n_in: int, std: float, outlier_frac: float, outlier_scale: float):
    w = _normal(rng_v, (n_out, n_in), std)
    count = int(round(outlier_frac * n_out * n_in))
    if count > 0:
        idx = rng_o.choice(n_out * n_in, size=count, replace=False)
        w.reshape(-1)[idx] *= np.float32(outlier_scale)
    return w


def _acts(rng_v, rng_o, m: int, k: int, outlier_channels: int, outlier_scale: float):
    x = _normal(rng_v, (m, k), 1.0)
    if outlier_channels > 0:
        ch = rng_o.choice(k, size=min(outlier_channels, k), replace=False)
        x[:, ch] *= np.float32(outlier_scale)
    return x


def make_linear(
    n_out: int,
    n_in: int,
    m_tokens: int,
    *,
    seed: int = 0,
    dtype: str = "bf16",
    w_std: float = 0.02,
    outlier_frac: float = 0.001,
    outlier_scale: float = 20.0,
    x_outlier_channels: int = 8,
    x_outlier_scale: float = 50.0,
) -> Dict[str, np.ndarray]:
    """One linear layer ``Y = X W^T``: weights ``W [n_out][n_in]`` and activations ``X [m_tokens][n_in]``.

    ``dtype="bf16"`` returns uint16 bf16 bit patterns; ``dtype="f32"`` returns float32.
    """
    r = _streams(seed)
    w = _weights(r[_S_W], r[_S_W_OUT], n_out, n_in, w_std, outlier_frac, outlier_scale)
    x = _acts(r[_S_X], r[_S_X_OUT], m_tokens, n_in, x_outlier_channels, x_outlier_scale)
    if dtype == "bf16":
        return {"W": to_bf16_bits(w), "X": to_bf16_bits(x)}
    if dtype == "f32":
        return {"W": w, "X": x}
    raise ValueError(f"unknown dtype {dtype!r}")


def make_mlp(
    hidden: int,
    inter: int,
    m_tokens: int,
    *,
    seed: int = 0,
    w_std: float = 0.02,
    outlier_frac: float = 0.001,
    outlier_scale: float = 20.0,
    x_outlier_channels: int = 8,
    x_outlier_scale: float = 50.0,
) -> Dict[str, np.ndarray]:
    """SwiGLU MLP block: gate/up ``[inter][hidden]``, down ``[hidden][inter]``, input ``X [m_tokens][hidden]`` (bf16 bits)."""
    r = _streams(seed)
    wg = _weights(r[_S_MLP_G], r[_S_W_OUT], inter, hidden, w_std, outlier_frac, outlier_scale)
    wu = _weights(r[_S_MLP_U], r[_S_W_OUT], inter, hidden, w_std, outlier_frac, outlier_scale)
    wd = _weights(r[_S_MLP_D], r[_S_W_OUT], hidden, inter, w_std, outlier_frac, outlier_scale)
    x = _acts(r[_S_X], r[_S_X_OUT], m_tokens, hidden, x_outlier_channels, x_outlier_scale)
    return {"Wg": to_bf16_bits(wg), "Wu": to_bf16_bits(wu), "Wd": to_bf16_bits(wd), "X": to_bf16_bits(x)}


def make_decoder(
    hidden: int,
    inter: int,
    m_tokens: int,
    *,
    seed: int = 0,
    w_std: float = 0.02,
    outlier_frac: float = 0.001,
    outlier_scale: float = 20.0,
    x_outlier_channels: int = 8,
    x_outlier_scale: float = 50.0,
    gamma_std: float = 0.1,
) -> Dict[str, np.ndarray]:
    """Decoder block: q, k, v, o ``[hidden][hidden]``, gate/up ``[inter][hidden]``, down ``[hidden][inter]``
    (bf16 bits, the linear layers' distribution), input ``X [m_tokens][hidden]`` (bf16 bits) and the two
    norm scales ``gamma1, gamma2 [hidden]`` ~ 1 + N(0, gamma_std), float32 values that bf16 holds exactly."""
    root = np.random.SeedSequence(seed).spawn(17)  # 0-13: the seven weights, 14: gammas, 15-16: X
    rng = lambda i: np.random.Generator(np.random.PCG64(root[i]))
    shapes = {"q": (hidden, hidden), "k": (hidden, hidden), "v": (hidden, hidden), "o": (hidden, hidden),
              "gate": (inter, hidden), "up": (inter, hidden), "down": (hidden, inter)}
    out = {}
    for i, (name, (n, k)) in enumerate(shapes.items()):
        out[name] = to_bf16_bits(_weights(rng(2 * i), rng(2 * i + 1), n, k, w_std, outlier_frac, outlier_scale))
    out["X"] = to_bf16_bits(_acts(rng(15), rng(16), m_tokens, hidden, x_outlier_channels, x_outlier_scale))
    g = rng(14)
    for name in ("gamma1", "gamma2"):
        out[name] = bf16_bits_to_f32(to_bf16_bits(1.0 + _normal(g, (hidden,), gamma_std)))
    return out


def make_activations(t: int, k: int, *, seed: int = 0) -> np.ndarray:
    """Decode-shaped activations ``A [t][k]`` ~N(0, 1) as bf16 bits (W4A16 inputs)."""
    r = _streams(seed)
    return to_bf16_bits(_normal(r[_S_ACT], (t, k), 1.0))


def make_state(n_out: int, n_in: int, group_size: int, *, seed: int = 0, spread: bool = False):
    """Tuning state ``V [n][k]``, ``alpha``, ``beta [n][k/g]``.

    ``spread=False`` is the method's initial state (V = 0, alpha = beta = 1).
    ``spread=True`` draws V ~ U[-0.5, 0.5] and alpha, beta ~ U[0.5, 1] so that
    parity cases exercise every branch of the quantizer, not only the start.
    """
    g = n_in // group_size
    if not spread:
        return (np.zeros((n_out, n_in), np.float32), np.ones((n_out, g), np.float32), np.ones((n_out, g), np.float32))
    r = _streams(seed)[_S_STATE]
    v = r.uniform(-0.5, 0.5, size=(n_out, n_in)).astype(np.float32)
    a = r.uniform(0.5, 1.0, size=(n_out, g)).astype(np.float32)
    b = r.uniform(0.5, 1.0, size=(n_out, g)).astype(np.float32)
    return v, a, b


@dataclasses.dataclass(frozen=True)
class Workload:
    """A named workload: shapes, quantizer settings and schedule."""

    name: str
    kind: str  # "linear" or "mlp"
    n_out: int
    n_in: int
    m_tokens: int
    bits: int = 4
    group_size: int = 128
    steps: int = 200
    lr: float = 0.005
    dtype: str = "bf16"
    x_outlier_channels: int = 8
    inter: Optional[int] = None
    seed: int = 0


WORKLOADS: Dict[str, Workload] = {
    # 256x256 fp32 layer, 32 fp32 tokens, 10 steps: small enough for the oracle in seconds.
    "linear_256": Workload("linear_256", "linear", 256, 256, 32, steps=10, dtype="f32", x_outlier_channels=0),
    # Llama-7B-shaped 4096x4096 projection, 8 samples x 2048 tokens.
    "linear_4096": Workload("linear_4096", "linear", 4096, 4096, 16384),
    # Llama-7B SwiGLU MLP block, tuned jointly.
    "mlp_4096_11008": Workload("mlp_4096_11008", "mlp", 4096, 4096, 16384, inter=11008),
    # Low-bit stress: 4096x4096, 2048 tokens.
    "lowbit_b3g32": Workload("lowbit_b3g32", "linear", 4096, 4096, 2048, bits=3, group_size=32, steps=500),
    "lowbit_b2g32": Workload("lowbit_b2g32", "linear", 4096, 4096, 2048, bits=2, group_size=32, steps=500),
    "lowbit_b8g256": Workload("lowbit_b8g256", "linear", 4096, 4096, 2048, bits=8, group_size=256, steps=500, lr=0.002),
    # Llama-70B-shaped down projection 8192x28672.
    "down_8192_28672": Workload("down_8192_28672", "linear", 8192, 28672, 16384),
}


def make_schedule(n_samples: int, batch: int, steps: int, seed: int = 0) -> np.ndarray:
    """Calibration samples each tuning step draws: int32 [steps][batch], ``batch``
    distinct indices in [0, n_samples) per step, uniformly at random (PCG64,
    seeded).  The draws are data: the GPU driver and the oracle take the same
    array."""
    if not (0 < batch <= n_samples):
        raise ValueError("need 0 < batch <= n_samples")
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 0x5A3D])))
    return np.stack([rng.choice(n_samples, size=batch, replace=False) for _ in range(steps)]).astype(np.int32)

