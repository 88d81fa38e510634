"""Seeded synthetic workloads for the W4A4 linear layer.

This module only draws random numbers and rounds them to bf16: it holds none of the
layer's arithmetic, so tests can feed the very same bytes to the CUDA path and to
the CPU oracle.

Recipe (one numpy PCG64 stream per tensor, spawned from SeedSequence(seed) in the
order x, W, s, outlier channels; fp32 draws rounded to bf16 with round-to-nearest-
even):

* x ~ N(0, 1) or Student-t(3); outlier channels multiplied in fp32 before the cast.
* W ~ N(0, sigma_w).
* s ~ exp(N(0, 0.5^2)), kept in fp32.

The shapes are those of real models (Llama-3-8B, Qwen3-32B) used as shapes only; no
weights or text are involved.
"""
from dataclasses import dataclass, replace
from typing import List, Optional, Tuple

import numpy as np


@dataclass(frozen=True)
class Linear:
    """One linear layer y[M, N] = x[M, K] W[N, K]^T and its input model."""
    name: str
    M: int
    N: int
    K: int
    x_dist: str = "normal"            # "normal" (N(0,1)) or "t3" (Student-t, nu=3)
    outlier_channels: Tuple[int, ...] = ()   # explicit channel indices
    outlier_frac: float = 0.0         # or a fraction of K drawn without replacement
    outlier_factor: float = 1.0
    w_std: float = 0.02
    s_sigma: float = 0.5
    seed: int = 0
    out_dtype: str = "bf16"           # "f32" or "bf16"


# The outlier model of the tiny layer: N(0, 1) with channels 3 and 77 times 50.
_TINY_X = dict(x_dist="normal", outlier_channels=(3, 77), outlier_factor=50.0)


def tiny_layer() -> Linear:
    """16x256 activations, 128x256 weight, fp32 output, seed 0."""
    return Linear("tiny_16x128x256", 16, 128, 256, w_std=0.02, out_dtype="f32", **_TINY_X)


def llama3_8b_gate_up_prefill() -> Linear:
    """Llama-3-8B gate/up projection, 4096-token prefill."""
    return Linear("llama3_8b_gate_up_prefill_4096x14336x4096", 4096, 14336, 4096,
                  x_dist="t3", outlier_frac=0.005, outlier_factor=20.0, w_std=0.02)


def qwen3_32b_up_decode(batch: int = 1) -> Linear:
    """Qwen3-32B MLP up projection at decode (weight-bandwidth bound)."""
    return Linear(f"qwen3_32b_up_decode_{batch}x25600x5120", batch, 25600, 5120,
                  w_std=0.02, **_TINY_X)


def qwen3_32b_up_decode_t3(batch: int = 1) -> Linear:
    """The same decode layer with the Llama prefill outlier model (labelled variant)."""
    return Linear(f"qwen3_32b_up_decode_t3_{batch}x25600x5120", batch, 25600, 5120,
                  x_dist="t3", outlier_frac=0.005, outlier_factor=20.0, w_std=0.02)


def qwen3_32b_down_prefill() -> Linear:
    """Qwen3-32B down projection, 8192-token prefill, K = 25600."""
    return Linear("qwen3_32b_down_prefill_8192x5120x25600", 8192, 5120, 25600,
                  x_dist="t3", outlier_frac=0.01, outlier_factor=30.0, w_std=0.01)


def qwen3_32b_layer_decode(batch: int = 256) -> List[Linear]:
    """All seven linears of one Qwen3-32B decoder layer at `batch` rows. Each has its
    own seed (hence its own s); the activations follow the tiny layer's outlier
    model."""
    shapes = [("q_proj", 8192, 5120), ("k_proj", 1024, 5120), ("v_proj", 1024, 5120),
              ("o_proj", 5120, 8192), ("gate_proj", 25600, 5120), ("up_proj", 25600, 5120),
              ("down_proj", 5120, 25600)]
    return [Linear(f"qwen3_32b_{n}_b{batch}", batch, N, K, w_std=0.02, seed=i, **_TINY_X)
            for i, (n, N, K) in enumerate(shapes)]


def all_single_layers() -> List[Linear]:
    """Every single-layer workload (the decoder-layer set is listed separately)."""
    return ([tiny_layer(), llama3_8b_gate_up_prefill()]
            + [qwen3_32b_up_decode(b) for b in (1, 8, 16, 64)]
            + [qwen3_32b_down_prefill()])


# ------------------------------------------------------------------ drawing ---

def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even) and return the uint16 bit patterns.
    Inputs are finite."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> 16) & 1
    return ((u + np.uint32(0x7FFF) + lsb) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class LayerInputs:
    layer: Linear
    x: np.ndarray          # uint16 bf16 bits [M, K]
    W: np.ndarray          # uint16 bf16 bits [N, K]
    s: np.ndarray          # float32 [K]
    outlier_channels: np.ndarray


def _streams(seed: int):
    return [np.random.Generator(np.random.PCG64(ss)) for ss in np.random.SeedSequence(seed).spawn(4)]


def outlier_channels(layer: Linear) -> np.ndarray:
    if layer.outlier_channels:
        ch = np.asarray(layer.outlier_channels, dtype=np.int64)
        return ch[ch < layer.K]
    if layer.outlier_frac > 0:
        n = int(round(layer.outlier_frac * layer.K))
        rng = _streams(layer.seed)[3]
        return np.sort(rng.choice(layer.K, size=n, replace=False)).astype(np.int64)
    return np.zeros(0, np.int64)


def draw_x(layer: Linear, rows: Optional[int] = None) -> np.ndarray:
    """bf16 bits of the activations (the first `rows` rows if given)."""
    M = layer.M if rows is None else rows
    rng = _streams(layer.seed)[0]
    if layer.x_dist == "normal":
        x = rng.standard_normal((M, layer.K), dtype=np.float32)
    elif layer.x_dist == "t3":
        x = rng.standard_t(3, size=(M, layer.K)).astype(np.float32)
    else:
        raise ValueError(layer.x_dist)
    ch = outlier_channels(layer)
    if ch.size:
        x[:, ch] *= np.float32(layer.outlier_factor)
    return f32_to_bf16_bits(x)


def draw_W(layer: Linear) -> np.ndarray:
    rng = _streams(layer.seed)[1]
    W = rng.standard_normal((layer.N, layer.K), dtype=np.float32) * np.float32(layer.w_std)
    return f32_to_bf16_bits(W)


def draw_s(layer: Linear) -> np.ndarray:
    rng = _streams(layer.seed)[2]
    return np.exp(rng.normal(0.0, layer.s_sigma, size=layer.K)).astype(np.float32)


def draw(layer: Linear) -> LayerInputs:
    return LayerInputs(layer, draw_x(layer), draw_W(layer), draw_s(layer), outlier_channels(layer))


def with_shape(layer: Linear, M=None, N=None, K=None, **kw) -> Linear:
    """Same input model at another shape (for ragged / edge-case tests)."""
    upd = {k: v for k, v in dict(M=M, N=N, K=K).items() if v is not None}
    upd.update(kw)
    return replace(layer, **upd)
