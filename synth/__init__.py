"""Seeded synthetic inputs for the SVDQuant W4A4 linear layer.

This module is shared by the tests and the benchmark.  It holds no arithmetic of
the method itself (no smoothing, SVD, quantization or GEMM): it only draws
deterministic bf16 tensors with the shapes and value distributions of the FLUX
DiT linears that the SVDQuant model card describes.

Generator (counter based, so any slice can be drawn independently):
  * SplitMix64 over the counter ``seed * 2**32 + i`` gives 64-bit words;
  * two consecutive words (2j, 2j+1) feed one Box-Muller draw in fp64;
  * fp64 -> fp32 (round to nearest) -> bf16 (round to nearest even).

Outlier channels: the ``n_out = round(frac * K)`` channels with the smallest
SplitMix64 hash of ``(seed_perm, k)`` are multiplied by the outlier factor.
The activation-outlier structure is what stage 1 of SVDQuant starts from
("both the activation X and weights W contain outliers", SVDQuant model card,
"Quantization Method").
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Tuple

import numpy as np

_MASK64 = np.uint64(0xFFFFFFFFFFFFFFFF)


def splitmix64(counter: np.ndarray) -> np.ndarray:
    """SplitMix64 finaliser applied to ``counter + golden_gamma`` (uint64, wraps)."""
    with np.errstate(over="ignore"):
        z = counter.astype(np.uint64) + np.uint64(0x9E3779B97F4A7C15)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        z = z ^ (z >> np.uint64(31))
    return z


def _counters(seed: int, start: int, count: int) -> np.ndarray:
    base = np.uint64((seed & 0xFFFFFFFF) << 32)
    return base + np.arange(start, start + count, dtype=np.uint64)


def normal_f64(seed: int, start: int, count: int) -> np.ndarray:
    """``count`` standard normal fp64 draws, draws ``start .. start+count-1``."""
    words = splitmix64(_counters(seed, 2 * start, 2 * count))
    w1 = words[0::2]
    w2 = words[1::2]
    u1 = ((w1 >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)  # (0, 1]
    u2 = (w2 >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)  # [0, 1)
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit pattern (uint16), round to nearest even.  Inputs are finite."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def gelu_erf(z: np.ndarray) -> np.ndarray:
    """Exact (erf) GELU in fp64; shapes the MLP-down input distribution."""
    from scipy.special import erf  # scipy is part of the image

    return 0.5 * z * (1.0 + erf(z / math.sqrt(2.0)))


def outlier_channels(seed_perm: int, K: int, frac: float) -> np.ndarray:
    n_out = int(round(frac * K))
    if n_out == 0:
        return np.zeros(0, dtype=np.int64)
    h = splitmix64(_counters(seed_perm, 0, K))
    return np.sort(np.argsort(h, kind="stable")[:n_out])


# ---------------------------------------------------------------------------
# Workloads: the FLUX-shaped layers.  Shapes are nn.Linear shapes: X is M x K,
# W is N x K (output features x input features), Y is M x N.
# ---------------------------------------------------------------------------


@dataclasses.dataclass(frozen=True)
class LayerSpec:
    name: str
    M: int
    K: int
    N: int
    rank: int
    out_frac: float = 0.005
    out_scale: float = 30.0
    w_std: float = 0.02
    b_std: float = 0.01
    x_kind: str = "normal"  # "normal" | "gelu" | "concat_gelu" (first 3072 normal, rest GELU)
    seed_x: int = 0
    seed_w: int = 0
    seed_b: int = 0
    seed_perm: int = 0

    @property
    def flops_4bit(self) -> int:
        return 2 * self.M * self.N * self.K

    @property
    def flops_lowrank(self) -> int:
        return 2 * self.M * self.rank * (self.K + self.N)

    @property
    def flops(self) -> int:
        return self.flops_4bit + self.flops_lowrank

    def with_rows(self, M: int) -> "LayerSpec":
        return dataclasses.replace(self, M=M)


def _spec(cfg: int, sub: int, name: str, M: int, K: int, N: int, rank: int, **kw) -> LayerSpec:
    off = 100 * sub
    return LayerSpec(name=name, M=M, K=K, N=N, rank=rank,
                     seed_x=1000 + cfg + off, seed_w=2000 + cfg + off,
                     seed_b=3000 + cfg + off, seed_perm=4000 + cfg + off, **kw)


def workloads() -> dict:
    """All FLUX-shaped layers, keyed by a name that states what the layer is."""
    w = {}
    w["tiny_256x512x512_r16"] = _spec(1, 0, "tiny_256x512x512_r16", 256, 512, 512, 16,
                                      out_frac=0.01, out_scale=50.0)
    w["flux_qkv_4608x3072x9216_r32"] = _spec(2, 0, "flux_qkv_4608x3072x9216_r32", 4608, 3072, 9216, 32)
    w["flux_mlp_up_4608x3072x12288_r32"] = _spec(3, 0, "flux_mlp_up_4608x3072x12288_r32", 4608, 3072, 12288, 32)
    w["flux_mlp_down_4608x12288x3072_r32"] = _spec(3, 1, "flux_mlp_down_4608x12288x3072_r32", 4608, 12288, 3072, 32,
                                                   x_kind="gelu")
    for M in (256, 1024, 4096, 16384):
        for r in (0, 16, 32, 64, 128):
            nm = f"sweep_{M}x3072x3072_r{r}"
            w[nm] = _spec(4, 0, nm, M, 3072, 3072, r)
    w["dit_qkv_mlp_in_16896x3072x21504_r32"] = _spec(5, 0, "dit_qkv_mlp_in_16896x3072x21504_r32",
                                                     16896, 3072, 21504, 32)
    w["dit_out_16896x15360x3072_r32"] = _spec(5, 1, "dit_out_16896x15360x3072_r32", 16896, 15360, 3072, 32,
                                              x_kind="concat_gelu")
    return w


def get(name: str) -> LayerSpec:
    return workloads()[name]


# ---------------------------------------------------------------------------
# Tensor draws
# ---------------------------------------------------------------------------


def _draw_rows_f64(seed: int, row0: int, nrows: int, ncols: int) -> np.ndarray:
    return normal_f64(seed, row0 * ncols, nrows * ncols).reshape(nrows, ncols)


def activations_bf16(spec: LayerSpec, rows: Optional[Tuple[int, int]] = None,
                     chunk_rows: int = 1024) -> np.ndarray:
    """X (M x K) as bf16 bits, or the row range ``rows=(r0, r1)`` of it."""
    r0, r1 = (0, spec.M) if rows is None else rows
    out = np.empty((r1 - r0, spec.K), dtype=np.uint16)
    oc = outlier_channels(spec.seed_perm, spec.K, spec.out_frac)
    for a in range(r0, r1, chunk_rows):
        b = min(r1, a + chunk_rows)
        z = _draw_rows_f64(spec.seed_x, a, b - a, spec.K)
        if spec.x_kind == "gelu":
            z = gelu_erf(z)
        elif spec.x_kind == "concat_gelu":
            split = 3072
            z[:, split:] = gelu_erf(z[:, split:])
        if oc.size:
            z[:, oc] *= spec.out_scale
        out[a - r0:b - r0] = f32_to_bf16_bits(z.astype(np.float32))
    return out


def weight_bf16(spec: LayerSpec) -> np.ndarray:
    """W (N x K, nn.Linear layout) as bf16 bits, ~N(0, w_std)."""
    out = np.empty((spec.N, spec.K), dtype=np.uint16)
    step = max(1, (1 << 24) // spec.K)
    for a in range(0, spec.N, step):
        b = min(spec.N, a + step)
        z = _draw_rows_f64(spec.seed_w, a, b - a, spec.K) * spec.w_std
        out[a:b] = f32_to_bf16_bits(z.astype(np.float32))
    return out


def bias_bf16(spec: LayerSpec) -> np.ndarray:
    z = normal_f64(spec.seed_b, 0, spec.N) * spec.b_std
    return f32_to_bf16_bits(z.astype(np.float32))


def act_absmax(x_bf16: np.ndarray) -> np.ndarray:
    """Per-input-channel calibration statistic max_m |X[m, k]| (fp32).

    This is bookkeeping over the drawn tensor (the calibration set is the same X
    that the forward consumes), not a step of the method.
    """
    return np.max(np.abs(bf16_bits_to_f32(x_bf16)), axis=0).astype(np.float32)


def rms_norm_weight(head_dim: int, seed: int) -> np.ndarray:
    """Per-channel weight of a Q or K RMS normalization: 1 + 0.1 N(0, 1), rounded to bf16 (a
    bf16 model's parameter), returned as fp32."""
    v = (1.0 + 0.1 * normal_f64(seed, 0, head_dim)).astype(np.float32)
    return bf16_bits_to_f32(f32_to_bf16_bits(v))


def rope_tables(M: int, head_dim: int = 128, text_tokens: int = 512, grid_w: int = 64,
                axes: Tuple[int, ...] = (16, 56, 56), theta: float = 10000.0) -> Tuple[np.ndarray, np.ndarray]:
    """cos and sin [M, head_dim / 2] (fp32) of FLUX-shaped rotary angles.

    Rows below ``text_tokens`` are text tokens (every position 0); row r above is image token
    r - text_tokens of a grid ``grid_w`` wide, at (h, w) = divmod(r - text_tokens, grid_w).  The
    pairs of channels are split over three position axes (index, h, w) with ``axes[a]`` channels
    each; pair i of axis a turns by pos_a * theta ** (-2 i / axes[a]).  Angles in fp64, cos and sin
    rounded to fp32 (they are inputs of the rotation, as a model precomputes them)."""
    assert sum(axes) == head_dim and all(a % 2 == 0 for a in axes)
    r = np.arange(M, dtype=np.int64)
    img = np.maximum(r - text_tokens, 0)
    is_img = r >= text_tokens
    pos = [np.zeros(M), np.where(is_img, img // grid_w, 0).astype(np.float64),
           np.where(is_img, img % grid_w, 0).astype(np.float64)]
    angles = []
    for a, dim in enumerate(axes):
        omega = theta ** (-np.arange(0, dim, 2, dtype=np.float64) / dim)
        angles.append(pos[a][:, None] * omega[None, :])
    ang = np.concatenate(angles, axis=1)
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def custom(name: str, M: int, K: int, N: int, rank: int, seed: int = 7, **kw) -> LayerSpec:
    """An ad-hoc layer (edge cases in tests): seeds derived from ``seed``."""
    return LayerSpec(name=name, M=M, K=K, N=N, rank=rank, seed_x=10000 + seed, seed_w=20000 + seed,
                     seed_b=30000 + seed, seed_perm=40000 + seed, **kw)


__all__: List[str] = [
    "LayerSpec", "workloads", "get", "custom", "activations_bf16", "weight_bf16", "bias_bf16",
    "act_absmax", "f32_to_bf16_bits", "bf16_bits_to_f32", "normal_f64", "splitmix64",
    "outlier_channels", "gelu_erf", "rms_norm_weight", "rope_tables",
]
