"""Workload descriptors: layer shapes, weight scale, input distribution, sparsities.

The shapes are those of well-known decoder FFNs (Llama-3-8B, Qwen3-14B,
Llama-3-70B) plus a tiny layer that a CPU reference finishes in seconds.
"""

from __future__ import annotations

from dataclasses import dataclass, field


def ffn_k(d_ff: int, s2_percent: int) -> int:
    """Number of channels kept at Stage-2 sparsity ``s2_percent`` (integer %).

    k = round((1 - s) * d_ff), evaluated in integers as (d_ff*(100-s) + 50) // 100
    so that no floating-point rounding enters the channel count.
    """
    if not 0 <= s2_percent <= 100:
        raise ValueError("s2_percent must be in [0, 100]")
    return (d_ff * (100 - s2_percent) + 50) // 100


@dataclass(frozen=True)
class WorkloadConfig:
    name: str
    index: int  # seed base = 1000 * index + layer
    d_model: int
    d_ff: int
    sigma: float  # weight standard deviation
    outlier_frac: float  # fraction of input channels that carry outliers
    outlier_scale: float  # multiplier applied to those channels
    s1_percent: tuple  # Stage-1 input sparsity targets (%)
    s2_percent: tuple  # Stage-2 channel sparsity targets (%)
    n_tokens: int  # eval tokens per layer
    n_cal: int = 256  # calibration tokens per layer
    n_layers: int = 1
    batch_sizes: tuple = (1,)
    group: int = 128
    notes: str = ""

    @property
    def n_outliers(self) -> int:
        return int(round(self.outlier_frac * self.d_model))

    def k(self, s2_percent: int | None = None) -> int:
        s = self.s2_percent[-1] if s2_percent is None else s2_percent
        return ffn_k(self.d_ff, s)

    def seed(self, layer: int = 0) -> int:
        return 1000 * self.index + layer

    def workload_name(self, s1_percent=None, s2_percent=None) -> str:
        s1 = self.s1_percent[0] if s1_percent is None else s1_percent
        s2 = self.s2_percent[-1] if s2_percent is None else s2_percent
        return (f"{self.name} ffn layer d_model={self.d_model} d_ff={self.d_ff} "
                f"s1={s1}% s2={s2}% k={ffn_k(self.d_ff, s2)}")


CONFIGS = {
    "tiny": WorkloadConfig(
        name="tiny", index=1, d_model=512, d_ff=1376, sigma=0.02,
        outlier_frac=0.01, outlier_scale=20.0, s1_percent=(50,), s2_percent=(70,),
        n_tokens=64,
        notes="single tiny SwiGLU layer; CPU reference finishes in seconds"),
    "llama3_8b": WorkloadConfig(
        name="llama3_8b", index=2, d_model=4096, d_ff=14336, sigma=0.02,
        outlier_frac=0.005, outlier_scale=30.0, s1_percent=(50,),
        s2_percent=(0, 50, 60, 70), n_tokens=256,
        notes="Llama-3-8B-shaped FFN layer"),
    "qwen3_14b": WorkloadConfig(
        name="qwen3_14b", index=3, d_model=5120, d_ff=17408, sigma=0.015,
        outlier_frac=0.005, outlier_scale=30.0, s1_percent=(40, 50, 60),
        s2_percent=(70,), n_tokens=256,
        notes="Qwen3-14B-shaped FFN layer"),
    "stack32": WorkloadConfig(
        name="stack32", index=4, d_model=4096, d_ff=14336, sigma=0.02,
        outlier_frac=0.005, outlier_scale=30.0, s1_percent=(50,), s2_percent=(70,),
        n_tokens=128, n_layers=32,
        notes="32 Llama-3-8B-shaped layers chained through RMSNorm"),
    "llama3_70b": WorkloadConfig(
        name="llama3_70b", index=5, d_model=8192, d_ff=28672, sigma=0.01,
        outlier_frac=0.005, outlier_scale=30.0, s1_percent=(50,), s2_percent=(70,),
        n_tokens=16, batch_sizes=(1, 2, 4, 8, 16),
        notes="Llama-3-70B-shaped FFN layer, per-token masks at batch 1..16"),
}


def get_config(name: str) -> WorkloadConfig:
    try:
        return CONFIGS[name]
    except KeyError as e:
        raise KeyError(f"unknown workload {name!r}; choose from {sorted(CONFIGS)}") from e
