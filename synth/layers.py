"""Seeded synthetic FFN layers and decode tokens.

Draw order for one layer, from ``numpy.random.Generator(PCG64(seed))`` with
``seed = 1000 * config_index + layer``:

1. the outlier channel set: ``round(f * d_model)`` distinct input channels;
2. W_gate [d_model, d_ff], then W_up [d_model, d_ff], then W_down [d_ff, d_model],
   each ``standard_normal(float32) * sigma`` rounded to bf16 (round to nearest even);
3. the calibration tokens [n_cal, d_model];
4. the eval tokens [n_tokens, d_model].

Tokens are Laplace(0, 1) in float64, cast to float32, and the outlier channels
are multiplied by the configured scale in every token (calibration and eval).
For the 32-layer stack only layer 0 draws tokens; later layers see the
normalised outputs of the layers before them.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .configs import WorkloadConfig, get_config


def bf16_round(a: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Round float32 values to bf16 storage (nearest, ties to even).

    Returns ``(bits, values)``: the uint16 bf16 bit patterns and the same values
    widened back to float32.  Inputs must be finite.
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    rounded = (u + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)
    bits = (rounded >> np.uint32(16)).astype(np.uint16)
    return bits, rounded.view(np.float32)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen uint16 bf16 bit patterns to float32 (exact)."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def outlier_channels(rng: np.random.Generator, d_model: int, n_out: int) -> np.ndarray:
    if n_out == 0:
        return np.zeros(0, dtype=np.int64)
    return np.sort(rng.choice(d_model, size=n_out, replace=False))


def _weights(rng, shape, sigma):
    w = rng.standard_normal(shape, dtype=np.float32) * np.float32(sigma)
    return bf16_round(w)


def _tokens(rng, n, d, outliers, scale):
    x = rng.laplace(0.0, 1.0, size=(n, d)).astype(np.float32)
    if outliers.size:
        x[:, outliers] *= np.float32(scale)
    return x


@dataclass
class SyntheticLayer:
    """One seeded layer.  Weight arrays are in math layout:
    W_gate, W_up: [d_model, d_ff]; W_down: [d_ff, d_model]."""

    config: WorkloadConfig
    layer: int
    outliers: np.ndarray
    w_gate_bits: np.ndarray
    w_up_bits: np.ndarray
    w_down_bits: np.ndarray
    w_gate: np.ndarray
    w_up: np.ndarray
    w_down: np.ndarray
    x_cal: np.ndarray | None
    x_eval: np.ndarray | None

    @property
    def d_model(self) -> int:
        return self.config.d_model

    @property
    def d_ff(self) -> int:
        return self.config.d_ff


def make_layer(config: WorkloadConfig | str, layer: int = 0, *, n_tokens: int | None = None,
               n_cal: int | None = None, draw_tokens: bool = True,
               keep_bits: bool = True) -> SyntheticLayer:
    """Draw one seeded layer (and its calibration + eval tokens)."""
    cfg = get_config(config) if isinstance(config, str) else config
    rng = np.random.Generator(np.random.PCG64(cfg.seed(layer)))
    d, f = cfg.d_model, cfg.d_ff
    outl = outlier_channels(rng, d, cfg.n_outliers)
    gb, gv = _weights(rng, (d, f), cfg.sigma)
    ub, uv = _weights(rng, (d, f), cfg.sigma)
    db, dv = _weights(rng, (f, d), cfg.sigma)
    x_cal = x_eval = None
    if draw_tokens:
        x_cal = _tokens(rng, cfg.n_cal if n_cal is None else n_cal, d, outl, cfg.outlier_scale)
        x_eval = _tokens(rng, cfg.n_tokens if n_tokens is None else n_tokens, d, outl,
                         cfg.outlier_scale)
    if not keep_bits:
        gb = ub = db = None
    return SyntheticLayer(cfg, layer, outl, gb, ub, db, gv, uv, dv, x_cal, x_eval)


def make_stack_layer(layer: int, *, n_tokens: int | None = None,
                     n_cal: int | None = None) -> SyntheticLayer:
    """Layer ``layer`` of the 32-layer stack; only layer 0 draws tokens."""
    cfg = get_config("stack32")
    return make_layer(cfg, layer, n_tokens=n_tokens, n_cal=n_cal, draw_tokens=(layer == 0))
