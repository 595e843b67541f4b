"""A stack of Prox layers chained through unit-gain RMSNorm, with sequential
threshold calibration (Prox App. A.7, Algorithm 1): layer l's input threshold
is the s1-quantile of the inputs it receives when the calibration tokens run
through layers 1..l-1 with their finalised rules.  Every step runs in the
library's kernels (calibration, the Prox step, RMSNorm)."""

from __future__ import annotations

import torch

from . import Layer, calibrate_thresholds, rmsnorm


class Stack:
    def __init__(self, weights, k: int, max_batch: int = 1, stream=None):
        """weights: sequence of (w_gate, w_up, w_down) bf16 CUDA tensors, math
        layout ([d, F], [d, F], [F, d]).  Thresholds start at 0 until
        calibrate() sets them."""
        self.layers = [Layer(wg, wu, wd, tau=0.0, k=k, max_batch=max_batch, stream=stream)
                       for (wg, wu, wd) in weights]
        self.taus = [0.0] * len(self.layers)
        self.k = k

    def calibrate(self, x_cal: torch.Tensor, s1: float, stream=None):
        """Algorithm 1 on fp32 calibration tokens [n, d] (n <= max_batch).
        Returns the thresholds and the calibration inputs each layer saw."""
        x = x_cal.contiguous()
        inputs = []
        for li, layer in enumerate(self.layers):
            inputs.append(x)
            tau = calibrate_thresholds(x, s1, stream=stream)
            layer.set_tau(tau)
            self.taus[li] = tau
            if li + 1 < len(self.layers):
                x = rmsnorm(layer.forward(x, stream=stream), stream=stream)
        return list(self.taus), inputs

    def forward(self, x: torch.Tensor, stream=None):
        """Tokens [B, d] through every layer; returns the per-layer inputs and
        the last layer's output."""
        xs = []
        y = None
        for li, layer in enumerate(self.layers):
            xs.append(x)
            y = layer.forward(x, stream=stream)
            if li + 1 < len(self.layers):
                x = rmsnorm(y, stream=stream)
        return xs, y

    def close(self):
        for layer in self.layers:
            layer.close()
        self.layers = []
