"""A stack of Prox layers chained through unit-gain RMSNorm, with sequential
threshold calibration (Prox App. A.7, Algorithm 1): layer l's input threshold
is the s1-quantile of the inputs it receives when the calibration tokens run
through layers 1..l-1 with their finalised rules, and -- when a Stage-2
sparsity s2 is given -- its score threshold is the s2-quantile of the proxy
scores of those same inputs.  Every step runs in the library's kernels
(calibration, proxy scores, the Prox step, RMSNorm)."""

from __future__ import annotations

import torch

from . import MASK_THRESHOLD, Layer, calibrate_thresholds, rmsnorm


class Stack:
    def __init__(self, weights, k: int, max_batch: int = 1, stream=None):
        """weights: sequence of (w_gate, w_up, w_down) bf16 CUDA tensors, math
        layout ([d, F], [d, F], [F, d]).  Thresholds start at 0 until
        calibrate() sets them."""
        self.layers = [Layer(wg, wu, wd, tau=0.0, k=k, max_batch=max_batch, stream=stream)
                       for (wg, wu, wd) in weights]
        self.taus = [0.0] * len(self.layers)
        self.k = k

    def calibrate(self, x_cal: torch.Tensor, s1: float, s2: float | None = None, stream=None):
        """Algorithm 1 on fp32 calibration tokens [n, d] (n <= max_batch).
        Returns (taus, inputs), or (taus, taus_s, inputs) when s2 is given and
        every layer switches to the score-threshold rule."""
        x = x_cal.contiguous()
        inputs = []
        taus_s = []
        for li, layer in enumerate(self.layers):
            inputs.append(x)
            tau = calibrate_thresholds(x, s1, stream=stream)
            layer.set_tau(tau)
            self.taus[li] = tau
            if s2 is not None:
                tau_s = calibrate_thresholds(layer.proxy_scores(x, stream=stream), s2,
                                             stream=stream)
                layer.set_mask(MASK_THRESHOLD, tau_s)
                taus_s.append(tau_s)
            if li + 1 < len(self.layers):
                x = rmsnorm(layer.forward(x, stream=stream), stream=stream)
        if s2 is not None:
            return list(self.taus), taus_s, inputs
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
