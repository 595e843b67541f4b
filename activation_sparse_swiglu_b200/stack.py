"""A stack of Prox layers chained through unit-gain RMSNorm, with sequential
threshold calibration (Prox App. A.7, Algorithm 1): layer l's input threshold
is the s1-quantile of the inputs it receives when the calibration tokens run
through layers 1..l-1 with their finalised rules, and -- when a Stage-2
sparsity s2 is given -- its score threshold is the s2-quantile of the proxy
scores of those same inputs.  Every step runs in the library's kernels
(calibration, proxy scores, the Prox step, RMSNorm)."""

from __future__ import annotations

import json
import math

import torch

from . import MASK_THRESHOLD, MASK_TOPK, Layer, calibrate_thresholds, rmsnorm

ARTEFACT_FORMAT = "prox-thresholds"
ARTEFACT_VERSION = 1


def thresholds_to_json(taus, taus_s=None, *, d_model: int, d_ff: int, k: int, s1: float,
                       s2: float | None = None) -> str:
    """The calibration artefact of a stack (Prox App. A.7: thresholds are
    calibrated once and never re-estimated at inference): per layer tau_x and,
    under the threshold rule, tau_s.  Floats are written so that they read back
    bit for bit."""
    if taus_s is not None and len(taus_s) != len(taus):
        raise ValueError("taus and taus_s differ in length")
    layers = [{"tau_x": float(t), "tau_s": None if taus_s is None else float(taus_s[i])}
              for i, t in enumerate(taus)]
    doc = {"format": ARTEFACT_FORMAT, "version": ARTEFACT_VERSION, "d_model": int(d_model),
           "d_ff": int(d_ff), "k": int(k), "s1": float(s1),
           "s2": None if s2 is None else float(s2), "layers": layers}
    _check_artefact(doc)
    return json.dumps(doc, indent=1)


def _check_artefact(doc) -> None:
    if doc.get("format") != ARTEFACT_FORMAT or doc.get("version") != ARTEFACT_VERSION:
        raise ValueError("not a prox-thresholds artefact of a known version")
    if not isinstance(doc.get("layers"), list) or not doc["layers"]:
        raise ValueError("the artefact holds no layers")
    if not 1 <= int(doc["k"]) <= int(doc["d_ff"]):
        raise ValueError("k must lie in [1, d_ff]")
    has_s = [ly.get("tau_s") is not None for ly in doc["layers"]]
    if any(has_s) and not all(has_s):
        raise ValueError("tau_s must be given for every layer or for none")
    for ly in doc["layers"]:
        for key in ("tau_x", "tau_s"):
            v = ly.get(key)
            if key == "tau_x" or v is not None:
                if not isinstance(v, (int, float)) or not math.isfinite(v) or v < 0:
                    raise ValueError(f"{key} must be a finite value >= 0, got {v!r}")


def thresholds_from_json(text: str) -> dict:
    """Parses and checks an artefact written by thresholds_to_json."""
    doc = json.loads(text)
    _check_artefact(doc)
    return doc


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

    def save_thresholds(self, path: str, s1: float, s2: float | None = None) -> None:
        """Writes the current per-layer thresholds as a calibration artefact."""
        infos = [layer.info() for layer in self.layers]
        taus = [inf["tau_x"] for inf in infos]
        taus_s = None
        if any(inf["mask_mode"] == MASK_THRESHOLD for inf in infos):
            taus_s = [inf["tau_s"] for inf in infos]
        text = thresholds_to_json(taus, taus_s, d_model=infos[0]["d_model"],
                                  d_ff=infos[0]["d_ff"], k=self.k, s1=s1, s2=s2)
        with open(path, "w") as fh:
            fh.write(text)

    def load_thresholds(self, path: str) -> dict:
        """Applies a calibration artefact: tau_x per layer and, when present,
        the score-threshold rule with tau_s (otherwise top-k with the
        artefact's k).  Shapes and layer count must match."""
        with open(path) as fh:
            doc = thresholds_from_json(fh.read())
        if len(doc["layers"]) != len(self.layers):
            raise ValueError("the artefact has a different number of layers")
        for layer, ly in zip(self.layers, doc["layers"]):
            inf = layer.info()
            if (inf["d_model"], inf["d_ff"]) != (doc["d_model"], doc["d_ff"]):
                raise ValueError("the artefact was calibrated for another layer shape")
        self.k = int(doc["k"])
        for li, (layer, ly) in enumerate(zip(self.layers, doc["layers"])):
            layer.set_tau(ly["tau_x"])
            layer.set_k(self.k)
            if ly["tau_s"] is None:
                layer.set_mask(MASK_TOPK)
            else:
                layer.set_mask(MASK_THRESHOLD, ly["tau_s"])
            self.taus[li] = ly["tau_x"]
        return doc

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
