"""Shared helpers for the GPU parity tests: device copies of seeded layers,
oracle-side packing, and the parity rules written once."""

from __future__ import annotations

import numpy as np
import torch

from oracle import prox_oracle as orc

# Parity bars (relative): Stage-1 scores and pre-activations; masks may differ
# only at channels whose oracle score is this close to the k-th value; outputs
# in relative L2 given the oracle's mask.
SCORE_RTOL = 1e-3
MASK_RTOL = 1e-3
OUT_RTOL = 5e-3


def bits_to_bf16(bits: np.ndarray, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device)
    return t.view(torch.bfloat16)


def device_layer(lay, tau, k, max_batch=1):
    import activation_sparse_swiglu_b200 as prox
    wg = bits_to_bf16(lay.w_gate_bits)
    wu = bits_to_bf16(lay.w_up_bits)
    wd = bits_to_bf16(lay.w_down_bits)
    layer = prox.Layer(wg, wu, wd, tau=float(tau), k=int(k), max_batch=max_batch)
    del wg, wu, wd
    return layer


class OracleLayer:
    """Oracle-side view of a seeded layer (packed proxies computed once)."""

    def __init__(self, lay):
        self.lay = lay
        self.qg, self.sg = orc.quantize_proxy(lay.w_gate)
        self.qu, self.su = orc.quantize_proxy(lay.w_up)

    def step(self, x, tau, k, **kw):
        """prox_ffn of the oracle; kw: tau_s, act, proxy_values."""
        lay = self.lay
        return orc.prox_ffn(x, lay.w_gate, lay.w_up, lay.w_down, self.qg, self.sg, self.qu,
                            self.su, tau=tau, k=k, **kw)

    def stage1(self, x, tau):
        return orc.proxy_intermediate(x, tau, self.qg, self.sg, self.qu, self.su)


def close_with_floor(gpu, ref, rtol=SCORE_RTOL):
    """|gpu - ref| <= rtol * max(|ref|, rtol * max|ref|) elementwise."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    floor = rtol * (np.max(np.abs(ref)) if ref.size else 0.0)
    bound = rtol * np.maximum(np.abs(ref), floor)
    bad = np.abs(gpu - ref) > bound
    return (not bad.any()), int(bad.sum())


def check_mask(gpu_idx, orc_idx, orc_scores, k):
    gpu_idx = np.asarray(gpu_idx, dtype=np.int64)
    assert gpu_idx.size == k
    assert np.all(np.diff(gpu_idx) > 0), "idx_s must be strictly ascending"
    kth = np.sort(np.asarray(orc_scores, dtype=np.float64))[::-1][k - 1]
    diff = np.setxor1d(gpu_idx, orc_idx)
    near = np.abs(np.asarray(orc_scores)[diff] - kth) <= MASK_RTOL * kth
    assert np.all(near), f"{int((~near).sum())} mask differences away from the k-th value"
    return int(diff.size)


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))
