"""fp64 CPU oracle for the Prox two-stage sparse SwiGLU FFN decode step.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module.  The
product path (``activation_sparse_swiglu_b200`` and its CUDA library) never
imports, links or calls it, and this module imports nothing from the product.

Source: "Prox: Training-Free FFN Activation Sparsity via Approximate
Intermediate-Channel Salience in LLMs" (Liu et al.), cited below as *Prox*
with the section, equation or algorithm each function follows.

Everything is evaluated in float64 on the exact stored values: bf16 weights
(passed as float32 arrays holding bf16 values), fp32 inputs, fp16 scales.
The code takes the method's steps in the paper's order and notation, with
library primitives (matmul, sort) as steps and no blocking or fusion.

Readings taken where the paper is silent or differs from the workload spec
(each one is listed in the design notes):

* proxy quantisation: symmetric INT4, groups of 128 consecutive input rows per
  output channel, fp16 scale ``S = fp16(amax / 7)``, codes
  ``clamp(round_half_even(W / S), -7, 7)``; a group with amax = 0 has S = 0 and
  codes 0.  (*Prox* §4.3 quantises "per row"; the workload uses group-128.)
* Stage-2 mask: per-token top-k of |s~| with ties going to the lower channel
  index (*Prox* App. A.6 "Per-token top-k selection"); the threshold rule of
  §4.1 is ``threshold_channels``.
* calibration: exact lower order statistic of |x| over all calibration values
  at rank floor(s1 * n) (0-based); s1 = 0 gives tau = 0.
* Stage 2 uses the full input x, not the sparsified one (*Prox* §4.1, Stage 2).
* GeGLU gate (*Prox* §5 names Gemma-3's GeGLU FFN, not the GELU form): both
  GELU(z) = z Phi(z), evaluated through erfc, and the tanh form.
* ablation A3 (*Prox* §5.2): the signed proxy values act(g~) u~ of the selected
  channels (same selection rule as Prox) go into W_down.
* allocation (*Prox* §4.2): a target whose re-solved s2 would leave [0, 1] has
  no allocation and raises.
* the Stage-2 score threshold tau_s: the same exact lower order statistic as
  tau_x, over the calibration tokens' scores held as fp32.
"""

from __future__ import annotations

import math

import numpy as np

F64 = np.float64
GROUP = 128
CODE_MAX = 7


# ---------------------------------------------------------------------------
# SwiGLU building blocks (Prox §2.1)
# ---------------------------------------------------------------------------

def silu(z):
    """SiLU(z) = z / (1 + e^{-z})  (Prox §2.1, SwiGLU definition)."""
    z = np.asarray(z, dtype=F64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def gelu(z):
    """GELU(z) = z Phi(z), Phi the standard normal CDF (Hendrycks & Gimpel,
    "Gaussian Error Linear Units", §2); the gate of a GeGLU FFN, the family
    Prox §5 sparsifies besides SwiGLU."""
    z = np.asarray(z, dtype=F64)
    # Phi(z) = erfc(-z / sqrt 2) / 2, which keeps its relative accuracy for z << 0
    return z * 0.5 * np.vectorize(math.erfc, otypes=[F64])(-z / math.sqrt(2.0))


def gelu_tanh(z):
    """The tanh form of GELU from the same paper:
    0.5 z (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3)))."""
    z = np.asarray(z, dtype=F64)
    return 0.5 * z * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (z + 0.044715 * z ** 3)))


# gate activations by name; the library's PROX_ACT_* codes are 0, 1, 2 in this order
ACTIVATIONS = {"silu": silu, "gelu_tanh": gelu_tanh, "gelu": gelu}


def dense_ffn(x, w_gate, w_up, w_down, act="silu"):
    """FFN(x) = (x W_up ⊙ SiLU(x W_gate)) W_down  (Prox §2.1, FFN equation);
    ``act`` swaps the gate activation (GeGLU with "gelu" / "gelu_tanh").

    x: [d_model]; W_gate, W_up: [d_model, d_ff]; W_down: [d_ff, d_model].
    """
    x = np.asarray(x, dtype=F64)
    u = x @ np.asarray(w_up, dtype=F64)
    h = ACTIVATIONS[act](x @ np.asarray(w_gate, dtype=F64))
    s = u * h
    return s @ np.asarray(w_down, dtype=F64)


def intermediate_state(x, w_gate, w_up, act="silu"):
    """s = u ⊙ h with u = x W_up, h = SiLU(x W_gate)  (Prox §2.1)."""
    x = np.asarray(x, dtype=F64)
    return (x @ np.asarray(w_up, dtype=F64)) * ACTIVATIONS[act](x @ np.asarray(w_gate, dtype=F64))


# ---------------------------------------------------------------------------
# Sparsity operators (Prox §2.2)
# ---------------------------------------------------------------------------

def pi_in(x, w, idx):
    """Input sparsity Π_in(x, W, m) = x[I(m)] W[I(m), :]  (Prox §2.2).

    ``idx`` is I(m), the retained input indices.
    """
    idx = np.asarray(idx, dtype=np.int64)
    return np.asarray(x, dtype=F64)[idx] @ np.asarray(w)[idx, :].astype(F64)


def pi_out(x, w, idx):
    """Output sparsity Π_out(x, W, m) = x W[:, I(m)]  (Prox §2.2)."""
    idx = np.asarray(idx, dtype=np.int64)
    return np.asarray(x, dtype=F64) @ np.asarray(w)[:, idx].astype(F64)


# ---------------------------------------------------------------------------
# INT4 proxy weights (Prox §4.3)
# ---------------------------------------------------------------------------

def quantize_proxy(w, group=GROUP):
    """Symmetric INT4 proxy of a [d_model, d_ff] weight (Prox §4.3).

    Returns ``(Q, S)``: Q int8 [d_model, d_ff] with codes in [-7, 7] and
    S float16 [d_model / group, d_ff], one scale per (row group, channel).
    """
    w = np.asarray(w, dtype=F64)
    d, f = w.shape
    if d % group:
        raise ValueError("d_model must be a multiple of the group size")
    g = d // group
    wg = w.reshape(g, group, f)
    amax = np.abs(wg).max(axis=1)                       # [G, F]
    scale = (amax / CODE_MAX).astype(np.float16)         # fp16, nearest-even
    s64 = scale.astype(F64)[:, None, :]
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(s64 > 0, wg / s64, 0.0)
    q = np.clip(np.rint(ratio), -CODE_MAX, CODE_MAX).astype(np.int8)
    return q.reshape(d, f), scale


def dequantize_proxy(q, scale, group=GROUP, rows=None):
    """W~ = Q * S broadcast over each group's rows (optionally only ``rows``)."""
    q = np.asarray(q)
    s = np.asarray(scale).astype(F64)
    if rows is None:
        return q.astype(F64) * np.repeat(s, group, axis=0)
    rows = np.asarray(rows, dtype=np.int64)
    return q[rows].astype(F64) * s[rows // group]


def code_near_tie(w, scale, group=GROUP, eps=2.0 ** -20):
    """Mask of weights whose W/S lies within ``eps`` of a rounding midpoint.

    Codes there may legitimately differ between an fp32 and an exact division.
    """
    w = np.asarray(w, dtype=F64)
    d, f = w.shape
    s = np.repeat(np.asarray(scale).astype(F64), group, axis=0)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(s > 0, w / s, 0.0)
    frac = np.abs(r - np.floor(r) - 0.5)
    return (s > 0) & (frac < eps)


def pack_nibbles(q):
    """Byte layout of the packed codes: byte b of row i holds channel 2b in its
    low nibble and channel 2b+1 in its high nibble, each as offset-binary q + 8."""
    u = (np.asarray(q).astype(np.int16) + 8).astype(np.uint8)
    return (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(b):
    b = np.asarray(b, dtype=np.uint8)
    d, half = b.shape
    q = np.empty((d, 2 * half), dtype=np.int8)
    q[:, 0::2] = (b & 0x0F).astype(np.int16) - 8
    q[:, 1::2] = (b >> 4).astype(np.int16) - 8
    return q


# ---------------------------------------------------------------------------
# Threshold calibration (Prox App. A.7, "Calibration data and scale")
# ---------------------------------------------------------------------------

def calibrate_tau(x_cal, s1):
    """Per-layer input threshold: the empirical s1-quantile of |x| over the
    calibration activations (Prox App. A.7).

    Exact lower order statistic at 0-based rank floor(s1 * n) of all n values;
    s1 = 0 gives tau = 0 (keep every input).  Returned as float32, the type the
    comparison |x_i| >= tau is made in.
    """
    s1 = np.float32(s1)
    if not (0.0 <= s1 <= 1.0):
        raise ValueError("s1 must be in [0, 1]")
    if s1 == 0:
        return np.float32(0.0)
    v = np.sort(np.abs(np.asarray(x_cal, dtype=np.float32)).ravel())
    if v.size == 0:
        raise ValueError("empty calibration set")
    r = min(int(np.floor(F64(s1) * v.size)), v.size - 1)
    return np.float32(v[r])


# ---------------------------------------------------------------------------
# Stage 1: input mask, INT4 proxy, proxy intermediate state (Prox §4.1)
# ---------------------------------------------------------------------------

def input_mask(x, tau):
    """I(m_x) for [m_x]_i = 1[|x_i| >= tau]  (Prox §4.1, Stage-1 input mask).

    Returned as ascending indices; the comparison is made in float32.
    """
    x = np.asarray(x, dtype=np.float32)
    return np.nonzero(np.abs(x) >= np.float32(tau))[0].astype(np.int64)


def proxy_intermediate(x, tau, q_gate, s_gate, q_up, s_up, group=GROUP, act="silu"):
    """Stage-1 proxy (Prox §4.1):
    u~ = Π_in(x, W~_up, m_x),  h~ = SiLU(Π_in(x, W~_gate, m_x)),  s~ = u~ ⊙ h~.

    Returns ``(idx_x, g~, u~, s~)`` where g~ is the gate pre-activation
    Π_in(x, W~_gate, m_x).
    """
    idx_x = input_mask(x, tau)
    x64 = np.asarray(x, dtype=F64)
    wg = dequantize_proxy(q_gate, s_gate, group, rows=idx_x)
    wu = dequantize_proxy(q_up, s_up, group, rows=idx_x)
    g_t = x64[idx_x] @ wg
    u_t = x64[idx_x] @ wu
    s_t = u_t * ACTIVATIONS[act](g_t)
    return idx_x, g_t, u_t, s_t


def proxy_scores(g_tilde, u_tilde, act="silu"):
    """Channel salience |s~_j| = |SiLU(g~_j) u~_j|  (Prox §4.1)."""
    return np.abs(ACTIVATIONS[act](g_tilde) * np.asarray(u_tilde, dtype=F64))


def topk_channels(scores, k):
    """TopKIndices(|z|, k) of Prox App. A.6 ("Per-token top-k selection").

    Larger score first, equal scores to the lower index; the k chosen indices
    are returned in ascending order.
    """
    scores = np.asarray(scores, dtype=F64)
    f = scores.size
    if not (0 <= k <= f):
        raise ValueError("k must be in [0, d_ff]")
    order = np.lexsort((np.arange(f), -scores))
    return np.sort(order[:k]).astype(np.int64)


def threshold_channels(scores, tau_s):
    """Threshold rule [m_s]_j = 1[|s~_j| >= tau_s]  (Prox §4.1, Stage-2 mask)."""
    return np.nonzero(np.asarray(scores, dtype=F64) >= F64(tau_s))[0].astype(np.int64)


def calibrate_tau_s(x_cal, tau_x, q_gate, s_gate, q_up, s_up, s2, group=GROUP, act="silu"):
    """Stage-2 score threshold (Prox App. A.7, Algorithm 1, steps 5-6): with the
    layer's input threshold fixed, the proxy scores |s~| of every calibration
    token, and their s2-quantile (the same exact lower order statistic as the
    input threshold, over the scores held as fp32)."""
    rows = []
    for x in np.asarray(x_cal):
        _, g_t, u_t, _ = proxy_intermediate(x, tau_x, q_gate, s_gate, q_up, s_up, group, act)
        rows.append(proxy_scores(g_t, u_t, act))
    return calibrate_tau(np.asarray(rows, dtype=np.float32), s2)


# ---------------------------------------------------------------------------
# Stage 2: exact computation of the selected channels (Prox §4.1)
# ---------------------------------------------------------------------------

def stage2(x, w_gate, w_up, w_down, idx_s, act="silu"):
    """Stage 2 (Prox §4.1):
    u_sp = Π_out(x, W_up, m_s), h_sp = SiLU(Π_out(x, W_gate, m_s)),
    s_sp = u_sp ⊙ h_sp,  y = Π_in(s_sp, W_down, m_s)  with the full x.

    Returns ``(y, s_sp)``; s_sp is indexed like ``idx_s``.
    """
    idx_s = np.asarray(idx_s, dtype=np.int64)
    u_sp = pi_out(x, w_up, idx_s)
    h_sp = ACTIVATIONS[act](pi_out(x, w_gate, idx_s))
    s_sp = u_sp * h_sp
    y = s_sp @ np.asarray(w_down)[idx_s, :].astype(F64)
    return y, s_sp


def stage2_proxy_values(w_down, idx_s, s_tilde):
    """Ablation A3 of Prox §5.2: no exact recomputation; the selected proxy
    values s~_j go straight into the down projection,
    y = Π_in(s~, W_down, m_s) = sum_{j in idx_s} s~_j W_down[j, :]."""
    idx_s = np.asarray(idx_s, dtype=np.int64)
    s_sel = np.asarray(s_tilde, dtype=F64)[idx_s]
    return s_sel @ np.asarray(w_down)[idx_s, :].astype(F64)


def oracle_s_mask(x, w_gate, w_up, k):
    """oracle-s of Prox §3.1: the k channels of the exact s with the largest
    magnitude (same tie rule as ``topk_channels``)."""
    return topk_channels(np.abs(intermediate_state(x, w_gate, w_up)), k)


# ---------------------------------------------------------------------------
# The whole decode step for one token
# ---------------------------------------------------------------------------

def prox_ffn(x, w_gate, w_up, w_down, q_gate, s_gate, q_up, s_up, tau, k,
             group=GROUP, tau_s=None, act="silu", proxy_values=False):
    """One token through both stages (Prox §4.1, with the top-k mask of App. A.6
    unless ``tau_s`` selects the §4.1 threshold rule; ``act`` the gate
    activation; ``proxy_values`` the A3 ablation of §5.2 in place of Stage 2).
    Returns a dict with idx_x, g_tilde, u_tilde, s_tilde, scores, idx_s, s_sp
    (None under A3) and y."""
    idx_x, g_t, u_t, s_t = proxy_intermediate(x, tau, q_gate, s_gate, q_up, s_up, group, act)
    scores = proxy_scores(g_t, u_t, act)
    if tau_s is None:
        idx_s = topk_channels(scores, k)
    else:
        idx_s = threshold_channels(scores, tau_s)
    if proxy_values:
        y, s_sp = stage2_proxy_values(w_down, idx_s, s_t), None
    else:
        y, s_sp = stage2(x, w_gate, w_up, w_down, idx_s, act)
    return dict(idx_x=idx_x, g_tilde=g_t, u_tilde=u_t, s_tilde=s_t, scores=scores,
                idx_s=idx_s, s_sp=s_sp, y=y)


def rmsnorm(y, eps=1e-6):
    """Unit-gain RMSNorm between stacked layers: y / sqrt(mean(y^2) + eps).

    Not part of the paper's FFN; used to chain synthetic layers.
    """
    y = np.asarray(y, dtype=F64)
    return y / np.sqrt(np.mean(y * y) + eps)


# ---------------------------------------------------------------------------
# A stack of layers (the synthetic multi-layer workload)
# ---------------------------------------------------------------------------

def stack_next_input(y, eps=1e-6):
    """Input of the next stacked layer: RMSNorm of the output, held in fp32 like
    every layer input."""
    return np.asarray(rmsnorm(y, eps), dtype=np.float32)


def calibrate_stack(layers, x_cal, s1, k, group=GROUP, eps=1e-6, s2=None):
    """Sequential threshold calibration (Prox App. A.7, Algorithm 1): layer l's
    input threshold is the s1-quantile of its own inputs, which are the
    calibration tokens run through layers 1..l-1 with their finalised rules
    (the current layer's inputs are collected before its own rule is fixed).
    With ``s2`` given, the layer's Stage-2 rule is the score threshold tau_s,
    the s2-quantile of its proxy scores (steps 5-6); otherwise it is top-k.

    ``layers``: sequence of (w_gate, w_up, w_down, q_gate, s_gate, q_up, s_up).
    Returns (taus, inputs) -- or (taus, taus_s, inputs) with ``s2`` -- the
    thresholds of every layer and the calibration inputs each layer saw.
    """
    x = np.asarray(x_cal, dtype=np.float32)
    taus, taus_s, inputs = [], [], []
    for li, (wg, wu, wd, qg, sg, qu, su) in enumerate(layers):
        inputs.append(x)
        tau = calibrate_tau(x, s1)
        taus.append(tau)
        tau_s = None
        if s2 is not None:
            tau_s = calibrate_tau_s(x, tau, qg, sg, qu, su, s2, group)
            taus_s.append(tau_s)
        if li + 1 < len(layers):
            ys = [prox_ffn(xt, wg, wu, wd, qg, sg, qu, su, tau=tau, k=k, group=group,
                           tau_s=tau_s)["y"] for xt in x]
            x = np.stack([stack_next_input(yt, eps) for yt in ys])
    if s2 is not None:
        return taus, taus_s, inputs
    return taus, inputs


def stack_forward(layers, taus, x, k, group=GROUP, eps=1e-6, taus_s=None):
    """One token through the stack: the Prox step of every layer (top-k, or
    the score threshold taus_s[l] when given), RMSNorm in between.  Returns
    the per-layer inputs and the last layer's output."""
    xs = []
    x = np.asarray(x, dtype=np.float32)
    y = None
    for li, ((wg, wu, wd, qg, sg, qu, su), tau) in enumerate(zip(layers, taus)):
        xs.append(x)
        tau_s = None if taus_s is None else taus_s[li]
        y = prox_ffn(x, wg, wu, wd, qg, sg, qu, su, tau=tau, k=k, group=group, tau_s=tau_s)["y"]
        if li + 1 < len(layers):
            x = stack_next_input(y, eps)
    return xs, y


# ---------------------------------------------------------------------------
# Cost model, allocation policy and runtime sparsity (Prox §4.2, App. A.4, A.7)
# ---------------------------------------------------------------------------

C_DENSE = 3.0  # gate, up and down projections at one unit each (Prox §4.2)


def prox_cost(s1, s2, alpha):
    """Normalised Prox FFN cost (Prox §4.2): two INT4 proxy projections of
    relative cost alpha over the kept (1 - s1) inputs plus three exact
    projections over the kept (1 - s2) channels."""
    return 2.0 * F64(alpha) * (1.0 - F64(s1)) + 3.0 * (1.0 - F64(s2))


def effective_sparsity(s1, s2, alpha):
    """e = 1 - C_Prox / C_Dense  (Prox §4.2)."""
    return 1.0 - prox_cost(s1, s2, alpha) / C_DENSE


def allocate_sparsity(e, alpha=1.0 / 3.0, s_ref=0.7, s1_min=0.0, s1_max=0.7):
    """Allocation policy of Prox §4.2 (operating points of App. A.4).

    Keep Stage 2 at the anchor s_ref and give Stage 1 whatever input sparsity
    makes the cost meet the budget C_Prox = C_Dense (1 - e); when that s1 is
    outside [s1_min, s1_max], pin s1 to the nearer bound and let s2 take up
    the budget instead.  Raises ValueError when no s2 in [0, 1] does.
    """
    e, alpha = F64(e), F64(alpha)
    if not alpha > 0:
        raise ValueError("alpha must be > 0")
    budget = C_DENSE * (1.0 - e)
    # Stage-1 share of the budget with s2 = s_ref: 2 alpha (1 - s1) = budget - 3 (1 - s_ref)
    s1 = 1.0 - (budget - 3.0 * (1.0 - F64(s_ref))) / (2.0 * alpha)
    if s1_min <= s1 <= s1_max:
        return float(s1), float(s_ref)
    s1 = F64(s1_min) if s1 < s1_min else F64(s1_max)
    # remaining budget for Stage 2: 3 (1 - s2) = budget - 2 alpha (1 - s1)
    s2 = 1.0 - (budget - 2.0 * alpha * (1.0 - s1)) / 3.0
    if not 0.0 <= s2 <= 1.0:
        raise ValueError(f"target e={float(e)} is out of reach with s1={float(s1)}")
    return float(s1), float(s2)


def runtime_sparsity(sum_nx, sum_sel, tokens, d_model, d_ff, alpha=1.0 / 3.0):
    """Realised (s1^, s2^, e^) from accumulated mask counts (Prox App. A.7,
    "Runtime sparsity"): the kept fractions of inputs and channels over all
    tokens, then the cost model of §4.2."""
    s1 = 1.0 - F64(sum_nx) / (F64(tokens) * d_model)
    s2 = 1.0 - F64(sum_sel) / (F64(tokens) * d_ff)
    return float(s1), float(s2), float(effective_sparsity(s1, s2, alpha))
