"""Pins for the fp64 oracle: each test ties an oracle function to something
other than itself -- a value printed in the paper, a closed form, a library
routine, an exact special case, or brute force on tiny inputs.

Paper: "Prox: Training-Free FFN Activation Sparsity via Approximate
Intermediate-Channel Salience in LLMs".
"""

import itertools
import os
import struct

import numpy as np
import pytest
from scipy import optimize, special, stats

from oracle import prox_oracle as orc
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if line:
                key, p, val = line.split()
                out[key] = (float(p), float(val))
    return out


# ---------------------------------------------------------------------------
# SwiGLU and the dense FFN (§2.1)
# ---------------------------------------------------------------------------

def test_silu_equals_z_times_logistic():
    z = np.concatenate([np.linspace(-50, 50, 2001), [-745.0, -1e3, 0.0, 1e-300, 700.0]])
    ref = z * special.expit(z)
    np.testing.assert_allclose(orc.silu(z), ref, rtol=1e-14, atol=1e-300)
    assert orc.silu(0.0) == 0.0


def test_dense_ffn_with_permutation_weights_is_elementwise():
    # W_up = P1, W_gate = c * P2, W_down = P3 are permutation matrices, so the
    # FFN reduces to an index shuffle of scalar SwiGLUs:
    # y[p3(j)] = x[p1^-1(j)] * SiLU(c * x[p2^-1(j)]).  A transposed operand or a
    # swapped branch changes the result.
    rng = np.random.default_rng(0)
    n = 7
    x = rng.standard_normal(n)
    p1, p2, p3 = (rng.permutation(n) for _ in range(3))
    c = 1.7
    w_up = np.zeros((n, n)); w_up[p1, np.arange(n)] = 1.0     # x@W_up [j] = x[p1[j]]
    w_gate = np.zeros((n, n)); w_gate[p2, np.arange(n)] = c
    w_down = np.zeros((n, n)); w_down[np.arange(n), p3] = 1.0  # s@W_down [p3[j]] = s[j]
    y = orc.dense_ffn(x, w_gate, w_up, w_down)
    expect = np.zeros(n)
    for j in range(n):
        z = c * x[p2[j]]
        expect[p3[j]] = x[p1[j]] * (z * special.expit(z))
    np.testing.assert_allclose(y, expect, rtol=1e-13, atol=1e-15)


def test_weighted_sum_view_of_the_ffn():
    # §3.1: FFN(x) = sum_i s_i W_down[i, :], evaluated as an explicit row loop.
    lay = synth.make_layer(_small_cfg(256, 96), n_tokens=2)
    x = lay.x_eval[0]
    s = orc.intermediate_state(x, lay.w_gate, lay.w_up)
    acc = np.zeros(lay.d_model)
    for i in range(lay.d_ff):
        acc += s[i] * lay.w_down[i].astype(np.float64)
    np.testing.assert_allclose(orc.dense_ffn(x, lay.w_gate, lay.w_up, lay.w_down), acc,
                               rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------------------
# Sparsity operators (§2.2) and the Appendix A.2 closed forms
# ---------------------------------------------------------------------------

def test_pi_in_and_pi_out_against_masked_matmul():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(40)
    w = rng.standard_normal((40, 30))
    idx = np.sort(rng.choice(40, 17, replace=False))
    xm = np.zeros(40); xm[idx] = x[idx]
    np.testing.assert_allclose(orc.pi_in(x, w, idx), xm @ w, rtol=1e-13, atol=1e-13)
    cols = np.array([29, 3, 3, 0])
    np.testing.assert_allclose(orc.pi_out(x, w, cols), (x @ w)[cols], rtol=1e-13)


def test_gaussian_input_sparsity_closed_forms():
    # Appendix A.2: X ~ N(0,1), prune the fraction p=0.7 of smallest |X|,
    # isotropic Gaussian weights.  Retained energy q_G, relative projection
    # error eta and correlation sqrt(q_G) are printed for p = 0.7.
    g = _golden("closed_forms_appendix_a2.txt")
    p = g["q_gauss"][0]
    rng = np.random.default_rng(2)
    d, n_out, n_tok = 2048, 256, 24
    w = rng.standard_normal((d, n_out))
    tau = stats.norm.ppf((1 + p) / 2)
    kept_energy, err2, y2, ys, yts = 0.0, 0.0, 0.0, [], []
    tot_energy = 0.0
    for _ in range(n_tok):
        x = rng.standard_normal(d).astype(np.float32)
        idx = orc.input_mask(x, tau)
        kept_energy += float(np.sum(x[idx].astype(np.float64) ** 2))
        tot_energy += float(np.sum(x.astype(np.float64) ** 2))
        y = orc.pi_in(x, w, np.arange(d))
        yt = orc.pi_in(x, w, idx)
        err2 += float(np.sum((y - yt) ** 2)); y2 += float(np.sum(y ** 2))
        ys.append(y); yts.append(yt)
    q = kept_energy / tot_energy
    eta = np.sqrt(err2 / y2)
    corr = np.corrcoef(np.concatenate(ys), np.concatenate(yts))[0, 1]
    assert abs(q - g["q_gauss"][1]) < 0.01
    assert abs(eta - g["eta_gauss"][1]) < 0.01
    assert abs(corr - g["corr_gauss"][1]) < 0.01
    # and the printed values are the closed forms themselves
    z = stats.norm.ppf((1 + p) / 2)
    qg = 1 - p + 2 * z * stats.norm.pdf(z)
    # printed to three decimals
    assert abs(qg - g["q_gauss"][1]) < 1e-3
    assert abs(np.sqrt(1 - qg) - g["eta_gauss"][1]) < 1e-3
    assert abs(np.sqrt(qg) - g["corr_gauss"][1]) < 1e-3


def test_laplace_energy_retention_through_topk():
    # Appendix A.2: keeping the top 30% magnitudes of Laplace samples keeps
    # q_Lap(0.7) = 87.9% of the squared energy.
    g = _golden("closed_forms_appendix_a2.txt")
    p, printed = g["q_lap"]
    rng = np.random.default_rng(3)
    s = rng.laplace(0, 1, 400_000)
    k = int(round((1 - p) * s.size))
    keep = orc.topk_channels(np.abs(s), k)
    q = np.sum(s[keep] ** 2) / np.sum(s ** 2)
    assert abs(q - printed) < 0.005
    a = -np.log(1 - p)
    assert abs((1 - p) / 2 * (a * a + 2 * a + 2) - printed) < 1e-3


# ---------------------------------------------------------------------------
# INT4 proxy quantisation (§4.3, group-128 reading)
# ---------------------------------------------------------------------------

def _grid_weights(rng, d, f, group=128):
    """Weights that lie exactly on a symmetric INT4 grid with power-of-two
    scales and at least one +/-7 code per (group, channel)."""
    g = d // group
    exps = rng.integers(-9, -5, size=(g, f))
    scale = np.ldexp(1.0, exps)
    codes = rng.integers(-7, 8, size=(g, group, f))
    pos = rng.integers(0, group, size=(g, f))
    sign = rng.choice([-7, 7], size=(g, f))
    for gi in range(g):
        codes[gi, pos[gi], np.arange(f)] = sign[gi]
    w = codes * scale[:, None, :]
    return w.reshape(d, f).astype(np.float32), codes.reshape(d, f), scale


def test_quantize_exact_grid_roundtrip():
    rng = np.random.default_rng(4)
    w, codes, scale = _grid_weights(rng, 256, 40)
    q, s = orc.quantize_proxy(w)
    np.testing.assert_array_equal(s.astype(np.float64), scale)
    np.testing.assert_array_equal(q, codes)
    np.testing.assert_array_equal(orc.dequantize_proxy(q, s), w.astype(np.float64))


def test_quantize_round_half_even_and_zero_group():
    w = np.zeros((128, 3), dtype=np.float32)
    sc = 2.0 ** -7
    col = np.array([7, 2.5, 3.5, -2.5, -3.5, 0.5, -0.5, 1.5, 6.5, -6.5])
    w[: col.size, 0] = col * sc
    w[0, 2] = -7 * sc
    w[5, 2] = 4.5 * sc  # column 1 stays all-zero
    q, s = orc.quantize_proxy(w)
    assert float(s[0, 0]) == sc and float(s[0, 1]) == 0.0 and float(s[0, 2]) == sc
    np.testing.assert_array_equal(q[: col.size, 0], [7, 2, 4, -2, -4, 0, 0, 2, 6, -6])
    assert np.all(q[:, 1] == 0)
    assert q[0, 2] == -7 and q[5, 2] == 4


def test_scale_is_fp16_nearest_even_of_amax_over_7():
    lay = synth.make_layer(_small_cfg(256, 64), draw_tokens=False)
    q, s = orc.quantize_proxy(lay.w_gate)
    amax = np.abs(lay.w_gate.astype(np.float64).reshape(2, 128, 64)).max(axis=1)
    # struct's 'e' format rounds a double to IEEE half, nearest-even.
    ref = np.array([[struct.unpack("<e", struct.pack("<e", v / 7.0))[0] for v in row]
                    for row in amax])
    np.testing.assert_array_equal(s.astype(np.float64), ref)


def test_quantize_invariants_on_random_weights():
    lay = synth.make_layer(_small_cfg(384, 160), draw_tokens=False)
    w = lay.w_up.astype(np.float64)
    q, s = orc.quantize_proxy(lay.w_up)
    assert q.min() >= -7 and q.max() <= 7
    s_rows = np.repeat(s.astype(np.float64), 128, axis=0)
    # |W - Q S| <= S/2 up to the fp16 rounding of S (relative 2^-11 of 7 S)
    err = np.abs(w - q * s_rows)
    assert np.all(err <= s_rows * (0.5 + 7 * 2.0 ** -11) + 1e-30)
    # the element that sets amax gets code +/-7 (ties of the fp16 scale aside)
    wg = np.abs(w).reshape(3, 128, 160)
    arg = wg.argmax(axis=1)
    for gi in range(3):
        codes = q.reshape(3, 128, 160)[gi, arg[gi], np.arange(160)]
        assert np.all(np.abs(codes) == 7)


def test_nibble_packing_layout():
    q = np.array([[-7, 7, 0, -8 + 1, 3, -3]], dtype=np.int8)
    b = orc.pack_nibbles(q)
    # channel 0 -> low nibble of byte 0 (-7+8 = 1), channel 1 -> high nibble (15)
    assert b.tolist() == [[0xF1, 0x18, 0x5B]]
    np.testing.assert_array_equal(orc.unpack_nibbles(b), q)


# ---------------------------------------------------------------------------
# Calibration (Appendix A.7) and the input mask (§4.1)
# ---------------------------------------------------------------------------

def test_calibrate_hand_example_and_special_cases():
    x = np.array([[0.1, -0.5], [0.3, 0.2]], dtype=np.float32)
    assert orc.calibrate_tau(x, 0.5) == np.float32(0.3)   # sorted |x|: .1 .2 .3 .5
    assert orc.calibrate_tau(x, 0.25) == np.float32(0.2)
    assert orc.calibrate_tau(x, 0.0) == 0.0
    assert orc.calibrate_tau(x, 1.0) == np.float32(0.5)


def test_calibrated_threshold_keeps_the_exact_fraction():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((64, 512)).astype(np.float32)
    for s1 in (0.4, 0.5, 0.6):
        tau = orc.calibrate_tau(x, s1)
        kept = int(np.sum(np.abs(x) >= tau))
        r = int(np.floor(np.float64(np.float32(s1)) * x.size))
        assert kept == x.size - r


@pytest.mark.parametrize("cfg_name,s1", [("tiny", 0.5), ("llama3_8b", 0.5),
                                         ("llama3_8b", 0.4), ("llama3_8b", 0.6)])
def test_calibrated_threshold_matches_mixture_quantile(cfg_name, s1):
    # |x| of Laplace(0,1) with a fixed fraction f of channels scaled by c has
    # CDF (1-f)(1-e^-t) + f(1-e^{-t/c}); the empirical quantile must sit at its root.
    cfg = synth.get_config(cfg_name)
    rng = np.random.Generator(np.random.PCG64(cfg.seed(0)))
    outl = synth.outlier_channels(rng, cfg.d_model, cfg.n_outliers)
    x = rng.laplace(0, 1, size=(256, cfg.d_model)).astype(np.float32)
    x[:, outl] *= np.float32(cfg.outlier_scale)
    f = cfg.n_outliers / cfg.d_model
    c = cfg.outlier_scale
    root = optimize.brentq(lambda t: (1 - f) * (1 - np.exp(-t)) + f * (1 - np.exp(-t / c)) - s1,
                           0, 50)
    tau = orc.calibrate_tau(x, s1)
    assert abs(tau - root) < 0.01


def test_input_mask_keeps_equality():
    x = np.array([0.5, -0.5, 0.49999997, -2.0, 0.0], dtype=np.float32)
    np.testing.assert_array_equal(orc.input_mask(x, np.float32(0.5)), [0, 1, 3])
    np.testing.assert_array_equal(orc.input_mask(x, 0.0), [0, 1, 2, 3, 4])


# ---------------------------------------------------------------------------
# Stage 1 proxy (§4.1) in the exact case
# ---------------------------------------------------------------------------

def test_proxy_equals_exact_projection_on_grid_weights():
    # With weights exactly on the INT4 grid the proxy is the exact projection
    # of the masked input: g~ = (x ⊙ m_x) W_gate, u~ = (x ⊙ m_x) W_up.
    rng = np.random.default_rng(6)
    wg, _, _ = _grid_weights(rng, 256, 64)
    wu, _, _ = _grid_weights(rng, 256, 64)
    qg, sg = orc.quantize_proxy(wg)
    qu, su = orc.quantize_proxy(wu)
    x = rng.laplace(0, 1, 256).astype(np.float32)
    for tau in (np.float32(0.0), np.float32(0.8)):
        idx, g_t, u_t, s_t = orc.proxy_intermediate(x, tau, qg, sg, qu, su)
        m = (np.abs(x) >= tau).astype(np.float64)
        xm = x.astype(np.float64) * m
        np.testing.assert_allclose(g_t, xm @ wg.astype(np.float64), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(u_t, xm @ wu.astype(np.float64), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(s_t, (xm @ wu) * (xm @ wg) * special.expit(xm @ wg),
                                   rtol=1e-11, atol=1e-12)
    # tau = 0 and grid weights: the proxy ranking is the exact oracle-s ranking
    k = 20
    _, g_t, u_t, _ = orc.proxy_intermediate(x, 0.0, qg, sg, qu, su)
    np.testing.assert_array_equal(orc.topk_channels(orc.proxy_scores(g_t, u_t), k),
                                  orc.oracle_s_mask(x, wg, wu, k))


def test_ranking_preservation_condition():
    # Appendix A.2: the order of i, j under |s| and |s~| is unchanged whenever
    # ||s_i| - |s_j|| > |delta_i| + |delta_j|.  Every flip must violate it.
    lay = synth.make_layer(_small_cfg(256, 128), n_tokens=3)
    qg, sg = orc.quantize_proxy(lay.w_gate)
    qu, su = orc.quantize_proxy(lay.w_up)
    tau = orc.calibrate_tau(lay.x_cal, 0.5)
    flips = 0
    for x in lay.x_eval:
        s = orc.intermediate_state(x, lay.w_gate, lay.w_up)
        _, _, _, st = orc.proxy_intermediate(x, tau, qg, sg, qu, su)
        a, b = np.abs(s), np.abs(st)
        delta = np.abs(st - s)
        flip = np.sign(a[:, None] - a[None, :]) * np.sign(b[:, None] - b[None, :]) < 0
        bound = np.abs(a[:, None] - a[None, :]) > delta[:, None] + delta[None, :]
        assert not np.any(flip & bound)
        flips += int(flip.sum())
    assert flips > 0  # the check is not vacuous


# ---------------------------------------------------------------------------
# Per-token top-k (Appendix A.6): brute force on tiny inputs
# ---------------------------------------------------------------------------

def _topk_brute(scores, k):
    f = len(scores)
    valid = []
    for sub in itertools.combinations(range(f), k):
        inside = set(sub)
        ok = all(scores[i] > scores[j] or (scores[i] == scores[j] and i < j)
                 for i in inside for j in range(f) if j not in inside)
        if ok:
            valid.append(sub)
    assert len(valid) == 1
    return list(valid[0])


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(7)
    for trial in range(60):
        f = int(rng.integers(1, 11))
        scores = rng.integers(0, 4, f).astype(np.float64) * 0.25  # many ties
        if trial % 3 == 0:
            scores = rng.random(f)
        for k in range(0, f + 1):
            got = orc.topk_channels(scores, k).tolist()
            assert got == _topk_brute(list(scores), k)


def test_threshold_rule_keeps_equality():
    s = np.array([0.1, 0.5, 0.5, 0.7, 0.0])
    np.testing.assert_array_equal(orc.threshold_channels(s, 0.5), [1, 2, 3])


# ---------------------------------------------------------------------------
# Stage 2 (§4.1) and the whole step
# ---------------------------------------------------------------------------

def _small_cfg(d, f, idx=90):
    return synth.WorkloadConfig(name=f"t{d}x{f}", index=idx, d_model=d, d_ff=f, sigma=0.05,
                                outlier_frac=0.01, outlier_scale=20.0, s1_percent=(50,),
                                s2_percent=(70,), n_tokens=4, n_cal=32)


def _packed(lay):
    qg, sg = orc.quantize_proxy(lay.w_gate)
    qu, su = orc.quantize_proxy(lay.w_up)
    return qg, sg, qu, su


def test_keep_all_equals_dense():
    # s1 = 0 (tau = 0) and k = d_ff: Stage 2 computes every channel exactly.
    lay = synth.make_layer(_small_cfg(256, 96), n_tokens=3)
    qg, sg, qu, su = _packed(lay)
    for x in lay.x_eval:
        r = orc.prox_ffn(x, lay.w_gate, lay.w_up, lay.w_down, qg, sg, qu, su,
                         tau=0.0, k=lay.d_ff)
        assert r["idx_x"].size == lay.d_model and r["idx_s"].size == lay.d_ff
        np.testing.assert_allclose(r["y"], orc.dense_ffn(x, lay.w_gate, lay.w_up, lay.w_down),
                                   rtol=1e-12, atol=1e-14)


def test_stage2_is_dense_with_s_zeroed_off_the_mask():
    lay = synth.make_layer(_small_cfg(256, 96), n_tokens=2)
    x = lay.x_eval[1]
    idx = np.array([0, 5, 17, 18, 95])
    y, s_sp = orc.stage2(x, lay.w_gate, lay.w_up, lay.w_down, idx)
    s = orc.intermediate_state(x, lay.w_gate, lay.w_up)
    np.testing.assert_allclose(s_sp, s[idx], rtol=1e-13)
    acc = np.zeros(lay.d_model)
    for j in idx:
        acc += s[j] * lay.w_down[j].astype(np.float64)
    np.testing.assert_allclose(y, acc, rtol=1e-12, atol=1e-15)


def test_stage2_uses_the_full_input():
    # Even when Stage 1 drops every input (tau above max |x|) the selected
    # channels are computed from the dense x.
    lay = synth.make_layer(_small_cfg(256, 96), n_tokens=1)
    qg, sg, qu, su = _packed(lay)
    x = lay.x_eval[0]
    r = orc.prox_ffn(x, lay.w_gate, lay.w_up, lay.w_down, qg, sg, qu, su,
                     tau=np.float32(1e9), k=10)
    assert r["idx_x"].size == 0
    np.testing.assert_array_equal(r["scores"], 0.0)
    np.testing.assert_array_equal(r["idx_s"], np.arange(10))  # ties -> lowest indices
    s = orc.intermediate_state(x, lay.w_gate, lay.w_up)
    np.testing.assert_allclose(r["s_sp"], s[:10], rtol=1e-13)


def test_rmsnorm_closed_form():
    c, eps = 0.37, 1e-6
    y = np.full(64, c)
    np.testing.assert_allclose(orc.rmsnorm(y, eps), c / np.sqrt(c * c + eps), rtol=1e-15)
    z = np.random.default_rng(8).standard_normal(4096) * 3
    assert abs(np.sqrt(np.mean(orc.rmsnorm(z, 0.0) ** 2)) - 1) < 1e-14


# ---------------------------------------------------------------------------
# the layer stack (sequential calibration, Prox App. A.7 Algorithm 1)
# ---------------------------------------------------------------------------

def _small_stack(n_layers=3, d=256, f=384, n_cal=24, n_tok=2):
    from synth.configs import WorkloadConfig
    cfg = WorkloadConfig(name="stack_small", index=61, d_model=d, d_ff=f, sigma=0.05,
                         outlier_frac=0.01, outlier_scale=20.0, s1_percent=(50,),
                         s2_percent=(70,), n_tokens=n_tok, n_cal=n_cal, n_layers=n_layers)
    layers = []
    x_cal = x_eval = None
    for li in range(n_layers):
        lay = synth.make_layer(cfg, li, draw_tokens=(li == 0))
        if li == 0:
            x_cal, x_eval = lay.x_cal, lay.x_eval
        qg, sg = orc.quantize_proxy(lay.w_gate)
        qu, su = orc.quantize_proxy(lay.w_up)
        layers.append((lay.w_gate, lay.w_up, lay.w_down, qg, sg, qu, su))
    return cfg, layers, x_cal, x_eval


def test_stack_keep_all_is_the_dense_chain():
    # s1 = 0 and k = d_ff: every layer is the dense SwiGLU, chained by RMSNorm
    cfg, layers, x_cal, x_eval = _small_stack()
    taus, _ = orc.calibrate_stack(layers, x_cal, 0.0, cfg.d_ff)
    assert taus == [0.0] * len(layers)
    _, y = orc.stack_forward(layers, taus, x_eval[0], cfg.d_ff)
    x = x_eval[0].astype(np.float64)
    for li, (wg, wu, wd, *_rest) in enumerate(layers):
        h = orc.dense_ffn(x, wg, wu, wd)
        if li + 1 < len(layers):
            x = (h / np.sqrt(np.mean(h * h) + 1e-6)).astype(np.float32).astype(np.float64)
    np.testing.assert_allclose(y, h, rtol=1e-12, atol=1e-12)


def test_stack_threshold_rule_keep_all_is_the_dense_chain():
    # s1 = 0 and s2 = 0: every tau and tau_s is 0, the score threshold keeps
    # every channel (scores are >= 0), and the stack is the dense chain
    cfg, layers, x_cal, x_eval = _small_stack()
    taus, taus_s, _ = orc.calibrate_stack(layers, x_cal, 0.0, 1, s2=0.0)
    assert taus == [0.0] * len(layers) and taus_s == [0.0] * len(layers)
    _, y = orc.stack_forward(layers, taus, x_eval[1], 1, taus_s=taus_s)
    _, y_dense = orc.stack_forward(layers, taus, x_eval[1], cfg.d_ff)
    np.testing.assert_allclose(y, y_dense, rtol=1e-12, atol=1e-12)


def test_stack_every_layer_keeps_the_target_fraction_of_its_own_inputs():
    cfg, layers, x_cal, _ = _small_stack()
    taus, inputs = orc.calibrate_stack(layers, x_cal, 0.5, cfg.k())
    n = x_cal.size
    r = int(np.floor(0.5 * n))
    for tau, xin in zip(taus, inputs):
        # tau is the order statistic of rank r of this layer's own |x|
        a = np.abs(xin.astype(np.float64)).ravel()
        assert np.count_nonzero(a < tau) <= r < np.count_nonzero(a <= tau)
    # later layers see the earlier sparse layers' outputs, not the raw tokens
    assert not np.array_equal(inputs[1], inputs[0])


# ---------------------------------------------------------------------------
# the Stage-2 score threshold (Prox §4.1 mask, App. A.7 calibration)
# ---------------------------------------------------------------------------

def test_threshold_rule_keeps_ties_at_tau():
    s = np.array([0.5, 0.25, 0.5, 0.75, 0.0])
    np.testing.assert_array_equal(orc.threshold_channels(s, 0.5), [0, 2, 3])
    np.testing.assert_array_equal(orc.threshold_channels(s, 0.0), [0, 1, 2, 3, 4])
    assert orc.threshold_channels(s, 0.8).size == 0


def test_tau_s_is_the_order_statistic_of_the_calibration_scores():
    lay = synth.make_layer("tiny", n_tokens=1, n_cal=16)
    qg, sg = orc.quantize_proxy(lay.w_gate)
    qu, su = orc.quantize_proxy(lay.w_up)
    tau_x = orc.calibrate_tau(lay.x_cal, 0.5)
    tau_s = orc.calibrate_tau_s(lay.x_cal, tau_x, qg, sg, qu, su, 0.7)
    scores = []
    for x in lay.x_cal:
        _, g, u, _ = orc.proxy_intermediate(x, tau_x, qg, sg, qu, su)
        scores.append(orc.proxy_scores(g, u))
    v = np.asarray(scores, dtype=np.float32).ravel().astype(np.float64)
    r = int(np.floor(np.float64(np.float32(0.7)) * v.size))
    assert np.count_nonzero(v < tau_s) <= r < np.count_nonzero(v <= tau_s)
    # the threshold rule then keeps about 30 % of the calibration channels
    kept = np.count_nonzero(v >= tau_s) / v.size
    assert abs(kept - 0.3) < 0.01


def test_stack_with_threshold_rule_calibrates_both_thresholds():
    cfg, layers, x_cal, _ = _small_stack()
    taus, taus_s, inputs = orc.calibrate_stack(layers, x_cal, 0.5, cfg.k(), s2=0.7)
    assert len(taus) == len(taus_s) == len(inputs) == len(layers)
    assert all(t > 0 for t in taus_s)
    # layer 1's thresholds depend only on the raw calibration tokens
    wg, wu, wd, qg, sg, qu, su = layers[0]
    assert taus_s[0] == orc.calibrate_tau_s(x_cal, taus[0], qg, sg, qu, su, 0.7)


# ---------------------------------------------------------------------------
# Cost model and allocation policy (§4.2, App. A.4, App. A.7)
# ---------------------------------------------------------------------------

def _allocation_table():
    rows = []
    with open(os.path.join(GOLDEN, "allocation_appendix_a4.txt")) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if line:
                e, s1, s2, clamp = line.split()
                rows.append((float(e) / 100, None if s1 == "-" else float(s1) / 100,
                             float(s2) / 100, clamp))
    return rows


def test_allocation_matches_the_printed_operating_points():
    rows = _allocation_table()
    assert len(rows) == 4
    for e, s1_p, s2_p, clamp in rows:
        s1, s2 = orc.allocate_sparsity(e)
        assert abs(s2 - s2_p) <= 5e-4 + 1e-12, (e, s2, s2_p)  # printed to 0.1 %
        if s1_p is not None:
            assert abs(s1 - s1_p) <= 5e-4 + 1e-12, (e, s1, s1_p)
        if clamp == "no":
            assert 0.0 < s1 < 0.7 and s2 == 0.7
        else:
            assert s1 == (0.0 if clamp == "low" else 0.7)


def test_cost_model_special_cases():
    a = 1.0 / 3.0
    # nothing skipped and no proxy: the dense cost, e = 0
    assert orc.prox_cost(1.0, 0.0, a) == orc.C_DENSE
    assert orc.effective_sparsity(1.0, 0.0, a) == 0.0
    # every input dropped: the proxy is free and e is the Stage-2 sparsity
    for s2 in (0.0, 0.3, 0.7, 1.0):
        assert orc.effective_sparsity(1.0, s2, a) == pytest.approx(s2, abs=1e-15)
    # keep every input and every channel: the proxy's two projections come on top
    assert orc.effective_sparsity(0.0, 0.0, a) == pytest.approx(-2.0 / 9.0, abs=1e-15)
    # each term on its own: one unit per dense projection, alpha per proxy projection
    assert orc.prox_cost(0.0, 1.0, 0.25) == pytest.approx(0.5, abs=1e-15)
    assert orc.prox_cost(1.0, 2.0 / 3.0, 0.25) == pytest.approx(1.0, abs=1e-15)


def test_allocation_meets_the_budget_and_respects_the_bounds():
    a = 1.0 / 3.0
    for e in np.linspace(0.0, 0.9, 91):
        s1, s2 = orc.allocate_sparsity(e)
        assert 0.0 <= s1 <= 0.7 and 0.0 <= s2 <= 1.0
        assert orc.effective_sparsity(s1, s2, a) == pytest.approx(e, abs=1e-12)
        # s2 is the anchor unless s1 sits on a bound
        assert s2 == 0.7 or s1 in (0.0, 0.7)
    # the switch points: with s2 = 0.7, s1 = 0 at e = 0.7 - 2a/3 and s1 = 0.7 at e = 0.7 - 0.6a/3
    lo = 0.7 - 2 * a / 3
    hi = 0.7 - 2 * a * 0.3 / 3
    assert orc.allocate_sparsity(lo) == pytest.approx((0.0, 0.7), abs=1e-12)
    assert orc.allocate_sparsity(hi) == pytest.approx((0.7, 0.7), abs=1e-12)
    # monotone: a larger target never lowers either sparsity
    prev = (-1.0, -1.0)
    for e in np.linspace(0.0, 0.9, 181):
        cur = orc.allocate_sparsity(e)
        assert cur[0] >= prev[0] - 1e-12 and cur[1] >= prev[1] - 1e-12
        prev = cur
    # out of reach: s2 would have to exceed 1
    with pytest.raises(ValueError):
        orc.allocate_sparsity(0.99)
    with pytest.raises(ValueError):
        orc.allocate_sparsity(-0.5)


def test_runtime_sparsity_from_counted_masks():
    rng = np.random.default_rng(7)
    d, f, t = 256, 640, 37
    mx = rng.random((t, d)) < 0.45
    ms = rng.random((t, f)) < 0.28
    s1, s2, e = orc.runtime_sparsity(int(mx.sum()), int(ms.sum()), t, d, f)
    assert s1 == pytest.approx(np.mean(~mx), abs=1e-15)
    assert s2 == pytest.approx(np.mean(~ms), abs=1e-15)
    # e^ with the realised pair equals the budget identity of §4.2
    assert e == pytest.approx(1.0 - orc.prox_cost(s1, s2, 1.0 / 3.0) / 3.0, abs=1e-15)


# ---------------------------------------------------------------------------
# GeGLU gate (§5: Gemma-3's GeGLU FFN) and the A3 ablation (§5.2)
# ---------------------------------------------------------------------------

def test_gelu_is_z_times_the_normal_cdf():
    z = np.linspace(-12, 12, 2401)
    np.testing.assert_allclose(orc.gelu(z), z * stats.norm.cdf(z), rtol=1e-13, atol=1e-300)
    # textbook values: Phi(0) = 1/2, Phi(1) = 0.8413447460685429
    assert orc.gelu(0.0) == 0.0
    assert orc.gelu(1.0) == pytest.approx(0.8413447460685429, rel=1e-15)
    assert orc.gelu(-1.0) == pytest.approx(-(1 - 0.8413447460685429), rel=1e-14)


@pytest.mark.parametrize("act", ["gelu", "gelu_tanh", "silu"])
def test_gate_activation_symmetry(act):
    # z Phi(z) - (-z) Phi(-z) = z, and the same holds for the tanh form (tanh is
    # odd) and for SiLU (the logistic function has the same symmetry)
    f = orc.ACTIVATIONS[act]
    z = np.linspace(-9, 9, 1801)
    np.testing.assert_allclose(f(z) - f(-z), z, rtol=1e-13, atol=1e-13)


def test_gelu_tanh_form_tracks_the_exact_gelu():
    z = np.linspace(-8, 8, 16001)
    err = np.abs(orc.gelu_tanh(z) - orc.gelu(z))
    assert err.max() < 5e-4  # the tanh form's known accuracy, a few 1e-4
    assert err.max() > 1e-5  # ... and it is an approximation, not a copy
    # derivative 1/2 at 0 for both: (f(h) - f(-h)) / 2h -> 1/2 ... and f(h)/h -> 1/2
    h = 1e-6
    assert orc.gelu_tanh(h) / h == pytest.approx(0.5, abs=1e-6)


def test_geglu_ffn_with_permutation_weights_is_elementwise():
    rng = np.random.default_rng(1)
    n = 9
    x = rng.standard_normal(n)
    p1, p2, p3 = (rng.permutation(n) for _ in range(3))
    c = -0.8
    w_up = np.zeros((n, n)); w_up[p1, np.arange(n)] = 1.0
    w_gate = np.zeros((n, n)); w_gate[p2, np.arange(n)] = c
    w_down = np.zeros((n, n)); w_down[np.arange(n), p3] = 1.0
    for act in ("gelu", "gelu_tanh"):
        y = orc.dense_ffn(x, w_gate, w_up, w_down, act=act)
        expect = np.zeros(n)
        for j in range(n):
            z = c * x[p2[j]]
            g = z * stats.norm.cdf(z) if act == "gelu" else \
                0.5 * z * (1 + np.tanh(np.sqrt(2 / np.pi) * (z + 0.044715 * z ** 3)))
            expect[p3[j]] = x[p1[j]] * g
        np.testing.assert_allclose(y, expect, rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("act", ["gelu", "gelu_tanh"])
def test_geglu_keep_all_equals_dense(act):
    lay = synth.make_layer(_small_cfg(256, 96), n_tokens=2)
    qg, sg, qu, su = _packed(lay)
    for x in lay.x_eval:
        r = orc.prox_ffn(x, lay.w_gate, lay.w_up, lay.w_down, qg, sg, qu, su,
                         tau=0.0, k=lay.d_ff, act=act)
        np.testing.assert_allclose(
            r["y"], orc.dense_ffn(x, lay.w_gate, lay.w_up, lay.w_down, act=act),
            rtol=1e-12, atol=1e-14)


def test_a3_equals_exact_stage2_when_the_proxy_is_exact():
    # Grid weights and tau = 0: the proxy values are the exact s, so the A3
    # output is the Prox output on the same mask.
    rng = np.random.default_rng(11)
    d, f = 256, 64
    wg, _, _ = _grid_weights(rng, d, f)
    wu, _, _ = _grid_weights(rng, d, f)
    wd = rng.standard_normal((f, d)).astype(np.float32)
    qg, sg = orc.quantize_proxy(wg)
    qu, su = orc.quantize_proxy(wu)
    x = rng.laplace(0, 1, d).astype(np.float32)
    for act in ("silu", "gelu"):
        ex = orc.prox_ffn(x, wg, wu, wd, qg, sg, qu, su, tau=0.0, k=20, act=act)
        a3 = orc.prox_ffn(x, wg, wu, wd, qg, sg, qu, su, tau=0.0, k=20, act=act,
                          proxy_values=True)
        np.testing.assert_array_equal(a3["idx_s"], ex["idx_s"])
        assert a3["s_sp"] is None
        np.testing.assert_allclose(a3["y"], ex["y"], rtol=1e-11, atol=1e-11)


def test_a3_is_the_masked_sum_of_proxy_values():
    # With an input threshold the A3 output differs from Prox and is exactly
    # the W_down rows of the selected channels weighted by s~.
    lay = synth.make_layer(_small_cfg(256, 96), n_tokens=1)
    qg, sg, qu, su = _packed(lay)
    x = lay.x_eval[0]
    tau = orc.calibrate_tau(lay.x_cal, 0.5)
    a3 = orc.prox_ffn(x, lay.w_gate, lay.w_up, lay.w_down, qg, sg, qu, su, tau=tau, k=30,
                      proxy_values=True)
    ex = orc.prox_ffn(x, lay.w_gate, lay.w_up, lay.w_down, qg, sg, qu, su, tau=tau, k=30)
    acc = np.zeros(lay.d_model)
    for j in a3["idx_s"]:
        acc += a3["s_tilde"][j] * lay.w_down[j].astype(np.float64)
    np.testing.assert_allclose(a3["y"], acc, rtol=1e-12, atol=1e-15)
    assert np.linalg.norm(a3["y"] - ex["y"]) > 1e-3 * np.linalg.norm(ex["y"])


def test_mask_overlap_report_runs():
    # the reporting script behind the quoted synthetic overlap (not a pin:
    # the paper's figure is for trained weights)
    from oracle import mask_overlap
    k, ov = mask_overlap.overlap("tiny", 2, 0.5, 70)
    assert k == 413 and ov.shape == (2,)
    assert np.all((ov > 0.5) & (ov <= 1.0))
