"""GPU parity on the remaining workloads: the Qwen3-14B-shaped layer at three
input sparsities, the Llama-3-70B-shaped layer at batch 1..16 (independent
per-token masks), and layer stacks chained through RMSNorm with sequential
threshold calibration (Prox App. A.7, Algorithm 1).

Bars as in test_gpu_parity.py.  Stacks are checked teacher-forced: each GPU
layer gets the oracle's inputs for that layer; the free-running GPU stack is
checked only loosely (its earlier layers round differently).
"""

import os
import tempfile

import numpy as np
import pytest
import torch

import synth
from oracle import prox_oracle as orc
from tests.gpu_helpers import (OUT_RTOL, OracleLayer, bits_to_bf16, check_mask,
                               close_with_floor, device_layer, rel_l2)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def prox():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import activation_sparse_swiglu_b200 as p
    return p


def _step_checks(layer, olay, x, tau, k):
    """Stage-1 taps, the mask rule and the output (given the oracle's mask)."""
    ref = olay.step(x, tau, k)
    xd = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    taps = layer.debug_stage1(xd)
    y_m, s_sp = layer.forward_with_mask(
        xd, torch.from_numpy(ref["idx_s"].astype(np.int32)).cuda(), want_s=True)
    torch.cuda.synchronize()
    n_x = int(taps["n_x"].item())
    np.testing.assert_array_equal(taps["idx_x"].cpu().numpy()[:n_x], ref["idx_x"])
    ok, nbad = close_with_floor(taps["g_tilde"].cpu().numpy(), ref["g_tilde"])
    assert ok, f"g~ off at {nbad} channels"
    ok, nbad = close_with_floor(taps["u_tilde"].cpu().numpy(), ref["u_tilde"])
    assert ok, f"u~ off at {nbad} channels"
    check_mask(taps["idx_s"].cpu().numpy(), ref["idx_s"], ref["scores"], k)
    assert rel_l2(y_m.cpu().numpy(), ref["y"]) <= OUT_RTOL
    assert rel_l2(s_sp.cpu().numpy(), ref["s_sp"]) <= OUT_RTOL
    return ref


# ---------------------------------------------------------------------------
# Qwen3-14B shape: s1 in {40, 50, 60} %
# ---------------------------------------------------------------------------

def test_qwen3_14b_three_input_sparsities(prox):
    lay = synth.make_layer("qwen3_14b", n_tokens=2, n_cal=64)
    olay = OracleLayer(lay)
    k = lay.config.k()
    layer = device_layer(lay, 0.0, k)
    xc = torch.from_numpy(lay.x_cal).cuda()
    for s1 in lay.config.s1_percent:
        tau = orc.calibrate_tau(lay.x_cal, s1 / 100)
        assert np.float32(prox.calibrate_thresholds(xc, s1 / 100)) == tau
        layer.set_tau(tau)
        _step_checks(layer, olay, lay.x_eval[0], tau, k)
    assert layer.error_word() == 0
    layer.close()


# ---------------------------------------------------------------------------
# Llama-3-70B shape at batch 1..16, per-token masks
# ---------------------------------------------------------------------------

def test_llama3_70b_batches(prox):
    lay = synth.make_layer("llama3_70b", n_cal=32)
    olay = OracleLayer(lay)
    k = lay.config.k()
    tau = orc.calibrate_tau(lay.x_cal, 0.5)
    layer = device_layer(lay, tau, k, max_batch=16)
    x = torch.from_numpy(lay.x_eval).cuda()
    singles = torch.stack([layer.forward(x[i]).reshape(-1) for i in range(16)])
    for b in lay.config.batch_sizes:
        yb = layer.forward(x[:b])
        torch.cuda.synchronize()
        assert torch.equal(yb, singles[:b])  # each token keeps its own mask
    for t in range(2):
        ref = _step_checks(layer, olay, lay.x_eval[t], tau, k)
        y_full = singles[t].cpu().numpy()
        if np.array_equal(layer.debug_stage1(x[t])["idx_s"].cpu().numpy(), ref["idx_s"]):
            assert rel_l2(y_full, ref["y"]) <= OUT_RTOL
    assert layer.error_word() == 0
    layer.close()


# ---------------------------------------------------------------------------
# Stacks with sequential calibration
# ---------------------------------------------------------------------------

def _stack_case(prox, cfg, n_layers, n_cal, n_tok):
    from activation_sparse_swiglu_b200.stack import Stack
    lays = [synth.make_layer(cfg, li, draw_tokens=(li == 0), n_cal=n_cal, n_tokens=n_tok)
            for li in range(n_layers)]
    x_cal, x_eval = lays[0].x_cal, lays[0].x_eval
    olays = [OracleLayer(lay) for lay in lays]
    layers = [(l.w_gate, l.w_up, l.w_down, o.qg, o.sg, o.qu, o.su) for l, o in zip(lays, olays)]
    k = cfg.k()
    taus, cal_inputs = orc.calibrate_stack(layers, x_cal, 0.5, k)
    weights = [(bits_to_bf16(l.w_gate_bits), bits_to_bf16(l.w_up_bits), bits_to_bf16(l.w_down_bits))
               for l in lays]
    stack = Stack(weights, k, max_batch=max(n_cal, n_tok))
    del weights
    # free-running GPU calibration: thresholds close to the oracle's
    g_taus, _ = stack.calibrate(torch.from_numpy(x_cal).cuda(), 0.5)
    for gt, ot in zip(g_taus, taus):
        assert abs(gt - ot) <= 1e-4 * ot, (gt, ot)
    # teacher-forced: every layer on the oracle's own inputs
    for li, (layer, olay) in enumerate(zip(stack.layers, olays)):
        tau_g = prox.calibrate_thresholds(torch.from_numpy(cal_inputs[li]).cuda(), 0.5)
        assert np.float32(tau_g) == taus[li]
        layer.set_tau(taus[li])
    for t in range(n_tok):
        xs, y_ref = orc.stack_forward(layers, taus, x_eval[t], k)
        for li, (layer, olay) in enumerate(zip(stack.layers, olays)):
            _step_checks(layer, olay, xs[li], taus[li], k)
        # free-running output, reported loosely
        _, y = stack.forward(torch.from_numpy(x_eval[t:t + 1]).cuda())
        assert rel_l2(y.cpu().numpy().reshape(-1), y_ref) <= 5e-2
    for layer in stack.layers:
        assert layer.error_word() == 0
    stack.close()


def test_stack_of_eight_small_layers(prox):
    cfg = synth.WorkloadConfig(name="stack_small", index=62, d_model=512, d_ff=1376, sigma=0.02,
                               outlier_frac=0.01, outlier_scale=20.0, s1_percent=(50,),
                               s2_percent=(70,), n_tokens=2, n_cal=32, n_layers=8)
    _stack_case(prox, cfg, n_layers=8, n_cal=32, n_tok=2)


def test_stack32_all_layers_teacher_forced(prox):
    """All 32 full-size layers of the stack workload, one token, teacher-forced:
    each layer is built, checked on the oracle's own input to it (its tau_x
    from Algorithm 1 on the oracle's calibration inputs, bit-exact on the GPU;
    mask and output as in every step check) and freed before the next, so
    only one layer's weights are held at a time."""
    cfg = synth.get_config("stack32")
    k = cfg.k()
    x_cal = x = None
    for li in range(cfg.n_layers):
        lay = synth.make_layer(cfg, li, draw_tokens=(li == 0), n_cal=2, n_tokens=1)
        if li == 0:
            x_cal, x = lay.x_cal, lay.x_eval[0]
        olay = OracleLayer(lay)
        tau = orc.calibrate_tau(x_cal, 0.5)
        assert np.float32(prox.calibrate_thresholds(torch.from_numpy(x_cal).cuda(), 0.5)) == tau
        layer = device_layer(lay, tau, k)
        ref = _step_checks(layer, olay, x, tau, k)
        assert layer.error_word() == 0
        layer.close()
        if li + 1 < cfg.n_layers:
            x_cal = np.stack([orc.stack_next_input(olay.step(xt, tau, k)["y"]) for xt in x_cal])
            x = orc.stack_next_input(ref["y"])
        del lay, olay
        torch.cuda.empty_cache()


def test_stack32_first_two_layers_full_size(prox):
    # the 32-layer workload's own seeds and shapes, first two layers
    _stack_case(prox, synth.get_config("stack32"), n_layers=2, n_cal=16, n_tok=1)


def test_stack_threshold_rule_small(prox):
    """Algorithm 1 with both thresholds: every layer's tau_x and then tau_s are
    fixed on the inputs that layer receives from the finalised layers before
    it.  Teacher-forced on the oracle's per-layer inputs the GPU's tau_x is
    bit-exact and its tau_s (from its own proxy scores) within the score
    tolerance; the free-running calibration tracks the oracle's."""
    from activation_sparse_swiglu_b200.stack import Stack
    cfg = synth.WorkloadConfig(name="stack_small", index=63, d_model=512, d_ff=1376, sigma=0.02,
                               outlier_frac=0.01, outlier_scale=20.0, s1_percent=(50,),
                               s2_percent=(70,), n_tokens=2, n_cal=32, n_layers=4)
    lays = [synth.make_layer(cfg, li, draw_tokens=(li == 0), n_cal=32, n_tokens=2)
            for li in range(4)]
    x_cal, x_eval = lays[0].x_cal, lays[0].x_eval
    olays = [OracleLayer(lay) for lay in lays]
    layers = [(l.w_gate, l.w_up, l.w_down, o.qg, o.sg, o.qu, o.su) for l, o in zip(lays, olays)]
    k = cfg.k()
    taus, taus_s, cal_inputs = orc.calibrate_stack(layers, x_cal, 0.5, k, s2=0.7)
    weights = [(bits_to_bf16(l.w_gate_bits), bits_to_bf16(l.w_up_bits), bits_to_bf16(l.w_down_bits))
               for l in lays]
    stack = Stack(weights, k, max_batch=32)
    del weights
    g_taus, g_taus_s, _ = stack.calibrate(torch.from_numpy(x_cal).cuda(), 0.5, s2=0.7)
    for gt, ot in zip(g_taus, taus):
        assert abs(gt - ot) <= 1e-4 * ot, (gt, ot)
    for gt, ot in zip(g_taus_s, taus_s):
        assert abs(gt - ot) <= 5e-3 * ot, (gt, ot)
    for li, layer in enumerate(stack.layers):
        assert layer.info()["mask_mode"] == prox.MASK_THRESHOLD
        xin = torch.from_numpy(cal_inputs[li]).cuda()
        assert np.float32(prox.calibrate_thresholds(xin, 0.5)) == taus[li]
        layer.set_tau(taus[li])
        tau_s_g = prox.calibrate_thresholds(layer.proxy_scores(xin), 0.7)
        assert abs(tau_s_g - taus_s[li]) <= 1e-3 * taus_s[li]
        layer.set_mask(prox.MASK_THRESHOLD, float(taus_s[li]))
    # teacher-forced forward under the threshold rule
    for t in range(2):
        xs, y_ref = orc.stack_forward(layers, taus, x_eval[t], k, taus_s=taus_s)
        for li, (layer, olay) in enumerate(zip(stack.layers, olays)):
            ref = olay.step(xs[li], taus[li], k, tau_s=taus_s[li])
            xd = torch.from_numpy(np.ascontiguousarray(xs[li], dtype=np.float32)).cuda()
            gpu_idx = layer.debug_mask(xd).cpu().numpy().astype(np.int64)
            diff = np.setxor1d(gpu_idx, ref["idx_s"])
            assert np.all(np.abs(ref["scores"][diff] - taus_s[li]) <= 1e-3 * taus_s[li])
            lay = lays[li]
            want, _ = orc.stage2(xs[li], lay.w_gate, lay.w_up, lay.w_down, gpu_idx)
            y_g = layer.forward(xd)
            torch.cuda.synchronize()
            assert rel_l2(y_g.cpu().numpy().reshape(-1), want) <= OUT_RTOL
    # the calibration artefact: saved, the layers reset, loaded back bit for bit
    with tempfile.TemporaryDirectory() as td:
        path = os.path.join(td, "thresholds.json")
        stack.save_thresholds(path, 0.5, 0.7)
        for layer in stack.layers:
            layer.set_tau(0.0)
            layer.set_mask(prox.MASK_TOPK)
        stack.load_thresholds(path)
    for li, layer in enumerate(stack.layers):
        inf = layer.info()
        assert inf["mask_mode"] == prox.MASK_THRESHOLD
        assert np.float32(inf["tau_x"]) == np.float32(taus[li])
        assert np.float32(inf["tau_s"]) == np.float32(taus_s[li])
    for layer in stack.layers:
        assert layer.error_word() == 0
    stack.close()



# ---------------------------------------------------------------------------
# The largest shape the header admits
# ---------------------------------------------------------------------------

def test_largest_shape_runs(prox):
    """d_model 16384, d_ff 32768 (the header's limits; Stage 1 then holds the
    most kept rows per CTA and its shallowest copy rings): the step runs with a
    clean error word, selects k channels
    and equals Stage 2 on its own mask bit for bit.  No oracle at this size:
    the properties hold at any size."""
    d, f = 16384, 32768
    k = (f * 30 + 50) // 100
    g = torch.Generator(device="cuda")
    g.manual_seed(123)
    w = [(torch.randn(shape, generator=g, device="cuda") * 0.01).to(torch.bfloat16)
         for shape in ((d, f), (d, f), (f, d))]
    x = torch.randn(d, generator=g, device="cuda")
    layer = prox.Layer(*w, tau=0.67, k=k, max_batch=1)
    del w
    torch.cuda.empty_cache()
    taps = layer.debug_stage1(x)
    idx = taps["idx_s"]
    y = layer.forward(x)
    y_m = layer.forward_with_mask(x, idx)
    torch.cuda.synchronize()
    sel = idx.cpu().numpy()
    assert sel.size == k and np.all(np.diff(sel) > 0)
    assert torch.isfinite(y).all()
    assert torch.equal(y_m, y.reshape(-1))
    assert layer.error_word() == 0
    layer.close()
