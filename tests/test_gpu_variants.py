"""GPU parity of the two method variants the paper evaluates besides SwiGLU +
exact Stage 2:

* GeGLU FFNs (Prox §5 applies the method to Gemma-3, whose FFN gate is GELU):
  the gate activation is switched in the Stage-1 score, Stage 2 and the dense
  baseline, with GELU as z Phi(z) or in its tanh form;
* ablation A3 (Prox §5.2): Stage 2 skips the exact gate/up projections and
  feeds the selected proxy values s~ straight into W_down.

Bars as in test_gpu_parity.py: Stage-1 scores within 1e-3 (with the floor),
masks equal except near the k-th score, outputs within 5e-3 relative L2 given a
mask, and the forward step equal bit for bit to Stage 2 on its own mask.
"""

import numpy as np
import pytest
import torch

import synth
from oracle import prox_oracle as orc
from tests.gpu_helpers import (OUT_RTOL, OracleLayer, check_mask, close_with_floor,
                               device_layer, rel_l2)

pytestmark = pytest.mark.gpu

ACT_NAMES = {0: "silu", 1: "gelu_tanh", 2: "gelu"}


@pytest.fixture(scope="module")
def prox():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import activation_sparse_swiglu_b200 as p
    return p


def _geglu_case(prox, name, act, tokens):
    lay = synth.make_layer(name, n_tokens=max(tokens) + 1, n_cal=32)
    olay = OracleLayer(lay)
    k = lay.config.k()
    tau = orc.calibrate_tau(lay.x_cal, 0.5)
    layer = device_layer(lay, tau, k)
    layer.set_activation(act)
    assert layer.info()["activation"] == act
    aname = ACT_NAMES[act]
    for t in tokens:
        x = lay.x_eval[t]
        ref = olay.step(x, tau, k, act=aname)
        xd = torch.from_numpy(x).cuda()
        sc = layer.proxy_scores(xd.reshape(1, -1)).cpu().numpy().reshape(-1)
        ok, nbad = close_with_floor(sc, ref["scores"])
        assert ok, f"{aname} scores off at {nbad} channels"
        gpu_idx = layer.debug_stage1(xd)["idx_s"].cpu().numpy()
        check_mask(gpu_idx, ref["idx_s"], ref["scores"], k)
        y_m, s_sp = layer.forward_with_mask(
            xd, torch.from_numpy(ref["idx_s"].astype(np.int32)).cuda(), want_s=True)
        y_full = layer.forward(xd)
        y_own = layer.forward_with_mask(xd, torch.from_numpy(gpu_idx.astype(np.int32)).cuda())
        y_dense = layer.dense(xd)
        torch.cuda.synchronize()
        assert rel_l2(y_m.cpu().numpy(), ref["y"]) <= OUT_RTOL
        assert rel_l2(s_sp.cpu().numpy(), ref["s_sp"]) <= OUT_RTOL
        assert torch.equal(y_own, y_full.reshape(-1))
        dense_ref = orc.dense_ffn(x, lay.w_gate, lay.w_up, lay.w_down, act=aname)
        assert rel_l2(y_dense.cpu().numpy().reshape(-1), dense_ref) <= OUT_RTOL
    assert layer.error_word() == 0
    layer.close()


@pytest.mark.parametrize("act", [1, 2])
def test_geglu_tiny(prox, act):
    _geglu_case(prox, "tiny", act, tokens=range(4))


def test_geglu_llama3_8b_sampled(prox):
    _geglu_case(prox, "llama3_8b", prox.ACT_GELU_TANH, tokens=[0])


def test_geglu_erf_llama3_8b_sampled(prox):
    # GELU as z Phi(z) (erf form) at full size
    _geglu_case(prox, "llama3_8b", prox.ACT_GELU_ERF, tokens=[0])


def _a3_case(prox, name, tokens, threshold=False, act=0):
    lay = synth.make_layer(name, n_tokens=max(tokens) + 1, n_cal=16)
    olay = OracleLayer(lay)
    k = lay.config.k()
    tau = orc.calibrate_tau(lay.x_cal, 0.5)
    layer = device_layer(lay, tau, k)
    layer.set_activation(act)
    aname = ACT_NAMES[act]
    kw = {"act": aname}
    if threshold:
        tau_s = orc.calibrate_tau_s(lay.x_cal, tau, olay.qg, olay.sg, olay.qu, olay.su, 0.7,
                                    act=aname)
        layer.set_mask(prox.MASK_THRESHOLD, float(tau_s))
        kw["tau_s"] = tau_s
    layer.set_stage2(prox.STAGE2_PROXY_VALUES)
    assert layer.info()["stage2_source"] == prox.STAGE2_PROXY_VALUES
    for t in tokens:
        x = lay.x_eval[t]
        xd = torch.from_numpy(x).cuda()
        ref = olay.step(x, tau, k, proxy_values=True, **kw)
        gpu_idx = layer.debug_mask(xd).cpu().numpy().astype(np.int64)
        if threshold:
            diff = np.setxor1d(gpu_idx, ref["idx_s"])
            assert np.all(np.abs(ref["scores"][diff] - kw["tau_s"]) <= 1e-3 * kw["tau_s"])
        else:
            check_mask(gpu_idx, ref["idx_s"], ref["scores"], k)
        y_a3 = layer.forward(xd)
        # the forward-with-mask tap stays exact in this mode
        y_exact_own = layer.forward_with_mask(xd, torch.from_numpy(gpu_idx.astype(np.int32)).cuda())
        torch.cuda.synchronize()
        # A3 on the GPU's own mask with the oracle's proxy values
        want = orc.stage2_proxy_values(lay.w_down, gpu_idx, ref["s_tilde"])
        assert rel_l2(y_a3.cpu().numpy().reshape(-1), want) <= OUT_RTOL
        exact = orc.stage2(x, lay.w_gate, lay.w_up, lay.w_down, gpu_idx, act=aname)[0]
        assert rel_l2(y_exact_own.cpu().numpy(), exact) <= OUT_RTOL
        # the ablation really changes the output (proxy values are not exact)
        assert rel_l2(want, exact) > 10 * OUT_RTOL
    layer.set_stage2(prox.STAGE2_EXACT)
    y_back = layer.forward(torch.from_numpy(lay.x_eval[tokens[0]]).cuda())
    ref = olay.step(lay.x_eval[tokens[0]], tau, k, **kw)
    gpu_idx = layer.debug_mask(torch.from_numpy(lay.x_eval[tokens[0]]).cuda()).cpu().numpy()
    if np.array_equal(gpu_idx, ref["idx_s"]):
        assert rel_l2(y_back.cpu().numpy().reshape(-1), ref["y"]) <= OUT_RTOL
    assert layer.error_word() == 0
    layer.close()


def test_a3_tiny_topk(prox):
    _a3_case(prox, "tiny", tokens=[0, 1, 2])


def test_a3_tiny_threshold_geglu(prox):
    _a3_case(prox, "tiny", tokens=[0, 1], threshold=True, act=2)


def test_a3_llama3_8b_sampled(prox):
    _a3_case(prox, "llama3_8b", tokens=[0])


def test_variant_setters_reject_bad_arguments(prox):
    lay = synth.make_layer("tiny", n_tokens=1, n_cal=8)
    layer = device_layer(lay, 0.5, 10)
    for bad in (-1, 3, 99):
        with pytest.raises(prox.ProxError):
            layer.set_activation(bad)
    for bad in (-1, 2):
        with pytest.raises(prox.ProxError):
            layer.set_stage2(bad)
    info = layer.info()
    assert info["activation"] == prox.ACT_SILU and info["stage2_source"] == prox.STAGE2_EXACT
    layer.close()
