"""GPU parity of the Stage-2 score-threshold rule (Prox §4.1: m_s = 1[|s~| >=
tau_s], tau_s calibrated as the s2-quantile of the calibration tokens' proxy
scores, Prox App. A.7).

Bars: proxy scores within 1e-3 (with the floor); tau_s bit-exact when the GPU
calibrates the oracle's own scores; masks equal except at channels whose oracle
score is within 1e-3 of tau_s; outputs within 5e-3 on the oracle's mask; the
forward step equal bit for bit to Stage 2 on its own mask.
"""

import numpy as np
import pytest
import torch

import synth
from oracle import prox_oracle as orc
from tests.gpu_helpers import (MASK_RTOL, OUT_RTOL, OracleLayer, close_with_floor,
                               device_layer, rel_l2)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def prox():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import activation_sparse_swiglu_b200 as p
    return p


def check_threshold_mask(gpu_idx, orc_idx, orc_scores, tau_s):
    gpu_idx = np.asarray(gpu_idx, dtype=np.int64)
    assert np.all(np.diff(gpu_idx) > 0), "idx_s must be strictly ascending"
    diff = np.setxor1d(gpu_idx, orc_idx)
    near = np.abs(np.asarray(orc_scores)[diff] - tau_s) <= MASK_RTOL * tau_s
    assert np.all(near), f"{int((~near).sum())} mask differences away from tau_s"
    return int(diff.size)


def _threshold_case(prox, name, n_cal, tokens, s2=0.7):
    lay = synth.make_layer(name, n_tokens=max(tokens) + 1, n_cal=n_cal)
    olay = OracleLayer(lay)
    tau_x = orc.calibrate_tau(lay.x_cal, 0.5)
    layer = device_layer(lay, tau_x, lay.config.k(), max_batch=n_cal)
    # proxy scores of the calibration tokens
    xc = torch.from_numpy(lay.x_cal).cuda()
    sc_gpu = layer.proxy_scores(xc).cpu().numpy()
    sc_orc = []
    for t in range(n_cal):
        _, g, u, _ = olay.stage1(lay.x_cal[t], tau_x)
        sc_orc.append(orc.proxy_scores(g, u))
        ok, nbad = close_with_floor(sc_gpu[t], sc_orc[t])
        assert ok, f"scores of calibration token {t} off at {nbad} channels"
    # tau_s: the GPU calibration of the oracle's scores is bit-exact
    tau_s = orc.calibrate_tau_s(lay.x_cal, tau_x, olay.qg, olay.sg, olay.qu, olay.su, s2)
    sc32 = torch.from_numpy(np.asarray(sc_orc, dtype=np.float32)).cuda()
    assert np.float32(prox.calibrate_thresholds(sc32, s2)) == tau_s
    # ... and from the GPU's own scores it is within the score tolerance
    tau_g = prox.calibrate_thresholds(torch.from_numpy(sc_gpu).cuda(), s2)
    assert abs(tau_g - tau_s) <= 1e-3 * tau_s
    layer.set_mask(prox.MASK_THRESHOLD, float(tau_s))
    assert layer.info()["mask_mode"] == prox.MASK_THRESHOLD
    layer.stats()
    n_sel = 0
    for t in tokens:
        x = lay.x_eval[t]
        ref = orc.prox_ffn(x, lay.w_gate, lay.w_up, lay.w_down, olay.qg, olay.sg, olay.qu,
                           olay.su, tau=tau_x, k=0, tau_s=tau_s)
        xd = torch.from_numpy(x).cuda()
        gpu_idx = layer.debug_mask(xd).cpu().numpy()
        check_threshold_mask(gpu_idx, ref["idx_s"], ref["scores"], tau_s)
        y_m, s_sp = layer.forward_with_mask(
            xd, torch.from_numpy(ref["idx_s"].astype(np.int32)).cuda(), want_s=True)
        y_full = layer.forward(xd)
        n_sel += gpu_idx.size
        y_own = layer.forward_with_mask(xd, torch.from_numpy(gpu_idx.astype(np.int32)).cuda())
        torch.cuda.synchronize()
        assert rel_l2(y_m.cpu().numpy(), ref["y"]) <= OUT_RTOL
        assert rel_l2(s_sp.cpu().numpy(), ref["s_sp"]) <= OUT_RTOL
        if np.array_equal(gpu_idx, ref["idx_s"]):
            assert rel_l2(y_full.cpu().numpy(), ref["y"]) <= OUT_RTOL
        assert torch.equal(y_own, y_full.reshape(-1))
    _, ntok, sum_sel = layer.stats(with_selected=True)
    assert ntok == len(tokens) and sum_sel == n_sel
    assert layer.error_word() == 0
    layer.close()


def test_threshold_rule_tiny(prox):
    _threshold_case(prox, "tiny", n_cal=64, tokens=range(8))


def test_threshold_rule_llama3_8b_sampled(prox):
    _threshold_case(prox, "llama3_8b", n_cal=16, tokens=range(2))


def test_set_mask_rejects_bad_arguments(prox):
    lay = synth.make_layer("tiny", n_tokens=1, n_cal=8)
    layer = device_layer(lay, 0.5, 10)
    for mode, tau_s in ((7, 0.0), (prox.MASK_THRESHOLD, -1.0), (prox.MASK_THRESHOLD, float("nan"))):
        with pytest.raises(prox.ProxError):
            layer.set_mask(mode, tau_s)
    layer.set_mask(prox.MASK_THRESHOLD, 0.1)
    with pytest.raises(prox.ProxError):  # idx_s of debug_stage1 holds k channels: top-k only
        layer.debug_stage1(torch.from_numpy(lay.x_eval[0]).cuda())
    layer.set_mask(prox.MASK_TOPK)
    layer.debug_stage1(torch.from_numpy(lay.x_eval[0]).cuda())
    layer.close()
