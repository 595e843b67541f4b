"""GPU parity of the batched step (prox_ffn_forward_batch, prox_dense_ffn_batch):
B tokens with per-token masks and union loads, against the fp64 oracle token
by token and against the batch-1 path.

Bars: each token's mask equal to the oracle's except at channels whose oracle
score is within 1e-3 of the k-th value; each output within 5e-3 relative L2
of the oracle given the oracle's mask; where the batch and the batch-1 path
select the same channels their outputs agree to 1e-4 relative L2 (the batched
products split x and h into two bf16 parts, 16 significant bits, and sum in
another order); union sizes equal the unions of the tokens' kept rows and
selected channels.
"""

import numpy as np
import pytest
import torch

import synth
from oracle import prox_oracle as orc
from tests.gpu_helpers import OUT_RTOL, OracleLayer, check_mask, device_layer, rel_l2

pytestmark = pytest.mark.gpu

AGREE_RTOL = 1e-4


@pytest.fixture(scope="module")
def prox():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import activation_sparse_swiglu_b200 as p
    return p


def _batch_case(layer, olay, x_eval, tau, k, B, oracle_tokens):
    x = torch.from_numpy(np.ascontiguousarray(x_eval[:B])).cuda()
    yb = layer.forward_batch(x)
    masks = layer.debug_batch_masks(B).cpu().numpy()
    rows, chans = layer.batch_union_sizes()
    torch.cuda.synchronize()
    kept = np.abs(x_eval[:B]) >= np.float32(tau)
    assert rows == int(kept.any(axis=0).sum())
    assert chans == int(masks.any(axis=0).sum())
    assert np.all(masks.sum(axis=1) == k)
    for b in range(B):
        idx_b = np.flatnonzero(masks[b])
        single_idx = layer.debug_stage1(x[b])["idx_s"].cpu().numpy()
        y_single = layer.forward(x[b]).reshape(-1)
        torch.cuda.synchronize()
        if np.array_equal(idx_b, single_idx):
            assert rel_l2(yb[b].cpu().numpy(), y_single.cpu().numpy()) <= AGREE_RTOL
        if b < oracle_tokens:
            ref = olay.step(x_eval[b], tau, k)
            check_mask(idx_b, ref["idx_s"], ref["scores"], k)
            if np.array_equal(idx_b, ref["idx_s"]):
                assert rel_l2(yb[b].cpu().numpy(), ref["y"]) <= OUT_RTOL
    return yb


def test_batch_tiny(prox):
    lay = synth.make_layer("tiny", n_tokens=16)
    olay = OracleLayer(lay)
    k = lay.config.k()
    tau = orc.calibrate_tau(lay.x_cal, 0.5)
    layer = device_layer(lay, tau, k, max_batch=16)
    for B in (1, 2, 5, 16):
        _batch_case(layer, olay, lay.x_eval, tau, k, B, oracle_tokens=B)
    assert layer.error_word() == 0
    layer.close()


def test_batch_dense_tiny(prox):
    lay = synth.make_layer("tiny", n_tokens=16)
    layer = device_layer(lay, 0.0, lay.config.k(), max_batch=16)
    x = torch.from_numpy(np.ascontiguousarray(lay.x_eval[:16])).cuda()
    yd = layer.dense_batch(x).cpu().numpy()
    for b in range(16):
        ref = orc.dense_ffn(lay.x_eval[b], lay.w_gate, lay.w_up, lay.w_down)
        assert rel_l2(yd[b], ref) <= OUT_RTOL
        y1 = layer.dense(x[b]).reshape(-1).cpu().numpy()
        assert rel_l2(yd[b], y1) <= AGREE_RTOL
    layer.close()


def test_batch_keep_all_equals_dense(prox):
    # tau_x = 0 and k = d_ff: every row and every channel, so the sparse batch
    # computes the dense FFN (with the INT4 proxies only deciding nothing).
    lay = synth.make_layer("tiny", n_tokens=16)
    layer = device_layer(lay, 0.0, lay.config.d_ff, max_batch=16)
    x = torch.from_numpy(np.ascontiguousarray(lay.x_eval[:4])).cuda()
    ys = layer.forward_batch(x).cpu().numpy()
    assert layer.batch_union_sizes() == (lay.config.d_model, lay.config.d_ff)
    yd = layer.dense_batch(x).cpu().numpy()
    for b in range(4):
        ref = orc.dense_ffn(lay.x_eval[b], lay.w_gate, lay.w_up, lay.w_down)
        assert rel_l2(ys[b], ref) <= OUT_RTOL
        assert rel_l2(ys[b], yd[b]) <= AGREE_RTOL
    layer.close()


def test_batch_threshold_rule(prox):
    lay = synth.make_layer("tiny", n_tokens=16)
    olay = OracleLayer(lay)
    k = lay.config.k()
    tau = orc.calibrate_tau(lay.x_cal, 0.5)
    layer = device_layer(lay, tau, k, max_batch=16)
    # tau_s at the median score of the first token: about half the channels
    s0 = olay.step(lay.x_eval[0], tau, k)["scores"]
    tau_s = float(np.float32(np.median(s0)))
    layer.set_mask(prox.MASK_THRESHOLD, tau_s)
    x = torch.from_numpy(np.ascontiguousarray(lay.x_eval[:8])).cuda()
    yb = layer.forward_batch(x).cpu().numpy()
    masks = layer.debug_batch_masks(8).cpu().numpy()
    for b in range(8):
        ref = olay.step(lay.x_eval[b], tau, k, tau_s=tau_s)
        diff = np.setxor1d(np.flatnonzero(masks[b]), ref["idx_s"])
        near = np.abs(ref["scores"][diff] - tau_s) <= 1e-3 * tau_s
        assert np.all(near)
        if diff.size == 0:
            assert rel_l2(yb[b], ref["y"]) <= OUT_RTOL
    layer.close()


def test_batch_llama3_70b(prox):
    lay = synth.make_layer("llama3_70b", n_cal=32)
    olay = OracleLayer(lay)
    k = lay.config.k()
    tau = orc.calibrate_tau(lay.x_cal, 0.5)
    layer = device_layer(lay, tau, k, max_batch=16)
    for B in lay.config.batch_sizes:
        _batch_case(layer, olay, lay.x_eval, tau, k, B, oracle_tokens=1 if B == 16 else 0)
    assert layer.error_word() == 0
    layer.close()


def test_batch_argument_errors(prox):
    lay = synth.make_layer("tiny", n_tokens=16)
    k = lay.config.k()
    one = device_layer(lay, 0.5, k, max_batch=1)
    x = torch.from_numpy(np.ascontiguousarray(lay.x_eval[:2])).cuda()
    with pytest.raises(prox.ProxError):
        one.forward_batch(x)
    one.close()
    many = device_layer(lay, 0.5, k, max_batch=32)
    x17 = torch.from_numpy(np.ascontiguousarray(np.tile(lay.x_eval[:1], (17, 1)))).cuda()
    with pytest.raises(prox.ProxError):
        many.forward_batch(x17)
    many.set_stage2(prox.STAGE2_PROXY_VALUES)
    with pytest.raises(prox.ProxError):
        many.forward_batch(x)
    many.close()
