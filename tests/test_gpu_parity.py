"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.

Bars: compacted input indices and packed codes bit-exact; Stage-1 scores
within 1e-3 relative (with a floor at 1e-3 of the largest score); masks equal
except at channels whose oracle score is within 1e-3 of the k-th value; FFN
outputs within 5e-3 relative L2 given the oracle's mask.
"""

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


def _custom(d, f, idx=70, sigma=0.05, n_tok=4, n_cal=32):
    return synth.WorkloadConfig(name=f"c{d}x{f}", index=idx, d_model=d, d_ff=f, sigma=sigma,
                                outlier_frac=0.01, outlier_scale=20.0, s1_percent=(50,),
                                s2_percent=(70,), n_tokens=n_tok, n_cal=n_cal)


_LAYERS = {}


def _layer(name, n_tok=None):
    key = (name, n_tok)
    if key not in _LAYERS:
        cfg = synth.get_config(name) if isinstance(name, str) else name
        lay = synth.make_layer(cfg, n_tokens=n_tok)
        _LAYERS[key] = (lay, OracleLayer(lay))
    return _LAYERS[key]


# ---------------------------------------------------------------------------
# Offline preparation
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("shape", [(128, 32), (384, 96), (512, 1376), (640, 256), (4096, 14336)])
def test_pack_proxy_bit_exact(prox, shape):
    d, f = shape
    lay = synth.make_layer(_custom(d, f, idx=71, sigma=0.02), draw_tokens=False)
    w = bits_to_bf16(lay.w_gate_bits)
    codes, scales = prox.pack_proxy(w)
    torch.cuda.synchronize()
    q, s = orc.quantize_proxy(lay.w_gate)
    np.testing.assert_array_equal(scales.cpu().numpy().view(np.uint16), s.view(np.uint16))
    got = codes.cpu().numpy()
    want = orc.pack_nibbles(q)
    if not np.array_equal(got, want):
        # only codes whose W/S sits within 2^-20 of a rounding midpoint may differ
        gq = orc.unpack_nibbles(got)
        bad = gq != q
        near = orc.code_near_tie(lay.w_gate, s)
        assert np.all(near[bad]) and np.all(np.abs(gq[bad].astype(int) - q[bad]) == 1)


def test_pack_proxy_special_values(prox):
    # exact grid, round-half-even ties and an all-zero group
    w = np.zeros((128, 64), dtype=np.float32)
    sc = 2.0 ** -7
    col = np.array([7, 2.5, 3.5, -2.5, -3.5, 0.5, -0.5, 1.5, 6.5, -6.5])
    w[: col.size, 0] = col * sc
    w[0, 2] = -7 * sc
    w[5, 2] = 4.5 * sc
    w[3, 5] = 1e-3
    bits, vals = synth.bf16_round(w)
    codes, scales = prox.pack_proxy(bits_to_bf16(bits))
    q, s = orc.quantize_proxy(vals)
    np.testing.assert_array_equal(codes.cpu().numpy(), orc.pack_nibbles(q))
    np.testing.assert_array_equal(scales.cpu().numpy().view(np.uint16), s.view(np.uint16))


@pytest.mark.parametrize("name,s1", [("tiny", 0.5), ("llama3_8b", 0.5), ("llama3_8b", 0.4),
                                     ("qwen3_14b", 0.6), ("tiny", 1.0), ("tiny", 1e-6)])
def test_calibrate_bit_exact(prox, name, s1):
    cfg = synth.get_config(name)
    rng = np.random.Generator(np.random.PCG64(cfg.seed(0) + 7))
    x = rng.laplace(0, 1, size=(256, cfg.d_model)).astype(np.float32)
    tau = prox.calibrate_thresholds(torch.from_numpy(x).cuda(), s1)
    assert np.float32(tau) == orc.calibrate_tau(x, s1)


def test_calibrate_with_ties(prox):
    x = np.repeat(np.array([[0.25, -0.5, 1.0, 0.5]], dtype=np.float32), 64, axis=0)
    for s1 in (0.1, 0.25, 0.5, 0.74, 0.75, 0.9):
        tau = prox.calibrate_thresholds(torch.from_numpy(x).cuda(), s1)
        assert np.float32(tau) == orc.calibrate_tau(x, s1)


# ---------------------------------------------------------------------------
# Stage 1 taps
# ---------------------------------------------------------------------------

def _stage1_case(prox, lay, olay, tau, k, tokens):
    layer = device_layer(lay, tau, k)
    n_diff = 0
    for t in tokens:
        x = lay.x_eval[t]
        taps = layer.debug_stage1(torch.from_numpy(x).cuda())
        torch.cuda.synchronize()
        idx_x, g_t, u_t, _ = olay.stage1(x, tau)
        n_x = int(taps["n_x"].item())
        assert n_x == idx_x.size
        np.testing.assert_array_equal(taps["idx_x"].cpu().numpy()[:n_x], idx_x)
        ok, nbad = close_with_floor(taps["g_tilde"].cpu().numpy(), g_t)
        assert ok, f"g~ off at {nbad} channels"
        ok, nbad = close_with_floor(taps["u_tilde"].cpu().numpy(), u_t)
        assert ok, f"u~ off at {nbad} channels"
        scores_o = orc.proxy_scores(g_t, u_t)
        scores_g = np.abs(orc.silu(taps["g_tilde"].cpu().numpy()) *
                          taps["u_tilde"].cpu().numpy().astype(np.float64))
        ok, nbad = close_with_floor(scores_g, scores_o)
        assert ok, f"scores off at {nbad} channels"
        # the scores the kernel itself ranks (device buffer, SiLU path)
        scores_dev = layer.proxy_scores(torch.from_numpy(x).cuda().reshape(1, -1))
        ok, nbad = close_with_floor(scores_dev.cpu().numpy().reshape(-1), scores_o)
        assert ok, f"device scores off at {nbad} channels"
        n_diff += check_mask(taps["idx_s"].cpu().numpy(), orc.topk_channels(scores_o, k),
                             scores_o, k)
    assert layer.error_word() == 0
    layer.close()
    return n_diff


def test_stage1_tiny_all_tokens(prox):
    lay, olay = _layer("tiny")
    tau = orc.calibrate_tau(lay.x_cal, 0.5)
    _stage1_case(prox, lay, olay, tau, lay.config.k(), range(lay.x_eval.shape[0]))


@pytest.mark.parametrize("shape", [(128, 32), (384, 96), (640, 256), (512, 1376)])
def test_stage1_ragged_shapes(prox, shape):
    lay, olay = _layer(_custom(*shape))
    tau = orc.calibrate_tau(lay.x_cal, 0.5)
    for k in (1, shape[1] // 3, shape[1]):
        _stage1_case(prox, lay, olay, tau, k, range(lay.x_eval.shape[0]))


def test_stage1_llama3_8b_sampled(prox):
    lay, olay = _layer("llama3_8b", n_tok=3)
    tau = orc.calibrate_tau(lay.x_cal, 0.5)
    for s2 in (70, 50):
        _stage1_case(prox, lay, olay, tau, lay.config.k(s2), range(3))


@pytest.mark.parametrize("shape,k", [((384, 96), 10), ((256, 8192), 3001)])
def test_stage1_no_input_kept(prox, shape, k):
    # tau above every |x|: n_x = 0, all proxy scores are 0, ties go to the lowest
    # indices (the second shape has more tied keys than the candidate buffer)
    lay, olay = _layer(_custom(*shape))
    layer = device_layer(lay, 1e30, k)
    x = torch.from_numpy(lay.x_eval[0]).cuda()
    taps = layer.debug_stage1(x)
    assert int(taps["n_x"].item()) == 0
    np.testing.assert_array_equal(taps["g_tilde"].cpu().numpy(), 0.0)
    np.testing.assert_array_equal(taps["idx_s"].cpu().numpy(), np.arange(k))
    # the full step selects the same channels
    ref_y, _ = orc.stage2(lay.x_eval[0], lay.w_gate, lay.w_up, lay.w_down, np.arange(k))
    assert rel_l2(layer.forward(x).cpu().numpy().reshape(-1), ref_y) <= OUT_RTOL
    assert layer.error_word() == 0


# ---------------------------------------------------------------------------
# Stage 2 and the whole step
# ---------------------------------------------------------------------------

def _stage2_case(lay, olay, tau, k, tokens, layer=None):
    own = layer is None
    if own:
        layer = device_layer(lay, tau, k)
    worst = 0.0
    for t in tokens:
        x = lay.x_eval[t]
        ref = olay.step(x, tau, k)
        xd = torch.from_numpy(x).cuda()
        idx = torch.from_numpy(ref["idx_s"].astype(np.int32)).cuda()
        y, s_sp = layer.forward_with_mask(xd, idx, want_s=True)
        torch.cuda.synchronize()
        err = rel_l2(y.cpu().numpy(), ref["y"])
        assert err <= OUT_RTOL, err
        assert rel_l2(s_sp.cpu().numpy(), ref["s_sp"]) <= OUT_RTOL
        worst = max(worst, err)
        # the full step: when the masks agree the outputs must agree too
        taps = layer.debug_stage1(xd)
        y_full = layer.forward(xd)
        torch.cuda.synchronize()
        gpu_idx = taps["idx_s"].cpu().numpy()
        check_mask(gpu_idx, ref["idx_s"], ref["scores"], k)
        if np.array_equal(gpu_idx, ref["idx_s"]):
            assert rel_l2(y_full.cpu().numpy(), ref["y"]) <= OUT_RTOL
        # forward == Stage 2 on its own mask, bit for bit
        y_m = layer.forward_with_mask(xd, taps["idx_s"])
        torch.cuda.synchronize()
        assert torch.equal(y_m, y_full.reshape(-1))
    assert layer.error_word() == 0
    if own:
        layer.close()
    return worst


def test_stage2_tiny_all_tokens(prox):
    lay, olay = _layer("tiny")
    tau = orc.calibrate_tau(lay.x_cal, 0.5)
    _stage2_case(lay, olay, tau, lay.config.k(), range(lay.x_eval.shape[0]))


@pytest.mark.parametrize("shape", [(128, 32), (384, 96), (640, 256)])
def test_stage2_ragged_shapes(prox, shape):
    lay, olay = _layer(_custom(*shape))
    tau = orc.calibrate_tau(lay.x_cal, 0.5)
    for k in (1, 7, shape[1]):
        _stage2_case(lay, olay, tau, k, range(2))


def test_llama3_8b_sampled_tokens(prox):
    lay, olay = _layer("llama3_8b", n_tok=3)
    tau = orc.calibrate_tau(lay.x_cal, 0.5)
    for s2 in (70, 0):
        _stage2_case(lay, olay, tau, lay.config.k(s2), range(2))


def test_keep_all_equals_dense(prox):
    # tau = 0 and k = d_ff: the sparse step is the dense SwiGLU (Prox §4.1 with m_s = 1)
    lay, olay = _layer("tiny")
    layer = device_layer(lay, 0.0, lay.d_ff)
    for t in range(4):
        x = lay.x_eval[t]
        xd = torch.from_numpy(x).cuda()
        dense_ref = orc.dense_ffn(x, lay.w_gate, lay.w_up, lay.w_down)
        y = layer.forward(xd).cpu().numpy()
        yd = layer.dense(xd).cpu().numpy()
        assert rel_l2(y, dense_ref) <= OUT_RTOL
        assert rel_l2(yd, dense_ref) <= OUT_RTOL
        np.testing.assert_array_equal(y, yd)  # same channels, same order, same kernels
    layer.close()


def test_dense_llama3_8b(prox):
    lay, _ = _layer("llama3_8b", n_tok=3)
    layer = device_layer(lay, 0.5, 100)
    x = lay.x_eval[0]
    y = layer.dense(torch.from_numpy(x).cuda()).cpu().numpy()
    assert rel_l2(y, orc.dense_ffn(x, lay.w_gate, lay.w_up, lay.w_down)) <= OUT_RTOL
    layer.close()


def test_batch_matches_single_tokens_and_is_deterministic(prox):
    lay, olay = _layer("tiny")
    tau = orc.calibrate_tau(lay.x_cal, 0.5)
    layer = device_layer(lay, tau, lay.config.k(), max_batch=8)
    xb = torch.from_numpy(lay.x_eval[:8]).cuda()
    yb = layer.forward(xb)
    yb2 = layer.forward(xb)
    singles = torch.stack([layer.forward(xb[i]).reshape(-1) for i in range(8)])
    torch.cuda.synchronize()
    assert torch.equal(yb, yb2)
    assert torch.equal(yb, singles)
    # realised input sparsity counters
    layer.stats()
    layer.forward(xb)
    sum_nx, ntok = layer.stats()
    want = sum(orc.input_mask(lay.x_eval[i], tau).size for i in range(8))
    assert ntok == 8 and sum_nx == want
    # host-buffer entry point
    xh = torch.from_numpy(lay.x_eval[:8]).pin_memory()
    yh = layer.forward_host(xh)
    assert torch.equal(yh, yb.cpu())
    layer.close()


def test_bad_mask_index_sets_error_word(prox):
    lay, _ = _layer(_custom(384, 96))
    layer = device_layer(lay, 0.5, 8)
    x = torch.from_numpy(lay.x_eval[0]).cuda()
    idx = torch.tensor([0, 5, 96, -3], dtype=torch.int32, device="cuda")  # 96, -3 out of range
    layer.forward_with_mask(x, idx)
    assert layer.error_word() & prox.DEVERR_MASK_INDEX
    assert layer.error_word() == 0  # reading clears it
    layer.close()


def test_rmsnorm(prox):
    rng = np.random.default_rng(3)
    y = rng.standard_normal((3, 4096)).astype(np.float32) * 5
    x = prox.rmsnorm(torch.from_numpy(y).cuda(), 1e-6).cpu().numpy()
    for r in range(3):
        assert rel_l2(x[r], orc.rmsnorm(y[r], 1e-6)) < 1e-6


def test_copy_kernel(prox):
    a = torch.randn(1 << 20, device="cuda")
    b = torch.empty_like(a)
    prox.copy(a, b)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
