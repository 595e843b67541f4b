"""Failure paths on a GPU without any GPU fault: an injected out-of-memory at
each of the nine device allocations of layer creation comes back as
PROX_ENOMEM, leaks nothing, and leaves the library usable; a device wait that
can never complete runs out after its bound, is reported in the layer's error
word, and the layer recovers."""

import gc

import pytest
import torch

import synth
from tests.gpu_helpers import bits_to_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def prox():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import activation_sparse_swiglu_b200 as p
    return p


def test_injected_allocation_failure_at_every_site(prox):
    cfg = synth.WorkloadConfig(name="fault_case", index=64, d_model=1024, d_ff=4096, sigma=0.02,
                               outlier_frac=0.01, outlier_scale=20.0, s1_percent=(50,),
                               s2_percent=(70,), n_tokens=1, n_cal=8)
    lay = synth.make_layer(cfg)
    wg, wu, wd = (bits_to_bf16(b) for b in (lay.w_gate_bits, lay.w_up_bits, lay.w_down_bits))
    x = torch.from_numpy(lay.x_eval[0]).cuda()
    k = cfg.k()
    # One good create, forward and comparison first, so that every kernel
    # module (the library's and torch's) is loaded before free memory is
    # measured; the bound then covers exactly the failed creates.
    good = prox.Layer(wg, wu, wd, tau=0.5, k=k)
    y_ref = good.forward(x).clone()
    assert torch.equal(y_ref, y_ref) and good.error_word() == 0
    good.close()
    gc.collect()  # layers an earlier test left to the collector are freed now
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0] + torch.cuda.memory_reserved()
    try:
        for rep in range(3):
            for nth in range(1, 10):
                prox.lib.prox_debug_fail_alloc(nth)
                with pytest.raises(prox.ProxError) as ei:
                    prox.Layer(wg, wu, wd, tau=0.5, k=k)
                assert ei.value.status == 2, (nth, str(ei.value))  # PROX_ENOMEM
        torch.cuda.synchronize()
        free1 = torch.cuda.mem_get_info()[0] + torch.cuda.memory_reserved()
        # 27 failed creates, each of which had allocated up to eight buffers of
        # 64 KB to 16 MB before the injected failure: a buffer left behind would
        # add up well past this bound (free memory net of torch's own reserve;
        # only a drop counts, memory returned meanwhile is not a leak)
        assert free0 - free1 < 2 ** 20, (free0, free1)
        # an injection past the last allocation does not fire during the create
        prox.lib.prox_debug_fail_alloc(10)
        layer = prox.Layer(wg, wu, wd, tau=0.5, k=k)
    finally:
        prox.lib.prox_debug_fail_alloc(0)
    y = layer.forward(x)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)
    assert layer.error_word() == 0
    layer.close()


def test_bounded_wait_runs_out_and_recovers(prox):
    """A grid-barrier wait that can never complete (the probe expects one more
    CTA than it launches) runs out after its bound, reports
    PROX_DEVERR_WAIT_TIMEOUT in the error word, and the layer computes the
    same output as before once the error word has been read."""
    lay = synth.make_layer("tiny", n_tokens=2, n_cal=8)
    wg, wu, wd = (bits_to_bf16(b) for b in (lay.w_gate_bits, lay.w_up_bits, lay.w_down_bits))
    layer = prox.Layer(wg, wu, wd, tau=0.5, k=lay.config.k())
    x = torch.from_numpy(lay.x_eval[0]).cuda()
    y_ref = layer.forward(x).clone()
    assert layer.error_word() == 0
    prox.check(prox.lib.prox_debug_wait_timeout(layer.handle, None))
    torch.cuda.synchronize()
    assert layer.error_word() & prox.DEVERR_WAIT_TIMEOUT
    y = layer.forward(x)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)
    assert layer.error_word() == 0
    layer.close()
