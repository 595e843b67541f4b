"""The allocation-free calibration entry point against the allocating one.

Collected last (file name) so that it also runs after every other GPU test;
it must pass on its own as well.
"""

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def prox():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import activation_sparse_swiglu_b200 as p
    return p


@pytest.mark.parametrize("name,s1s", [("tiny", (0.0, 0.3, 0.5, 1.0)),
                                      ("llama3_8b", (0.5, 0.9))])
def test_noalloc_matches_allocating_calibration_twice(prox, name, s1s):
    lay = synth.make_layer(name, n_tokens=1)
    x = torch.from_numpy(np.ascontiguousarray(lay.x_cal)).cuda()
    tau = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    for s1 in s1s:
        ref = prox.calibrate_thresholds(x, s1)
        for _ in range(2):  # two calls in a row reuse the same static scratch
            tau.fill_(-1.0)
            prox.calibrate_thresholds_noalloc(x, s1, tau)
            torch.cuda.synchronize()
            got = float(tau.item())
            assert np.float32(got).view(np.uint32) == np.float32(ref).view(np.uint32), (s1, got, ref)


def test_noalloc_rejects_bad_arguments(prox):
    x = torch.zeros((4, 128), dtype=torch.float32, device="cuda")
    tau = torch.zeros(1, dtype=torch.float32, device="cuda")
    with pytest.raises(prox.ProxError):
        prox.calibrate_thresholds_noalloc(x, 1.5, tau)
    flat = torch.zeros(4 * 128 + 1, dtype=torch.float32, device="cuda")
    with pytest.raises(prox.ProxError):  # contiguous, but 4 bytes past a 16-byte boundary
        prox.calibrate_thresholds_noalloc(flat[1:].view(4, 128), 0.5, tau)


def test_noalloc_allocates_nothing(prox):
    x = torch.randn((64, 512), dtype=torch.float32, device="cuda")
    tau = torch.zeros(1, dtype=torch.float32, device="cuda")
    prox.calibrate_thresholds_noalloc(x, 0.5, tau)  # first call: symbol lookup
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(4):
        prox.calibrate_thresholds_noalloc(x, 0.5, tau)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
