"""The allocation-free calibration entry point against the allocating one.

It serves callers that cannot allocate device memory when they calibrate
(their device memory belongs to another allocator, or an allocation's implicit
synchronisation is not acceptable), so besides its result these tests check
that it takes nothing from the device, the stream-ordered pool included, and
that it refuses memory that is not on the current device.

Collected last (file name) so that it also runs after every other GPU test;
it must pass on its own as well.
"""

import ctypes

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


CU_MEMPOOL_ATTR_USED_MEM_HIGH = 8  # cuda.h, CUmemPool_attribute


def _pool_used_high(dev: int, reset: bool = False) -> int:
    """High watermark of the device's default stream-ordered memory pool
    (where cudaMallocAsync takes memory unless told otherwise)."""
    cu = ctypes.CDLL("libcuda.so.1")
    cudev = ctypes.c_int(0)
    assert cu.cuDeviceGet(ctypes.byref(cudev), dev) == 0
    pool = ctypes.c_void_p(0)
    assert cu.cuDeviceGetDefaultMemPool(ctypes.byref(pool), cudev) == 0
    val = ctypes.c_uint64(0)
    if reset:
        assert cu.cuMemPoolSetAttribute(pool, CU_MEMPOOL_ATTR_USED_MEM_HIGH, ctypes.byref(val)) == 0
    assert cu.cuMemPoolGetAttribute(pool, CU_MEMPOOL_ATTR_USED_MEM_HIGH, ctypes.byref(val)) == 0
    return int(val.value)


def test_noalloc_takes_nothing_from_the_stream_ordered_pool(prox):
    dev = torch.cuda.current_device()
    x = torch.randn((64, 512), dtype=torch.float32, device="cuda")
    tau = torch.zeros(1, dtype=torch.float32, device="cuda")
    prox.calibrate_thresholds_noalloc(x, 0.5, tau)  # first call: symbol lookup
    torch.cuda.synchronize()
    assert _pool_used_high(dev, reset=True) == 0
    for _ in range(2):
        prox.calibrate_thresholds_noalloc(x, 0.5, tau)
    torch.cuda.synchronize()
    assert _pool_used_high(dev) == 0
    # the watermark does see a stream-ordered allocation: the allocating
    # entry point takes its scratch from that pool
    prox.calibrate_thresholds(x, 0.5)
    torch.cuda.synchronize()
    assert _pool_used_high(dev) > 0


def test_noalloc_refuses_memory_off_the_device(prox):
    x = torch.randn((8, 128), dtype=torch.float32, device="cuda")
    tau = torch.zeros(1, dtype=torch.float32, device="cuda")
    x_host = np.zeros((8, 128), dtype=np.float32)
    tau_host = np.zeros(4, dtype=np.float32)
    assert x_host.ctypes.data % 16 == 0
    fn = prox.lib.prox_calibrate_thresholds_noalloc
    st = fn(ctypes.c_void_p(x_host.ctypes.data), 8, 128, 0.5, ctypes.c_void_p(tau.data_ptr()), None)
    assert st == 1  # PROX_EINVAL, before any launch
    st = fn(ctypes.c_void_p(x.data_ptr()), 8, 128, 0.5, ctypes.c_void_p(tau_host.ctypes.data), None)
    assert st == 1
    assert "current device" in prox.last_error()
    # the entry point still works afterwards
    prox.calibrate_thresholds_noalloc(x, 0.5, tau)
    torch.cuda.synchronize()
    assert float(tau.item()) == prox.calibrate_thresholds(x, 0.5)
