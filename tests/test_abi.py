"""The C-ABI library loads, exports every symbol include/prox.h declares, and
rejects bad arguments on the host before touching a GPU."""

import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "prox.h")).read()
    return sorted(set(re.findall(r"PROX_API\s+[\w\s\*]+?\b(prox_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def plib():
    from activation_sparse_swiglu_b200 import _lib
    return _lib


def test_header_symbols_are_exported(plib):
    declared = _declared()
    assert len(declared) >= 15
    raw = ctypes.CDLL(plib.LIB_PATH)
    for name in declared:
        assert hasattr(raw, name), name
    assert set(declared) == set(plib.SIGNATURES)


def test_version(plib):
    assert b"sm_100a" in plib.lib.prox_version()


def test_host_side_argument_checks(plib):
    lib = plib.lib
    h = ctypes.c_void_p(0)
    p = ctypes.c_void_p(16)
    # d_model not a multiple of 128
    st = lib.prox_layer_create(p, p, p, 100, 64, 0.5, 8, 1, None, ctypes.byref(h))
    assert st == plib.PROX_EINVAL and "d_model" in plib.last_error()
    # d_ff not a multiple of 32
    st = lib.prox_layer_create(p, p, p, 128, 40, 0.5, 8, 1, None, ctypes.byref(h))
    assert st == plib.PROX_EINVAL and "d_ff" in plib.last_error()
    # k out of range
    st = lib.prox_layer_create(p, p, p, 128, 64, 0.5, 65, 1, None, ctypes.byref(h))
    assert st == plib.PROX_EINVAL and "k=" in plib.last_error()
    st = lib.prox_layer_create(p, p, p, 128, 64, 0.5, 0, 1, None, ctypes.byref(h))
    assert st == plib.PROX_EINVAL
    # negative threshold, unaligned pointer
    st = lib.prox_layer_create(p, p, p, 128, 64, -1.0, 8, 1, None, ctypes.byref(h))
    assert st == plib.PROX_EINVAL
    st = lib.prox_layer_create(ctypes.c_void_p(18), p, p, 128, 64, 0.5, 8, 1, None,
                               ctypes.byref(h))
    assert st == plib.PROX_EINVAL and "aligned" in plib.last_error()
    # packer: only group 128
    assert lib.prox_pack_proxy(p, 128, 64, 64, p, p, None) == plib.PROX_EINVAL
    # calibration: s1 outside [0, 1]
    tau = ctypes.c_float(1.0)
    assert lib.prox_calibrate_thresholds(p, 4, 128, 1.5, ctypes.byref(tau), None) == plib.PROX_EINVAL
    # s1 = 0 needs no device work and gives tau = 0
    assert lib.prox_calibrate_thresholds(p, 4, 128, 0.0, ctypes.byref(tau), None) == plib.PROX_OK
    assert tau.value == 0.0
    # allocation-free calibration: oversize input, bad s1, misaligned outputs,
    # all refused on the host before any device work
    assert lib.prox_calibrate_thresholds_noalloc(p, 65536, 32768, 0.5, p, None) == plib.PROX_EINVAL
    assert "2^31" in plib.last_error()
    assert lib.prox_calibrate_thresholds_noalloc(p, 4, 128, -0.1, p, None) == plib.PROX_EINVAL
    assert lib.prox_calibrate_thresholds_noalloc(p, 4, 128, 0.5, ctypes.c_void_p(18), None) == plib.PROX_EINVAL
    assert lib.prox_calibrate_thresholds_noalloc(ctypes.c_void_p(20), 4, 128, 0.5, p, None) == plib.PROX_EINVAL
    # NULL handles
    assert lib.prox_ffn_forward(None, p, p, 1, None) == plib.PROX_EINVAL
    assert lib.prox_dense_ffn(None, p, p, 1, None) == plib.PROX_EINVAL
    assert lib.prox_layer_set_k(None, 3) == plib.PROX_EINVAL
    assert lib.prox_layer_destroy(None) == plib.PROX_OK
    # copy: size must be a multiple of 16
    assert lib.prox_copy(p, p, 20, None) == plib.PROX_EINVAL


def test_cost_model_host_functions_match_the_oracle(plib):
    """The library's host-only cost model (Prox §4.2, App. A.7) against the
    oracle's restatement, and its argument checks."""
    from oracle import prox_oracle as orc
    lib = plib.lib
    D = ctypes.c_double
    a, b, c = D(), D(), D()
    for alpha in (1.0 / 3.0, 0.285, 0.5):
        for e in np.linspace(0.0, 0.9, 37):
            try:
                want = orc.allocate_sparsity(e, alpha)
            except ValueError:
                assert lib.prox_allocate_sparsity(e, alpha, 0.7, 0.0, 0.7, ctypes.byref(a),
                                                  ctypes.byref(b)) == plib.PROX_EINVAL
                continue
            assert lib.prox_allocate_sparsity(e, alpha, 0.7, 0.0, 0.7, ctypes.byref(a),
                                              ctypes.byref(b)) == plib.PROX_OK
            assert a.value == pytest.approx(want[0], abs=1e-12)
            assert b.value == pytest.approx(want[1], abs=1e-12)
            assert lib.prox_effective_sparsity(a.value, b.value, alpha, ctypes.byref(c)) == plib.PROX_OK
            assert c.value == pytest.approx(orc.effective_sparsity(a.value, b.value, alpha), abs=1e-12)
    assert lib.prox_runtime_sparsity(1000, 300, 4, 512, 1024, 1.0 / 3.0, ctypes.byref(a),
                                     ctypes.byref(b), ctypes.byref(c)) == plib.PROX_OK
    want = orc.runtime_sparsity(1000, 300, 4, 512, 1024)
    assert (a.value, b.value, c.value) == pytest.approx(want, abs=1e-15)
    # bad arguments
    assert lib.prox_allocate_sparsity(0.5, 0.0, 0.7, 0.0, 0.7, ctypes.byref(a), ctypes.byref(b)) == plib.PROX_EINVAL
    assert lib.prox_allocate_sparsity(0.5, 1 / 3, 0.7, 0.5, 0.2, ctypes.byref(a), ctypes.byref(b)) == plib.PROX_EINVAL
    assert lib.prox_allocate_sparsity(float("nan"), 1 / 3, 0.7, 0.0, 0.7, ctypes.byref(a),
                                      ctypes.byref(b)) == plib.PROX_EINVAL
    assert lib.prox_allocate_sparsity(0.99, 1 / 3, 0.7, 0.0, 0.7, ctypes.byref(a), ctypes.byref(b)) == plib.PROX_EINVAL
    assert "out of reach" in plib.last_error()
    assert lib.prox_effective_sparsity(1.2, 0.5, 1 / 3, ctypes.byref(c)) == plib.PROX_EINVAL
    assert lib.prox_runtime_sparsity(5000, 0, 4, 512, 1024, 1 / 3, None, None, None) == plib.PROX_EINVAL
    assert lib.prox_runtime_sparsity(0, 0, 0, 512, 1024, 1 / 3, None, None, None) == plib.PROX_EINVAL


def test_fault_injection_arguments(plib):
    lib = plib.lib
    assert lib.prox_debug_fail_alloc(-1) == plib.PROX_EINVAL
    assert lib.prox_debug_fail_alloc(3) == plib.PROX_OK
    assert lib.prox_debug_fail_alloc(0) == plib.PROX_OK  # cancelled again


def test_every_entry_point_is_documented():
    """Each PROX_API declaration in include/prox.h follows a comment block (a
    declaration may share the comment of the one right above it)."""
    lines = open(os.path.join(ROOT, "include", "prox.h")).read().splitlines()
    undocumented = []
    for i, line in enumerate(lines):
        m = re.search(r"PROX_API\s+[\w\s\*]+?\b(prox_\w+)\s*\(", line)
        if not m:
            continue
        j = i - 1
        while j >= 0 and lines[j].strip().startswith("PROX_API"):
            j -= 1  # grouped declarations share one comment
        if j < 0 or not lines[j].strip().endswith("*/"):
            undocumented.append(m.group(1))
    assert not undocumented, undocumented


def test_binding_refuses_short_or_host_buffers():
    """The Python binding checks what the C ABI cannot see (tensor sizes and
    memory spaces) before any library call."""
    import torch
    import activation_sparse_swiglu_b200 as prox
    with pytest.raises(ValueError):
        prox._need(torch.empty(10), 11, "out")
    prox._need(torch.empty(10), 10, "out")
    with pytest.raises(ValueError):
        prox._one_token(torch.empty(2, 512), 512)
    prox._one_token(torch.empty(512), 512)
    with pytest.raises(TypeError):  # host tensors never reach the copy kernel
        prox.copy(torch.empty(16), torch.empty(16))
    with pytest.raises(TypeError):
        prox.rmsnorm(torch.empty(4, 8))


def test_noalloc_binding_checks_the_device(monkeypatch):
    """The binding refuses tensors that are not on the current CUDA device
    before the allocation-free calibration runs (checked with stand-ins for
    tensors, no GPU needed)."""
    import types

    import torch

    import activation_sparse_swiglu_b200 as prox
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    here = types.SimpleNamespace(device=torch.device("cuda", 0))
    other = types.SimpleNamespace(device=torch.device("cuda", 1))
    host = types.SimpleNamespace(device=torch.device("cpu"))
    prox._on_current_device(x_cal=here, tau=here)
    for bad in (other, host):
        with pytest.raises(ValueError, match="current CUDA device"):
            prox._on_current_device(x_cal=here, tau=bad)
        with pytest.raises(ValueError, match="current CUDA device"):
            prox._on_current_device(x_cal=bad, tau=here)
