"""The per-token kernel's host-side plan (prox_debug_token_geometry, the same
planning code prox_layer_create runs) against the shape rules of
include/prox.h, on the CPU: every shape the rules admit fits one CTA's shared
memory on a 148-SM B200 with at least two Stage-1 tiles per warp; on devices
with fewer SMs every shape within the stated Stage-1 bound
ceil(d_ff/512) * d_model <= 15535 * SMs (and d_ff <= 512 * SMs) is planned,
and the largest shape is refused where it exceeds that bound."""

import ctypes
import math

import pytest

PROX_OK, PROX_EINVAL, PROX_EUNSUPPORTED = 0, 1, 4
SMEM_PER_CTA = 232448  # opt-in dynamic shared memory per CTA on sm_100
D_MODELS = (128, 256, 512, 1024, 2048, 4096, 5120, 8192, 12288, 16384)
D_FFS = (32, 1376, 4096, 11008, 14336, 17408, 28672, 32768)


@pytest.fixture(scope="module")
def geometry():
    from activation_sparse_swiglu_b200 import _lib

    def plan(d, f, sms):
        out = (ctypes.c_int32 * 6)()
        st = _lib.lib.prox_debug_token_geometry(d, f, sms, out)
        return st, list(out)

    return plan


def test_every_admitted_shape_fits_148_sms(geometry):
    for d in D_MODELS:
        for f in D_FFS:
            st, (c, lmax, depth, slots, groups, smem) = geometry(d, f, 148)
            assert st == PROX_OK, (d, f)
            assert c == math.ceil(f / 512)
            assert lmax >= math.ceil(c * d / 148)
            assert depth >= 2 and slots >= 2 and groups in (1, 2, 4)
            assert 0 < smem <= SMEM_PER_CTA


def test_stated_bound_on_fewer_sms(geometry):
    for sms in (24, 40, 60, 80, 100, 132):
        for d in D_MODELS:
            for f in D_FFS:
                within = math.ceil(f / 512) * d <= 15535 * sms and math.ceil(f / sms) <= 512
                if within:
                    st, out = geometry(d, f, sms)
                    assert st == PROX_OK, (sms, d, f)
                    assert out[2] >= 2 and out[5] <= SMEM_PER_CTA
    # 64 * 16384 = 1.05 M > 15535 * 60: refused, not run past shared memory
    st, _ = geometry(16384, 32768, 60)
    assert st == PROX_EUNSUPPORTED


def test_channels_per_cta_rule(geometry):
    # scoring takes one channel per thread: d_ff <= 512 * SMs
    assert geometry(4096, 32768, 64)[0] == PROX_OK
    assert geometry(4096, 32768, 63)[0] == PROX_EUNSUPPORTED


def test_bad_arguments(geometry):
    assert geometry(100, 14336, 148)[0] == PROX_EINVAL      # d_model not a multiple of 128
    assert geometry(4096, 14340, 148)[0] == PROX_EINVAL     # d_ff not a multiple of 32
    assert geometry(16512, 14336, 148)[0] == PROX_EINVAL    # d_model above 16384
    assert geometry(4096, 32800, 148)[0] == PROX_EINVAL     # d_ff above 32768
    assert geometry(4096, 14336, 0)[0] == PROX_EUNSUPPORTED
    assert geometry(4096, 14336, 300)[0] == PROX_EUNSUPPORTED  # more SMs than the kernel's grid takes
