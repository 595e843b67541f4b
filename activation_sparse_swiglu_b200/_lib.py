"""ctypes loader for libprox.so (the C ABI declared in include/prox.h).

Argument marshalling only: every step of the decode step runs in the CUDA
library.  Importing this module fails loudly when the library is missing.
"""

from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libprox.so")

PROX_OK, PROX_EINVAL, PROX_ENOMEM, PROX_ECUDA, PROX_EUNSUPPORTED, PROX_EDEVICE = range(6)
STATUS_NAMES = {0: "PROX_OK", 1: "PROX_EINVAL", 2: "PROX_ENOMEM", 3: "PROX_ECUDA",
                4: "PROX_EUNSUPPORTED", 5: "PROX_EDEVICE"}
DEVERR_MASK_INDEX = 0x1
DEVERR_WAIT_TIMEOUT = 0x2


class ProxError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class LayerInfo(ctypes.Structure):
    _fields_ = [
        ("d_model", ctypes.c_int), ("d_ff", ctypes.c_int), ("group", ctypes.c_int),
        ("k", ctypes.c_int), ("max_batch", ctypes.c_int), ("tau_x", ctypes.c_float),
        ("stage1_col_slices", ctypes.c_int), ("stage1_ctas", ctypes.c_int),
        ("stage2_ctas", ctypes.c_int), ("stage2_ring_slots", ctypes.c_int),
        ("weight_bytes", ctypes.c_size_t), ("proxy_bytes", ctypes.c_size_t),
        ("workspace_bytes", ctypes.c_size_t),
        ("mask_mode", ctypes.c_int), ("tau_s", ctypes.c_float),
        ("activation", ctypes.c_int), ("stage2_source", ctypes.c_int),
    ]


MASK_TOPK = 0
MASK_THRESHOLD = 1
ACT_SILU, ACT_GELU_TANH, ACT_GELU_ERF = 0, 1, 2
STAGE2_EXACT, STAGE2_PROXY_VALUES = 0, 1


_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_S = ctypes.c_size_t
_D = ctypes.c_double
_L = ctypes.c_int64

# name -> (restype, argtypes); the order follows include/prox.h
SIGNATURES = {
    "prox_pack_proxy": (_I, [_P, _I, _I, _I, _P, _P, _P]),
    "prox_calibrate_thresholds": (_I, [_P, _I, _I, _F, ctypes.POINTER(_F), _P]),
    "prox_calibrate_thresholds_noalloc": (_I, [_P, _I, _I, _F, _P, _P]),
    "prox_layer_create": (_I, [_P, _P, _P, _I, _I, _F, _I, _I, _P, ctypes.POINTER(_P)]),
    "prox_layer_destroy": (_I, [_P]),
    "prox_layer_set_tau": (_I, [_P, _F]),
    "prox_layer_set_k": (_I, [_P, _I]),
    "prox_layer_set_mask": (_I, [_P, _I, _F]),
    "prox_layer_set_activation": (_I, [_P, _I]),
    "prox_layer_set_stage2": (_I, [_P, _I]),
    "prox_layer_get_info": (_I, [_P, ctypes.POINTER(LayerInfo)]),
    "prox_layer_error": (_I, [_P, ctypes.POINTER(ctypes.c_int32), _P]),
    "prox_layer_stats": (_I, [_P, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64),
                              ctypes.POINTER(ctypes.c_int64), _P]),
    "prox_effective_sparsity": (_I, [_D, _D, _D, ctypes.POINTER(_D)]),
    "prox_allocate_sparsity": (_I, [_D, _D, _D, _D, _D, ctypes.POINTER(_D), ctypes.POINTER(_D)]),
    "prox_runtime_sparsity": (_I, [_L, _L, _L, _I, _I, _D, ctypes.POINTER(_D), ctypes.POINTER(_D),
                                   ctypes.POINTER(_D)]),
    "prox_ffn_forward": (_I, [_P, _P, _P, _I, _P]),
    "prox_dense_ffn": (_I, [_P, _P, _P, _I, _P]),
    "prox_ffn_forward_batch": (_I, [_P, _P, _P, _I, _P]),
    "prox_dense_ffn_batch": (_I, [_P, _P, _P, _I, _P]),
    "prox_batch_union_sizes": (_I, [_P, _P, _P, _P]),
    "prox_debug_batch_masks": (_I, [_P, _P, _I, _P]),
    "prox_ffn_forward_host": (_I, [_P, _P, _P, _I, _P]),
    "prox_ffn_forward_profiled": (_I, [_P, _P, _P, ctypes.POINTER(_P), _P, _P]),
    "prox_debug_stage1": (_I, [_P, _P, _P, _P, _P, _P, _P, _P]),
    "prox_layer_proxy_scores": (_I, [_P, _P, _I, _P, _P]),
    "prox_debug_mask": (_I, [_P, _P, _P, _P, _P]),
    "prox_forward_with_mask": (_I, [_P, _P, _P, _I, _P, _P, _P]),
    "prox_debug_fail_alloc": (_I, [_I]),
    "prox_debug_wait_timeout": (_I, [_P, _P]),
    "prox_debug_token_geometry": (_I, [_I, _I, _I, _P]),
    "prox_rmsnorm": (_I, [_P, _P, _I, _I, _F, _P]),
    "prox_copy": (_I, [_P, _P, _S, _P]),
    "prox_last_error": (_S, [ctypes.c_char_p, _S]),
    "prox_version": (ctypes.c_char_p, []),
}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m activation_sparse_swiglu_b200.build` "
            "(the CUDA library is required; there is no fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def last_error() -> str:
    buf = ctypes.create_string_buffer(1024)
    lib.prox_last_error(buf, len(buf))
    return buf.value.decode(errors="replace")


def check(status: int) -> None:
    if status != PROX_OK:
        raise ProxError(status, last_error())
