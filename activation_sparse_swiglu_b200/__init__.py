"""B200-native Prox two-stage sparse SwiGLU FFN decode step.

Python binding over the C ABI of libprox.so (include/prox.h).  PyTorch is used
only for device memory and CUDA streams; every step of the computation runs
in the library's sm_100a kernels.

    import activation_sparse_swiglu_b200 as prox
    tau = prox.calibrate_thresholds(x_cal, s1=0.5)
    layer = prox.Layer(w_gate, w_up, w_down, tau=tau, k=4301)
    y = layer.forward(x)          # x: fp32 [B, d_model] on the GPU
"""

from __future__ import annotations

import ctypes

import torch

from ._lib import (ACT_GELU_ERF, ACT_GELU_TANH, ACT_SILU, DEVERR_MASK_INDEX, DEVERR_WAIT_TIMEOUT,
                   MASK_THRESHOLD, MASK_TOPK, STAGE2_EXACT, STAGE2_PROXY_VALUES, LayerInfo,
                   ProxError, check, last_error, lib)

__all__ = ["Layer", "phase_times_us", "pack_proxy", "calibrate_thresholds", "rmsnorm", "copy", "version",
           "effective_sparsity", "allocate_sparsity", "runtime_sparsity", "ALPHA",
           "ACT_SILU", "ACT_GELU_TANH", "ACT_GELU_ERF", "STAGE2_EXACT", "STAGE2_PROXY_VALUES",
           "ProxError", "DEVERR_MASK_INDEX", "DEVERR_WAIT_TIMEOUT", "MASK_TOPK", "MASK_THRESHOLD",
           "last_error", "lib"]

GROUP = 128


def version() -> str:
    return lib.prox_version().decode()


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _ptr(t: torch.Tensor | None) -> ctypes.c_void_p:
    if t is None:
        return ctypes.c_void_p(0)
    return ctypes.c_void_p(t.data_ptr())


def _dev(t: torch.Tensor, dtype: torch.dtype, name: str) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _need(t: torch.Tensor, numel: int, name: str) -> None:
    """The library writes `numel` values through t's pointer: t must hold them."""
    if t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} values, {numel} needed")


def _on_current_device(**tensors) -> None:
    """Every named tensor lives on the current CUDA device (the library
    launches on that device and reads the pointers there)."""
    cur = torch.cuda.current_device()
    for name, t in tensors.items():
        if t.device.type != "cuda" or t.device.index != cur:
            raise ValueError(f"{name} is on {t.device}, not on the current CUDA device cuda:{cur}")


def _one_token(x: torch.Tensor, d_model: int, name: str = "x") -> None:
    if x.numel() != d_model:
        raise ValueError(f"{name} must hold one token of d_model={d_model} values, "
                         f"got {x.numel()}")


def pack_proxy(w: torch.Tensor, group: int = GROUP, stream=None):
    """INT4 proxy of a bf16 [d_model, d_ff] weight: (codes uint8 [d, d_ff/2],
    scales fp16 [d/group, d_ff])."""
    _dev(w, torch.bfloat16, "w")
    d, f = w.shape
    codes = torch.empty((d, f // 2), dtype=torch.uint8, device=w.device)
    scales = torch.empty((d // group, f), dtype=torch.float16, device=w.device)
    check(lib.prox_pack_proxy(_ptr(w), d, f, group, _ptr(codes), _ptr(scales), _stream(stream)))
    return codes, scales


def calibrate_thresholds(x_cal: torch.Tensor, s1: float, stream=None) -> float:
    """Exact s1-quantile of |x_cal| (fp32 [n_tok, d_model] on the GPU)."""
    _dev(x_cal, torch.float32, "x_cal")
    n, d = x_cal.shape
    tau = ctypes.c_float(0.0)
    check(lib.prox_calibrate_thresholds(_ptr(x_cal), n, d, float(s1), ctypes.byref(tau),
                                        _stream(stream)))
    return float(tau.value)


def calibrate_thresholds_noalloc(x_cal: torch.Tensor, s1: float, tau: torch.Tensor,
                                 stream=None) -> torch.Tensor:
    """The same quantile written to the 1-element fp32 device tensor `tau` in
    stream order, with no device allocation, for callers that cannot allocate
    at that point (their device memory belongs to another allocator, or the
    implicit synchronisation of an allocation is not acceptable).  The scratch
    is a fixed static array per device; concurrent calls on one device race.
    x_cal and tau must live on the current CUDA device."""
    _dev(x_cal, torch.float32, "x_cal")
    _dev(tau, torch.float32, "tau")
    if tau.numel() < 1:
        raise ValueError("tau needs one element")
    _on_current_device(x_cal=x_cal, tau=tau)
    n, d = x_cal.shape
    check(lib.prox_calibrate_thresholds_noalloc(_ptr(x_cal), n, d, float(s1), _ptr(tau),
                                                _stream(stream)))
    return tau


def rmsnorm(y: torch.Tensor, eps: float = 1e-6, out: torch.Tensor | None = None, stream=None):
    _dev(y, torch.float32, "y")
    y2 = y.reshape(-1, y.shape[-1])
    if out is None:
        out = torch.empty_like(y)
    else:
        _dev(out, torch.float32, "out")
        _need(out, y2.numel(), "out")
    check(lib.prox_rmsnorm(_ptr(y2), _ptr(out), y2.shape[0], y2.shape[1], float(eps),
                           _stream(stream)))
    return out


def copy(src: torch.Tensor, dst: torch.Tensor, stream=None) -> None:
    for t, name in ((src, "src"), (dst, "dst")):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous CUDA tensor")
    nbytes = src.numel() * src.element_size()
    if dst.numel() * dst.element_size() < nbytes:
        raise ValueError("dst is smaller than src")
    check(lib.prox_copy(_ptr(src), _ptr(dst), nbytes, _stream(stream)))


ALPHA = 1.0 / 3.0  # proxy-projection cost the paper allocates with (Prox §4.2)


def phase_times_us(stamps) -> "np.ndarray":
    """Raw stamps of Layer.forward_profiled ([P, 24] int64, host or device) as
    float64 microseconds from the earliest CTA entry, NaN where a CTA wrote no
    stamp; slot 13 (a channel count) is passed through.  Each CTA's cycle
    counts are placed on the global-timer line by its entry and exit readings
    (slots 0 / 22 and 21 / 23)."""
    import numpy as np
    a = np.asarray(stamps.cpu() if hasattr(stamps, "cpu") else stamps).astype(np.float64)
    clk0, clk1, gt0, gt1 = a[:, 0:1], a[:, 21:22], a[:, 22:23], a[:, 23:24]
    ns_per_clk = (gt1 - gt0) / np.maximum(clk1 - clk0, 1.0)
    t = gt0 + (a - clk0) * ns_per_clk
    t[a == 0] = np.nan
    t[:, 22], t[:, 23] = a[:, 22], a[:, 23]
    out = (t - np.nanmin(gt0)) / 1e3
    out[:, 13] = a[:, 13]
    return out


def effective_sparsity(s1: float, s2: float, alpha: float = ALPHA) -> float:
    """e = s2 - 2 alpha (1 - s1) / 3 (Prox §4.2 cost model)."""
    e = ctypes.c_double(0.0)
    check(lib.prox_effective_sparsity(float(s1), float(s2), float(alpha), ctypes.byref(e)))
    return e.value


def allocate_sparsity(e: float, alpha: float = ALPHA, s_ref: float = 0.7,
                      s1_bounds: tuple[float, float] = (0.0, 0.7)) -> tuple[float, float]:
    """(s1, s2) for a target effective sparsity e (Prox §4.2 allocation policy)."""
    s1, s2 = ctypes.c_double(0.0), ctypes.c_double(0.0)
    check(lib.prox_allocate_sparsity(float(e), float(alpha), float(s_ref), float(s1_bounds[0]),
                                     float(s1_bounds[1]), ctypes.byref(s1), ctypes.byref(s2)))
    return s1.value, s2.value


def runtime_sparsity(sum_nx: int, sum_sel: int, tokens: int, d_model: int, d_ff: int,
                     alpha: float = ALPHA) -> tuple[float, float, float]:
    """(s1^, s2^, e^) from accumulated mask counts (Prox App. A.7)."""
    a, b, c = ctypes.c_double(0.0), ctypes.c_double(0.0), ctypes.c_double(0.0)
    check(lib.prox_runtime_sparsity(int(sum_nx), int(sum_sel), int(tokens), int(d_model), int(d_ff),
                                    float(alpha), ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)))
    return a.value, b.value, c.value


class Layer:
    """One Prox FFN layer resident on the current CUDA device.

    w_gate, w_up: bf16 [d_model, d_ff]; w_down: bf16 [d_ff, d_model] (math
    layout, CUDA tensors).  The library repacks them into its own buffers, so
    the tensors may be freed afterwards.
    """

    def __init__(self, w_gate, w_up, w_down, tau: float, k: int, max_batch: int = 1,
                 stream=None):
        _dev(w_gate, torch.bfloat16, "w_gate")
        _dev(w_up, torch.bfloat16, "w_up")
        _dev(w_down, torch.bfloat16, "w_down")
        d, f = w_gate.shape
        if tuple(w_up.shape) != (d, f) or tuple(w_down.shape) != (f, d):
            raise ValueError("inconsistent weight shapes")
        self.d_model, self.d_ff = d, f
        self.device = w_gate.device
        h = ctypes.c_void_p(0)
        check(lib.prox_layer_create(_ptr(w_gate), _ptr(w_up), _ptr(w_down), d, f, float(tau),
                                    int(k), int(max_batch), _stream(stream), ctypes.byref(h)))
        self._h = h

    # -- lifetime --------------------------------------------------------
    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            with torch.cuda.device(self.device):
                lib.prox_layer_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def handle(self) -> ctypes.c_void_p:
        if self._h is None:
            raise RuntimeError("layer is closed")
        return self._h

    # -- parameters ------------------------------------------------------
    def info(self) -> dict:
        inf = LayerInfo()
        check(lib.prox_layer_get_info(self.handle, ctypes.byref(inf)))
        return {name: getattr(inf, name) for name, _ in LayerInfo._fields_}

    @property
    def k(self) -> int:
        return self.info()["k"]

    @property
    def tau(self) -> float:
        return self.info()["tau_x"]

    def set_tau(self, tau: float) -> None:
        check(lib.prox_layer_set_tau(self.handle, float(tau)))

    def set_k(self, k: int) -> None:
        check(lib.prox_layer_set_k(self.handle, int(k)))

    def set_mask(self, mode: int, tau_s: float = 0.0) -> None:
        """Stage-2 rule: MASK_TOPK (uses k) or MASK_THRESHOLD (score >= tau_s)."""
        check(lib.prox_layer_set_mask(self.handle, int(mode), float(tau_s)))

    def set_activation(self, act: int) -> None:
        """Gate activation: ACT_SILU (SwiGLU), ACT_GELU_TANH or ACT_GELU_ERF (GeGLU)."""
        check(lib.prox_layer_set_activation(self.handle, int(act)))

    def set_stage2(self, source: int) -> None:
        """STAGE2_EXACT (the method) or STAGE2_PROXY_VALUES (ablation A3)."""
        check(lib.prox_layer_set_stage2(self.handle, int(source)))

    def error_word(self, stream=None) -> int:
        v = ctypes.c_int32(0)
        check(lib.prox_layer_error(self.handle, ctypes.byref(v), _stream(stream)))
        return int(v.value)

    def stats(self, stream=None, with_selected: bool = False):
        """(sum of n_x, tokens[, sum of selected Stage-2 channels]) since the last call."""
        s, t, c = ctypes.c_int64(0), ctypes.c_int64(0), ctypes.c_int64(0)
        check(lib.prox_layer_stats(self.handle, ctypes.byref(s), ctypes.byref(t), ctypes.byref(c),
                                   _stream(stream)))
        if with_selected:
            return int(s.value), int(t.value), int(c.value)
        return int(s.value), int(t.value)

    def runtime_sparsity(self, alpha: float = ALPHA, stream=None) -> dict:
        """Realised s1^, s2^ and e^ of the tokens run since the last stats read
        (Prox App. A.7 "Runtime sparsity"); resets the counters."""
        s, t, c = self.stats(stream, with_selected=True)
        inf = self.info()
        s1, s2, e = runtime_sparsity(s, c, t, inf["d_model"], inf["d_ff"], alpha)
        return {"tokens": t, "s1": s1, "s2": s2, "e": e}

    def proxy_scores(self, x: torch.Tensor, stream=None) -> torch.Tensor:
        """Stage-1 scores |act(g~) u~| of tokens x [B, d] as fp32 [B, d_ff]."""
        _dev(x, torch.float32, "x")
        x2 = x.reshape(-1, self.d_model)
        out = torch.empty((x2.shape[0], self.d_ff), dtype=torch.float32, device=x.device)
        check(lib.prox_layer_proxy_scores(self.handle, _ptr(x2), x2.shape[0], _ptr(out),
                                          _stream(stream)))
        return out

    def debug_mask(self, x: torch.Tensor, stream=None) -> torch.Tensor:
        """The Stage-2 channels one token selects under the current rule (int32, ascending)."""
        _dev(x, torch.float32, "x")
        _one_token(x, self.d_model)
        idx = torch.empty(self.d_ff, dtype=torch.int32, device=x.device)
        n = torch.zeros(1, dtype=torch.int32, device=x.device)
        check(lib.prox_debug_mask(self.handle, _ptr(x), _ptr(idx), _ptr(n), _stream(stream)))
        return idx[: int(n.item())]

    # -- compute ---------------------------------------------------------
    def _io(self, x, out):
        _dev(x, torch.float32, "x")
        x2 = x.reshape(-1, self.d_model)
        if out is None:
            out = torch.empty_like(x2)
        else:
            _dev(out, torch.float32, "out")
            _need(out, x2.numel(), "out")
        return x2, out

    def forward(self, x: torch.Tensor, out: torch.Tensor | None = None, stream=None):
        x2, out = self._io(x, out)
        check(lib.prox_ffn_forward(self.handle, _ptr(x2), _ptr(out), x2.shape[0], _stream(stream)))
        return out

    __call__ = forward

    def dense(self, x: torch.Tensor, out: torch.Tensor | None = None, stream=None):
        x2, out = self._io(x, out)
        check(lib.prox_dense_ffn(self.handle, _ptr(x2), _ptr(out), x2.shape[0], _stream(stream)))
        return out

    def forward_batch(self, x: torch.Tensor, out: torch.Tensor | None = None, stream=None):
        """B <= 16 tokens in one batched step (union loads; needs max_batch > 1)."""
        x2, out = self._io(x, out)
        check(lib.prox_ffn_forward_batch(self.handle, _ptr(x2), _ptr(out), x2.shape[0],
                                         _stream(stream)))
        return out

    def dense_batch(self, x: torch.Tensor, out: torch.Tensor | None = None, stream=None):
        """Dense baseline for B <= 16 tokens reading every weight once."""
        x2, out = self._io(x, out)
        check(lib.prox_dense_ffn_batch(self.handle, _ptr(x2), _ptr(out), x2.shape[0],
                                       _stream(stream)))
        return out

    def batch_union_sizes(self, stream=None) -> tuple[int, int]:
        """(union input rows, union channels) of the last forward_batch."""
        rows, chans = ctypes.c_int32(0), ctypes.c_int32(0)
        check(lib.prox_batch_union_sizes(self.handle, ctypes.byref(rows), ctypes.byref(chans),
                                         _stream(stream)))
        return rows.value, chans.value

    def debug_batch_masks(self, B: int, stream=None) -> torch.Tensor:
        """int32 [B, d_ff] per-token masks of the last forward_batch (CUDA)."""
        m = torch.empty((B, self.d_ff), dtype=torch.int32, device="cuda")
        check(lib.prox_debug_batch_masks(self.handle, _ptr(m), B, _stream(stream)))
        return m

    def forward_host(self, x_host: torch.Tensor, out_host: torch.Tensor | None = None,
                     stream=None):
        """Tokens whose inputs/outputs live in host memory (pinned for async copies)."""
        if x_host.is_cuda or x_host.dtype != torch.float32 or not x_host.is_contiguous():
            raise TypeError("x_host must be a contiguous fp32 CPU tensor")
        x2 = x_host.reshape(-1, self.d_model)
        if out_host is None:
            out_host = torch.empty_like(x2)
        elif (out_host.is_cuda or out_host.dtype != torch.float32
              or not out_host.is_contiguous()):
            raise TypeError("out_host must be a contiguous fp32 CPU tensor")
        else:
            _need(out_host, x2.numel(), "out_host")
        check(lib.prox_ffn_forward_host(self.handle, _ptr(x2), _ptr(out_host), x2.shape[0],
                                        _stream(stream)))
        return out_host

    def forward_profiled(self, x: torch.Tensor, out: torch.Tensor, events,
                         phase_ns: torch.Tensor | None = None, stream=None):
        """One token with its kernel bracketed by 2 torch.cuda.Event(enable_timing=True)
        (no programmatic overlap).  phase_ns: optional int64 CUDA tensor
        [stage1_ctas, 24] receiving each CTA's raw phase stamps (SM cycle counts
        plus the global timer at entry and exit; slot meanings in
        include/prox.h); phase_times_us turns them into one time line."""
        _dev(x, torch.float32, "x")
        _dev(out, torch.float32, "out")
        _one_token(x, self.d_model)
        _need(out, self.d_model, "out")
        if len(events) != 2:
            raise ValueError("forward_profiled needs 2 events")
        if phase_ns is not None:
            _dev(phase_ns, torch.int64, "phase_ns")
            _need(phase_ns, self.info()["stage1_ctas"] * 24, "phase_ns")
        arr = (ctypes.c_void_p * 2)(*[ctypes.c_void_p(e.cuda_event) for e in events])
        check(lib.prox_ffn_forward_profiled(self.handle, _ptr(x), _ptr(out), arr, _ptr(phase_ns),
                                            _stream(stream)))

    def debug_stage1(self, x: torch.Tensor, stream=None) -> dict:
        """Stage 1 of one token: idx_x, n_x, g_tilde, u_tilde, idx_s (CUDA tensors)."""
        _dev(x, torch.float32, "x")
        _one_token(x, self.d_model)
        dev = x.device
        k = self.k
        idx_x = torch.full((self.d_model,), -1, dtype=torch.int32, device=dev)
        n_x = torch.zeros(1, dtype=torch.int32, device=dev)
        g = torch.empty(self.d_ff, dtype=torch.float32, device=dev)
        u = torch.empty(self.d_ff, dtype=torch.float32, device=dev)
        idx_s = torch.empty(k, dtype=torch.int32, device=dev)
        check(lib.prox_debug_stage1(self.handle, _ptr(x), _ptr(idx_x), _ptr(n_x), _ptr(g), _ptr(u),
                                    _ptr(idx_s), _stream(stream)))
        return dict(idx_x=idx_x, n_x=n_x, g_tilde=g, u_tilde=u, idx_s=idx_s)

    def forward_with_mask(self, x: torch.Tensor, idx_s: torch.Tensor,
                          out: torch.Tensor | None = None, want_s: bool = False, stream=None):
        """Stage 2 on a given channel list (int32 CUDA tensor)."""
        _dev(x, torch.float32, "x")
        _dev(idx_s, torch.int32, "idx_s")
        _one_token(x, self.d_model)
        if out is None:
            out = torch.empty(self.d_model, dtype=torch.float32, device=x.device)
        else:
            _dev(out, torch.float32, "out")
            _need(out, self.d_model, "out")
        s_sp = torch.empty(idx_s.numel(), dtype=torch.float32, device=x.device) if want_s else None
        check(lib.prox_forward_with_mask(self.handle, _ptr(x), _ptr(idx_s), idx_s.numel(), _ptr(out),
                                         _ptr(s_sp), _stream(stream)))
        return (out, s_sp) if want_s else out
