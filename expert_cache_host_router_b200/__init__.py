"""Python binding of libmoe (include/moe_cache.h): argument marshalling only.

Every step of the decode path runs in the CUDA library; this module converts numpy
arrays and torch tensors to pointers and status codes to exceptions.  There is no
Python or CPU implementation of the path here: if libmoe.so is missing the import of
the binding's functions raises.
"""
from __future__ import annotations

import atexit
import ctypes
import os
import re
import weakref

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_lib", "libmoe.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "moe_cache.h")

MOE_OK = 0
MOE_ERR_INVALID = -1
MOE_ERR_NOMEM = -2
MOE_ERR_CUDA = -3
MOE_ERR_TIMEOUT = -4
MOE_ERR_STATE = -5
MOE_ERR_UNSUPPORTED = -6
MOE_ERR_DEVICE = -7
MOE_PIN_HIT, MOE_RING_HIT, MOE_MISS = 0, 1, 2
MOE_PLACE_CALIBRATED, MOE_PLACE_UNIFORM = 0, 1
MOE_MISS_COPY_ENGINE, MOE_MISS_SM_PULL = 0, 1


class MoEError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status} ({status_string(status)})")


class Config(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("hidden", ctypes.c_int32),
                ("n_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("inter", ctypes.c_int32), ("shared_inter", ctypes.c_int32),
                ("ring_slots", ctypes.c_int32), ("use_rmsnorm", ctypes.c_int32),
                ("rms_eps", ctypes.c_float), ("device", ctypes.c_int32),
                ("log_steps", ctypes.c_int32), ("wait_timeout_ms", ctypes.c_uint32)]


class Weights(ctypes.Structure):
    _fields_ = [("expert_q4_0", ctypes.POINTER(ctypes.c_void_p)),
                ("shared_q4_0", ctypes.POINTER(ctypes.c_void_p)),
                ("router_bf16", ctypes.c_void_p), ("router_bias", ctypes.c_void_p),
                ("rms_gain", ctypes.c_void_p)]


class NoAllocWeights(ctypes.Structure):
    _fields_ = [("experts_dev", ctypes.c_void_p), ("shared_dev", ctypes.c_void_p),
                ("router_dev", ctypes.c_void_p), ("bias_dev", ctypes.c_void_p),
                ("gain_dev", ctypes.c_void_p)]


class Event(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("step", "layer", "rank", "expert", "kind", "slot", "evicted")]


EVENT_DTYPE = np.dtype([(n, np.int32) for n in
                        ("step", "layer", "rank", "expert", "kind", "slot", "evicted")])


class Stats(ctypes.Structure):
    _fields_ = [("steps", ctypes.c_uint64), ("accesses", ctypes.c_uint64),
                ("pin_hits", ctypes.c_uint64), ("ring_hits", ctypes.c_uint64),
                ("misses", ctypes.c_uint64), ("evictions", ctypes.c_uint64),
                ("bytes_copied", ctypes.c_uint64), ("staged_misses", ctypes.c_uint64),
                ("log_dropped", ctypes.c_uint64), ("device_error", ctypes.c_int32),
                ("n_pinned", ctypes.c_int32), ("residency", ctypes.c_float),
                ("placement", ctypes.c_int32), ("repins", ctypes.c_uint64),
                ("repin_copies", ctypes.c_uint64), ("miss_requests", ctypes.c_uint64),
                ("miss_served", ctypes.c_uint64), ("proxy_error", ctypes.c_int32),
                ("miss_path", ctypes.c_int32), ("pulled_misses", ctypes.c_uint64),
                ("copies_timed", ctypes.c_uint64), ("copy_ns_timed", ctypes.c_uint64)]

    def as_dict(self) -> dict:
        return {n: getattr(self, n) for n, _ in self._fields_}


_P = ctypes.c_void_p
_SIGS = {
    "moe_create": (ctypes.c_int, [ctypes.POINTER(Config), ctypes.POINTER(Weights), ctypes.POINTER(_P)]),
    "moe_load_layer": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.POINTER(ctypes.c_void_p), _P, _P, _P, _P]),
    "moe_set_residency": (ctypes.c_int, [_P, ctypes.c_float, _P, ctypes.c_int32]),
    "moe_decode_step": (ctypes.c_int, [_P, _P, _P, _P]),
    "moe_decode_step_host": (ctypes.c_int, [_P, _P, _P]),
    "moe_prefill": (ctypes.c_int, [_P, _P, ctypes.c_int32, _P, _P]),
    "moe_sync": (ctypes.c_int, [_P]),
    "moe_clear_error": (ctypes.c_int, [_P]),
    "moe_stats": (ctypes.c_int, [_P, ctypes.POINTER(Stats), _P, _P, ctypes.c_size_t,
                                 ctypes.POINTER(ctypes.c_size_t), ctypes.c_int32]),
    "moe_set_trace": (ctypes.c_int, [_P, _P, _P]),
    "moe_set_prefill_trace": (ctypes.c_int, [_P, _P, _P]),
    "moe_recalibrate": (ctypes.c_int, [_P]),
    "moe_set_router_bias": (ctypes.c_int, [_P, ctypes.c_int32, _P]),
    "moe_set_phase_trace": (ctypes.c_int, [_P, _P, ctypes.c_size_t]),
    "moe_set_miss_path": (ctypes.c_int, [_P, ctypes.c_int32]),
    "moe_measure_h2d": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.POINTER(ctypes.c_double)]),
    "moe_set_prefetch": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.c_int32]),
    "moe_debug_drop_signals": (ctypes.c_int, [_P, ctypes.c_int32]),
    "moe_decode_step_noalloc": (ctypes.c_int, [ctypes.POINTER(Config), ctypes.POINTER(NoAllocWeights),
                                                _P, _P, _P]),
    "moe_destroy": (None, [_P]),
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libmoe.so (built in-tree by expert_cache_host_router_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libmoe.so not built ({LIB_PATH}); run expert_cache_host_router_b200/build.py")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def header_symbols() -> list[str]:
    """Entry points declared in include/moe_cache.h."""
    with open(HEADER) as f:
        return re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", f.read())


def status_string(status: int) -> str:
    return lib().moe_status_string(status).decode()


def _check(status: int, what: str) -> None:
    if status != MOE_OK:
        raise MoEError(status, what)


def _arr(a, dtype) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(a), dtype=dtype)
    return a


def _ptr(a) -> int | None:
    return None if a is None else a.ctypes.data


# ------------------------------------------------------------------ C-ABI mirrors

def moe_create(cfg: Config) -> int:
    h = _P()
    _check(lib().moe_create(ctypes.byref(cfg), None, ctypes.byref(h)), "moe_create")
    return h.value


def moe_load_layer(ctx: int, layer: int, experts, shared, router, bias=None, gain=None) -> None:
    ex = [_arr(e, np.uint8) for e in experts]
    ptrs = (ctypes.c_void_p * len(ex))(*[e.ctypes.data for e in ex])
    sh = None if shared is None else _arr(shared, np.uint8)
    rt = _arr(router, np.uint16)
    bs = None if bias is None else _arr(bias, np.float32)
    gn = None if gain is None else _arr(gain, np.float32)
    _check(lib().moe_load_layer(ctx, layer, ptrs, _ptr(sh), _ptr(rt), _ptr(bs), _ptr(gn)),
           "moe_load_layer")


def moe_set_residency(ctx: int, fraction: float, hist=None, placement: int = MOE_PLACE_CALIBRATED) -> None:
    h = None if hist is None else _arr(hist, np.uint32)
    _check(lib().moe_set_residency(ctx, fraction, _ptr(h), placement), "moe_set_residency")


def moe_decode_step(ctx: int, x_dev: int, y_dev: int, stream: int) -> None:
    _check(lib().moe_decode_step(ctx, x_dev, y_dev, stream), "moe_decode_step")


def moe_decode_step_host(ctx: int, x: np.ndarray, y: np.ndarray) -> None:
    assert x.dtype == np.float32 and y.dtype == np.float32 and x.flags.c_contiguous and y.flags.c_contiguous
    _check(lib().moe_decode_step_host(ctx, x.ctypes.data, y.ctypes.data), "moe_decode_step_host")


def moe_prefill(ctx: int, x_dev: int, n_tokens: int, y_dev: int, stream: int) -> None:
    _check(lib().moe_prefill(ctx, x_dev, n_tokens, y_dev, stream), "moe_prefill")


def moe_sync(ctx: int) -> None:
    _check(lib().moe_sync(ctx), "moe_sync")


def moe_clear_error(ctx: int) -> None:
    _check(lib().moe_clear_error(ctx), "moe_clear_error")


def moe_stats(ctx: int, n_layers: int, n_experts: int, log_cap: int = 0, reset: bool = False):
    st = Stats()
    hist = np.zeros((n_layers, n_experts), np.uint32)
    log = np.zeros(log_cap, EVENT_DTYPE)
    n = ctypes.c_size_t(0)
    _check(lib().moe_stats(ctx, ctypes.byref(st), hist.ctypes.data, log.ctypes.data if log_cap else None,
                           log_cap, ctypes.byref(n), int(reset)), "moe_stats")
    return st.as_dict(), hist, log[: n.value]


def moe_recalibrate(ctx: int) -> None:
    _check(lib().moe_recalibrate(ctx), "moe_recalibrate")


def moe_set_router_bias(ctx: int, layer: int, bias) -> None:
    b = None if bias is None else _arr(bias, np.float32)
    _check(lib().moe_set_router_bias(ctx, layer, _ptr(b)), "moe_set_router_bias")


def moe_set_trace(ctx: int, h_trace_dev: int | None, w_trace_dev: int | None) -> None:
    _check(lib().moe_set_trace(ctx, h_trace_dev, w_trace_dev), "moe_set_trace")


def moe_set_prefill_trace(ctx: int, h_trace_dev: int | None, sel_trace_dev: int | None) -> None:
    _check(lib().moe_set_prefill_trace(ctx, h_trace_dev, sel_trace_dev), "moe_set_prefill_trace")


def moe_set_phase_trace(ctx: int, stamps_dev: int | None, n_words: int = 0) -> None:
    _check(lib().moe_set_phase_trace(ctx, stamps_dev, n_words), "moe_set_phase_trace")


def moe_set_miss_path(ctx: int, mode: int) -> None:
    _check(lib().moe_set_miss_path(ctx, mode), "moe_set_miss_path")


def moe_set_prefetch(ctx: int, n_preload: int, n_l2: int = 0) -> None:
    _check(lib().moe_set_prefetch(ctx, n_preload, n_l2), "moe_set_prefetch")


def moe_measure_h2d(ctx: int, n_copies: int) -> float:
    g = ctypes.c_double(0.0)
    _check(lib().moe_measure_h2d(ctx, n_copies, ctypes.byref(g)), "moe_measure_h2d")
    return g.value


def phase_trace_words(n_layers: int, n_sm: int) -> int:
    """Length (uint64 words) moe_set_phase_trace needs: [(L+1)][32] + [L][n_sm][4]."""
    return (n_layers + 1) * 32 + n_layers * n_sm * 4


def moe_debug_drop_signals(ctx: int, n: int) -> None:
    _check(lib().moe_debug_drop_signals(ctx, n), "moe_debug_drop_signals")


def moe_decode_step_noalloc(cfg: Config, weights: NoAllocWeights, x_dev: int, y_dev: int,
                            stream: int) -> None:
    _check(lib().moe_decode_step_noalloc(ctypes.byref(cfg), ctypes.byref(weights), x_dev, y_dev, stream),
           "moe_decode_step_noalloc")


def moe_destroy(ctx: int) -> None:
    lib().moe_destroy(ctx)


# ------------------------------------------------------------------ convenience wrapper

_live = weakref.WeakSet()  # contexts still open, closed at interpreter exit


@atexit.register
def _close_live_contexts() -> None:
    for m in list(_live):
        m.close()


class ExpertCacheMoE:
    """One libmoe context plus the torch plumbing (device buffers, current stream).

    shape: synthetic.Shape-like object (n_layers, hidden, n_experts, top_k, inter,
    shared_inter, ring_slots, use_rmsnorm, rms_eps).
    """

    def __init__(self, shape, device: int = 0, log_steps: int = 0, wait_timeout_ms: int = 0):
        self.shape = shape
        self.cfg = Config(shape.n_layers, shape.hidden, shape.n_experts, shape.top_k, shape.inter,
                          shape.shared_inter, shape.ring_slots, shape.use_rmsnorm, shape.rms_eps,
                          device, log_steps, wait_timeout_ms)
        self.device = device
        self.ctx = moe_create(self.cfg)
        _live.add(self)

    def close(self):
        ctx = getattr(self, "ctx", None)
        if ctx:
            self.ctx = None
            moe_destroy(ctx)

    def __del__(self):
        # contexts left open at exit are closed by the atexit hook while the module is
        # intact; a finaliser that runs during interpreter teardown has nothing to do
        try:
            self.close()
        except Exception:
            pass

    def load_layer(self, layer: int, lw) -> None:
        moe_load_layer(self.ctx, layer, lw.experts, lw.shared, lw.router, lw.bias, lw.gain)

    def set_residency(self, fraction: float, hist=None, placement: int = MOE_PLACE_CALIBRATED) -> None:
        moe_set_residency(self.ctx, fraction, hist, placement)

    def decode(self, x, y=None, stream=None):
        """x: torch float32 [H] on this device.  Returns y (torch, same device)."""
        import torch
        assert x.dtype == torch.float32 and x.is_cuda and x.is_contiguous()
        if y is None:
            y = torch.empty_like(x)
        s = torch.cuda.current_stream(x.device) if stream is None else stream
        moe_decode_step(self.ctx, x.data_ptr(), y.data_ptr(), s.cuda_stream)
        return y

    def prefill(self, x, y=None, stream=None):
        """x: torch float32 [T, H] on this device.  Returns y [T, H] (torch, same device)."""
        import torch
        assert x.dtype == torch.float32 and x.is_cuda and x.is_contiguous() and x.dim() == 2
        if y is None:
            y = torch.empty_like(x)
        s = torch.cuda.current_stream(x.device) if stream is None else stream
        moe_prefill(self.ctx, x.data_ptr(), x.shape[0], y.data_ptr(), s.cuda_stream)
        return y

    def set_prefill_trace(self, h_trace=None, sel_trace=None):
        """h_trace: torch float32 [L+1, T, H]; sel_trace: torch int32 [L, T, k]; or None."""
        moe_set_prefill_trace(self.ctx, None if h_trace is None else h_trace.data_ptr(),
                              None if sel_trace is None else sel_trace.data_ptr())

    def decode_host(self, x: np.ndarray) -> np.ndarray:
        x = _arr(x, np.float32)
        y = np.empty_like(x)
        moe_decode_step_host(self.ctx, x, y)
        return y

    def stats(self, log_cap: int = 0, reset: bool = False):
        return moe_stats(self.ctx, self.shape.n_layers, self.shape.n_experts, log_cap, reset)

    def sync(self):
        moe_sync(self.ctx)

    def recalibrate(self) -> None:
        moe_recalibrate(self.ctx)

    def set_router_bias(self, layer: int, bias) -> None:
        moe_set_router_bias(self.ctx, layer, bias)

    def set_phase_trace(self, stamps=None):
        """stamps: contiguous torch int64 tensor on the device with at least
        phase_trace_words(L, n_sm) elements (n_sm = the device's SM count), or None."""
        if stamps is None:
            moe_set_phase_trace(self.ctx, None, 0)
        else:
            assert stamps.is_contiguous() and stamps.element_size() == 8
            moe_set_phase_trace(self.ctx, stamps.data_ptr(), stamps.numel())

    def set_miss_path(self, mode: int) -> None:
        moe_set_miss_path(self.ctx, mode)

    def set_prefetch(self, n_preload: int, n_l2: int = 0) -> None:
        moe_set_prefetch(self.ctx, n_preload, n_l2)

    def measure_h2d(self, n_copies: int = 64) -> float:
        return moe_measure_h2d(self.ctx, n_copies)

    def set_trace(self, h_trace=None, w_trace=None):
        moe_set_trace(self.ctx, None if h_trace is None else h_trace.data_ptr(),
                      None if w_trace is None else w_trace.data_ptr())
