"""CPU oracle of the sparse MoE decode step with a bounded expert cache.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the bench's CPU-baseline
leg may import this package; the product library never does.  The arithmetic lives in
``moe_oracle.c`` (plain single-threaded C); this module only compiles it with gcc and
marshals numpy arrays through ctypes.  See the header of ``moe_oracle.c`` for what each
function computes and which passage or reading it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")
_lock = threading.Lock()
_lib = None

PIN_HIT, RING_HIT, MISS = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile moe_oracle.c with gcc (single-threaded, no FP contraction).

    ``ORACLE_LIB`` in the environment names an already built copy to load instead; the
    mutation check of the pins uses it to run them against deliberately broken copies."""
    override = os.environ.get("ORACLE_LIB")
    if override:
        return override
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        compile_c(_SRC, tmp)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def compile_c(src: str, out: str) -> None:
    """gcc flags of the oracle: -O2, no FP contraction, no fast-math, C11."""
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
                           "-shared", "-fPIC", "-o", out, src, "-lm"])


class Dims(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("inter", ctypes.c_int32),
                ("shared_inter", ctypes.c_int32), ("use_rmsnorm", ctypes.c_int32),
                ("rms_eps", ctypes.c_float)]


class LayerW(ctypes.Structure):
    _fields_ = [("experts", ctypes.POINTER(ctypes.c_void_p)), ("shared", ctypes.c_void_p),
                ("router", ctypes.c_void_p), ("bias", ctypes.c_void_p),
                ("gain", ctypes.c_void_p)]


class Event(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("step", "layer", "rank", "expert", "kind", "slot", "evicted")]


EVENT_DTYPE = np.dtype([(n, np.int32) for n in
                        ("step", "layer", "rank", "expert", "kind", "slot", "evicted")])

_P = ctypes.c_void_p


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            sig = {
                "orc_f16_to_f32": (ctypes.c_float, [ctypes.c_uint16]),
                "orc_bf16_to_f32": (ctypes.c_float, [ctypes.c_uint16]),
                "orc_dequant_q4_0": (None, [_P, ctypes.c_int64, _P]),
                "orc_canonical_sum": (ctypes.c_float, [_P, ctypes.c_int]),
                "orc_rms_inv": (ctypes.c_float, [_P, ctypes.c_int, ctypes.c_float]),
                "orc_router_logits": (None, [_P, _P, _P, ctypes.c_float, _P, ctypes.c_int,
                                             ctypes.c_int, _P]),
                "orc_topk": (None, [_P, ctypes.c_int, ctypes.c_int, _P]),
                "orc_route_weights": (None, [_P, _P, ctypes.c_int, _P]),
                "orc_silu": (ctypes.c_double, [ctypes.c_double]),
                "orc_expert_ffn": (None, [_P, ctypes.c_int, ctypes.c_int, _P, _P]),
                "orc_moe_layer": (None, [ctypes.POINTER(Dims), ctypes.POINTER(LayerW), _P, _P,
                                         _P, _P, _P, _P, _P]),
                "orc_decode_token": (None, [ctypes.POINTER(Dims), ctypes.c_int,
                                            ctypes.POINTER(LayerW), _P, _P, _P, _P]),
                "orc_select_pinned": (None, [_P, ctypes.c_int, ctypes.c_int, _P]),
                "orc_recal_score": (None, [_P, _P, ctypes.c_int]),
                "orc_cache_create": (_P, [ctypes.c_int, ctypes.c_int, ctypes.c_int]),
                "orc_cache_destroy": (None, [_P]),
                "orc_cache_set_pinned": (None, [_P, ctypes.c_int, _P]),
                "orc_cache_access": (None, [_P, ctypes.c_int, ctypes.c_int, _P, ctypes.c_int, _P]),
                "orc_cache_ring": (None, [_P, ctypes.c_int, _P]),
            }
            for name, (res, args) in sig.items():
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
    return _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a), dtype=dtype)


# ------------------------------------------------------------------ thin wrappers

def f16_to_f32(bits: int) -> float:
    return lib().orc_f16_to_f32(bits)


def bf16_to_f32(bits: int) -> float:
    return lib().orc_bf16_to_f32(bits)


def dequant_q4_0(blocks) -> np.ndarray:
    blocks = _c(blocks, np.uint8)
    n = blocks.size // 18
    out = np.empty(32 * n, np.float64)
    lib().orc_dequant_q4_0(_ptr(blocks), n, _ptr(out))
    return out


def canonical_sum(parts) -> np.float32:
    parts = _c(parts, np.float32)
    return np.float32(lib().orc_canonical_sum(_ptr(parts), parts.size))


def rms_inv(h, eps: float) -> np.float32:
    h = _c(h, np.float32)
    return np.float32(lib().orc_rms_inv(_ptr(h), h.size, ctypes.c_float(eps)))


def router_logits(w_bf16, h, gain, inv, bias) -> np.ndarray:
    w = _c(w_bf16, np.uint16)
    E, H = w.shape
    h = _c(h, np.float32)
    gain = None if gain is None else _c(gain, np.float32)
    bias = None if bias is None else _c(bias, np.float32)
    z = np.empty(E, np.float32)
    lib().orc_router_logits(_ptr(w), _ptr(h), _ptr(gain), ctypes.c_float(inv), _ptr(bias), E, H,
                            _ptr(z))
    return z


def topk(z, k: int) -> np.ndarray:
    z = _c(z, np.float32)
    sel = np.empty(k, np.int32)
    lib().orc_topk(_ptr(z), z.size, k, _ptr(sel))
    return sel


def route_weights(z, sel) -> np.ndarray:
    z = _c(z, np.float32)
    sel = _c(sel, np.int32)
    w = np.empty(sel.size, np.float64)
    lib().orc_route_weights(_ptr(z), _ptr(sel), sel.size, _ptr(w))
    return w


def silu(t: float) -> float:
    return lib().orc_silu(t)


def expert_ffn(q4, hidden: int, inter: int, x) -> np.ndarray:
    q4 = _c(q4, np.uint8)
    x = _c(x, np.float64)
    out = np.empty(hidden, np.float64)
    lib().orc_expert_ffn(_ptr(q4), hidden, inter, _ptr(x), _ptr(out))
    return out


def select_pinned(hist, P: int) -> np.ndarray:
    hist = _c(hist, np.uint32)
    mask = np.empty(hist.size, np.uint8)
    lib().orc_select_pinned(_ptr(hist), hist.size, P, _ptr(mask))
    return mask


def recal_score(score, window) -> np.ndarray:
    """New recalibration scores (uint32) from the old ones and a window of counts."""
    out = _c(score, np.uint32).copy()
    window = _c(window, np.uint32)
    assert out.shape == window.shape
    lib().orc_recal_score(_ptr(out), _ptr(window), out.size)
    return out


class _LayerRef:
    """Keeps the numpy arrays of one layer alive while C holds pointers to them."""

    def __init__(self, lw):
        self.experts = [_c(e, np.uint8) for e in lw.experts]
        self.shared = None if lw.shared is None else _c(lw.shared, np.uint8)
        self.router = _c(lw.router, np.uint16)
        self.bias = None if lw.bias is None else _c(lw.bias, np.float32)
        self.gain = None if lw.gain is None else _c(lw.gain, np.float32)
        self.ptrs = (ctypes.c_void_p * len(self.experts))(*[e.ctypes.data for e in self.experts])
        self.c = LayerW(ctypes.cast(self.ptrs, ctypes.POINTER(ctypes.c_void_p)),
                        _ptr(self.shared), _ptr(self.router), _ptr(self.bias), _ptr(self.gain))


def dims_of(shape) -> Dims:
    return Dims(shape.hidden, shape.n_experts, shape.top_k, shape.inter, shape.shared_inter,
                shape.use_rmsnorm, shape.rms_eps)


class Model:
    """The oracle's view of an MoE stack: shape plus per-layer weights (synthetic.LayerWeights)."""

    def __init__(self, shape, layers):
        self.shape = shape
        self.dims = dims_of(shape)
        self.refs = [_LayerRef(lw) for lw in layers]
        self.carr = (LayerW * len(self.refs))(*[r.c for r in self.refs])

    def layer(self, l: int, h32, h64=None):
        """One layer on fp32 input h32 (h64 defaults to h32).  Returns dict of outputs."""
        s = self.shape
        h32 = _c(h32, np.float32)
        h64 = _c(h32 if h64 is None else h64, np.float64)
        z = np.empty(s.n_experts, np.float32)
        sel = np.empty(s.top_k, np.int32)
        w = np.empty(s.top_k, np.float64)
        y = np.empty(s.hidden, np.float64)
        h_out = np.empty(s.hidden, np.float64)
        lib().orc_moe_layer(ctypes.byref(self.dims), ctypes.byref(self.refs[l].c), _ptr(h32),
                            _ptr(h64), _ptr(z), _ptr(sel), _ptr(w), _ptr(y), _ptr(h_out))
        return {"z": z, "sel": sel, "w": w, "y": y, "h_out": h_out}

    def decode(self, x, n_layers: int | None = None, trace: bool = False):
        """Free-running decode of one token.  Returns (h_out, sel[L,k], trace or None)."""
        s = self.shape
        L = len(self.refs) if n_layers is None else n_layers
        x = _c(x, np.float32)
        h = np.empty(s.hidden, np.float64)
        sel = np.empty((L, s.top_k), np.int32)
        tr = np.empty((L + 1, s.hidden), np.float64) if trace else None
        lib().orc_decode_token(ctypes.byref(self.dims), L, self.carr, _ptr(x), _ptr(h), _ptr(sel),
                               _ptr(tr))
        return h, sel, tr


class Cache:
    """The oracle's expert-cache simulator (pinned set + LRU ring per layer)."""

    def __init__(self, n_layers: int, n_experts: int, ring_slots: int):
        self.k_max = 0
        self.h = lib().orc_cache_create(n_layers, n_experts, ring_slots)
        self.n_experts, self.ring_slots = n_experts, ring_slots

    def __del__(self):
        if getattr(self, "h", None):
            lib().orc_cache_destroy(self.h)
            self.h = None

    def set_pinned(self, layer: int, mask):
        mask = _c(mask, np.uint8)
        assert mask.size == self.n_experts
        lib().orc_cache_set_pinned(self.h, layer, _ptr(mask))

    def access(self, step: int, layer: int, sel) -> np.ndarray:
        sel = _c(sel, np.int32)
        ev = np.zeros(sel.size, EVENT_DTYPE)
        lib().orc_cache_access(self.h, step, layer, _ptr(sel), sel.size, ev.ctypes.data)
        return ev

    def ring(self, layer: int) -> np.ndarray:
        out = np.empty(self.ring_slots, np.int32)
        lib().orc_cache_ring(self.h, layer, _ptr(out))
        return out
