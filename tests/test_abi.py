"""The C-ABI library builds, loads and exports every entry point its header declares.

No GPU needed: only symbol lookup, status strings and host-side argument validation
(every rejected configuration returns before any device call)."""
import ctypes
import subprocess

import pytest

import expert_cache_host_router_b200 as moe
from expert_cache_host_router_b200 import build


@pytest.fixture(scope="module")
def lib():
    build.build()
    return moe.lib()


def test_header_declares_the_boundary():
    names = moe.header_symbols()
    for required in ("moe_create", "moe_set_residency", "moe_decode_step", "moe_prefill", "moe_stats"):
        assert required in names
    assert len(names) == len(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = moe.header_symbols()
    for n in names:
        assert hasattr(lib, n), n
    out = subprocess.check_output(["nm", "-D", "--defined-only", moe.LIB_PATH], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert set(names) <= exported
    # nothing else leaks out of the library as a global function
    assert {e for e in exported if e.startswith("moe_")} == set(names)


def test_status_strings(lib):
    for s in range(0, -8, -1):
        assert moe.status_string(s) and moe.status_string(s) != "unknown status"
    assert moe.status_string(-99) == "unknown status"


def _cfg(**kw):
    base = dict(n_layers=1, hidden=512, n_experts=64, top_k=4, inter=256, shared_inter=0,
                ring_slots=8, use_rmsnorm=0, rms_eps=1e-6, device=0, log_steps=0, wait_timeout_ms=0)
    base.update(kw)
    return moe.Config(**base)


@pytest.mark.parametrize("bad", [
    dict(n_layers=0), dict(hidden=500), dict(hidden=8192), dict(top_k=0), dict(top_k=33),
    dict(n_experts=3), dict(n_experts=2048), dict(inter=48), dict(shared_inter=-32),
    dict(shared_inter=40), dict(ring_slots=-1), dict(ring_slots=33), dict(use_rmsnorm=2),
    dict(rms_eps=float("nan")), dict(log_steps=-1), dict(device=-1),
])
def test_create_rejects_bad_config(lib, bad):
    h = ctypes.c_void_p()
    st = lib.moe_create(ctypes.byref(_cfg(**bad)), None, ctypes.byref(h))
    assert st == moe.MOE_ERR_INVALID
    assert h.value is None


def test_null_arguments_are_rejected(lib):
    assert lib.moe_create(None, None, None) == moe.MOE_ERR_INVALID
    assert lib.moe_set_residency(None, 1.0, None, 0) == moe.MOE_ERR_INVALID
    assert lib.moe_decode_step(None, None, None, None) == moe.MOE_ERR_INVALID
    assert lib.moe_decode_step_host(None, None, None) == moe.MOE_ERR_INVALID
    assert lib.moe_prefill(None, None, 0, None, None) == moe.MOE_ERR_INVALID
    assert lib.moe_sync(None) == moe.MOE_ERR_INVALID
    assert lib.moe_clear_error(None) == moe.MOE_ERR_INVALID
    assert lib.moe_stats(None, None, None, None, 0, None, 0) == moe.MOE_ERR_INVALID
    assert lib.moe_set_trace(None, None, None) == moe.MOE_ERR_INVALID
    assert lib.moe_debug_drop_signals(None, 1) == moe.MOE_ERR_INVALID
    assert lib.moe_load_layer(None, 0, None, None, None, None, None) == moe.MOE_ERR_INVALID
    assert lib.moe_decode_step_noalloc(None, None, None, None, None) == moe.MOE_ERR_INVALID
    assert lib.moe_recalibrate(None) == moe.MOE_ERR_INVALID
    assert lib.moe_set_router_bias(None, 0, None) == moe.MOE_ERR_INVALID
    assert lib.moe_set_prefill_trace(None, None, None) == moe.MOE_ERR_INVALID
    assert lib.moe_set_phase_trace(None, None, 0) == moe.MOE_ERR_INVALID
    assert lib.moe_set_miss_path(None, 0) == moe.MOE_ERR_INVALID
    assert lib.moe_measure_h2d(None, 1, None) == moe.MOE_ERR_INVALID
    assert lib.moe_set_prefetch(None, 0, 0) == moe.MOE_ERR_INVALID
    lib.moe_destroy(None)  # no-op


_STRUCTS = {
    "moe_config": ("Config", ["n_layers", "hidden", "n_experts", "top_k", "inter", "shared_inter", "ring_slots",
                              "use_rmsnorm", "rms_eps", "device", "log_steps", "wait_timeout_ms"]),
    "moe_weights": ("Weights", ["expert_q4_0", "shared_q4_0", "router_bf16", "router_bias", "rms_gain"]),
    "moe_noalloc_weights": ("NoAllocWeights", ["experts_dev", "shared_dev", "router_dev", "bias_dev", "gain_dev"]),
    "moe_event": ("Event", ["step", "layer", "rank", "expert", "kind", "slot", "evicted"]),
    "moe_stats_t": ("Stats", ["steps", "accesses", "pin_hits", "ring_hits", "misses", "evictions", "bytes_copied",
                              "staged_misses", "log_dropped", "device_error", "n_pinned", "residency", "placement",
                              "repins", "repin_copies", "miss_requests", "miss_served", "proxy_error",
                              "miss_path", "pulled_misses", "copies_timed", "copy_ns_timed"]),
}


def test_struct_layouts_match_the_header(tmp_path):
    """The binding's ctypes structures have the header's sizes and field offsets (a C
    program compiled against include/moe_cache.h prints them)."""
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    lines = ["#include <stddef.h>", "#include <stdio.h>", '#include "moe_cache.h"', "int main(void) {"]
    for c, (_, fields) in _STRUCTS.items():
        lines.append(f'  printf("{c} size %zu\\n", sizeof({c}));')
        for f in fields:
            lines.append(f'  printf("{c} {f} %zu\\n", offsetof({c}, {f}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c11", f"-I{os.path.join(root, 'include')}", str(src), "-o", str(exe)])
    out = subprocess.check_output([str(exe)], text=True).split("\n")
    got = {}
    for ln in out:
        if ln:
            c, f, v = ln.split()
            got[(c, f)] = int(v)
    for c, (py, fields) in _STRUCTS.items():
        cls = getattr(moe, py)
        assert ctypes.sizeof(cls) == got[(c, "size")], c
        assert [n for n, _ in cls._fields_] == fields, c
        for f in fields:
            assert getattr(cls, f).offset == got[(c, f)], (c, f)
