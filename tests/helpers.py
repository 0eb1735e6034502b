"""Shared helpers for the GPU parity tests: build the same synthetic model for the CPU
oracle and for libmoe, run tokens, and compare."""
from __future__ import annotations

import numpy as np

import oracle
import synthetic

# Layer outputs must match the oracle within this fraction of the output RMS, element
# by element (the stated float tolerance of the decode path).
LAYER_TOL = 2e-3
# End of a free-running stack: relative L2 error.
STACK_TOL = 1e-2


def make_layers(shape, gain_kind="ones", bias_seed=synthetic.SEED_PERM):
    return [synthetic.layer_weights(l, shape, gain_kind, bias_seed) for l in range(shape.n_layers)]


def build_gpu(shape, layers, **kw):
    import expert_cache_host_router_b200 as moe
    m = moe.ExpertCacheMoE(shape, **kw)
    for l, lw in enumerate(layers):
        m.load_layer(l, lw)
    return m


def max_rel_err(got, ref) -> float:
    rms = float(np.sqrt(np.mean(np.square(ref))))
    return float(np.max(np.abs(np.asarray(got, np.float64) - ref))) / max(rms, 1e-30)


def oracle_events(shape, sels, masks, first_step=0, cache=None):
    """Oracle cache log for the selections sels[step][layer] (rank order) given pinned masks."""
    if cache is None:
        cache = oracle.Cache(shape.n_layers, shape.n_experts, shape.ring_slots)
        for l in range(shape.n_layers):
            cache.set_pinned(l, masks[l])
    evs = []
    for t, sel_t in enumerate(sels):
        for l in range(shape.n_layers):
            evs.append(cache.access(first_step + t, l, sel_t[l]))
    return np.concatenate(evs) if evs else np.zeros(0, oracle.EVENT_DTYPE), cache


def n_pinned(shape, fraction) -> int:
    """P = round(fraction * E), half away from zero, on the fp32 fraction the ABI takes."""
    return int(np.floor(float(np.float32(fraction)) * shape.n_experts + 0.5))


def pinned_masks(shape, hist, fraction, placement):
    P = n_pinned(shape, fraction)
    masks = []
    for l in range(shape.n_layers):
        if placement == 1:
            m = np.zeros(shape.n_experts, np.uint8)
            m[:P] = 1
        else:
            m = oracle.select_pinned(hist[l], P)
        masks.append(m)
    return masks


def events_equal(gpu_log, orc_log) -> bool:
    if len(gpu_log) != len(orc_log):
        return False
    return all(np.array_equal(gpu_log[f], orc_log[f]) for f in oracle.EVENT_DTYPE.names)
