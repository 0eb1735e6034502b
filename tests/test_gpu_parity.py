"""Parity of the CUDA decode path (through the C ABI) with the CPU oracle.

Bars: routing choices, histograms and cache event logs bit-exact; every layer's output
within 2e-3 x its RMS element by element (teacher-forced: the oracle runs layer l on
the GPU's own h_l); the end of a free-running stack within 1e-2 relative; GPU outputs
bit-identical across residency levels (the write-up's full-residency-equals-all-GPU
claim)."""
import numpy as np
import pytest

import oracle
import synthetic
from helpers import (LAYER_TOL, STACK_TOL, build_gpu, events_equal, make_layers, max_rel_err,
                     oracle_events, pinned_masks)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _run_tokens(m, xs, trace=False):
    """Decode tokens one by one; returns y [T,H] and, with trace, h [T,L+1,H], w [T,L,k]."""
    s = m.shape
    ys, hs, ws = [], [], []
    if trace:
        ht = torch.zeros((s.n_layers + 1, s.hidden), dtype=torch.float32, device=DEV)
        wt = torch.zeros((s.n_layers, s.top_k), dtype=torch.float32, device=DEV)
        m.set_trace(ht, wt)
    for x in xs:
        y = m.decode(torch.from_numpy(np.ascontiguousarray(x)).to(DEV))
        torch.cuda.synchronize()
        ys.append(y.cpu().numpy())
        if trace:
            hs.append(ht.cpu().numpy().copy())
            ws.append(wt.cpu().numpy().copy())
    if trace:
        m.set_trace(None, None)
    m.sync()
    return np.stack(ys), (np.stack(hs) if trace else None), (np.stack(ws) if trace else None)


def _sels_from_log(log, n_steps, shape):
    sel = log["expert"].reshape(n_steps, shape.n_layers, shape.top_k)
    assert np.array_equal(log["rank"].reshape(sel.shape), np.broadcast_to(np.arange(shape.top_k), sel.shape))
    return sel


def _check_teacher_forced(orc, shape, xs, ys, hs, ws, sels):
    for t in range(len(xs)):
        assert np.array_equal(hs[t, 0], xs[t])
        for l in range(shape.n_layers):
            ref = orc.layer(l, hs[t, l])
            assert np.array_equal(ref["sel"], sels[t, l]), (t, l, ref["sel"], sels[t, l])
            assert np.allclose(ws[t, l], ref["w"], rtol=2e-6, atol=1e-7), (t, l)
            err = np.max(np.abs(hs[t, l + 1].astype(np.float64) - ref["h_out"]))
            rms = np.sqrt(np.mean(ref["y"] ** 2))
            assert err <= LAYER_TOL * rms, (t, l, err / rms)
        assert np.array_equal(ys[t], hs[t, -1])


# ------------------------------------------------------------------ single layers

def test_small_layer_all_resident():
    """1 layer, hidden 512, 64 experts, top-4, SwiGLU 256, no shared, 8 tokens."""
    s = synthetic.SMALL
    layers = make_layers(s)
    orc = oracle.Model(s, layers)
    m = build_gpu(s, layers)
    m.set_residency(1.0)
    xs = synthetic.tokens(0, 8, s.hidden)
    ys, hs, ws = _run_tokens(m, xs, trace=True)
    st, hist, log = m.stats(log_cap=8 * s.top_k)
    sels = _sels_from_log(log, 8, s)
    for t, x in enumerate(xs):
        ref = orc.layer(0, x)
        assert np.array_equal(sels[t, 0], ref["sel"])
        assert max_rel_err(ys[t], ref["y"]) <= LAYER_TOL
    _check_teacher_forced(orc, s, xs, ys, hs, ws, sels)
    assert np.array_equal(hist[0], np.bincount(sels.reshape(-1), minlength=s.n_experts))
    assert st["pin_hits"] == 8 * s.top_k and st["misses"] == 0 and st["steps"] == 8
    m.close()


def test_full_shape_layer_with_shared_expert():
    """1 layer, hidden 2048, 256 experts, top-8, 512 + shared 512, Zipf-biased router."""
    s = synthetic.FULL_LAYER
    layers = make_layers(s)
    orc = oracle.Model(s, layers)
    m = build_gpu(s, layers)
    m.set_residency(1.0)
    xs = synthetic.tokens(100, 4, s.hidden)
    ys, hs, ws = _run_tokens(m, xs, trace=True)
    _, hist, log = m.stats(log_cap=4 * s.top_k)
    sels = _sels_from_log(log, 4, s)
    _check_teacher_forced(orc, s, xs, ys, hs, ws, sels)
    assert int(hist.sum()) == 4 * s.top_k
    m.close()


@pytest.mark.parametrize("shape", [
    synthetic.Shape(3, 96, 40, 3, 64, 32, ring_slots=2, use_rmsnorm=1, zipf_s=1.0),
    synthetic.Shape(2, 64, 9, 1, 32, 0, ring_slots=1, use_rmsnorm=1, zipf_s=0.5),
    synthetic.Shape(1, 4096, 33, 32, 32, 96, ring_slots=4, use_rmsnorm=0, zipf_s=1.0),
    synthetic.Shape(2, 544, 70, 5, 96, 0, ring_slots=3, use_rmsnorm=1, zipf_s=1.0),
    # the compile-time hidden-size instances (1024 and 3072) with the k = 8 top-k over a
    # ragged expert count
    synthetic.Shape(2, 3072, 24, 8, 64, 32, ring_slots=2, use_rmsnorm=1, zipf_s=1.0),
    synthetic.Shape(2, 1024, 200, 8, 96, 0, ring_slots=4, use_rmsnorm=1, zipf_s=1.0),
])
def test_ragged_shapes(shape):
    """Shapes that leave partial warps, odd block counts and single-block rows, and the
    kernel instances compiled for a fixed hidden size."""
    layers = make_layers(shape, gain_kind="random")
    orc = oracle.Model(shape, layers)
    m = build_gpu(shape, layers)
    m.set_residency(1.0)
    xs = synthetic.tokens(7, 3, shape.hidden)
    ys, hs, ws = _run_tokens(m, xs, trace=True)
    _, _, log = m.stats(log_cap=3 * shape.n_layers * shape.top_k)
    _check_teacher_forced(orc, shape, xs, ys, hs, ws, _sels_from_log(log, 3, shape))
    m.close()


# ------------------------------------------------------------------ stacks and the cache

STACK = synthetic.Shape(n_layers=4, hidden=2048, n_experts=256, top_k=8, inter=512,
                        shared_inter=512, ring_slots=8, use_rmsnorm=1)


def test_stack_teacher_forced_and_free_running():
    s = STACK
    layers = make_layers(s, gain_kind="random")
    orc = oracle.Model(s, layers)
    m = build_gpu(s, layers)
    m.set_residency(1.0)
    xs = synthetic.tokens(0, 3, s.hidden)
    ys, hs, ws = _run_tokens(m, xs, trace=True)
    _, _, log = m.stats(log_cap=3 * s.n_layers * s.top_k)
    sels = _sels_from_log(log, 3, s)
    _check_teacher_forced(orc, s, xs, ys, hs, ws, sels)
    compared = 0
    for t, x in enumerate(xs):
        h, sel, _ = orc.decode(x)
        # a free-running stack may legitimately route differently after a near-tie (the
        # teacher-forced check above holds every layer exactly); compare where it agreed
        if np.array_equal(sel, sels[t]):
            assert np.linalg.norm(ys[t] - h) <= STACK_TOL * np.linalg.norm(h), t
            compared += 1
    assert compared >= 1, "no token's free-running routing agreed with the oracle's"
    m.close()


@pytest.mark.parametrize("miss_path", ["copy_engine", "sm_pull"])
def test_residency_levels_bit_identical_and_cache_log_exact(miss_path):
    import expert_cache_host_router_b200 as moe
    s = STACK
    layers = make_layers(s)
    m = build_gpu(s, layers, log_steps=64)
    m.set_miss_path(moe.MOE_MISS_SM_PULL if miss_path == "sm_pull" else moe.MOE_MISS_COPY_ENGINE)
    m.set_residency(1.0)
    calib = synthetic.tokens(0, 16, s.hidden, synthetic.SEED_CALIB)
    _run_tokens(m, calib)
    _, hist, calib_log = m.stats(log_cap=16 * s.n_layers * s.top_k, reset=True)
    csel = _sels_from_log(calib_log, 16, s)
    ref_hist = np.stack([np.bincount(csel[:, l].reshape(-1), minlength=s.n_experts) for l in range(s.n_layers)])
    assert np.array_equal(hist, ref_hist)

    xs = synthetic.tokens(0, 12, s.hidden)
    outs = {}
    for frac, place in [(1.0, 0), (0.6, 0), (0.4, 0), (0.6, 1)]:
        m.set_residency(frac, hist, place)
        ys, _, _ = _run_tokens(m, xs)
        st, _, log = m.stats(log_cap=12 * s.n_layers * s.top_k, reset=True)
        sels = _sels_from_log(log, 12, s)
        masks = pinned_masks(s, hist, frac, place)
        ref_log, _ = oracle_events(s, sels, masks, first_step=int(log["step"][0]))
        assert events_equal(log, ref_log), (frac, place)
        assert st["misses"] == int(np.sum(log["kind"] == 2))
        assert st["pulled_misses"] == (st["misses"] if miss_path == "sm_pull" else 0)
        outs[(frac, place)] = ys
    base = outs[(1.0, 0)]
    for key, ys in outs.items():
        assert np.array_equal(ys.view(np.uint32), base.view(np.uint32)), key
    m.close()


@pytest.mark.parametrize("miss_path", ["copy_engine", "sm_pull"])
def test_ring_smaller_than_top_k_stages_misses(miss_path):
    """R=2 < k=4: a layer can miss more often than it has ring slots; the log still
    follows the oracle's LRU exactly and the output stays bit-identical."""
    import expert_cache_host_router_b200 as moe
    s = synthetic.Shape(n_layers=2, hidden=512, n_experts=64, top_k=4, inter=256, shared_inter=0,
                        ring_slots=2, use_rmsnorm=1, zipf_s=0.0)
    layers = make_layers(s)
    m = build_gpu(s, layers)
    m.set_miss_path(moe.MOE_MISS_SM_PULL if miss_path == "sm_pull" else moe.MOE_MISS_COPY_ENGINE)
    m.set_residency(1.0)
    xs = synthetic.tokens(3, 10, s.hidden)
    base, _, _ = _run_tokens(m, xs)
    m.stats(reset=True, log_cap=10 * s.n_layers * s.top_k)
    m.set_residency(0.0)
    ys, _, _ = _run_tokens(m, xs)
    st, _, log = m.stats(log_cap=10 * s.n_layers * s.top_k)
    sels = _sels_from_log(log, 10, s)
    ref_log, _ = oracle_events(s, sels, pinned_masks(s, None, 0.0, 1), first_step=int(log["step"][0]))
    assert events_equal(log, ref_log)
    assert st["staged_misses"] > 0
    assert np.array_equal(ys.view(np.uint32), base.view(np.uint32))
    m.close()


def test_host_buffer_entry_point_matches_device_entry_point():
    s = synthetic.SMALL
    layers = make_layers(s)
    m = build_gpu(s, layers)
    m.set_residency(1.0)
    xs = synthetic.tokens(0, 4, s.hidden)
    ys, _, _ = _run_tokens(m, xs)
    for t, x in enumerate(xs):
        assert np.array_equal(m.decode_host(x).view(np.uint32), ys[t].view(np.uint32))
    m.close()


def test_lost_miss_signal_times_out_and_recovers():
    """Failure detection without a GPU fault: the proxy stops signalling completed miss
    copies (the completion word is monotonic, so every signal of the step is dropped), the
    kernel's bounded wait runs out, the step reports MOE_ERR_TIMEOUT, and after
    moe_clear_error decoding resumes with correct results."""
    import expert_cache_host_router_b200 as moe
    s = synthetic.Shape(n_layers=2, hidden=512, n_experts=64, top_k=4, inter=256, shared_inter=0,
                        ring_slots=4, use_rmsnorm=1)
    layers = make_layers(s)
    m = build_gpu(s, layers, wait_timeout_ms=200)
    m.set_residency(1.0)
    xs = synthetic.tokens(0, 2, s.hidden)
    base, _, _ = _run_tokens(m, xs)
    m.set_residency(0.0)
    moe.moe_debug_drop_signals(m.ctx, 1000)
    m.decode(torch.from_numpy(xs[0]).to(DEV))
    with pytest.raises(moe.MoEError) as ei:
        m.sync()
    assert ei.value.status == moe.MOE_ERR_TIMEOUT
    moe.moe_clear_error(m.ctx)
    ys, _, _ = _run_tokens(m, xs)
    assert np.array_equal(ys.view(np.uint32), base.view(np.uint32))
    m.close()


def test_invalid_calls_on_a_live_context():
    import expert_cache_host_router_b200 as moe
    s = synthetic.SMALL
    m = moe.ExpertCacheMoE(s)
    x = torch.zeros(s.hidden, device=DEV)
    with pytest.raises(moe.MoEError) as ei:
        m.decode(x)  # weights not loaded, no residency
    assert ei.value.status == moe.MOE_ERR_STATE
    with pytest.raises(moe.MoEError):
        m.set_residency(1.0)  # layers not loaded
    layers = make_layers(s)
    m.load_layer(0, layers[0])
    with pytest.raises(moe.MoEError):
        m.set_residency(1.5)
    with pytest.raises(moe.MoEError):
        moe.moe_set_residency(m.ctx, 0.5, None, 7)
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_prefill(m.ctx, x.data_ptr(), 1, x.data_ptr(), 0)  # no residency set yet
    assert ei.value.status == moe.MOE_ERR_STATE
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_prefill(m.ctx, x.data_ptr(), 0, x.data_ptr(), 0)
    assert ei.value.status == moe.MOE_ERR_INVALID
    m.close()


@pytest.mark.parametrize("frac", [1.0, 0.6])
def test_speculative_loads_change_nothing(frac):
    """Preloading likely experts into shared memory (and prefetching more into L2) only
    moves where and when bytes are read: outputs bit-identical, the same event log."""
    s = STACK
    layers = make_layers(s, gain_kind="random")
    m = build_gpu(s, layers, log_steps=64)
    m.set_residency(1.0)
    calib = synthetic.tokens(0, 16, s.hidden, synthetic.SEED_CALIB)
    _run_tokens(m, calib)
    _, hist, _ = m.stats(log_cap=16 * s.n_layers * s.top_k, reset=True)
    xs = synthetic.tokens(40, 8, s.hidden)
    outs, logs = {}, {}
    for pre, l2 in [(0, 0), (8, 0), (4, 6), (8, 8)]:
        m.set_prefetch(pre, l2)
        m.set_residency(frac, hist)
        ys, _, _ = _run_tokens(m, xs)
        _, _, log = m.stats(log_cap=8 * s.n_layers * s.top_k, reset=True)
        outs[(pre, l2)] = ys
        logs[(pre, l2)] = log
    base = outs[(0, 0)]
    for key, ys in outs.items():
        assert np.array_equal(ys.view(np.uint32), base.view(np.uint32)), key
        for f in ("layer", "rank", "expert", "kind", "slot", "evicted"):
            assert np.array_equal(logs[key][f], logs[(0, 0)][f]), (key, f)
    m.close()
