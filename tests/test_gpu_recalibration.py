"""Online recalibration on the GPU against the oracle's policy.

A small stack runs at 40% residency with a 4-slot ring; the router bias (the traffic's
popularity) switches to a reshuffled Zipf permutation halfway; moe_recalibrate runs
every 8 tokens.  The oracle replays the same policy from the routing the GPU logged
(score <- floor(score / 2) + window counts, re-pin top-P, ring emptied) and must produce
the same cache event log bit for bit; routing after the switch must match the oracle run
with the new bias; outputs must equal a full-residency run bit for bit.
"""
import numpy as np
import pytest

import oracle
import synthetic
from helpers import build_gpu, events_equal, make_layers, n_pinned

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

DEV = "cuda:0"
N_TOK, SWITCH, EVERY = 48, 24, 8


def test_recalibration_log_matches_oracle_across_drift():
    s = synthetic.Shape(n_layers=2, hidden=512, n_experts=64, top_k=4, inter=256, shared_inter=0,
                        ring_slots=4, use_rmsnorm=1, zipf_s=1.0)
    layers = make_layers(s)
    drifted = make_layers(s, bias_seed=synthetic.SEED_RESHUFFLE)
    m = build_gpu(s, layers, log_steps=256)
    m.set_residency(1.0)
    for x in synthetic.tokens(0, 16, s.hidden, synthetic.SEED_CALIB):
        m.decode(torch.from_numpy(x).to(DEV))
    m.sync()
    _, hist, _ = m.stats(reset=True, log_cap=16 * s.n_layers * s.top_k)

    xs = synthetic.tokens(0, N_TOK, s.hidden)

    def run(fraction):
        for l in range(s.n_layers):
            m.set_router_bias(l, layers[l].bias)
        m.set_residency(fraction, hist)
        m.stats(reset=True, log_cap=4096)
        ht = torch.zeros((s.n_layers + 1, s.hidden), dtype=torch.float32, device=DEV)
        ys, traced = [], None
        for t, x in enumerate(xs):
            if t == SWITCH:
                for l in range(s.n_layers):
                    m.set_router_bias(l, drifted[l].bias)
            if fraction < 1.0 and t and t % EVERY == 0:
                m.recalibrate()
            if t == SWITCH + 3:
                m.set_trace(ht, None)
            y = m.decode(torch.from_numpy(x).to(DEV))
            try:  # wait for the step before any blocking copy (see moe_decode_step's notes)
                m.sync()
            except Exception as ex:  # report which wait ran out, and the miss queue's state
                st, _, lg = m.stats(log_cap=4096)
                raise AssertionError(f"fraction {fraction} token {t}: {ex}; stats {st}; "
                                     f"last events {lg[-8:].tolist()}") from ex
            ys.append(y.cpu().numpy())
            if t == SWITCH + 3:
                traced = ht.cpu().numpy().copy()
                m.set_trace(None, None)
        m.sync()
        st, _, log = m.stats(log_cap=N_TOK * s.n_layers * s.top_k)
        return np.stack(ys), st, log, traced

    ys_full, _, _, _ = run(1.0)
    ys, st, log, traced = run(0.4)
    assert np.array_equal(ys.view(np.uint32), ys_full.view(np.uint32))
    assert st["repins"] == (N_TOK - 1) // EVERY

    # routing after the switch follows the drifted bias (teacher-forced oracle)
    orc_new = oracle.Model(s, drifted)
    sel = log["expert"].reshape(N_TOK, s.n_layers, s.top_k)
    for l in range(s.n_layers):
        assert np.array_equal(orc_new.layer(l, traced[l])["sel"], sel[SWITCH + 3, l])

    # the oracle replays the recalibration policy on the logged routing
    P = n_pinned(s, 0.4)
    cache = oracle.Cache(s.n_layers, s.n_experts, s.ring_slots)
    score = hist.astype(np.uint32).copy()
    for l in range(s.n_layers):
        cache.set_pinned(l, oracle.select_pinned(score[l], P))
    window = np.zeros_like(score)
    first = int(log["step"][0])
    ref = []
    for t in range(N_TOK):
        if t and t % EVERY == 0:
            score = np.stack([oracle.recal_score(score[l], window[l]) for l in range(s.n_layers)])
            window[:] = 0
            for l in range(s.n_layers):
                cache.set_pinned(l, oracle.select_pinned(score[l], P))
        for l in range(s.n_layers):
            ref.append(cache.access(first + t, l, sel[t, l]))
            window[l, sel[t, l]] += 1
    ref = np.concatenate(ref)
    assert events_equal(log, ref)
    assert st["misses"] == int(np.sum(log["kind"] == oracle.MISS))
    m.close()
