"""The 40-layer full-shape stack in the configurations bench.py times (decode at 60%
calibrated residency with 8-slot rings and at 100%; batched prefill at 100%), checked
against the oracle on sampled outputs: every layer of the sampled tokens teacher-forced
(routing bit-exact, layer outputs within 2e-3 x RMS), decode outputs bit-identical across
residency, the cache log equal to the oracle's replay of the logged selections, and the
free-running end of the stack within 1e-2 relative L2 of the oracle's own decode."""
import numpy as np
import pytest

import oracle
import synthetic
from helpers import LAYER_TOL, STACK_TOL, build_gpu, events_equal, make_layers, oracle_events, pinned_masks

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _check_layer(orc, l, h_in, h_out, sel):
    ref = orc.layer(l, h_in)
    assert np.array_equal(ref["sel"], sel), (l, ref["sel"], sel)
    err = np.max(np.abs(h_out.astype(np.float64) - ref["h_out"]))
    rms = np.sqrt(np.mean(ref["y"] ** 2))
    assert err <= LAYER_TOL * rms, (l, err / rms)


def test_full_stack_40_layers_decode_and_prefill():
    s = synthetic.FULL_STACK
    assert s.n_layers == 40
    layers = make_layers(s)
    orc = oracle.Model(s, layers)
    m = build_gpu(s, layers, log_steps=512)
    y = torch.empty(s.hidden, dtype=torch.float32, device=DEV)

    # calibration at full residency
    m.set_residency(1.0)
    for x in synthetic.tokens(0, 32, s.hidden, synthetic.SEED_CALIB):
        m.decode(torch.from_numpy(x).to(DEV), y)
    m.sync()
    _, hist, _ = m.stats(log_cap=32 * s.n_layers * s.top_k, reset=True)  # reads the calibration log too

    xs = synthetic.tokens(0, 4, s.hidden)
    outs = {}
    for frac in (0.6, 1.0):
        m.set_residency(frac, hist)
        ht = torch.zeros((s.n_layers + 1, s.hidden), dtype=torch.float32, device=DEV)
        ys, traced = [], None
        for t, x in enumerate(xs):
            if t == 1:
                m.set_trace(ht, None)
            m.decode(torch.from_numpy(x).to(DEV), y)
            m.sync()
            ys.append(y.cpu().numpy().copy())
            if t == 1:
                traced = ht.cpu().numpy().copy()
                m.set_trace(None, None)
        st, _, log = m.stats(log_cap=len(xs) * s.n_layers * s.top_k, reset=True)
        assert len(log) == len(xs) * s.n_layers * s.top_k
        sels = log["expert"].reshape(len(xs), s.n_layers, s.top_k)
        masks = pinned_masks(s, hist, frac, 0)
        ref_log, _ = oracle_events(s, sels, masks, first_step=int(log["step"][0]))
        assert events_equal(log, ref_log), frac
        assert np.array_equal(traced[0], xs[1])
        for l in range(s.n_layers):
            _check_layer(orc, l, traced[l], traced[l + 1], sels[1, l])
        assert np.array_equal(ys[1], traced[-1])
        outs[frac] = np.stack(ys)
        assert st["misses"] == int(np.sum(log["kind"] == oracle.MISS))
    assert np.array_equal(outs[0.6].view(np.uint32), outs[1.0].view(np.uint32))

    # the free-running end of the stack: the oracle decodes the same tokens through all
    # 40 layers on its own (fp64 between layers); where its routing agrees with the
    # GPU's at every layer, the final states agree within 1e-2 relative L2
    compared = 0
    for t, x in enumerate(xs):
        h_ref, sel_ref, _ = orc.decode(x)
        if np.array_equal(sel_ref, sels[t]):
            rel = np.linalg.norm(outs[1.0][t] - h_ref) / np.linalg.norm(h_ref)
            assert rel <= STACK_TOL, (t, rel)
            compared += 1
        else:
            first = int(np.argmax(np.any(sel_ref != sels[t], axis=1)))
            print(f"token {t}: free-running routing first differs at layer {first}")
    assert compared >= len(xs) // 2, compared

    # batched prefill through the same 40 layers
    T = 256
    xp = synthetic.tokens(7000, T, s.hidden)
    hp = torch.zeros((s.n_layers + 1, T, s.hidden), dtype=torch.float32, device=DEV)
    sp = torch.zeros((s.n_layers, T, s.top_k), dtype=torch.int32, device=DEV)
    m.set_prefill_trace(hp, sp)
    yp = m.prefill(torch.from_numpy(xp).to(DEV))
    m.sync()
    m.set_prefill_trace(None, None)
    h, sel = hp.cpu().numpy(), sp.cpu().numpy()
    assert np.array_equal(yp.cpu().numpy(), h[-1])
    for t in (0, 131, 255):
        for l in range(s.n_layers):
            _check_layer(orc, l, h[l, t], h[l + 1, t], sel[l, t])
    m.close()
