"""The calibration stream's length and the cold share at 60% residency (CPU).

The placement pins the top-P experts of a layer by routing count (oracle.select_pinned:
ties -> lower index).  How well a histogram of N calibration tokens finds the hot set
is a property of the synthetic workload, checked here with a plain model of the
benchmark layer's router: unit-RMS Gaussian inputs, the layer's bf16 router rows and its
Zipf(1) bias, top-8 by logit.  Pinning 154 of 256 experts from 2048 calibration tokens
must leave far fewer selections outside the pinned set than pinning from 128 tokens
(the model gives about 0.2% against 1%), and no histogram can beat pinning from the
test stream's own counts."""
import numpy as np

import oracle
import synthetic

E, H, K = 256, 2048, 8
P = round(0.6 * E)


def _router(layer: int):
    w = (synthetic.router_bf16(layer, E, H).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    b = synthetic.zipf_bias(layer, E, 1.0).astype(np.float64)
    return w, b


def _selections(w, b, rng, n: int) -> np.ndarray:
    x = rng.standard_normal((n, H))
    x /= np.sqrt(np.mean(x * x, axis=1, keepdims=True))
    z = x @ w.T + b
    return np.argsort(-z, axis=1, kind="stable")[:, :K]


def _cold_share(hist: np.ndarray, test_sel: np.ndarray) -> float:
    mask = oracle.select_pinned(hist.astype(np.uint32), P).astype(bool)
    return float(np.mean(~mask[test_sel]))


def test_longer_calibration_pins_the_hot_set_better():
    short, long_, best = [], [], []
    for layer in (0, 7):
        w, b = _router(layer)
        rng = np.random.default_rng(1000 + layer)
        test_sel = _selections(w, b, rng, 2000)
        for n, out in ((128, short), (2048, long_)):
            hist = np.bincount(_selections(w, b, rng, n).ravel(), minlength=E)
            out.append(_cold_share(hist, test_sel))
        best.append(_cold_share(np.bincount(test_sel.ravel(), minlength=E), test_sel))
    short_m, long_m, best_m = np.mean(short), np.mean(long_), np.mean(best)
    assert 0.0 < long_m < 0.6 * short_m, (short_m, long_m)
    assert best_m <= long_m
    assert short_m < 0.05  # the Zipf bias makes even a short calibration mostly right
