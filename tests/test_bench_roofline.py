"""bench.py's prefill roofline against hand-computed cases (host arithmetic only)."""
import dataclasses
import importlib.util
import os

import numpy as np

_ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(_ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@dataclasses.dataclass
class _Shape:
    n_layers: int
    hidden: int
    inter: int
    shared_inter: int


def test_prefill_roofline_hand_computed():
    b = _bench()
    s = _Shape(n_layers=1, hidden=256, inter=256, shared_inter=0)
    tflops, hbm = 1.0, 1.0  # 1e12 FLOP/s, 1e9 B/s: flop time = flops * 1e-12, byte time = bytes * 1e-9
    fl_tok = 2 * 3 * 256 * 256  # 393,216 FLOPs per token and expert
    by_exp = 3 * 256 * 256 * 18 / 32  # 110,592 B of Q4_0 weights per expert
    # expert 0: 10 tokens (byte-bound), expert 1: 10^6 tokens (flop-bound), expert 2: unused
    r = b.prefill_roofline([[10, 1e6, 0]], n_tokens=10, shape=s, tflops=tflops, hbm_gbs=hbm)
    want = max(10 * fl_tok * 1e-12, by_exp * 1e-9) + max(1e6 * fl_tok * 1e-12, by_exp * 1e-9)
    assert abs(r["time_s"] - want) <= 1e-15 * want + 1e-18
    assert r["useful_flops"] == (10 + 1e6) * fl_tok
    # issued: 1 + 7813 tiles of 128 rows, every K step twice
    assert r["issued_flops"] == (1 + np.ceil(1e6 / 128)) * 128 * fl_tok * 2


def test_prefill_roofline_shared_expert_every_token():
    b = _bench()
    s = _Shape(n_layers=2, hidden=256, inter=256, shared_inter=512)
    r0 = b.prefill_roofline(np.zeros((2, 4)), n_tokens=300, shape=s, tflops=1.0, hbm_gbs=1.0)
    fl = 300 * 2 * 3 * 256 * 512
    by = 3 * 256 * 512 * 18 / 32
    assert abs(r0["time_s"] - 2 * max(fl * 1e-12, by * 1e-9)) < 1e-18
    assert r0["useful_flops"] == 2 * fl
    assert r0["issued_flops"] == 2 * np.ceil(300 / 128) * 128 * 2 * 3 * 256 * 512 * 2
