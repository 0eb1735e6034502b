"""Mutation check of the oracle's pins.

Each entry plants one plausible slip in a copy of the oracle's C source (on the CPU,
in a temporary folder), compiles it with the oracle's own flags and runs the pins of
test_oracle_pins.py against it: every mutant must make at least one pin fail.  A mutant
that survives is a part of the oracle the pins do not hold.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

# (name, text in moe_oracle.c, replacement)
MUTANTS = [
    # conversions and Q4_0
    ("fp16 exponent bias off by one", "ldexpf((float)(man | 0x400), exp - 25)",
     "ldexpf((float)(man | 0x400), exp - 24)"),
    ("fp16 subnormal scale", "ldexpf((float)man, -24)", "ldexpf((float)man, -23)"),
    ("bf16 placed one bit low", "uint32_t u = (uint32_t)b << 16;", "uint32_t u = (uint32_t)b << 15;"),
    ("low half reads the high nibble", "out[32 * b + j] = (double)((qs[j] & 15) - 8) * d;",
     "out[32 * b + j] = (double)((qs[j] >> 4) - 8) * d;"),
    ("Q4_0 offset 7", "out[32 * b + 16 + j] = (double)((qs[j] >> 4) - 8) * d;",
     "out[32 * b + 16 + j] = (double)((qs[j] >> 4) - 7) * d;"),
    # canonical fold
    ("fold drops the last part", "for (int m = l; m < n; m += ORC_LANES)",
     "for (int m = l; m < n - 1; m += ORC_LANES)"),
    ("butterfly offsets ascending", "for (int off = ORC_LANES / 2; off >= 1; off /= 2)",
     "for (int off = 1; off < ORC_LANES; off *= 2)"),
    ("lane chain accumulates in reverse", "for (int m = l; m < n; m += ORC_LANES) acc = acc + parts[m];",
     "for (int m = l + ((n - 1 - l) / ORC_LANES) * ORC_LANES; m >= l && m < n; m -= ORC_LANES) "
     "acc = acc + parts[m];"),
    # RMSNorm scale
    ("sum of squares by multiply then add",
     "p = fmaf(h[c * ORC_CHUNK + t], h[c * ORC_CHUNK + t], p);",
     "p = h[c * ORC_CHUNK + t] * h[c * ORC_CHUNK + t] + p;"),
    ("mean over H + 1", "float mean = ss / (float)H;", "float mean = ss / (float)(H + 1);"),
    ("eps added after the root", "float r = sqrtf(mean + eps);", "float r = sqrtf(mean) + eps;"),
    # router
    ("router chunks of 32", "#define ORC_CHUNK 16", "#define ORC_CHUNK 32"),
    ("router weight transposed", "p = fmaf(orc_bf16_to_f32(row[j]), u[j], p);",
     "p = fmaf(orc_bf16_to_f32(w[(size_t)j * E + e]), u[j], p);"),
    ("router products rounded before the add", "p = fmaf(orc_bf16_to_f32(row[j]), u[j], p);",
     "p = orc_bf16_to_f32(row[j]) * u[j] + p;"),
    ("norm scale rounded before the bias", "z[e] = fmaf(s, inv, bias ? bias[e] : 0.0f);",
     "z[e] = s * inv + (bias ? bias[e] : 0.0f);"),
    ("router bias dropped", "z[e] = fmaf(s, inv, bias ? bias[e] : 0.0f);", "z[e] = fmaf(s, inv, 0.0f);"),
    ("router gain dropped", "u[j] = gain ? gain[j] * h[j] : h[j];", "u[j] = h[j];"),
    # top-k and weights
    ("top-k ties to the higher index", "if (best < 0 || z[e] > z[best]) best = e;",
     "if (best < 0 || z[e] >= z[best]) best = e;"),
    ("top-k smallest logits", "if (best < 0 || z[e] > z[best]) best = e;",
     "if (best < 0 || z[e] < z[best]) best = e;"),
    ("weights not renormalised", "for (int i = 0; i < k; ++i) w[i] = exp((double)z[sel[i]] - zmax) / s;",
     "for (int i = 0; i < k; ++i) w[i] = exp((double)z[sel[i]] - zmax);"),
    # experts and combine
    ("silu sign", "return t / (1.0 + exp(-t));", "return t / (1.0 + exp(t));"),
    ("gate and up swapped", "a[r] = orc_silu(g) * u;", "a[r] = orc_silu(u) * g;"),
    ("up read from the gate matrix", "*U = q4 + (size_t)I * rowblk_gu * 18,", "*U = q4,"),
    ("combine weights in reverse rank order", "for (int j = 0; j < H; ++j) y[j] += w[i] * o[j];",
     "for (int j = 0; j < H; ++j) y[j] += w[k - 1 - i] * o[j];"),
    ("shared expert halved", "for (int j = 0; j < H; ++j) y[j] += o[j];",
     "for (int j = 0; j < H; ++j) y[j] += 0.5 * o[j];"),
    ("residual dropped", "h_out[j] = d->use_rmsnorm ? h64[j] + y[j] : y[j];", "h_out[j] = y[j];"),
    ("norm gain dropped from the expert input", "x[j] = h64[j] * inv64 * (double)gain[j];",
     "x[j] = h64[j] * inv64;"),
    ("norm eps dropped from the expert input", "double inv64 = 1.0 / sqrt(ss / H + (double)d->rms_eps);",
     "double inv64 = 1.0 / sqrt(ss / H);"),
    # placement and recalibration
    ("pinning ties to the higher index", "if (best < 0 || hist[e] > hist[best]) best = e;",
     "if (best < 0 || hist[e] >= hist[best]) best = e;"),
    ("recalibration without decay", "score[i] = (score[i] >> 1) + window[i];",
     "score[i] = score[i] + window[i];"),
    # cache simulator
    ("LRU evicts the most recent", "if (used[r] < used[victim]) victim = r;",
     "if (used[r] > used[victim]) victim = r;"),
    ("ring hit does not refresh recency", "used[hit] = ++c->clock[layer];", "(void)c->clock[layer];"),
    ("empty ring slots filled from the top", "for (int r = 0; r < R && victim < 0; ++r)",
     "for (int r = R - 1; r >= 0 && victim < 0; --r)"),
    ("eviction not logged", "v->evicted = owner[victim];", "v->evicted = -1;"),
    ("ring slots numbered without the pinned offset", "v->slot = P + victim;", "v->slot = victim;"),
    ("pinned slots numbered from 1", "mask[e] ? p++ : -1", "mask[e] ? ++p : -1"),
    ("re-pin keeps the ring", "c->ring_owner[(size_t)layer * c->ring_slots + r] = -1;", "(void)0;"),
]


def _run_pins(lib_path: str) -> subprocess.CompletedProcess:
    env = dict(os.environ, ORACLE_LIB=lib_path)
    return subprocess.run([sys.executable, "-m", "pytest", PINS, "-x", "-q", "-p", "no:cacheprovider"],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_every_planted_slip_fails_a_pin(tmp_path):
    src = open(oracle._SRC).read()
    libs = []
    for i, (name, old, new) in enumerate(MUTANTS):
        assert src.count(old) == 1, f"{name}: text not found exactly once"
        c_path = tmp_path / f"mutant{i}.c"
        c_path.write_text(src.replace(old, new))
        so_path = str(tmp_path / f"mutant{i}.so")
        oracle.compile_c(str(c_path), so_path)
        libs.append(so_path)
    workers = max(1, min(4, (os.cpu_count() or 2)))
    with ThreadPoolExecutor(workers) as ex:
        results = list(ex.map(_run_pins, libs))
    survivors = [name for (name, _, _), r in zip(MUTANTS, results) if r.returncode == 0]
    crashed = [(name, r.returncode) for (name, _, _), r in zip(MUTANTS, results)
               if r.returncode not in (0, 1)]
    assert not survivors, f"mutants not caught by any pin: {survivors}"
    assert not crashed, f"mutants that crashed the pin run instead of failing a pin: {crashed}"


def test_unmutated_copy_passes_the_pins(tmp_path):
    """The harness itself: the oracle's source compiled the same way passes every pin."""
    so_path = str(tmp_path / "copy.so")
    oracle.compile_c(oracle._SRC, so_path)
    r = _run_pins(so_path)
    assert r.returncode == 0, r.stdout[-2000:]
