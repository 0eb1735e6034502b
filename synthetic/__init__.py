"""Seeded synthetic inputs for the MoE decode path: expert weights, router, tokens.

This module is shared by the CPU oracle's tests, the CUDA path's tests and the bench.
It draws random numbers and packs bytes; it holds none of the MoE layer's arithmetic
(no dequantisation, no dot products, no routing, no cache policy).

Workload shapes follow the pages' description of an A3B-class MoE (Luce Spark write-up,
"runs 35B MoE models on 16GB GPU", key components paragraph): about 8 of 256 experts
routed per token, 40 layers.  Every stream is keyed by (seed, layer, expert, matrix) or
(seed, step) through numpy's SeedSequence, so any single expert or token can be
regenerated on its own.

Recipe (stated once, used everywhere):
  * Q4_0 expert matrices, GGUF block layout (18 bytes per 32 weights: fp16 scale d,
    then 16 bytes; byte j holds weight j in its low nibble and weight j+16 in its high
    nibble).  Nibbles q are uniform on 0..15; d = fp16(0.0043 * U(0.5, 1.5)), so the
    weight std is about 0.02.
  * Router weights W_r ~ N(0, 0.02) rounded to bf16 (round to nearest even).
  * Router bias b_e = s * ln(p_e), p_e = (1/rank_e) / H_E with rank_e the position of
    expert e in a seeded per-layer permutation (Zipf exponent 1.0), s = 1.0.
  * Tokens x ~ N(0, 1) fp32, one independent stream per decode step.
  * RMSNorm gains: ones by default, or U(0.5, 1.5) when a test wants them non-trivial.
"""
from __future__ import annotations

import dataclasses

import numpy as np

SEED_WEIGHTS = 0x5EED0000
SEED_PERM = 0x9E3779B9
SEED_TOKENS = 42
SEED_CALIB = 7
SEED_RESHUFFLE = 1337
SEED_GAIN = 0x6A1
SEED_ROUTER = 0x2047

MAT_GATE, MAT_UP, MAT_DOWN = 0, 1, 2
Q4_0_BLOCK_BYTES = 18
Q4_0_BLOCK_ELEMS = 32


@dataclasses.dataclass(frozen=True)
class Shape:
    """Dimensions of one MoE stack."""

    n_layers: int
    hidden: int
    n_experts: int
    top_k: int
    inter: int
    shared_inter: int  # 0: no shared expert
    ring_slots: int = 8
    use_rmsnorm: int = 0
    zipf_s: float = 1.0  # 0.0: zero router bias
    rms_eps: float = 1e-6

    def expert_bytes(self) -> int:
        return 3 * self.hidden * self.inter * Q4_0_BLOCK_BYTES // Q4_0_BLOCK_ELEMS

    def shared_bytes(self) -> int:
        return 3 * self.hidden * self.shared_inter * Q4_0_BLOCK_BYTES // Q4_0_BLOCK_ELEMS


# The two shapes the pages' workload is described at: a small single layer and the
# full A3B-class layer (hidden 2048, 256 experts, top-8, 512-wide SwiGLU, one shared).
SMALL = Shape(n_layers=1, hidden=512, n_experts=64, top_k=4, inter=256, shared_inter=0,
              zipf_s=0.0)
FULL_LAYER = Shape(n_layers=1, hidden=2048, n_experts=256, top_k=8, inter=512,
                   shared_inter=512)
FULL_STACK = Shape(n_layers=40, hidden=2048, n_experts=256, top_k=8, inter=512,
                   shared_inter=512, ring_slots=8, use_rmsnorm=1)


def _stream(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.SFC64(np.random.SeedSequence([int(k) for k in key])))


def q4_0_matrix(layer: int, expert: int, matrix: int, rows: int, cols: int,
                seed: int = SEED_WEIGHTS) -> np.ndarray:
    """One Q4_0 matrix [rows x cols], row-major, canonical 18-byte blocks, as uint8."""
    if cols % Q4_0_BLOCK_ELEMS:
        raise ValueError("cols must be a multiple of 32")
    nblk = rows * cols // Q4_0_BLOCK_ELEMS
    raw = np.random.SFC64(np.random.SeedSequence([seed, layer, expert, matrix])).random_raw(3 * nblk)
    out = np.empty((nblk, Q4_0_BLOCK_BYTES), np.uint8)
    out[:, 2:] = raw[: 2 * nblk].view(np.uint8).reshape(nblk, 16)
    u = (raw[2 * nblk:] >> np.uint64(40)).astype(np.float64) * (1.0 / (1 << 24))
    d = (0.0043 * (0.5 + u)).astype(np.float16)
    out[:, :2] = d.view(np.uint8).reshape(nblk, 2)
    return out.reshape(-1)


def expert_q4_0(layer: int, expert: int, hidden: int, inter: int,
                seed: int = SEED_WEIGHTS) -> np.ndarray:
    """Gate [inter x hidden] | up [inter x hidden] | down [hidden x inter], concatenated."""
    return np.concatenate([
        q4_0_matrix(layer, expert, MAT_GATE, inter, hidden, seed),
        q4_0_matrix(layer, expert, MAT_UP, inter, hidden, seed),
        q4_0_matrix(layer, expert, MAT_DOWN, hidden, inter, seed),
    ])


def shared_q4_0(layer: int, shape: Shape, seed: int = SEED_WEIGHTS) -> np.ndarray | None:
    """The shared expert of a layer (keyed as expert index n_experts)."""
    if shape.shared_inter == 0:
        return None
    return expert_q4_0(layer, shape.n_experts, shape.hidden, shape.shared_inter, seed)


def router_bf16(layer: int, n_experts: int, hidden: int, seed: int = SEED_ROUTER) -> np.ndarray:
    """Router weights [E x H] as bf16 bit patterns (uint16), N(0, 0.02) rounded to nearest even."""
    w = _stream(seed, layer).standard_normal(n_experts * hidden, dtype=np.float32) * np.float32(0.02)
    bits = w.view(np.uint32).astype(np.uint64)
    rounded = (bits + np.uint64(0x7FFF) + ((bits >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return rounded.astype(np.uint16).reshape(n_experts, hidden)


def zipf_perm(layer: int, n_experts: int, seed: int = SEED_PERM) -> np.ndarray:
    """Seeded permutation: perm[r] is the expert of popularity rank r+1."""
    return _stream(seed, layer).permutation(n_experts)


def zipf_bias(layer: int, n_experts: int, s: float = 1.0, seed: int = SEED_PERM) -> np.ndarray:
    """Router bias b_e = s * ln(p_e) with Zipf(1.0) p_e over a seeded permutation (fp32)."""
    if s == 0.0:
        return np.zeros(n_experts, np.float32)
    perm = zipf_perm(layer, n_experts, seed)
    rank = np.empty(n_experts, np.int64)
    rank[perm] = np.arange(1, n_experts + 1)
    harmonic = np.sum(1.0 / np.arange(1, n_experts + 1, dtype=np.float64))
    p = (1.0 / rank) / harmonic
    return (s * np.log(p)).astype(np.float32)


def rms_gain(layer: int, hidden: int, kind: str = "ones", seed: int = SEED_GAIN) -> np.ndarray:
    if kind == "ones":
        return np.ones(hidden, np.float32)
    return (0.5 + _stream(seed, layer).random(hidden, dtype=np.float64)).astype(np.float32)


def token(step: int, hidden: int, seed: int = SEED_TOKENS) -> np.ndarray:
    """Decode input of one step, x ~ N(0, 1) fp32."""
    return _stream(seed, step).standard_normal(hidden, dtype=np.float32)


def tokens(first_step: int, n: int, hidden: int, seed: int = SEED_TOKENS) -> np.ndarray:
    return np.stack([token(first_step + i, hidden, seed) for i in range(n)])


@dataclasses.dataclass
class LayerWeights:
    experts: list  # n_experts arrays of uint8 (canonical Q4_0, gate|up|down)
    shared: np.ndarray | None
    router: np.ndarray  # uint16 [E, H]
    bias: np.ndarray  # float32 [E]
    gain: np.ndarray  # float32 [H]


def layer_weights(layer: int, shape: Shape, gain_kind: str = "ones",
                  bias_seed: int = SEED_PERM, threads: int = 8) -> LayerWeights:
    from concurrent.futures import ThreadPoolExecutor

    def one(e):
        return expert_q4_0(layer, e, shape.hidden, shape.inter)

    if threads > 1 and shape.n_experts >= 16:
        with ThreadPoolExecutor(threads) as ex:
            experts = list(ex.map(one, range(shape.n_experts)))
    else:
        experts = [one(e) for e in range(shape.n_experts)]
    return LayerWeights(
        experts=experts,
        shared=shared_q4_0(layer, shape),
        router=router_bf16(layer, shape.n_experts, shape.hidden),
        bias=zipf_bias(layer, shape.n_experts, shape.zipf_s, bias_seed),
        gain=rms_gain(layer, shape.hidden, gain_kind),
    )
