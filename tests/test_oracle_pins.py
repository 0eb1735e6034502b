"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test ties one oracle function to a hand-built value, a brute-force search, a
closed form, an invariant or a library routine, chosen so that a plausible slip in the
oracle (a dropped term, a wrong sign or index, a transposed operand) fails.
"""
import itertools
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
U24 = 2.0 ** -24


# ------------------------------------------------------------------ conversions

def test_f16_all_bit_patterns_match_numpy():
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float32)
    got = np.array([oracle.f16_to_f32(int(b)) for b in bits], np.float32)
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite].view(np.uint32), ref[finite].view(np.uint32))
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(np.isinf(got), np.isinf(ref))


def test_bf16_all_bit_patterns_match_torch():
    bits = np.arange(65536, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    got = np.array([oracle.bf16_to_f32(int(b)) for b in bits], np.float32)
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite].view(np.uint32), ref[finite].view(np.uint32))
    assert np.array_equal(np.isnan(got), np.isnan(ref))


# ------------------------------------------------------------------ Q4_0

def _golden_blocks():
    blocks, expects = [], []
    with open(os.path.join(GOLDEN, "q4_0_blocks.txt")) as f:
        for line in f:
            if line.startswith("block"):
                hexs = "".join(line.split()[1:])
                blocks.append(bytes.fromhex(hexs))
            elif line.startswith("expect"):
                expects.append([float(v) for v in line.split()[1:]])
    assert len(blocks) == len(expects) == 5
    return blocks, expects


def test_q4_0_hand_built_blocks():
    blocks, expects = _golden_blocks()
    for blk, exp in zip(blocks, expects):
        assert len(blk) == 18 and len(exp) == 32
        got = oracle.dequant_q4_0(np.frombuffer(blk, np.uint8))
        assert np.array_equal(got, np.array(exp)), (blk.hex(), got)
    # all five in one call: blocks are independent and in order
    got = oracle.dequant_q4_0(np.frombuffer(b"".join(blocks), np.uint8))
    assert np.array_equal(got, np.array(sum(expects, [])))


def test_q4_0_extremes_and_roundtrip_on_synthetic_blocks():
    m = synthetic.q4_0_matrix(0, 3, synthetic.MAT_GATE, 4, 64)
    blk = m.reshape(-1, 18)
    d = blk[:, :2].copy().view(np.float16).astype(np.float64).reshape(-1)
    w = oracle.dequant_q4_0(m).reshape(-1, 32)
    q = w / d[:, None] + 8
    assert np.array_equal(q, np.round(q)) and q.min() >= 0 and q.max() <= 15
    # nibble placement: the recovered q equals the byte's low / high nibble
    qs = blk[:, 2:]
    assert np.array_equal(q[:, :16].astype(np.uint8), qs & 15)
    assert np.array_equal(q[:, 16:].astype(np.uint8), qs >> 4)


# ------------------------------------------------------------------ canonical fp32 fold

def test_canonical_sum_exact_cases():
    assert oracle.canonical_sum(np.zeros(0, np.float32)) == 0.0
    assert oracle.canonical_sum(np.array([-3.25], np.float32)) == -3.25
    # distinct powers of two: any dropped or doubled term changes the exact sum
    parts = np.array([2.0 ** i for i in range(24)], np.float32)
    assert oracle.canonical_sum(parts) == 2.0 ** 24 - 1
    # 128 small integers (every partial sum exact): lane strides must cover all parts
    parts = np.arange(1, 129, dtype=np.float32)
    assert oracle.canonical_sum(parts) == 128 * 129 / 2
    parts = np.arange(1, 33, dtype=np.float32) * 3
    assert oracle.canonical_sum(parts) == 3 * 32 * 33 / 2


def test_canonical_sum_order_hand_computed():
    # Lane 0 adds parts 0, 32, 64 in that order: 2^24 + 1 rounds to 2^24 (ties to even),
    # and again, so the fold gives 2^24; adding the two ones first would give 2^24 + 2.
    p = np.zeros(128, np.float32)
    p[0], p[32], p[64] = 2.0 ** 24, 1.0, 1.0
    assert oracle.canonical_sum(p) == 2.0 ** 24
    # Butterfly: lanes 0 and 16 meet first (2^24 + 1 -> 2^24), then lane 8 joins
    # (2^24 + 1 -> 2^24); a tree pairing lanes 8 and 16 first would give 2^24 + 2.
    p = np.zeros(32, np.float32)
    p[0], p[16], p[8] = 2.0 ** 24, 1.0, 1.0
    assert oracle.canonical_sum(p) == 2.0 ** 24
    # Lane 1 holds 2^24 + 2 + 2 = 2^24 + 4 exactly, lane 17 holds 1: lane 1 + lane 17 =
    # 2^24 + 5 -> 2^24 + 4 (ties to even); then lane 0's 1.0 joins at offset 1:
    # 2^24 + 4 + 1 -> 2^24 + 4.
    p = np.zeros(64, np.float32)
    p[1], p[33], p[17], p[0] = 2.0 ** 24 + 2, 2.0, 1.0, 1.0
    assert oracle.canonical_sum(p) == 2.0 ** 24 + 4
    # Offset 16 comes first: lanes 1 and 17 meet (1 + 1 = 2) before lane 1 joins lane 0
    # at offset 1, giving 2^24 + 2 exactly; offsets taken from 1 upwards would add each
    # 1.0 to 2^24 on its own and lose both (2^24).
    p = np.zeros(32, np.float32)
    p[0], p[1], p[17] = 2.0 ** 24, 1.0, 1.0
    assert oracle.canonical_sum(p) == 2.0 ** 24 + 2


def test_canonical_sum_within_error_bound():
    rng = np.random.default_rng(0)
    for n in (1, 7, 32, 33, 96, 128, 200):
        p = rng.standard_normal(n).astype(np.float32)
        exact = np.sum(p.astype(np.float64))
        depth = (n + 31) // 32 + 5
        bound = depth * U24 * np.sum(np.abs(p.astype(np.float64))) * 1.01
        assert abs(float(oracle.canonical_sum(p)) - exact) <= bound


# ------------------------------------------------------------------ RMSNorm scale

@pytest.mark.parametrize("H", [16, 512, 2048])
def test_rms_inv_closed_forms(H):
    assert oracle.rms_inv(np.ones(H, np.float32), 0.0) == 1.0
    assert oracle.rms_inv(np.full(H, 2.0, np.float32), 0.0) == 0.5
    assert oracle.rms_inv(np.full(H, -4.0, np.float32), 0.0) == 0.25
    # mean h^2 = 1, eps = 3: 1/sqrt(4)
    h = np.ones(H, np.float32)
    h[::2] = -1
    assert oracle.rms_inv(h, 3.0) == 0.5


def test_rms_inv_sum_of_squares_is_one_fused_chain():
    # One 16-element chunk, h = (a, b, 0, ...) with a = 2051/1024 and b = 1 + 2^-23.
    # a^2 = 4206601 * 2^-20 is exact in fp32; b^2 = 1 + 2^-22 + 2^-46.  The fused step
    # fmaf(b, b, a^2) rounds a^2 + 1 + 2^-22 + 2^-46 once, where a^2 + 1 = 10510354 * 2^-21
    # and fp32 steps by 2^-21 here: just above halfway, so ss = 10510355 * 2^-21.
    # Rounding b^2 first (to 1 + 2^-22) would leave an exact tie, resolved to the even
    # 10510354 * 2^-21, and a different 1/sqrt(ss/16).
    h = np.zeros(16, np.float32)
    h[0], h[1] = 2051 / 1024, 1 + 2.0 ** -23
    ss_fused = np.float32(10510355 * 2.0 ** -21)
    ss_split = np.float32(10510354 * 2.0 ** -21)

    def inv_of(ss):
        return np.float32(1) / np.sqrt(ss / np.float32(16))

    assert inv_of(ss_fused) != inv_of(ss_split)
    assert oracle.rms_inv(h, 0.0) == inv_of(ss_fused)


def test_rms_inv_matches_fp64_within_bound():
    rng = np.random.default_rng(1)
    for H in (32, 512, 2048):
        h = (rng.standard_normal(H) * 3).astype(np.float32)
        ref = 1.0 / np.sqrt(np.mean(h.astype(np.float64) ** 2) + 1e-6)
        got = float(oracle.rms_inv(h, 1e-6))
        # fold error (16 + H/512 + 5 adds) then div, add, sqrt, div roundings
        rel = (16 + H // 512 + 5) * U24 + 6 * U24
        assert abs(got - ref) <= rel * ref


# ------------------------------------------------------------------ router logits

def _bf16(x):
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_router_identity_rows_catch_transpose():
    E, H = 24, 64
    w = np.zeros((E, H), np.uint16)
    for e in range(E):
        w[e, 2 * e + 1] = _bf16(1.0)
    h = np.arange(H, dtype=np.float32) * 0.5 - 7
    b = np.arange(E, dtype=np.float32) * 0.25
    z = oracle.router_logits(w, h, None, 1.0, b)
    assert np.array_equal(z, h[2 * np.arange(E) + 1] + b)


def test_router_gain_and_scale_closed_form():
    E, H = 8, 256
    w = np.full((E, H), _bf16(1.0), np.uint16)
    h = np.ones(H, np.float32)
    g = np.full(H, 0.5, np.float32)
    b = np.full(E, -1.0, np.float32)
    z = oracle.router_logits(w, h, g, 0.25, b)
    assert np.all(z == H * 0.5 * 0.25 - 1.0)


def test_router_rounding_hand_computed():
    one = _bf16(1.0)
    # Each product joins its chunk's chain in one rounding (fmaf): w = (-1, 1 + 2^-7),
    # u = (1 + 2^-7 + 2^-23, 1 + 2^-23).  The chain is -(1 + 2^-7 + 2^-23), then
    # (1 + 2^-7)(1 + 2^-23) - (1 + 2^-7 + 2^-23) = 2^-30 exactly; rounding the product
    # first would drop its 2^-30 and give 0.
    w = np.zeros((1, 16), np.uint16)
    w[0, 0], w[0, 1] = _bf16(-1.0), _bf16(1 + 2.0 ** -7)
    h = np.zeros(16, np.float32)
    h[0], h[1] = 1 + 2.0 ** -7 + 2.0 ** -23, 1 + 2.0 ** -23
    assert oracle.router_logits(w, h, None, 1.0, None)[0] == 2.0 ** -30
    # Chunks of 16 columns: u = (2^24, 1, ..., 1) over 32 columns of ones.  The first
    # chunk's fifteen ones each round away against 2^24 (ties to even); the second chunk
    # sums its sixteen ones to 16 on its own; the fold gives 2^24 + 16.  One chain over
    # all 32 columns would give 2^24, chunks of 8 would give 2^24 + 24.
    w = np.full((1, 32), one, np.uint16)
    h = np.ones(32, np.float32)
    h[0] = 2.0 ** 24
    assert oracle.router_logits(w, h, None, 1.0, None)[0] == 2.0 ** 24 + 16
    # The norm scale and the bias join the folded sum in one rounding:
    # S = 1 + 2^-23, inv = 1 + 2^-23, b = -(1 + 2^-22): S * inv + b = 2^-46 exactly;
    # rounding S * inv first gives 1 + 2^-22 and then 0.
    w = np.zeros((1, 16), np.uint16)
    w[0, 0] = one
    h = np.zeros(16, np.float32)
    h[0] = 1 + 2.0 ** -23
    b = np.array([-(1 + 2.0 ** -22)], np.float32)
    assert oracle.router_logits(w, h, None, np.float32(1 + 2.0 ** -23), b)[0] == 2.0 ** -46


def test_router_matches_fp64_within_bound():
    for layer, (E, H) in enumerate([(64, 512), (256, 2048), (17, 96)]):
        w = synthetic.router_bf16(layer, E, H)
        h = synthetic.token(layer, H)
        g = synthetic.rms_gain(layer, H, "random")
        inv = np.float32(0.8)
        b = synthetic.zipf_bias(layer, E, 1.0)
        z = oracle.router_logits(w, h, g, inv, b)
        wf = torch.from_numpy(w.view(np.int16)).view(torch.bfloat16).double().numpy()
        u = (g.astype(np.float64) * h)
        exact = wf @ u * float(inv) + b
        mag = np.abs(wf) @ np.abs(u) * float(inv) + np.abs(b)
        depth = 16 + H // 512 + 5 + 3
        assert np.all(np.abs(z - exact) <= depth * U24 * mag * 1.01)


# ------------------------------------------------------------------ top-k + weights

def _brute_topk(z, k):
    return np.array(sorted(range(len(z)), key=lambda e: (-float(z[e]), e))[:k], np.int32)


def test_topk_matches_brute_force_sort_with_ties():
    rng = np.random.default_rng(2)
    for trial in range(200):
        E = int(rng.integers(1, 300))
        k = int(rng.integers(1, min(E, 16) + 1))
        z = np.round(rng.standard_normal(E) * 2).astype(np.float32)  # many ties
        assert np.array_equal(oracle.topk(z, k), _brute_topk(z, k))
    # all equal -> the k lowest indices
    assert np.array_equal(oracle.topk(np.full(256, 0.3, np.float32), 8), np.arange(8))
    # -0 and +0 tie -> lower index first
    z = np.array([0.0, -0.0, -1.0, -0.0, 0.0], np.float32)
    assert np.array_equal(oracle.topk(z, 4), [0, 1, 3, 4])


def test_route_weights_are_renormalised_softmax():
    rng = np.random.default_rng(3)
    for E, k in [(64, 4), (256, 8), (10, 10), (5, 1)]:
        z = (rng.standard_normal(E) * 3).astype(np.float32)
        sel = oracle.topk(z, k)
        w = oracle.route_weights(z, sel)
        full = scipy.special.softmax(z.astype(np.float64))
        ref = full[sel] / full[sel].sum()
        assert np.allclose(w, ref, rtol=1e-12, atol=1e-15)
        assert abs(w.sum() - 1.0) <= k * 2.0 ** -52
        assert np.all(np.diff(w) <= 0)  # rank order == weight order
        if k == E:
            assert np.allclose(w, full[sel], rtol=1e-12)
        if k == 1:
            assert w[0] == 1.0


def test_silu_values():
    assert oracle.silu(0.0) == 0.0
    for t in (-30.0, -3.0, -0.5, 0.25, 2.0, 40.0):
        assert oracle.silu(t) == pytest.approx(t * scipy.special.expit(t), rel=1e-14, abs=1e-300)
    assert oracle.silu(50.0) == pytest.approx(50.0, rel=1e-20)


# ------------------------------------------------------------------ experts

def _dense(q4, H, I):
    n_gu = I * H // 32 * 18
    G = oracle.dequant_q4_0(q4[:n_gu]).reshape(I, H)
    U = oracle.dequant_q4_0(q4[n_gu:2 * n_gu]).reshape(I, H)
    D = oracle.dequant_q4_0(q4[2 * n_gu:]).reshape(H, I)
    return G, U, D


@pytest.mark.parametrize("H,I", [(64, 96), (96, 32), (512, 256)])
def test_expert_ffn_equals_dense_swiglu(H, I):
    q4 = synthetic.expert_q4_0(0, 5, H, I)
    assert q4.size == 3 * H * I // 32 * 18
    x = synthetic.token(9, H).astype(np.float64)
    G, U, D = _dense(q4, H, I)
    g, u = G @ x, U @ x
    ref = D @ (g * scipy.special.expit(g) * u)
    got = oracle.expert_ffn(q4, H, I, x)
    assert np.allclose(got, ref, rtol=1e-11, atol=1e-13)


def _model(shape, gain_kind="ones", n_layers=None):
    L = shape.n_layers if n_layers is None else n_layers
    layers = [synthetic.layer_weights(l, shape, gain_kind) for l in range(L)]
    return oracle.Model(shape, layers), layers


def test_top1_layer_reduces_to_dense_ffn_of_argmax_expert():
    s = synthetic.Shape(1, 128, 16, 1, 64, 0, zipf_s=1.0)
    m, layers = _model(s)
    x = synthetic.token(0, s.hidden)
    out = m.layer(0, x)
    assert out["w"][0] == 1.0
    assert out["sel"][0] == int(np.argmax(out["z"]))
    G, U, D = _dense(layers[0].experts[out["sel"][0]], s.hidden, s.inter)
    xd = x.astype(np.float64)
    g = G @ xd
    ref = D @ (g * scipy.special.expit(g) * (U @ xd))
    assert np.allclose(out["y"], ref, rtol=1e-11, atol=1e-13)
    assert np.array_equal(out["h_out"], out["y"])  # no residual without the norm


def test_layer_is_weighted_sum_of_experts_plus_shared():
    s = synthetic.Shape(1, 128, 12, 3, 64, 96, zipf_s=1.0)
    m, layers = _model(s)
    x = synthetic.token(4, s.hidden)
    out = m.layer(0, x)
    xd = x.astype(np.float64)

    def ffn(q4, I):
        G, U, D = _dense(q4, s.hidden, I)
        g = G @ xd
        return D @ (g * scipy.special.expit(g) * (U @ xd))

    ref = sum(out["w"][i] * ffn(layers[0].experts[out["sel"][i]], s.inter) for i in range(s.top_k))
    ref = ref + ffn(layers[0].shared, s.shared_inter)
    assert np.allclose(out["y"], ref, rtol=1e-11, atol=1e-13)
    # the shared expert is additive: removing it removes exactly its FFN
    s0 = synthetic.Shape(1, 128, 12, 3, 64, 0, zipf_s=1.0)
    m0 = oracle.Model(s0, [synthetic.LayerWeights(layers[0].experts, None, layers[0].router,
                                                  layers[0].bias, layers[0].gain)])
    out0 = m0.layer(0, x)
    assert np.array_equal(out0["sel"], out["sel"])
    assert np.allclose(out["y"] - out0["y"], ffn(layers[0].shared, 96), rtol=1e-10, atol=1e-12)


def test_norm_layer_special_cases():
    s = synthetic.Shape(1, 256, 16, 4, 64, 64, use_rmsnorm=1, zipf_s=1.0, rms_eps=0.0)
    m, layers = _model(s)
    rng = np.random.default_rng(5)
    # h with mean(h^2) == 1 exactly: the norm is the identity, so the stack layer's
    # update equals the plain layer's output on h itself
    h = rng.choice([-1.0, 1.0], size=s.hidden).astype(np.float32)
    out = m.layer(0, h)
    plain = oracle.Model(synthetic.Shape(1, 256, 16, 4, 64, 64, zipf_s=1.0), layers).layer(0, h)
    assert np.array_equal(out["sel"], plain["sel"])
    assert np.allclose(out["h_out"] - h, plain["y"], rtol=1e-12, atol=1e-12)
    # with a non-uniform power-of-two gain g on the same unit-RMS h, the norm reduces to
    # x = g * h exactly, so the update equals the plain layer on g * h
    g = np.where(np.arange(s.hidden) % 3 == 0, 2.0, 0.5).astype(np.float32)
    lw_g = [synthetic.LayerWeights(layers[0].experts, layers[0].shared, layers[0].router,
                                   layers[0].bias, g)]
    out_g = oracle.Model(s, lw_g).layer(0, h)
    plain_g = oracle.Model(synthetic.Shape(1, 256, 16, 4, 64, 64, zipf_s=1.0), lw_g).layer(0, g * h)
    assert np.array_equal(out_g["z"], plain_g["z"])
    assert np.array_equal(out_g["sel"], plain_g["sel"])
    assert np.allclose(out_g["h_out"] - h, plain_g["y"], rtol=1e-12, atol=1e-12)
    # eps = 3 on the same unit-RMS h: mean(h^2) + eps = 4, so the norm is x = g * h / 2
    # exactly, routing included (a power-of-two scale passes through every fmaf)
    s3 = synthetic.Shape(1, 256, 16, 4, 64, 64, use_rmsnorm=1, zipf_s=1.0, rms_eps=3.0)
    out_e = oracle.Model(s3, lw_g).layer(0, h)
    plain_e = oracle.Model(synthetic.Shape(1, 256, 16, 4, 64, 64, zipf_s=1.0), lw_g).layer(0, g * h / 2)
    assert np.array_equal(out_e["z"], plain_e["z"])
    assert np.array_equal(out_e["sel"], plain_e["sel"])
    assert np.allclose(out_e["h_out"] - h, plain_e["y"], rtol=1e-12, atol=1e-12)
    # scale invariance of RMSNorm (eps = 0): y(4h) == y(h) and routing is unchanged
    h = rng.standard_normal(s.hidden).astype(np.float32)
    a, b = m.layer(0, h), m.layer(0, 4 * h)
    assert np.array_equal(a["sel"], b["sel"])
    assert np.allclose(a["y"], b["y"], rtol=1e-12, atol=1e-12)
    assert np.allclose(b["h_out"], 4 * h + a["y"], rtol=1e-12, atol=1e-12)


def test_stack_decode_is_composition_of_layers():
    s = synthetic.Shape(3, 128, 16, 4, 64, 32, use_rmsnorm=1, zipf_s=1.0)
    m, _ = _model(s, gain_kind="random")
    x = synthetic.token(11, s.hidden)
    h, sel, tr = m.decode(x, trace=True)
    cur = x.astype(np.float64)
    for l in range(s.n_layers):
        out = m.layer(l, cur.astype(np.float32), cur)
        assert np.array_equal(out["sel"], sel[l])
        cur = out["h_out"]
        assert np.array_equal(cur, tr[l + 1])
    assert np.array_equal(cur, h)


# ------------------------------------------------------------------ placement + cache

def test_select_pinned_brute_force():
    rng = np.random.default_rng(6)
    for _ in range(100):
        E = int(rng.integers(1, 80))
        P = int(rng.integers(0, E + 1))
        hist = rng.integers(0, 5, E).astype(np.uint32)
        ref = np.zeros(E, np.uint8)
        ref[sorted(range(E), key=lambda e: (-int(hist[e]), e))[:P]] = 1
        assert np.array_equal(oracle.select_pinned(hist, P), ref)


def _brute_cache(pinned, R, accesses):
    """Brute-force LRU ring: recency recomputed from the full history at every miss."""
    P = int(pinned.sum())
    pin_slot = np.cumsum(pinned) - 1
    owner = [-1] * R
    history = []  # (time, expert) of every ring hit and ring fill
    events = []
    for t, e in enumerate(accesses):
        if pinned[e]:
            events.append((0, int(pin_slot[e]), -1))
            continue
        if e in owner:
            r = owner.index(e)
            history.append((t, e))
            events.append((1, P + r, -1))
            continue
        empty = [r for r in range(R) if owner[r] < 0]
        if empty:
            r = empty[0]
        else:
            def last_use(r):
                return max(tt for tt, ee in history if ee == owner[r])
            r = min(range(R), key=last_use)
        events.append((2, P + r, owner[r]))
        owner[r] = e
        history.append((t, e))
    return events, owner


def test_cache_matches_brute_force_lru():
    rng = np.random.default_rng(7)
    for trial in range(60):
        E = int(rng.integers(4, 40))
        R = int(rng.integers(1, 6))
        k = int(rng.integers(1, min(E, 8) + 1))
        pinned = (rng.random(E) < 0.4).astype(np.uint8)
        c = oracle.Cache(1, E, R)
        c.set_pinned(0, pinned)
        seq = []
        got = []
        for step in range(30):
            sel = rng.choice(E, size=k, replace=False).astype(np.int32)
            ev = c.access(step, 0, sel)
            assert np.array_equal(ev["rank"], np.arange(k)) and np.all(ev["step"] == step)
            assert np.array_equal(ev["expert"], sel)
            seq.extend(sel.tolist())
            got.extend(zip(ev["kind"].tolist(), ev["slot"].tolist(), ev["evicted"].tolist()))
        ref, owner = _brute_cache(pinned, R, seq)
        assert got == ref
        assert np.array_equal(c.ring(0), owner)
        kinds = np.array([g[0] for g in got])
        assert len(kinds) == len(seq)  # hits + misses == accesses
        assert len(set(o for o in owner if o >= 0)) <= R


def test_cache_full_residency_never_misses_and_layers_are_independent():
    E, R, k = 32, 4, 4
    c = oracle.Cache(2, E, R)
    c.set_pinned(0, np.ones(E, np.uint8))
    c.set_pinned(1, np.zeros(E, np.uint8))
    rng = np.random.default_rng(8)
    for step in range(50):
        sel = rng.choice(E, size=k, replace=False).astype(np.int32)
        e0 = c.access(step, 0, sel)
        assert np.all(e0["kind"] == oracle.PIN_HIT)
        assert np.array_equal(e0["slot"], sel)  # all pinned: slot == expert index
        e1 = c.access(step, 1, sel)
        assert np.all(e1["kind"] != oracle.PIN_HIT)


def test_ring_reused_within_one_token_when_misses_exceed_ring():
    c = oracle.Cache(1, 16, 2)
    c.set_pinned(0, np.zeros(16, np.uint8))
    ev = c.access(0, 0, np.array([3, 5, 7, 9], np.int32))
    assert ev["kind"].tolist() == [2, 2, 2, 2]
    assert ev["slot"].tolist() == [0, 1, 0, 1]
    assert ev["evicted"].tolist() == [-1, -1, 3, 5]
    assert c.ring(0).tolist() == [7, 9]


def test_repin_empties_the_ring():
    """A new pinned set starts with an empty ring: an expert the ring held before misses
    again, into the first ring slot, with nothing evicted."""
    c = oracle.Cache(1, 8, 2)
    c.set_pinned(0, np.zeros(8, np.uint8))
    c.access(0, 0, np.array([1, 2], np.int32))
    assert c.ring(0).tolist() == [1, 2]
    mask = np.zeros(8, np.uint8)
    mask[5] = 1
    c.set_pinned(0, mask)
    assert c.ring(0).tolist() == [-1, -1]
    ev = c.access(1, 0, np.array([1, 5], np.int32))
    assert ev["kind"].tolist() == [oracle.MISS, oracle.PIN_HIT]
    assert ev["slot"].tolist() == [1, 0] and ev["evicted"].tolist() == [-1, -1]


def test_calibrated_placement_cuts_cold_hits_vs_uniform():
    """The write-up's direction (cold-hit rate 36% -> ~7%): pinning the most-routed
    experts must beat an uninformed split on Zipf-skewed routing."""
    s = synthetic.Shape(1, 256, 64, 4, 32, 0, zipf_s=1.0)
    m, _ = _model(s)
    calib = np.zeros(s.n_experts, np.uint32)
    for t in range(64):
        calib[m.layer(0, synthetic.token(t, s.hidden, synthetic.SEED_CALIB))["sel"]] += 1
    P = round(0.6 * s.n_experts)
    cal_mask = oracle.select_pinned(calib, P)
    uni_mask = np.zeros(s.n_experts, np.uint8)
    uni_mask[:P] = 1
    cold = {}
    for name, mask in (("cal", cal_mask), ("uni", uni_mask)):
        c = oracle.Cache(1, s.n_experts, 4)
        c.set_pinned(0, mask)
        kinds = []
        for t in range(64):
            kinds += c.access(t, 0, m.layer(0, synthetic.token(t, s.hidden))["sel"])["kind"].tolist()
        cold[name] = np.mean(np.array(kinds) != oracle.PIN_HIT)
    assert cold["cal"] < cold["uni"]
    assert cold["cal"] < 0.15 and cold["uni"] > 0.2


# ------------------------------------------------------------------ recalibration

def test_recal_score_closed_forms():
    # a constant window w = 2^10 from zero: s_n = 2w - w / 2^(n-1), exactly
    w = np.full(5, 1024, np.uint32)
    s = np.zeros(5, np.uint32)
    for n in range(1, 11):
        s = oracle.recal_score(s, w)
        assert np.all(s == 2048 - 1024 // 2 ** (n - 1))
    # fixed points of s = floor(s/2) + w are 2w and 2w - 1
    for w0 in (1, 7, 1000):
        for fp in (2 * w0, 2 * w0 - 1):
            assert oracle.recal_score(np.array([fp]), np.array([w0]))[0] == fp
    # a one-off burst B then quiet windows: s_n = floor(B / 2^n)
    s = oracle.recal_score(np.zeros(1, np.uint32), np.array([1000]))
    for n in range(1, 12):
        s = oracle.recal_score(s, np.zeros(1, np.uint32))
        assert s[0] == 1000 >> n


def test_recalibration_follows_drifted_popularity():
    """The write-up's "self-tunes over time": after the popularity permutation changes,
    re-pinning from decayed routing counts cuts cold hits below a placement frozen at the
    first calibration."""
    s = synthetic.Shape(1, 256, 64, 4, 32, 0, ring_slots=4, zipf_s=1.0)
    layers = [synthetic.layer_weights(0, s)]
    drifted = [synthetic.layer_weights(0, s, bias_seed=synthetic.SEED_RESHUFFLE)]
    m_old, m_new = oracle.Model(s, layers), oracle.Model(s, drifted)
    P = round(0.4 * s.n_experts)
    calib = np.zeros(s.n_experts, np.uint32)
    for t in range(64):
        calib[m_old.layer(0, synthetic.token(t, s.hidden, synthetic.SEED_CALIB))["sel"]] += 1
    cold = {}
    for name in ("static", "recal"):
        c = oracle.Cache(1, s.n_experts, 4)
        c.set_pinned(0, oracle.select_pinned(calib, P))
        score, window, kinds = calib.copy(), np.zeros(s.n_experts, np.uint32), []
        for t in range(256):
            if name == "recal" and t % 16 == 0 and t:
                score = oracle.recal_score(score, window)
                window[:] = 0
                c.set_pinned(0, oracle.select_pinned(score, P))
            sel = (m_old if t < 96 else m_new).layer(0, synthetic.token(t, s.hidden))["sel"]
            window[sel] += 1
            kinds.append(c.access(t, 0, sel)["kind"])
        k = np.concatenate(kinds[128:])
        cold[name] = np.mean(k != oracle.PIN_HIT)
    assert cold["recal"] < 0.5 * cold["static"]
