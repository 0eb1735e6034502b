"""Edge cases of the CUDA path against the CPU oracle: exact logit ties, zero logits of
either sign, duplicate router rows, and extreme Q4_0 scales.

Ties: the reading "equal logits -> lower expert index" must hold on the GPU's top-k
(decode) and on the prefill's certified candidate rule.  A layer with an all-zero router
makes every logit exactly its bias (z = fmaf(+0, inv, b) = b), so the biases set exact
ties: at the k-th place (0.5, 0.5, 0.5 for two places) and, in a second layer, sixty-one
experts tied at zero with biases of both signs (-0 and +0 compare equal; the plus-zero
sum of the canonical fold makes every such logit +0).  A third layer has random router
rows of which two are identical and carry the same large bias: their logits are equal to
the bit, both are selected, the lower index ranks first.

Extreme scales: the golden blocks of tests/golden/q4_0_blocks.txt with the smallest
subnormal fp16 scale (2^-24, block D) and the largest finite one (65504, block E: every
weight -524032) are written into gate, up and down rows of the expert every token
routes to and of the shared expert, plus a down block of scale 65504 with one weight
+65504; the layer output is checked against the oracle in fp64 as every other layer is.
Where the 65504 scale sits decides what the kernel's int16 activation codes (error up to
half a code, 2^-16 of the block's largest |value|) can carry within 2e-3 x RMS(y): in an
up row it scales one activation that then reaches every output, so the error stays a
small fraction of RMS(y); a down row full of +-65504 weights would multiply the code
error of a whole normal block into a single output and exceed the bar, so that row has
one such weight."""
import os

import numpy as np
import pytest

import oracle
import synthetic
from helpers import LAYER_TOL, build_gpu, make_layers

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

DEV = "cuda:0"
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "q4_0_blocks.txt")

SHAPE = synthetic.Shape(n_layers=3, hidden=512, n_experts=64, top_k=4, inter=256, shared_inter=256,
                        ring_slots=2, use_rmsnorm=1, zipf_s=1.0)


def _golden_blocks():
    out = []
    with open(GOLDEN) as f:
        for line in f:
            if line.startswith("block"):
                out.append(np.frombuffer(bytes.fromhex("".join(line.split()[1:])), np.uint8))
    return out


def _tie_layers():
    s = SHAPE
    layers = make_layers(s, gain_kind="random")
    E, H = s.n_experts, s.hidden
    # layer 0: zero router; ties at the 4th place: 5 (2.0), 0 (1.0), then 9, 12, 30 at 0.5
    layers[0].router = np.zeros((E, H), np.uint16)
    b = np.zeros(E, np.float32)
    b[5], b[0], b[9], b[12], b[30] = 2.0, 1.0, 0.5, 0.5, 0.5
    layers[0].bias = b
    # layer 1: zero router; 7, 2, 50 above, the rest tied at zero with mixed signs
    layers[1].router = np.zeros((E, H), np.uint16)
    b = np.full(E, -0.0, np.float32)
    b[1::3] = 0.0
    b[7], b[2], b[50] = 3.0, 2.0, 1.0
    layers[1].bias = b
    # layer 2: rows 23 and 11 identical with the same large bias
    r = layers[2].router.copy()
    r[23] = r[11]
    layers[2].router = r
    b = layers[2].bias.copy()
    b[11] = b[23] = 6.0
    layers[2].bias = b
    return layers


def _decode_traced(m, xs):
    s = m.shape
    ht = torch.zeros((s.n_layers + 1, s.hidden), dtype=torch.float32, device=DEV)
    wt = torch.zeros((s.n_layers, s.top_k), dtype=torch.float32, device=DEV)
    m.set_trace(ht, wt)
    hs, ws = [], []
    for x in xs:
        m.decode(torch.from_numpy(x).to(DEV))
        m.sync()
        hs.append(ht.cpu().numpy().copy())
        ws.append(wt.cpu().numpy().copy())
    m.set_trace(None, None)
    _, _, log = m.stats(log_cap=len(xs) * s.n_layers * s.top_k, reset=True)
    return np.stack(hs), np.stack(ws), log["expert"].reshape(len(xs), s.n_layers, s.top_k)


def _check_layer(orc, l, h_in, h_out, sel, w=None):
    ref = orc.layer(l, h_in)
    assert np.array_equal(ref["sel"], sel), (l, ref["sel"], sel)
    if w is not None:
        assert np.allclose(w, ref["w"], rtol=2e-6, atol=1e-7), l
    err = np.max(np.abs(h_out.astype(np.float64) - ref["h_out"]))
    rms = np.sqrt(np.mean(ref["y"] ** 2))
    assert err <= LAYER_TOL * rms, (l, err / rms)


def test_ties_decode_and_prefill():
    s = SHAPE
    layers = _tie_layers()
    orc = oracle.Model(s, layers)
    m = build_gpu(s, layers)
    m.set_residency(1.0)
    xs = synthetic.tokens(21, 3, s.hidden)
    hs, ws, sels = _decode_traced(m, xs)
    for t in range(len(xs)):
        assert list(sels[t, 0]) == [5, 0, 9, 12]
        assert list(sels[t, 1]) == [7, 2, 50, 0]
        row = list(sels[t, 2])
        assert 11 in row and 23 in row and row.index(11) < row.index(23), row
        for l in range(s.n_layers):
            _check_layer(orc, l, hs[t, l], hs[t, l + 1], sels[t, l], ws[t, l])

    T = 40
    xp = synthetic.tokens(300, T, s.hidden)
    hp = torch.zeros((s.n_layers + 1, T, s.hidden), dtype=torch.float32, device=DEV)
    sp = torch.full((s.n_layers, T, s.top_k), -1, dtype=torch.int32, device=DEV)
    m.set_prefill_trace(hp, sp)
    m.prefill(torch.from_numpy(xp).to(DEV))
    m.sync()
    m.set_prefill_trace(None, None)
    h, sel = hp.cpu().numpy(), sp.cpu().numpy()
    assert np.all(sel[0] == np.array([5, 0, 9, 12]))
    assert np.all(sel[1] == np.array([7, 2, 50, 0]))
    for t in range(T):
        row = list(sel[2, t])
        assert 11 in row and 23 in row and row.index(11) < row.index(23), (t, row)
        for l in range(s.n_layers):
            ref = orc.layer(l, h[l, t])
            assert np.array_equal(ref["sel"], sel[l, t]), (l, t)
    for t in (0, T - 1):
        for l in range(s.n_layers):
            _check_layer(orc, l, h[l, t], h[l + 1, t], sel[l, t])
    m.close()


def _put_block(q4, byte_off, blk):
    q4[byte_off:byte_off + 18] = blk


def test_extreme_q4_0_scales_through_the_kernel():
    s = synthetic.Shape(n_layers=1, hidden=512, n_experts=64, top_k=4, inter=256, shared_inter=256,
                        ring_slots=2, use_rmsnorm=1, zipf_s=1.0)
    layers = make_layers(s)
    lw = layers[0]
    H, I = s.hidden, s.inter
    nb, nbd = H // 32, I // 32
    g = _golden_blocks()
    sub, big = g[3], g[4]  # d = 2^-24 (q 15 / 9) and d = 65504 (q 0: weights -524032)
    assert sub[0] == 0x01 and sub[1] == 0x00 and big[0] == 0xFF and big[1] == 0x7B
    one = big.copy()
    one[2:] = np.uint8(0x88)  # d = 65504, every weight 0 ...
    one[2] = np.uint8(0x89)   # ... but weight 0: +65504
    hot = 17
    lw.bias = lw.bias.copy()
    lw.bias[hot] = 8.0  # every token routes to it
    gu = I * nb * 18
    lw.experts[hot] = lw.experts[hot].copy()
    lw.shared = lw.shared.copy()
    for q4 in (lw.experts[hot], lw.shared):  # canonical gate | up | down blocks
        _put_block(q4, (3 * nb + 1) * 18, sub)                # gate row 3, block 1
        _put_block(q4, gu + (40 * nb + 2) * 18, sub)          # up row 40, block 2
        _put_block(q4, gu + (41 * nb + 0) * 18, big)          # up row 41, block 0: |u| ~ 1e6
        _put_block(q4, 2 * gu + (100 * nbd + 3) * 18, one)    # down row 100, block 3 (rows 96..127)
        _put_block(q4, 2 * gu + (7 * nbd + 1) * 18, sub)      # down row 7, block 1
    orc = oracle.Model(s, layers)
    m = build_gpu(s, layers)
    m.set_residency(1.0)
    xs = synthetic.tokens(77, 3, s.hidden)
    hs, ws, sels = _decode_traced(m, xs)
    for t in range(len(xs)):
        assert hot in sels[t, 0]
        assert np.all(np.isfinite(hs[t]))
        _check_layer(orc, 0, hs[t, 0], hs[t, 1], sels[t, 0], ws[t, 0])
    m.sync()
    m.close()
