"""The seeded synthetic inputs have the stated recipe: Q4_0 nibbles uniform over 0..15 and
scales fp16(0.0043 * U(0.5, 1.5)) (weight RMS 0.0043 * sqrt(13/12) * sqrt(21.5) = 0.0208);
router weights N(0, 0.02) rounded to nearest-even bf16; router bias s * ln p with Zipf(1)
popularity over a seeded permutation; tokens N(0, 1); everything reproducible from its
seeds."""
import numpy as np

import oracle
import synthetic


def test_q4_0_nibbles_scales_and_weight_rms():
    m = synthetic.q4_0_matrix(3, 5, synthetic.MAT_UP, 512, 2048)
    blocks = m.reshape(-1, 18)
    qs = blocks[:, 2:]
    nib = np.concatenate([(qs & 15).ravel(), (qs >> 4).ravel()])
    freq = np.bincount(nib, minlength=16) / nib.size
    assert np.all(np.abs(freq - 1 / 16) < 0.002)
    d = blocks[:, :2].copy().view(np.float16).astype(np.float64).ravel()
    assert d.min() >= float(np.float16(0.0043 * 0.5)) and d.max() <= float(np.float16(0.0043 * 1.5))
    w = oracle.dequant_q4_0(m)
    rms_expected = 0.0043 * np.sqrt(13 / 12) * np.sqrt(21.5)
    assert abs(np.sqrt(np.mean(w ** 2)) / rms_expected - 1) < 0.01


def test_router_weights_are_rounded_gaussians():
    bits = synthetic.router_bf16(2, 256, 2048)
    w = (bits.astype(np.uint32) << 16).view(np.float32)
    assert abs(w.std() / 0.02 - 1) < 0.01 and abs(w.mean()) < 2e-4
    # nearest-even rounding of the fp32 draw: re-derive a few from the same stream
    raw = synthetic._stream(synthetic.SEED_ROUTER, 2).standard_normal(8, dtype=np.float32) * np.float32(0.02)
    for x, b in zip(raw, bits.ravel()[:8]):
        lo = np.float32((np.uint32(x.view(np.uint32)) >> 16 << 16).view(np.float32))
        hi = np.float32(np.uint32((int(x.view(np.uint32)) >> 16) + 1 << 16).view(np.float32))
        got = np.uint32(int(b) << 16).view(np.float32)
        assert got in (lo, hi)
        assert abs(float(got) - float(x)) <= abs(float(lo if got == hi else hi) - float(x))


def test_zipf_bias_is_log_popularity():
    E = 256
    b = synthetic.zipf_bias(4, E, 1.0).astype(np.float64)
    perm = synthetic.zipf_perm(4, E)
    assert abs(np.exp(b).sum() - 1.0) < 1e-5  # p_e sums to one
    ranks = np.empty(E, np.int64)
    ranks[perm] = np.arange(1, E + 1)
    assert np.allclose(b - b[perm[0]], -np.log(ranks), atol=1e-5)  # b_e - b_top = -ln rank
    assert np.array_equal(synthetic.zipf_bias(4, E, 0.0), np.zeros(E, np.float32))
    assert np.allclose(synthetic.zipf_bias(4, E, 0.5), 0.5 * b, atol=1e-6)


def test_tokens_and_weights_are_reproducible():
    assert np.array_equal(synthetic.tokens(10, 3, 512), synthetic.tokens(10, 3, 512))
    x = synthetic.tokens(0, 64, 2048)
    assert abs(x.std() - 1) < 0.01 and abs(x.mean()) < 0.01
    assert not np.array_equal(x[0], x[1])
    a = synthetic.expert_q4_0(1, 2, 512, 256)
    assert np.array_equal(a, synthetic.expert_q4_0(1, 2, 512, 256))
    assert not np.array_equal(a, synthetic.expert_q4_0(1, 3, 512, 256))
