"""The prefill router's candidate rule, restated on the CPU (no GPU needed).

The kernel knows approximate logits z~ with |z~ - z| <= delta / 2 (delta is twice its
error bound) and takes as candidates the k best approximate logits plus every expert with
z~ >= z~(k) - 2 delta, then ranks the candidates by their exact logits.  This checks that
the resulting top-k always equals the exact top-k (larger first, equal -> lower index),
with errors drawn up to the bound, pushed to the bound against the order, and with ties."""
import numpy as np


def topk_exact(z, k):
    order = sorted(range(len(z)), key=lambda e: (-z[e], e))
    return order[:k]


def select(z, za, k, delta):
    a = sorted(range(len(za)), key=lambda e: (-za[e], e))[:k]
    thr = np.float32(za[a[-1]] - np.float32(2.0) * np.float32(delta))
    cand = set(a) | {e for e in range(len(za)) if za[e] >= thr}
    return sorted(cand, key=lambda e: (-z[e], e))[:k], len(cand)


def test_candidate_rule_random_errors_within_bound():
    rng = np.random.default_rng(11)
    for trial in range(3000):
        E = int(rng.choice([16, 32, 64, 256]))
        k = int(rng.integers(1, min(E, 9)))
        delta = np.float32(10.0 ** rng.uniform(-3, -0.5))
        z = (rng.standard_normal(E) + np.log(1.0 / np.arange(1, E + 1)) * rng.uniform(0, 1)).astype(np.float32)
        if trial % 5 == 0:  # ties and near-ties
            z[rng.integers(0, E, E // 4)] = z[rng.integers(0, E)]
        err = (rng.uniform(-0.5, 0.5, E) * delta).astype(np.float32)
        za = (z + err).astype(np.float32)
        got, _ = select(z, za, k, delta)
        assert got == topk_exact(z, k)


def test_candidate_rule_adversarial_errors_at_the_bound():
    """Errors at +-delta/2 pushed against the exact order: the experts just outside the
    exact top-k look better, the top-k ones look worse."""
    rng = np.random.default_rng(12)
    for trial in range(2000):
        E, k = 64, 8
        delta = np.float32(0.05)
        z = np.sort(rng.standard_normal(E).astype(np.float32))[::-1].copy()
        z[k:k + 3] = z[k - 1] - np.float32(rng.uniform(0, 2.5)) * delta  # crowd the boundary
        exact = topk_exact(z, k)
        za = z.copy()
        for e in range(E):
            za[e] = z[e] - delta / 2 if e in exact else z[e] + delta / 2
        got, n = select(z, za, k, delta)
        assert got == exact
        assert n >= k


def test_candidate_set_is_small_when_logits_are_spread():
    rng = np.random.default_rng(13)
    sizes = []
    for _ in range(500):
        z = (rng.standard_normal(256) * 0.9 + np.log(1.0 / np.arange(1, 257))).astype(np.float32)
        za = (z + rng.uniform(-1e-5, 1e-5, 256)).astype(np.float32)
        _, n = select(z, za, 8, np.float32(0.08))
        sizes.append(n)
    assert np.mean(sizes) < 12  # about k + 2 at the bound the kernel uses for this shape
