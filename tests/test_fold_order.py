"""The prefill router evaluates the canonical fold (32 lane sums combined by the xor
butterfly 16, 8, 4, 2, 1) as four residue subtrees (lanes r, r+4, ... combined in
bit-reversed order by a 3-deep binary counter) followed by two shuffle levels.  In fp32
that must give the butterfly's lane-0 value bit for bit for any inputs: this checks the
restated order on the CPU (no GPU needed)."""
import numpy as np

f32 = np.float32


def butterfly(lanes):
    v = lanes.astype(np.float32).copy()
    for off in (16, 8, 4, 2, 1):
        v = (v + v[np.arange(32) ^ off]).astype(np.float32)
    return v


def residue_then_shuffles(lanes):
    def brev3(i):
        return int(f"{i:03b}"[::-1], 2)

    cr = []
    for r in range(4):
        stk, out = [None] * 3, None
        for i in range(8):
            v, carry = f32(lanes[r + 4 * brev3(i)]), True
            for b in range(3):
                if not carry:
                    break
                if (i >> b) & 1:
                    v = f32(stk[b] + v)
                else:
                    stk[b], carry = v, False
            if carry:
                out = v
        cr.append(out)
    c2 = [f32(cr[r] + cr[r ^ 2]) for r in range(4)]
    return [f32(c2[r] + c2[r ^ 1]) for r in range(4)]


def test_residue_fold_equals_butterfly():
    rng = np.random.default_rng(20261202)
    for _ in range(3000):
        lanes = (rng.standard_normal(32) * 10.0 ** rng.integers(-4, 5, 32)).astype(np.float32)
        ref = butterfly(lanes)
        got = residue_then_shuffles(lanes)
        assert all(np.float32(g).view(np.uint32) == ref[r].view(np.uint32) for r, g in enumerate(got))


def test_residue_fold_with_empty_lanes():
    """hidden < 512: lanes without chunks hold +0 and must not change the order."""
    rng = np.random.default_rng(7)
    for n in (8, 16, 24):
        lanes = np.zeros(32, np.float32)
        lanes[:n] = rng.standard_normal(n).astype(np.float32)
        assert residue_then_shuffles(lanes)[0].view(np.uint32) == butterfly(lanes)[0].view(np.uint32)
