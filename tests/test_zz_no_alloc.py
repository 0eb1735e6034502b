"""The allocation-free decode entry point against the regular one.

moe_decode_step_noalloc serves callers that cannot allocate device memory (a fixed
memory budget or their own allocator, a stream-capture region, a real-time path): it
keeps its scratch in a static device array and takes every weight resident in device
memory the caller owns.  This test packs the weights into the library's documented
slot layout itself (a byte regrouping done here with numpy), calls the entry point twice
in a row, and checks each output against moe_decode_step's on the same token, within
the per-layer tolerance the parity tests use (the two share one kernel, so the results
are expected to be equal bit for bit).  It sits last in collection order so that a run
stopping at the first failure has already run every other test.
"""
import numpy as np
import pytest

import synthetic
from helpers import LAYER_TOL, build_gpu, make_layers

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _slot_bytes(H, W):
    return (3 * H * W * 9 // 16 + 255) // 256 * 256


def _tiles(rows):
    """[n, 16, nb, 18] canonical blocks -> [n, 16*nb*16 nibble bytes + 16*nb*2 scale bytes]."""
    n = rows.shape[0]
    return np.concatenate([rows[..., 2:].reshape(n, -1), rows[..., :2].reshape(n, -1)], axis=1)


def _pack_expert(q4, H, W):
    nb, nbd = H // 32, W // 32
    n_gu = W * nb * 18
    gate = q4[:n_gu].reshape(W // 32, 2, 16, nb, 18)
    up = q4[n_gu:2 * n_gu].reshape(W // 32, 2, 16, nb, 18)
    down = q4[2 * n_gu:].reshape(H // 16, 16, nbd, 18)
    gu = np.stack([_tiles(gate[:, 0]), _tiles(gate[:, 1]), _tiles(up[:, 0]), _tiles(up[:, 1])], axis=1)
    out = np.zeros(_slot_bytes(H, W), np.uint8)
    body = np.concatenate([gu.reshape(-1), _tiles(down).reshape(-1)])
    out[: body.size] = body
    return out


def _pack_router(w, H):
    E = w.shape[0]
    return np.ascontiguousarray(w.reshape(E, H // 16, 16).transpose(1, 0, 2))


def test_noalloc_entry_point_matches_decode_step():
    import expert_cache_host_router_b200 as moe
    s = synthetic.Shape(n_layers=3, hidden=1024, n_experts=64, top_k=6, inter=256, shared_inter=256,
                        ring_slots=4, use_rmsnorm=1, zipf_s=1.0)
    layers = make_layers(s, gain_kind="random")
    xs = synthetic.tokens(5, 2, s.hidden)

    ref = build_gpu(s, layers)
    ref.set_residency(1.0)
    y_ref = []
    for x in xs:
        y_ref.append(ref.decode(torch.from_numpy(x).to(DEV)).cpu().numpy())
    ref.sync()
    ref.close()

    experts = torch.from_numpy(np.concatenate(
        [_pack_expert(e, s.hidden, s.inter) for lw in layers for e in lw.experts])).to(DEV)
    shared = torch.from_numpy(np.concatenate(
        [_pack_expert(lw.shared, s.hidden, s.shared_inter) for lw in layers])).to(DEV)
    router = torch.from_numpy(np.concatenate(
        [_pack_router(lw.router, s.hidden).reshape(-1) for lw in layers]).view(np.int16)).to(DEV)
    bias = torch.from_numpy(np.concatenate([lw.bias for lw in layers])).to(DEV)
    gain = torch.from_numpy(np.concatenate([lw.gain for lw in layers])).to(DEV)
    cfg = moe.Config(s.n_layers, s.hidden, s.n_experts, s.top_k, s.inter, s.shared_inter, s.ring_slots,
                     s.use_rmsnorm, s.rms_eps, 0, 0, 0)
    w = moe.NoAllocWeights(experts.data_ptr(), shared.data_ptr(), router.data_ptr(), bias.data_ptr(),
                           gain.data_ptr())
    stream = torch.cuda.current_stream().cuda_stream
    for t, x in enumerate(xs):  # two calls in a row share the static scratch
        xd = torch.from_numpy(x).to(DEV)
        y = torch.full_like(xd, float("nan"))
        moe.moe_decode_step_noalloc(cfg, w, xd.data_ptr(), y.data_ptr(), stream)
        torch.cuda.synchronize()
        got = y.cpu().numpy().astype(np.float64)
        want = y_ref[t].astype(np.float64)
        delta = want - xs[t]  # the stack's update; its RMS sets the scale of the tolerance
        rms = float(np.sqrt(np.mean(delta ** 2)))
        assert np.max(np.abs(got - want)) <= LAYER_TOL * rms, t
        assert np.array_equal(got, want), t


def test_noalloc_rejects_oversized_shapes():
    import expert_cache_host_router_b200 as moe
    cfg = moe.Config(64, 4096, 1024, 8, 512, 0, 0, 1, 1e-6, 0, 0, 0)
    w = moe.NoAllocWeights(16, None, 16, None, None)  # never dereferenced: rejected first
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_decode_step_noalloc(cfg, w, 16, 16, 0)
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED
