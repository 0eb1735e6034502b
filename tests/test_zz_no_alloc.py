"""The allocation-free decode entry point against the regular one.

moe_decode_step_noalloc serves callers that cannot allocate device memory (a fixed
memory budget or their own allocator, a stream-capture region, a real-time path): it
keeps its scratch in a static device array and takes every weight resident in device
memory the caller owns.  These tests pack the weights into the library's documented
slot layout themselves (a byte regrouping done here with numpy), call the entry point
twice in a row, and check each output against moe_decode_step's on the same token,
within the per-layer tolerance the parity tests use (the two share one kernel, so the
results are expected to be equal bit for bit).  The file sits last in collection order
so that a run stopping at the first failure has already run every other test.
"""
import numpy as np
import pytest

import synthetic
from helpers import LAYER_TOL, build_gpu, make_layers

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _slot_bytes(H, W):
    return ((W // 32) * 54 * H + 255) // 256 * 256


def _tiles(rows):
    """[n, 16, nb, 18] canonical blocks -> [n, 16*nb*16 nibble bytes + 16*nb*2 scale bytes]."""
    n = rows.shape[0]
    return np.concatenate([rows[..., 2:].reshape(n, -1), rows[..., :2].reshape(n, -1)], axis=1)


def _pack_expert(q4, H, W):
    """Canonical gate | up | down of width W -> W/32 units of 54 H bytes each."""
    nb, nbd = H // 32, W // 32
    n_gu = W * nb * 18
    gate = q4[:n_gu].reshape(nbd, 2, 16, nb, 18)
    up = q4[n_gu:2 * n_gu].reshape(nbd, 2, 16, nb, 18)
    down = q4[2 * n_gu:].reshape(H, nbd, 18)
    gu = np.stack([_tiles(gate[:, 0]), _tiles(gate[:, 1]), _tiles(up[:, 0]), _tiles(up[:, 1])], axis=1)
    dn = down[:, :, 2:].transpose(1, 0, 2).reshape(nbd, 16 * H)
    ds = down[:, :, :2].transpose(1, 0, 2).reshape(nbd, 2 * H)
    body = np.concatenate([gu.reshape(nbd, 36 * H), dn, ds], axis=1).reshape(-1)
    out = np.zeros(_slot_bytes(H, W), np.uint8)
    out[: body.size] = body
    return out


def _reference(s, layers, xs):
    ref = build_gpu(s, layers)
    ref.set_residency(1.0)
    ys = [ref.decode(torch.from_numpy(x).to(DEV)).cpu().numpy() for x in xs]
    ref.sync()
    ref.close()
    return ys


def _noalloc_weights(moe, s, layers):
    experts = torch.from_numpy(np.concatenate(
        [_pack_expert(e, s.hidden, s.inter) for lw in layers for e in lw.experts])).to(DEV)
    shared = None if s.shared_inter == 0 else torch.from_numpy(np.concatenate(
        [_pack_expert(lw.shared, s.hidden, s.shared_inter) for lw in layers])).to(DEV)
    router = torch.from_numpy(np.concatenate([lw.router.reshape(-1) for lw in layers]).view(np.int16)).to(DEV)
    bias = torch.from_numpy(np.concatenate([lw.bias for lw in layers])).to(DEV)
    gain = torch.from_numpy(np.concatenate([lw.gain for lw in layers])).to(DEV)
    keep = (experts, shared, router, bias, gain)  # the caller owns the device memory
    w = moe.NoAllocWeights(experts.data_ptr(), None if shared is None else shared.data_ptr(), router.data_ptr(),
                           bias.data_ptr(), gain.data_ptr())
    cfg = moe.Config(s.n_layers, s.hidden, s.n_experts, s.top_k, s.inter, s.shared_inter, s.ring_slots,
                     s.use_rmsnorm, s.rms_eps, 0, 0, 0)
    return cfg, w, keep


def _check_calls(moe, s, layers, xs, y_ref):
    cfg, w, keep = _noalloc_weights(moe, s, layers)
    stream = torch.cuda.current_stream().cuda_stream
    for t, x in enumerate(xs):  # calls in a row share the static scratch
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
    del keep


def test_noalloc_entry_point_matches_decode_step():
    import expert_cache_host_router_b200 as moe
    s = synthetic.Shape(n_layers=3, hidden=1024, n_experts=64, top_k=6, inter=256, shared_inter=256,
                        ring_slots=4, use_rmsnorm=1, zipf_s=1.0)
    layers = make_layers(s, gain_kind="random")
    xs = synthetic.tokens(5, 2, s.hidden)
    _check_calls(moe, s, layers, xs, _reference(s, layers, xs))


def test_noalloc_shapes_of_different_kernel_instances_in_a_row():
    """hidden 2048 then hidden 1024 (two kernel instances), then hidden 1024 again after
    a context of a smaller shape was created: every call must launch and match."""
    import expert_cache_host_router_b200 as moe
    big = synthetic.Shape(n_layers=2, hidden=2048, n_experts=32, top_k=4, inter=256, shared_inter=256,
                          ring_slots=2, use_rmsnorm=1, zipf_s=1.0)
    small = synthetic.Shape(n_layers=2, hidden=1024, n_experts=64, top_k=6, inter=256, shared_inter=0,
                            ring_slots=2, use_rmsnorm=1, zipf_s=1.0)
    xb = synthetic.tokens(11, 2, big.hidden)
    xsm = synthetic.tokens(12, 2, small.hidden)
    lb = make_layers(big, gain_kind="random")
    ls = make_layers(small, gain_kind="random")
    yb, ys = _reference(big, lb, xb), _reference(small, ls, xsm)
    _check_calls(moe, big, lb, xb, yb)
    _check_calls(moe, small, ls, xsm, ys)
    tiny = synthetic.Shape(n_layers=1, hidden=256, n_experts=16, top_k=2, inter=64, shared_inter=0,
                           ring_slots=2, use_rmsnorm=1, zipf_s=1.0)
    ctx = build_gpu(tiny, make_layers(tiny))
    _check_calls(moe, small, ls, xsm, ys)
    ctx.close()


def test_noalloc_rejects_oversized_shapes():
    """A shape whose scratch does not fit the static array is refused before anything
    is launched; real (small) device buffers are passed all the same."""
    import expert_cache_host_router_b200 as moe
    buf = torch.zeros(4096, dtype=torch.float32, device=DEV)
    p = buf.data_ptr()
    cfg = moe.Config(512, 4096, 1024, 8, 512, 0, 0, 1, 1e-6, 0, 0, 0)  # 2 MiB of slot tables alone
    w = moe.NoAllocWeights(p, None, p, None, None)
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_decode_step_noalloc(cfg, w, p, p, 0)
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED
    torch.cuda.synchronize()
