"""Parity of the batched prefill (moe_prefill, tcgen05 grouped GEMM) with the CPU oracle.

Bars: every token's top-k choices bit-exact at every layer (teacher-forced: the oracle
routes the GPU's own fp32 input of the layer); every layer's output within 2e-3 x the
RMS of the MoE output, element by element; the end of a free-running stack within 1e-2
relative; the routing histogram equal to the counts of the choices; results
independent of the batch a token is prefilled in (bit for bit)."""
import numpy as np
import pytest

import oracle
import synthetic
from helpers import LAYER_TOL, STACK_TOL, build_gpu, make_layers

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _prefill(m, xs, trace=False):
    s = m.shape
    x = torch.from_numpy(np.ascontiguousarray(xs, dtype=np.float32)).to(DEV)
    ht = st = None
    if trace:
        ht = torch.zeros((s.n_layers + 1, len(xs), s.hidden), dtype=torch.float32, device=DEV)
        st = torch.full((s.n_layers, len(xs), s.top_k), -1, dtype=torch.int32, device=DEV)
        m.set_prefill_trace(ht, st)
    y = m.prefill(x)
    m.sync()
    if trace:
        m.set_prefill_trace(None, None)
        return y.cpu().numpy(), ht.cpu().numpy(), st.cpu().numpy()
    return y.cpu().numpy(), None, None


def _oracle_sel(shape, lw, h32):
    """Top-k of one layer on fp32 input h32, from the oracle's routing functions."""
    if shape.use_rmsnorm:
        inv, gain = oracle.rms_inv(h32, shape.rms_eps), lw.gain
    else:
        inv, gain = np.float32(1.0), None
    z = oracle.router_logits(lw.router, h32, gain, inv, lw.bias)
    return oracle.topk(z, shape.top_k)


def _check_layers(shape, layers, xs, hs, sels, sample):
    """Routing of every token at every layer; outputs of the sampled tokens."""
    orc = oracle.Model(shape, layers)
    assert np.array_equal(hs[0], xs)
    for l in range(shape.n_layers):
        for t in range(len(xs)):
            ref = _oracle_sel(shape, layers[l], hs[l, t])
            assert np.array_equal(ref, sels[l, t]), (l, t, ref, sels[l, t])
        for t in sample:
            ref = orc.layer(l, hs[l, t])
            assert np.array_equal(ref["sel"], sels[l, t])
            err = np.max(np.abs(hs[l + 1, t].astype(np.float64) - ref["h_out"]))
            rms = np.sqrt(np.mean(ref["y"] ** 2))
            assert err <= LAYER_TOL * rms, (l, t, err / rms)


def test_prefill_small_layer():
    """1 layer, hidden 512, 64 experts, top-4, SwiGLU 256, no shared; 300 tokens (ragged)."""
    s = synthetic.SMALL
    layers = make_layers(s)
    m = build_gpu(s, layers)
    m.set_residency(1.0)
    xs = synthetic.tokens(0, 300, s.hidden)
    y, hs, sels = _prefill(m, xs, trace=True)
    assert np.array_equal(y, hs[-1])
    _check_layers(s, layers, xs, hs, sels, sample=range(0, 300, 7))
    _, hist, _ = m.stats()
    assert np.array_equal(hist[0], np.bincount(sels[0].reshape(-1), minlength=s.n_experts))
    m.close()


STACK = synthetic.Shape(n_layers=3, hidden=512, n_experts=64, top_k=8, inter=512, shared_inter=256,
                        use_rmsnorm=1, zipf_s=1.0)


def test_prefill_stack_teacher_forced_and_free_running():
    """3-layer pre-norm stack with a narrower shared expert and Zipf routing (experts with
    several 128-row tiles next to experts with none), 333 tokens."""
    s = STACK
    layers = make_layers(s, gain_kind="random")
    m = build_gpu(s, layers)
    m.set_residency(1.0)
    xs = synthetic.tokens(0, 333, s.hidden)
    y, hs, sels = _prefill(m, xs, trace=True)
    counts = np.bincount(sels[0].reshape(-1), minlength=s.n_experts)
    assert counts.max() > 128 and (counts == 0).any()  # multi-tile and empty experts both occur
    _check_layers(s, layers, xs, hs, sels, sample=list(range(0, 333, 11)) + [332])
    orc = oracle.Model(s, layers)
    for t in (0, 100, 332):
        h_ref, _, _ = orc.decode(xs[t])
        rel = np.linalg.norm(y[t] - h_ref) / np.linalg.norm(h_ref)
        assert rel <= STACK_TOL, (t, rel)
    # the first layer's routing agrees with decode's on the same input
    m.set_residency(1.0)
    m.stats(reset=True)
    for t in range(4):
        m.decode(torch.from_numpy(xs[t]).to(DEV))
    m.sync()
    _, _, log = m.stats(log_cap=4 * s.n_layers * s.top_k)
    dsel = log["expert"].reshape(4, s.n_layers, s.top_k)
    assert np.array_equal(dsel[:, 0], sels[0, :4])
    m.close()


def test_prefill_full_shape_layer():
    """hidden 2048, 256 experts, top-8, 512 + shared 512, Zipf router; 2048 tokens: every
    token's routing, sampled tokens' outputs, the histogram."""
    s = synthetic.FULL_LAYER
    layers = make_layers(s)
    m = build_gpu(s, layers)
    m.set_residency(1.0)
    m.stats(reset=True)
    xs = synthetic.tokens(1000, 2048, s.hidden)
    y, hs, sels = _prefill(m, xs, trace=True)
    _check_layers(s, layers, xs, hs, sels, sample=[0, 1, 517, 1024, 1500, 2046, 2047])
    _, hist, _ = m.stats()
    assert np.array_equal(hist[0], np.bincount(sels[0].reshape(-1), minlength=s.n_experts))
    m.close()


def test_prefill_batch_independent_and_repeatable():
    """A token's result does not depend on the batch it is prefilled in, nor on the run."""
    s = STACK
    layers = make_layers(s, gain_kind="random")
    m = build_gpu(s, layers)
    m.set_residency(1.0)
    xs = synthetic.tokens(50, 257, s.hidden)
    y_all, _, _ = _prefill(m, xs)
    y_again, _, _ = _prefill(m, xs)
    assert np.array_equal(y_all.view(np.uint32), y_again.view(np.uint32))
    for n in (1, 17, 130):
        y_n, _, _ = _prefill(m, xs[:n])
        assert np.array_equal(y_n.view(np.uint32), y_all[:n].view(np.uint32)), n
    m.close()


def test_prefill_needs_full_residency_and_supported_shape():
    import expert_cache_host_router_b200 as moe
    s = synthetic.Shape(n_layers=1, hidden=512, n_experts=64, top_k=4, inter=256, shared_inter=0,
                        ring_slots=4)
    m = build_gpu(s, make_layers(s))
    x = torch.zeros((4, s.hidden), dtype=torch.float32, device=DEV)
    with pytest.raises(moe.MoEError) as ei:
        m.prefill(x)  # no residency set yet
    assert ei.value.status == moe.MOE_ERR_STATE
    m.set_residency(0.5)
    with pytest.raises(moe.MoEError) as ei:
        m.prefill(x)
    assert ei.value.status == moe.MOE_ERR_STATE
    m.close()
    s2 = synthetic.Shape(n_layers=1, hidden=96, n_experts=16, top_k=2, inter=64, shared_inter=0)
    m2 = build_gpu(s2, make_layers(s2))
    m2.set_residency(1.0)
    with pytest.raises(moe.MoEError) as ei:
        m2.prefill(torch.zeros((2, s2.hidden), dtype=torch.float32, device=DEV))
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED
    m2.close()


@pytest.mark.parametrize("shape", [
    # two router tiles of 256 experts; shared expert as wide as the routed ones
    synthetic.Shape(n_layers=1, hidden=512, n_experts=512, top_k=8, inter=256, shared_inter=256,
                    use_rmsnorm=1, zipf_s=1.0),
    # hidden 256: fold lanes 16..31 hold no chunk; top-1 routing; 32 experts (N = 32 router tile)
    synthetic.Shape(n_layers=2, hidden=256, n_experts=32, top_k=1, inter=256, shared_inter=0,
                    use_rmsnorm=1, zipf_s=0.5),
])
def test_prefill_other_shapes(shape):
    layers = make_layers(shape, gain_kind="random")
    m = build_gpu(shape, layers)
    m.set_residency(1.0)
    xs = synthetic.tokens(3, 200, shape.hidden)
    y, hs, sels = _prefill(m, xs, trace=True)
    assert np.array_equal(y, hs[-1])
    _check_layers(shape, layers, xs, hs, sels, sample=[0, 1, 99, 130, 199])
    m.close()
