"""Exact ties of router logits on the GPU: the lowest expert index wins.

The top-K selection orders experts by router probability descending and breaks
exact ties towards the lower expert index (the softmax-then-top-K routing of
intelliparadigm.com, section 2.1, router snippet, and tinai-dev README, "Pipeline
mỗi lớp"; the tie rule is the oracle's sort-based definition).  Every case here
builds logits that tie exactly -- in the fp64 sums of both the GPU and the oracle
-- and checks the single-token routing (fmoe_route), the whole layer
(fmoe_layer_forward) and the batched routing (fmoe_route_batched) against the
oracle's order, bit for bit.

The ties are placed so that both levels of the GPU's rank selection decide them:
experts 5 (group 0 of 32), 33 and 40 (group 1) tie for the top, and experts 31
(group 0), 32 and 50 (group 1) tie across the K/K+1 boundary.
"""
import numpy as np
import pytest
import torch

import fmoe_synth as synth
import oracle
from _ties import index_mismatch

pytestmark = pytest.mark.gpu

TOP = (5, 33, 40)
NEXT = (31, 32, 50)


def _bf(t):
    return oracle.bf16_to_f64(t.view(torch.int16).cpu().numpy().view(np.uint16))


def _layer(fm, shape, seed, router, rbias):
    """Device layer with the generator's expert records and shared gate, and the
    given router (fp32 [E, H]) and router bias (fp32 [E] or None); plus the oracle
    layer over the same inputs."""
    from fmoe_synth.torch_layer import make_device_layer
    w = make_device_layer(shape, seed, 0)
    w.router.copy_(torch.from_numpy(router))
    if rbias is not None:
        w.router_bias.copy_(torch.from_numpy(rbias))
    cfg = fm.fmoe_config(shape.hidden, shape.inter, shape.n_experts, shape.top_k, shape.bits,
                         shape.has_shared, shape.router_bias)
    L = fm.Layer.create(cfg, w.experts, w.router, w.router_bias, w.shared_gate)
    olay = oracle.OracleLayer(shape.hidden, shape.inter, shape.n_experts, shape.top_k, shape.bits,
                              synth.gen_layer_records(seed, 0, shape), router,
                              synth.gen_shared_gate(seed, 0, shape.hidden), rbias,
                              has_shared=bool(shape.has_shared))
    return w, L, olay


def _check(fm, L, olay, x, want_first=None):
    T = x.shape[0]
    idx, wts, sig = L.route(x)
    y = torch.empty_like(x)
    for t in range(T):
        fm.fmoe_layer_forward(L.handle, x[t:t + 1], x[t:t + 1], 1, y[t:t + 1])
    L.attach_batch(T)
    ib, wb, sb = L.route_batched(x)
    torch.cuda.synchronize()
    assert L.error() == 0
    xs, ys = _bf(x), _bf(y)
    idx, ib = idx.cpu().numpy(), ib.cpu().numpy()
    for t in range(T):
        r = olay.forward(xs[t])
        if t == 0 and want_first is not None:
            assert list(r.idx) == list(want_first), "the oracle's own tie order"
        assert list(idx[t]) == list(r.idx), index_mismatch(f"fmoe_route token {t}", idx[t], r.idx, r.logits)
        assert list(ib[t]) == list(r.idx), index_mismatch(f"fmoe_route_batched token {t}", ib[t], r.idx,
                                                          r.logits)
        assert np.allclose(wts.cpu().numpy()[t], r.w, rtol=1e-6, atol=1e-7)
        assert np.allclose(wb.cpu().numpy()[t], r.w, rtol=1e-6, atol=1e-7)
        ok, worst = oracle.within_tolerance(ys[t], r.y)
        assert ok, f"token {t}: worst error/bound {worst:.3f}"


@pytest.mark.parametrize("K", [4, 2, 5])
def test_tied_router_bias(cuda_lib, K):
    """Zero router, so every logit is its router bias exactly; the biases of TOP tie,
    those of NEXT tie below them, every other expert is lower and distinct."""
    shape = synth.LayerShape(256, 128, 64, K, 4, 1, 1)
    E = shape.n_experts
    router = np.zeros((E, shape.hidden), dtype=np.float32)
    rbias = (-1.0 - 1e-3 * np.arange(E)).astype(np.float32)
    rbias[list(TOP)] = 2.0
    rbias[list(NEXT)] = 1.0
    _, L, olay = _layer(cuda_lib, shape, 11, router, rbias)
    from fmoe_synth.torch_layer import make_device_x
    x = make_device_x(11, 0, 4, shape.hidden)
    want = list(TOP + NEXT)[:K]
    _check(cuda_lib, L, olay, x, want_first=want)
    L.close()


def test_duplicated_router_rows(cuda_lib):
    """No router bias: router rows of TOP are one vector aligned with token 0's x, those
    of NEXT a smaller multiple of it, so token 0's logits tie exactly within each set
    (identical rows give identical fp64 sums on both sides)."""
    from fmoe_synth.torch_layer import make_device_x
    shape = synth.LayerShape(256, 128, 64, 4, 4, 1, 0)
    seed = 12
    x = make_device_x(seed, 0, 6, shape.hidden)
    x0 = _bf(x)[0].astype(np.float32)
    router = synth.gen_router(seed, 0, shape.n_experts, shape.hidden).astype(np.float32).copy()
    router[list(TOP)] = 0.05 * x0
    router[list(NEXT)] = 0.03 * x0
    _, L, olay = _layer(cuda_lib, shape, seed, router, None)
    l0 = olay.route(_bf(x)[0])[3]
    assert l0[5] == l0[33] == l0[40] and l0[31] == l0[32] == l0[50], "the oracle's logits tie exactly"
    _check(cuda_lib, L, olay, x, want_first=[5, 33, 40, 31])
    L.close()


def test_all_logits_zero(cuda_lib):
    """A zero router without bias: all E logits are +0.0, the selection is experts
    0 .. K-1 in order and the weights are 1/K."""
    from fmoe_synth.torch_layer import make_device_x
    shape = synth.LayerShape(128, 64, 40, 3, 2, 1, 0)
    router = np.zeros((shape.n_experts, shape.hidden), dtype=np.float32)
    _, L, olay = _layer(cuda_lib, shape, 13, router, None)
    x = make_device_x(13, 0, 3, shape.hidden)
    _check(cuda_lib, L, olay, x, want_first=[0, 1, 2])
    idx, w, _ = L.route(x)
    torch.cuda.synchronize()
    assert np.all(w.cpu().numpy() == np.float32(1.0 / 3.0))
    L.close()
