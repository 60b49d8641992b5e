"""The batched (grouped-by-expert) path on the GPU against the fp64 oracle.

Routing of a batch must equal the single-token routing bit for bit (same logits,
same selection); outputs are checked per token against the oracle under the layer
tolerance (2e-3 * (|y| + rms(y)) before the bf16 rounding, plus bf16's half-ulp) and
against the oracle rounded to nearest-even bf16: no output more than one bf16 ulp
away and at most max(2, 2 %) of them one ulp away.  (The batched path multiplies on
the tensor cores with each code entered as 1 + c/2^b and the offset removed per
64-column group; the fp32 sums of those larger terms leave ~1e-5 relative error,
measured as 0.3-0.4 % of outputs one ulp from the rounded oracle on average, 1.04 %
at most, against ~0 % for the single-token path's smaller partial sums: 100 times
inside the stated bound either way.)
"""
import multiprocessing
from concurrent.futures import ProcessPoolExecutor
from types import SimpleNamespace

import numpy as np
import pytest
import torch

import fmoe_synth as synth
import oracle
from _ties import index_mismatch
from _stack_oracle import block_case, shape_fields

pytestmark = pytest.mark.gpu

EPS = 1e-6


def _bf(t):
    return oracle.bf16_to_f64(t.view(torch.int16).cpu().numpy().view(np.uint16))


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _layer(fm, shape, seed, layer=0, max_tokens=64):
    from fmoe_synth.torch_layer import make_device_layer
    w = make_device_layer(shape, seed, layer)
    cfg = fm.fmoe_config(shape.hidden, shape.inter, shape.n_experts, shape.top_k, shape.bits,
                         shape.has_shared, shape.router_bias)
    return fm.Layer.create(cfg, w.experts, w.router, w.router_bias, w.shared_gate).attach_batch(max_tokens)


def _x(seed, t0, T, H):
    from fmoe_synth.torch_layer import make_device_x
    return make_device_x(seed, t0, T, H)


def _assert_token(ctx, y, idx, w, sig, t, r, has_shared):
    assert list(idx[t]) == list(r.idx), index_mismatch(ctx, idx[t], r.idx, r.logits)
    assert np.allclose(w[t], r.w, rtol=1e-6, atol=1e-7), f"{ctx}: w"
    if has_shared:
        assert abs(float(sig[t]) - r.sigma) <= 1e-6 * abs(r.sigma), f"{ctx}: sigma"
    ok, ratio = oracle.within_tolerance(y, r.y)
    assert ok, f"{ctx}: worst error/bound {ratio:.3f}"
    same, ulps = oracle.bf16_agreement(y, r.y, min_rel_rms=1.0 / 16)
    n_diff = round((1.0 - same) * y.shape[0])
    assert n_diff <= max(2, 0.02 * y.shape[0]) and ulps <= 1.0, f"{ctx}: {n_diff} differ, {ulps} ulps"


SHAPES = {
    "tiny": synth.LayerShape(512, 128, 32, 4, 4, 1, 0),
    "tiny_2bit": synth.LayerShape(512, 128, 32, 4, 2, 1, 0),
    "h64_k_eq_e": synth.LayerShape(64, 64, 4, 4, 4, 1, 0),
    "e40_noshared": synth.LayerShape(256, 192, 40, 3, 4, 0, 0),
    "rbias_k10": synth.LayerShape(1024, 256, 64, 10, 4, 1, 1),
    "mid_2bit": synth.LayerShape(2048, 512, 128, 6, 2, 1, 0),
}


@pytest.mark.parametrize("name", list(SHAPES))
@pytest.mark.parametrize("T", [1, 7, 32])
def test_batched_layer_matches_oracle(cuda_lib, name, T):
    shape = SHAPES[name]
    L = _layer(cuda_lib, shape, seed=21)
    x = _x(21, 0, T, shape.hidden)
    y = L.forward_batched(x)
    ib, wb, sb = L.route_batched(x)
    i1, w1, s1 = L.route(x)
    torch.cuda.synchronize()
    assert L.error() == 0
    assert torch.equal(ib, i1) and torch.equal(wb, w1)
    if shape.has_shared:
        assert torch.equal(sb, s1)
    olay = oracle.synthetic_layer(21, 0, shape, lazy=True)
    xs, ys = _bf(x), _bf(y)
    idx, w, sig = ib.cpu().numpy(), wb.cpu().numpy(), sb.cpu().numpy()
    for t in range(T):
        _assert_token(f"{name} T={T} token {t}", ys[t], idx, w, sig, t, olay.forward(xs[t]), shape.has_shared)


def _umma_shape(shape):
    pc = 256 if shape.bits == 4 else 512
    return shape.hidden % pc == 0 and shape.inter % pc == 0


def _layer_kind(cuda_lib, shape, seed, env, monkeypatch, max_tokens=64):
    """A layer attached with the environment variable `env` set to "1" (or none)."""
    if env:
        monkeypatch.setenv(env, "1")
    try:
        return _layer(cuda_lib, shape, seed=seed, max_tokens=max_tokens)
    finally:
        if env:
            monkeypatch.delenv(env)


def test_batched_kind_follows_the_shape(cuda_lib, monkeypatch):
    """mma.sync by default; CUDA-core small tiles or tcgen05 on request (tcgen05 where
    the shape allows it)."""
    for name, shape in SHAPES.items():
        for env, want in ((None, 1), ("FMOE_GROUPED_SMALL", 3),
                          ("FMOE_GROUPED_TCGEN05", 2 if _umma_shape(shape) else 1)):
            L = _layer_kind(cuda_lib, shape, 20, env, monkeypatch, max_tokens=8)
            assert L.batched_kind() == want, (name, env)
            L.close()


@pytest.mark.parametrize("name", ["rbias_k10", "mid_2bit", "tiny", "e40_noshared"])
@pytest.mark.parametrize("T", [1, 7, 32])
def test_batched_kernel_variants(cuda_lib, name, T, monkeypatch):
    """The same layer on each kernel configuration of the grouped matvecs (mma.sync,
    CUDA-core small tiles + mma.sync, tcgen05 where the shape allows it): each against
    the oracle, routing identical."""
    shape = SHAPES[name]
    envs = [None, "FMOE_GROUPED_SMALL"] + (["FMOE_GROUPED_TCGEN05"] if _umma_shape(shape) else [])
    x = _x(28, 0, T, shape.hidden)
    olay = oracle.synthetic_layer(28, 0, shape, lazy=True)
    xs = _bf(x)
    refs = [olay.forward(xs[t]) for t in range(T)]
    for env in envs:
        L = _layer_kind(cuda_lib, shape, 28, env, monkeypatch)
        y = L.forward_batched(x)
        ib, wb, sb = (a.cpu().numpy() for a in L.route_batched(x))
        torch.cuda.synchronize()
        assert L.error() == 0, env
        ys = _bf(y)
        for t in range(T):
            _assert_token(f"{name} T={T} {env or 'default'} token {t}", ys[t], ib, wb, sb, t, refs[t],
                          shape.has_shared)
        L.close()


def test_batched_in_place_deterministic_and_graph(cuda_lib):
    shape = SHAPES["rbias_k10"]
    L = _layer(cuda_lib, shape, seed=22)
    x = _x(22, 0, 32, shape.hidden)
    resid = _x(22, 500, 32, shape.hidden)
    ya = L.forward_batched(x, resid=resid)
    yb = L.forward_batched(x, resid=resid)
    xi = x.clone()
    L.forward_batched(xi, resid=resid, y=xi)  # y aliases x
    ri = resid.clone()
    L.forward_batched(x, resid=ri, y=ri)  # y aliases resid
    yg = torch.empty_like(x)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        cuda_lib.fmoe_layer_forward_batched(L.handle, x, resid, 32, yg, stream=s)
    g.replay()
    torch.cuda.synchronize()
    assert L.error() == 0
    for other in (yb, xi, ri, yg):
        assert torch.equal(ya.view(torch.int16), other.view(torch.int16))


def test_batched_max_tokens_and_limits(cuda_lib):
    shape = SHAPES["mid_2bit"]
    L = _layer(cuda_lib, shape, seed=23, max_tokens=64)
    x = _x(23, 0, 64, shape.hidden)
    y = L.forward_batched(x)
    torch.cuda.synchronize()
    assert L.error() == 0
    olay = oracle.synthetic_layer(23, 0, shape, lazy=True)
    ib, wb, sb = L.route_batched(x)
    xs, ys = _bf(x), _bf(y)
    for t in (0, 17, 63):
        _assert_token(f"mid_2bit T=64 token {t}", ys[t], ib.cpu().numpy(), wb.cpu().numpy(), sb.cpu().numpy(), t,
                      olay.forward(xs[t]), True)
    small = _layer(cuda_lib, shape, seed=23, max_tokens=8)
    with pytest.raises(cuda_lib.FmoeError):
        small.forward_batched(_x(23, 0, 9, shape.hidden))
    cfg = cuda_lib.fmoe_config(shape.hidden, shape.inter, shape.n_experts, shape.top_k, shape.bits, 1, 0)
    assert cuda_lib.fmoe_batch_workspace_bytes(cfg, 65) == 0
    assert cuda_lib.fmoe_batch_workspace_bytes(cfg, 0) == 0


def test_batched_block_equals_norm_then_layer(cuda_lib):
    shape = SHAPES["tiny"]
    L = _layer(cuda_lib, shape, seed=24)
    h = (_x(24, 0, 20, shape.hidden).float() * 3.0).to(torch.bfloat16)
    yb = L.block_batched(h)
    n = torch.empty_like(h)
    cuda_lib.fmoe_rmsnorm(h, n, 20, shape.hidden, EPS)
    yl = L.forward_batched(n, resid=h)
    hi = h.clone()
    L.block_batched(hi, h_out=hi)
    torch.cuda.synchronize()
    assert torch.equal(yb.view(torch.int16), yl.view(torch.int16))
    assert torch.equal(yb.view(torch.int16), hi.view(torch.int16))


def test_batched_small_stack_graph(cuda_lib):
    """3 tiny layers, 12 tokens in steps of 5 (a ragged last step): graph == direct
    stack == layer after layer per step; every (layer, token) block against the
    oracle, teacher-forced."""
    shape = SHAPES["rbias_k10"]
    NL, T, B = 3, 12, 5
    layers = [_layer(cuda_lib, shape, 25, l, max_tokens=B) for l in range(NL)]
    h0 = _x(25, 0, T, shape.hidden)
    hs = [h0.clone()]
    for L in layers:
        nxt = hs[-1].clone()
        for t0 in range(0, T, B):
            L.block_batched(nxt[t0:t0 + B], h_out=nxt[t0:t0 + B])
        hs.append(nxt)
    stack = cuda_lib.Stack(layers, EPS)
    hg = h0.clone()
    g = stack.graph(hg, batch=B)
    g.launch()
    hf = stack.forward(h0.clone(), batch=B)
    torch.cuda.synchronize()
    assert all(L.error() == 0 for L in layers)
    assert torch.equal(hg.view(torch.int16), hs[-1].view(torch.int16))
    assert torch.equal(hf.view(torch.int16), hs[-1].view(torch.int16))
    g.close()
    stack.close()
    for l, L in enumerate(layers):
        n = torch.empty_like(hs[l])
        cuda_lib.fmoe_rmsnorm(hs[l], n, T, shape.hidden, EPS)
        idx, w, sig = (a.cpu().numpy() for a in L.route(n))
        olay = oracle.synthetic_layer(25, l, shape, lazy=True)
        hin, hout = _bf(hs[l]), _bf(hs[l + 1])
        for t in range(T):
            _assert_token(f"layer {l} token {t}", hout[t], idx, w, sig, t, oracle.block_forward(olay, hin[t], EPS),
                          True)


def _stack16_gpu(cuda_lib, samples):
    cfg = synth.CONFIGS["stack16_batched"]
    shape, NL, T, B = cfg["shape"], cfg["layers"], cfg["tokens"], cfg["batch"]
    layers = [_layer(cuda_lib, shape, 0, l, max_tokens=B) for l in range(NL)]
    h0 = _x(0, 0, T, shape.hidden)
    steps = sorted({t // B for (_, t) in samples})
    keep = {}  # (layer, step) -> h_l of the step's tokens
    hd = h0.clone()
    for s0 in range(0, T, B):
        hsl = hd[s0:s0 + B]
        for l, L in enumerate(layers):
            if s0 // B in steps:
                keep[(l, s0 // B)] = hsl.clone()
            L.block_batched(hsl, h_out=hsl)
        if s0 // B in steps:
            keep[(NL, s0 // B)] = hsl.clone()
    stack = cuda_lib.Stack(layers, EPS)
    hg = h0.clone()
    g = stack.graph(hg, batch=B)
    g.launch()
    torch.cuda.synchronize()
    assert all(L.error() == 0 for L in layers)
    assert torch.equal(hg.view(torch.int16), hd.view(torch.int16))
    g.close()
    stack.close()
    jobs, gpu = [], []
    for (l, t) in samples:
        s, j = t // B, t % B
        hin = keep[(l, s)]
        n = torch.empty_like(hin)
        cuda_lib.fmoe_rmsnorm(hin, n, B, shape.hidden, EPS)
        ib, wb, sb = layers[l].route_batched(n)
        i1, w1, s1 = layers[l].route(n)
        assert torch.equal(ib, i1) and torch.equal(wb, w1) and torch.equal(sb, s1)
        jobs.append((0, l, shape_fields(shape), _bits(hin[j])))
        gpu.append((l, t, j, _bf(keep[(l + 1, s)][j]), tuple(a.cpu().numpy() for a in (ib, wb, sb))))
    for L in layers:
        L.close()
    return jobs, gpu


def test_stack16_batched_full_size(cuda_lib):
    """16 full-size 4-bit layers with K = 10 and router bias (58 GB resident), 2048
    tokens decoded in steps of 32 through the captured graph; sampled blocks against
    the oracle."""
    samples = [(0, 0), (0, 31), (7, 1000), (15, 2047), (15, 2016), (11, 77)]
    try:
        jobs, gpu = _stack16_gpu(cuda_lib, samples)
    finally:
        torch.cuda.empty_cache()
    with ProcessPoolExecutor(max_workers=len(jobs), mp_context=multiprocessing.get_context("spawn")) as ex:
        refs = list(ex.map(block_case, jobs))
    for (l, t, j, y, (idx, w, sig)), (r_idx, r_w, r_sig, r_y, r_logits) in zip(gpu, refs):
        r = SimpleNamespace(idx=r_idx, w=r_w, sigma=r_sig, y=r_y, logits=r_logits)
        _assert_token(f"stack16 layer {l} token {t}", y, idx, w, sig, j, r, True)


def test_batched_layers_of_different_shapes_interleaved(cuda_lib):
    """A large and a small layer, attached one after the other, run alternately (the
    kernels' shared-memory limit is shared by all layers)."""
    big, small = SHAPES["mid_2bit"], SHAPES["tiny"]
    Lb = _layer(cuda_lib, big, seed=26, max_tokens=16)
    Ls = _layer(cuda_lib, small, seed=27, max_tokens=16)
    xb = _x(26, 0, 16, big.hidden)
    xs = _x(27, 0, 16, small.hidden)
    yb1 = Lb.forward_batched(xb)
    ys1 = Ls.forward_batched(xs)
    yb2 = Lb.forward_batched(xb)
    torch.cuda.synchronize()
    assert Lb.error() == 0 and Ls.error() == 0
    assert torch.equal(yb1.view(torch.int16), yb2.view(torch.int16))
    ob = oracle.synthetic_layer(26, 0, big, lazy=True)
    osm = oracle.synthetic_layer(27, 0, small, lazy=True)
    ib, wb, sb = (a.cpu().numpy() for a in Lb.route_batched(xb))
    is_, ws, ss = (a.cpu().numpy() for a in Ls.route_batched(xs))
    for t in (0, 15):
        _assert_token(f"big token {t}", _bf(yb1)[t], ib, wb, sb, t, ob.forward(_bf(xb)[t]), True)
        _assert_token(f"small token {t}", _bf(ys1)[t], is_, ws, ss, t, osm.forward(_bf(xs)[t]), True)
