"""Parity of the CUDA layer (through the C ABI) with the fp64 oracle.

Expert indices must match exactly and in order; routing weights within 1e-6
relative (fp64 softmax rounded to fp32); layer outputs per element within
|gpu - oracle| <= 2e-3 * (|oracle| + rms(oracle)) applied before the bf16 output
rounding (plus bf16's half-ulp), and all but max(2, 1%) of the outputs equal to
the oracle rounded to nearest-even bf16, none more than one bf16 ulp away (an
fp32 result within ~1e-6 of a bf16 rounding midpoint may round either way); the
ulp check covers outputs with |oracle| >= rms/16, where the bf16 ulp exceeds the
fp32 sum's absolute rounding error.
"""
import math
import multiprocessing
import os
from concurrent.futures import ProcessPoolExecutor

import numpy as np
import pytest
import torch

import fmoe_synth as synth
import oracle
from _stack_oracle import layer_tokens, shape_fields
from _ties import index_mismatch

pytestmark = pytest.mark.gpu


def _mk(fm, shape, seed=0, layer=0):
    from fmoe_synth.torch_layer import make_device_layer
    w = make_device_layer(shape, seed, layer)
    cfg = fm.fmoe_config(shape.hidden, shape.inter, shape.n_experts, shape.top_k, shape.bits,
                         shape.has_shared, shape.router_bias)
    L = fm.Layer.create(cfg, w.experts, w.router, w.router_bias, w.shared_gate)
    return w, L


def _x(seed, t0, T, H):
    from fmoe_synth.torch_layer import make_device_x
    return make_device_x(seed, t0, T, H)


def _bf(t):
    return oracle.bf16_to_f64(t.view(torch.int16).cpu().numpy().view(np.uint16))


def _check_token(t, ref, xs, ys, idx, w, sig, has_shared, ctx=""):
    """One token's GPU routing and output against the oracle's (idx, w, sigma, y,
    logits); returns the worst error/bound ratio."""
    r_idx, r_w, r_sigma, r_y, r_logits = ref
    assert list(idx[t]) == list(r_idx), index_mismatch(f"{ctx} token {t}", idx[t], r_idx, r_logits)
    assert np.allclose(w[t], r_w, rtol=1e-6, atol=1e-7), f"{ctx} token {t}: w"
    if has_shared and sig is not None:
        assert math.isclose(float(sig[t]), r_sigma, rel_tol=1e-6), f"{ctx} token {t}: sigma"
    ok, ratio = oracle.within_tolerance(ys[t], r_y)
    assert ok, f"{ctx} token {t}: worst error/bound {ratio:.3f}"
    same, ulps = oracle.bf16_agreement(ys[t], r_y, min_rel_rms=1.0 / 16)
    n_diff = round((1.0 - same) * ys.shape[1])
    assert n_diff <= max(2, 0.01 * ys.shape[1]) and ulps <= 1.0, \
        f"{ctx} token {t}: {n_diff} outputs differ from the rounded oracle, max {ulps} ulps"
    return ratio


def _check_tokens(olay, xg, yg, idxg, wg, sigg, tokens, ctx=""):
    xs = _bf(xg)
    ys = _bf(yg)
    idx = idxg.cpu().numpy()
    w = wg.cpu().numpy()
    sig = None if sigg is None else sigg.cpu().numpy()
    worst = 0.0
    for t in tokens:
        r = olay.forward(xs[t])
        ref = (r.idx, r.w, r.sigma, r.y, r.logits)
        worst = max(worst, _check_token(t, ref, xs, ys, idx, w, sig, olay.has_shared, ctx))
    return worst


SHAPES = {
    "tiny": synth.LayerShape(512, 128, 32, 4, 4, 1, 0),
    "tiny_2bit": synth.LayerShape(512, 128, 32, 4, 2, 1, 0),
    "h64_k1": synth.LayerShape(64, 64, 8, 1, 4, 1, 0),
    "h64_k_eq_e": synth.LayerShape(64, 64, 4, 4, 4, 1, 0),
    "e40_noshared": synth.LayerShape(256, 192, 40, 3, 4, 0, 0),
    "rbias_k10": synth.LayerShape(1024, 256, 64, 10, 4, 1, 1),
    "mid_2bit": synth.LayerShape(2048, 512, 128, 6, 2, 1, 0),
}


@pytest.mark.parametrize("name", list(SHAPES))
def test_layer_forward_matches_oracle(cuda_lib, name):
    shape = SHAPES[name]
    T = 24
    _, L = _mk(cuda_lib, shape, seed=1)
    x = _x(1, 0, T, shape.hidden)
    y = torch.empty_like(x)
    for t in range(T):  # single-token decode calls
        cuda_lib.fmoe_layer_forward(L.handle, x[t:t + 1], x[t:t + 1], 1, y[t:t + 1])
    idx, w, sig = L.route(x)
    torch.cuda.synchronize()
    assert L.error() == 0
    olay = oracle.synthetic_layer(1, 0, shape, lazy=True)
    _check_tokens(olay, x, y, idx, w, sig, range(T), name)


def test_multi_token_call_equals_single_token_calls(cuda_lib):
    shape = SHAPES["tiny"]
    _, L = _mk(cuda_lib, shape, seed=2)
    x = _x(2, 0, 40, shape.hidden)
    y1 = L.forward(x)
    y2 = torch.empty_like(x)
    for t in range(40):
        L.forward(x[t:t + 1], y=y2[t:t + 1])
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    assert L.error() == 0


def test_split_api_equals_fused_and_oracle(cuda_lib):
    shape = SHAPES["tiny"]
    _, L = _mk(cuda_lib, shape, seed=3)
    x = _x(3, 0, 16, shape.hidden)
    yf = L.forward(x)
    idx, w, sig = L.route(x)
    ys = L.expert_forward(x, x, idx, w, sig)
    torch.cuda.synchronize()
    assert torch.equal(yf.view(torch.int16), ys.view(torch.int16))
    olay = oracle.synthetic_layer(3, 0, shape, lazy=True)
    xs = _bf(x)
    for t in range(16):
        r = olay.forward(xs[t])
        ye = olay.expert_forward(xs[t], xs[t], idx[t].cpu().numpy(), w[t].cpu().numpy(), float(sig[t]))
        assert oracle.within_tolerance(_bf(ys)[t], ye)[0]
        assert list(idx[t].cpu().numpy()) == list(r.idx), index_mismatch(f"token {t}", idx[t].cpu().numpy(), r.idx,
                                                                         r.logits)


def test_resid_differs_from_x_and_in_place(cuda_lib):
    shape = SHAPES["tiny"]
    _, L = _mk(cuda_lib, shape, seed=4)
    x = _x(4, 0, 8, shape.hidden)
    resid = _x(4, 100, 8, shape.hidden)
    y = L.forward(x, resid=resid)
    r2 = resid.clone()
    L.forward(x, resid=r2, y=r2)  # y aliases resid
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), r2.view(torch.int16))
    olay = oracle.synthetic_layer(4, 0, shape, lazy=True)
    xs, rs, ys = _bf(x), _bf(resid), _bf(y)
    for t in range(8):
        assert oracle.within_tolerance(ys[t], olay.forward(xs[t], rs[t]).y)[0]


def test_deterministic_and_graph_replay(cuda_lib):
    shape = SHAPES["tiny"]
    _, L = _mk(cuda_lib, shape, seed=5)
    x = _x(5, 0, 8, shape.hidden)
    ya = L.forward(x)
    yb = L.forward(x)
    yg = torch.empty_like(x)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for t in range(8):
            cuda_lib.fmoe_layer_forward(L.handle, x[t:t + 1], x[t:t + 1], 1, yg[t:t + 1], stream=s)
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(ya.view(torch.int16), yb.view(torch.int16))
    assert torch.equal(ya.view(torch.int16), yg.view(torch.int16))
    assert L.error() == 0


def test_full_size_layer_64_tokens(cuda_lib):
    """hidden 4096, intermediate 1024, 512 experts + shared, top-4, 4-bit (the
    full-size decode layer), single-token calls as the benchmark times them; all 64
    tokens (the first and the last among them) against the oracle, which runs in a
    spawned process pool."""
    shape = synth.CONFIGS["layer4096"]["shape"]
    _, L = _mk(cuda_lib, shape, seed=0)
    T = 64
    x = _x(0, 0, T, shape.hidden)
    y = torch.empty_like(x)
    for t in range(T):
        cuda_lib.fmoe_layer_forward(L.handle, x[t:t + 1], x[t:t + 1], 1, y[t:t + 1])
    idx, w, sig = L.route(x)
    torch.cuda.synchronize()
    assert L.error() == 0
    L.close()
    xb = x.view(torch.int16).cpu().numpy().view(np.uint16)
    workers = max(1, min(16, os.cpu_count() or 1))
    jobs = [(0, 0, shape_fields(shape), [xb[t] for t in range(T) if t % workers == j]) for j in range(workers)]
    with ProcessPoolExecutor(max_workers=workers, mp_context=multiprocessing.get_context("spawn")) as ex:
        parts = list(ex.map(layer_tokens, jobs))
    refs = {}
    for j, part in enumerate(parts):
        for t, ref in zip([t for t in range(T) if t % workers == j], part):
            refs[t] = ref
    xs, ys = _bf(x), _bf(y)
    idx, w, sig = idx.cpu().numpy(), w.cpu().numpy(), sig.cpu().numpy()
    worst = 0.0
    for t in range(T):
        worst = max(worst, _check_token(t, refs[t], xs, ys, idx, w, sig, True, "layer4096"))
    print(f"layer4096 worst error/bound over {T} tokens {worst:.3f}")


@pytest.mark.parametrize("scale,zero_resid", [(2.0 ** 20, False), (1e-20, False), (2.0 ** -40, True),
                                              (1e-10, True)])
@pytest.mark.parametrize("name", ["tiny", "tiny_2bit"])
def test_activation_magnitudes(cuda_lib, name, scale, zero_resid):
    """Activations far from unit size: x scaled by 2^20 (the hidden h reaches about
    2^46), by 1e-20, and by 2^-40 and 1e-10 with a zero residual (so that y is the MoE
    output alone, of the order of scale^2).  The dequantising dot products pick their
    power-of-two pre-scale per chunk of activations, so the single-token and the
    batched path both stay within the tolerance of the oracle."""
    shape = SHAPES[name]
    T = 8
    _, L = _mk(cuda_lib, shape, seed=14)
    x = (_x(14, 0, T, shape.hidden).float() * scale).to(torch.bfloat16)
    resid = torch.zeros_like(x) if zero_resid else x
    y = torch.empty_like(x)
    for t in range(T):
        cuda_lib.fmoe_layer_forward(L.handle, x[t:t + 1], resid[t:t + 1], 1, y[t:t + 1])
    idx, w, sig = L.route(x)
    L.attach_batch(T)
    yb = L.forward_batched(x, resid=resid)
    torch.cuda.synchronize()
    assert L.error() == 0
    olay = oracle.synthetic_layer(14, 0, shape, lazy=True)
    xs, rs, ys, ybs = _bf(x), _bf(resid), _bf(y), _bf(yb)
    idx, w = idx.cpu().numpy(), w.cpu().numpy()
    for t in range(T):
        r = olay.forward(xs[t], rs[t])
        assert list(idx[t]) == list(r.idx), index_mismatch(f"{name} x*{scale:g} token {t}", idx[t], r.idx, r.logits)
        assert np.allclose(w[t], r.w, rtol=1e-6, atol=1e-7)
        if zero_resid:  # y is the MoE output alone: nonzero, of the order of scale^2
            assert 0.0 < np.max(np.abs(r.y)) < 1e4 * scale * scale
        for label, got in (("single-token", ys[t]), ("batched", ybs[t])):
            ok, worst = oracle.within_tolerance(got, r.y)
            assert ok, f"{label} {name} x*{scale:g} token {t}: worst error/bound {worst:.3f}"


def test_rmsnorm_matches_oracle(cuda_lib):
    T, H = 16, 4096
    g = torch.Generator().manual_seed(0)
    h = (torch.randn(T, H, generator=g, dtype=torch.float64) * 3).to(torch.bfloat16).cuda()
    out = torch.empty_like(h)
    cuda_lib.fmoe_rmsnorm(h, out, T, H, 1e-6)
    torch.cuda.synchronize()
    hs = _bf(h)
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    for t in range(T):
        assert np.array_equal(got[t], oracle.rmsnorm_bf16(hs[t], 1e-6))


def test_empty_batch_is_noop(cuda_lib):
    shape = SHAPES["tiny"]
    _, L = _mk(cuda_lib, shape, seed=6)
    x = _x(6, 0, 1, shape.hidden)
    y = torch.zeros_like(x)
    cuda_lib.fmoe_layer_forward(L.handle, x, x, 0, y)
    torch.cuda.synchronize()
    assert int(y.view(torch.int16).abs().sum()) == 0


def test_bad_expert_index_sets_error(cuda_lib):
    shape = SHAPES["tiny"]
    _, L = _mk(cuda_lib, shape, seed=7)
    x = _x(7, 0, 2, shape.hidden)
    idx, w, sig = L.route(x)
    idx[1, 2] = shape.n_experts  # out of range
    y = torch.zeros_like(x)
    L.expert_forward(x, x, idx, w, sig, y=y)
    torch.cuda.synchronize()
    assert L.error() & cuda_lib.DEVERR_BAD_EXPERT
    assert int(y[1].view(torch.int16).abs().sum()) == 0
    assert L.error() == 0  # cleared


def test_barrier_wait_limit_reports_timeout(cuda_lib):
    """A block that never arrives makes the others' bounded grid wait run out: the
    kernel returns with an error bit, the context stays usable."""
    shape = SHAPES["tiny"]
    _, L = _mk(cuda_lib, shape, seed=8)
    x = _x(8, 0, 1, shape.hidden)
    cuda_lib.fmoe_layer_set_wait_limit(L.handle, 50_000_000)  # 50 ms
    cuda_lib.fmoe_layer_debug_hold_block(L.handle, 3)
    y = L.forward(x)
    torch.cuda.synchronize()
    assert L.error() & cuda_lib.DEVERR_BARRIER_TIMEOUT
    cuda_lib.fmoe_layer_debug_hold_block(L.handle, -1)
    y = L.forward(x)
    torch.cuda.synchronize()
    assert L.error() == 0
    olay = oracle.synthetic_layer(8, 0, shape, lazy=True)
    assert oracle.within_tolerance(_bf(y)[0], olay.forward(_bf(x)[0]).y)[0]
