"""Pre-norm layer stacks on the GPU: the fused RMSNorm block, the token-by-token
stack decode and its captured CUDA graph, against the fp64 oracle.

A block computes h + MoE(RMSNorm(h)); the stack check is teacher-forced: the stack's
own h_l (read back after each layer) is the oracle block's input, and the oracle's
unrounded output is compared with the GPU's h_{l+1} under the layer tolerance
(2e-3 * (|y| + rms(y)) before the bf16 rounding, plus bf16's half-ulp, and agreement
with the rounded oracle).  Routing of a block is checked bit-exactly through the
separate entry points: fmoe_rmsnorm (bit-exact with the oracle's normalisation) and
fmoe_route on its output, after the fused block has been shown to equal
normalise-then-layer bit for bit.
"""
import multiprocessing
from concurrent.futures import ProcessPoolExecutor

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


def _layers(fm, shape, seed, n):
    from fmoe_synth.torch_layer import make_device_layer
    out = []
    for l in range(n):
        w = make_device_layer(shape, seed, l)
        cfg = fm.fmoe_config(shape.hidden, shape.inter, shape.n_experts, shape.top_k, shape.bits,
                             shape.has_shared, shape.router_bias)
        out.append(fm.Layer.create(cfg, w.experts, w.router, w.router_bias, w.shared_gate))
    return out


def _h0(seed, T, H, scale=1.0):
    from fmoe_synth.torch_layer import make_device_x
    x = make_device_x(seed, 0, T, H)
    return (x.float() * scale).to(torch.bfloat16) if scale != 1.0 else x


def _gpu_routing(fm, L, h):
    """Routing of the block input h through the separate entry points."""
    n = torch.empty_like(h)
    fm.fmoe_rmsnorm(h, n, h.shape[0], h.shape[1], EPS)
    return n, L.route(n)


def _assert_block(ctx, y_gpu, route, t, ref):
    idx, w, sig = route
    r_idx, r_w, r_sig, r_y = ref[:4]
    r_logits = ref[4] if len(ref) > 4 else None
    assert list(idx[t].cpu().numpy()) == list(r_idx), index_mismatch(ctx, idx[t].cpu().numpy(), r_idx, r_logits)
    assert np.allclose(w[t].cpu().numpy(), r_w, rtol=1e-6, atol=1e-7), f"{ctx}: w"
    ok, ratio = oracle.within_tolerance(y_gpu, r_y)
    assert ok, f"{ctx}: worst error/bound {ratio:.3f}"
    same, ulps = oracle.bf16_agreement(y_gpu, r_y, min_rel_rms=1.0 / 16)
    n_diff = round((1.0 - same) * y_gpu.shape[0])
    assert n_diff <= max(2, 0.01 * y_gpu.shape[0]) and ulps <= 1.0, f"{ctx}: {n_diff} differ, {ulps} ulps"


SMALL = {
    "tiny": synth.LayerShape(512, 128, 32, 4, 4, 1, 0),
    "tiny_2bit": synth.LayerShape(512, 128, 32, 4, 2, 1, 0),
    "rbias_k10": synth.LayerShape(1024, 256, 64, 10, 4, 1, 1),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_block_equals_norm_then_layer_and_oracle(cuda_lib, name):
    shape = SMALL[name]
    T = 12
    (L,) = _layers(cuda_lib, shape, 11, 1)
    h = _h0(11, T, shape.hidden, scale=2.5)  # not already normalised
    y = L.block(h)
    n, route = _gpu_routing(cuda_lib, L, h)
    y2 = L.forward(n, resid=h)
    hi = h.clone()
    L.block(hi, h_out=hi)  # in place
    torch.cuda.synchronize()
    assert L.error() == 0
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    assert torch.equal(y.view(torch.int16), hi.view(torch.int16))
    olay = oracle.synthetic_layer(11, 0, shape, lazy=True)
    hs, ys = _bf(h), _bf(y)
    for t in range(T):
        r = oracle.block_forward(olay, hs[t], EPS)
        _assert_block(f"{name} token {t}", ys[t], route, t, (r.idx, r.w, r.sigma, r.y, r.logits))


@pytest.mark.parametrize("name", ["tiny", "tiny_2bit"])
def test_small_stack_graph_teacher_forced(cuda_lib, name):
    shape = SMALL[name]
    T, NL = 6, 3
    layers = _layers(cuda_lib, shape, 12, NL)
    h0 = _h0(12, T, shape.hidden)
    hs = [h0.clone()]
    for L in layers:  # layer after layer, all tokens per launch
        hs.append(L.block(hs[-1]))
    stack = cuda_lib.Stack(layers, EPS)
    hg = h0.clone()
    g = stack.graph(hg)
    g.launch()
    hf = stack.forward(h0.clone())
    torch.cuda.synchronize()
    assert all(L.error() == 0 for L in layers)
    assert torch.equal(hg.view(torch.int16), hs[-1].view(torch.int16))
    assert torch.equal(hf.view(torch.int16), hs[-1].view(torch.int16))
    g.launch()  # replay continues from the first replay's output
    torch.cuda.synchronize()
    ref = hs[-1].clone()
    for L in layers:
        ref = L.block(ref)
    torch.cuda.synchronize()
    assert torch.equal(hg.view(torch.int16), ref.view(torch.int16))
    g.close()
    stack.close()
    for l, L in enumerate(layers):
        olay = oracle.synthetic_layer(12, l, shape, lazy=True)
        _, route = _gpu_routing(cuda_lib, L, hs[l])
        hin, hout = _bf(hs[l]), _bf(hs[l + 1])
        for t in range(T):
            r = oracle.block_forward(olay, hin[t], EPS)
            _assert_block(f"{name} layer {l} token {t}", hout[t], route, t, (r.idx, r.w, r.sigma, r.y, r.logits))


def _full_stack_gpu(cuda_lib, shape, NL, T, seed, samples):
    layers = _layers(cuda_lib, shape, seed, NL)
    h0 = _h0(seed, T, shape.hidden)
    hs = [h0.clone()]
    for lay in layers:
        hs.append(lay.block(hs[-1]))
    stack = cuda_lib.Stack(layers, EPS)
    hg = h0.clone()
    g = stack.graph(hg)
    g.launch()
    torch.cuda.synchronize()
    assert all(lay.error() == 0 for lay in layers)
    assert torch.equal(hg.view(torch.int16), hs[-1].view(torch.int16))
    g.close()
    stack.close()
    jobs, gpu = [], []
    for (l, t) in samples:
        _, route = _gpu_routing(cuda_lib, layers[l], hs[l])
        jobs.append((seed, l, shape_fields(shape), _bits(hs[l][t])))
        gpu.append((l, t, _bf(hs[l + 1][t]), tuple(r.cpu() for r in route)))
    for lay in layers:
        lay.close()
    return jobs, gpu


def _full_stack(cuda_lib, config, seed, samples):
    """The full-size stack of `config`: every token decoded through the captured graph
    must equal the layer-after-layer run bit for bit; sampled (layer, token) blocks are
    checked against the oracle (evaluated in a spawned process pool)."""
    cfg = synth.CONFIGS[config]
    shape, NL, T = cfg["shape"], cfg["layers"], cfg["tokens"]
    try:
        jobs, gpu = _full_stack_gpu(cuda_lib, shape, NL, T, seed, samples)
    finally:
        torch.cuda.empty_cache()  # the weights died with the helper's frame
    with ProcessPoolExecutor(max_workers=len(jobs), mp_context=multiprocessing.get_context("spawn")) as ex:
        refs = list(ex.map(block_case, jobs))
    for (l, t, y, route), ref in zip(gpu, refs):
        _assert_block(f"{config} layer {l} token {t}", y, route, t, ref)


def test_stack24_4bit_full_size(cuda_lib):
    """24 full-size 4-bit layers (87 GB resident), 256 tokens."""
    _full_stack(cuda_lib, "stack24_4bit", 0, [(0, 0), (0, 255), (11, 100), (23, 0), (23, 255), (17, 37)])


def test_stack60_2bit_full_size(cuda_lib):
    """60 full-size 2-bit layers (121.5 GB resident), 128 tokens."""
    _full_stack(cuda_lib, "stack60_2bit", 0, [(0, 0), (0, 127), (29, 64), (59, 0), (59, 127), (44, 9)])
