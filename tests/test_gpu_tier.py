"""The host-memory expert tier on the GPU: routed expert records in pinned host memory,
an HBM cache of a few slots (least recently used evicted), the routing and the expert
kernels of the layer.

The outputs must equal fmoe_layer_forward's on the same weights bit for bit (the same
kernels on byte-identical records), and match the fp64 oracle within the layer
tolerance; the hit and miss counts must add up and every miss must have copied one
record.
"""
import numpy as np
import pytest
import torch

import fmoe_synth as synth
import oracle

pytestmark = pytest.mark.gpu


def _bf(t):
    return oracle.bf16_to_f64(t.view(torch.int16).cpu().numpy().view(np.uint16))


def _setup(fm, shape, seed, slots, max_tokens):
    from fmoe_synth.torch_layer import make_device_layer
    w = make_device_layer(shape, seed, 0)
    cfg = fm.fmoe_config(shape.hidden, shape.inter, shape.n_experts, shape.top_k, shape.bits,
                         shape.has_shared, shape.router_bias)
    ref = fm.Layer.create(cfg, w.experts, w.router, w.router_bias, w.shared_gate)
    rb = fm.fmoe_record_bytes(shape.hidden, shape.inter, shape.bits)
    E = shape.n_experts
    host = w.experts[:E * rb].cpu().pin_memory()          # the routed records, in host memory
    shared = w.experts[E * rb:(E + 1) * rb] if shape.has_shared else None
    tier = fm.Tier(cfg, host, shared, w.router, w.router_bias, w.shared_gate, slots, max_tokens)
    return w, ref, tier, rb


@pytest.mark.parametrize("name,slots", [("tiny", 8), ("tiny_2bit", 5), ("rbias_k10", 12)])
def test_tier_equals_hbm_layer_and_oracle(cuda_lib, name, slots):
    shapes = {"tiny": synth.LayerShape(512, 128, 32, 4, 4, 1, 0),
              "tiny_2bit": synth.LayerShape(512, 128, 32, 4, 2, 1, 0),
              "rbias_k10": synth.LayerShape(1024, 256, 64, 10, 4, 1, 1)}
    shape = shapes[name]
    fm = cuda_lib
    w, ref, tier, rb = _setup(fm, shape, 31, slots, 1)
    from fmoe_synth.torch_layer import make_device_x
    T = 24
    x = make_device_x(31, 0, T, shape.hidden)
    y_ref = torch.empty_like(x)
    y = torch.empty_like(x)
    for t in range(T):  # single-token decode calls, as the HBM layer runs them
        fm.fmoe_layer_forward(ref.handle, x[t:t + 1], x[t:t + 1], 1, y_ref[t:t + 1])
        tier.forward(x[t:t + 1], y=y[t:t + 1])
    torch.cuda.synchronize()
    assert ref.error() == 0 and tier.error() == 0
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    st = tier.stats()
    assert st["hits"] + st["misses"] == T * shape.top_k
    assert st["bytes_h2d"] == st["misses"] * rb
    assert st["misses"] >= min(shape.n_experts, slots)  # the cache starts empty
    olay = oracle.synthetic_layer(31, 0, shape, lazy=True)
    xs, ys = _bf(x), _bf(y)
    for t in (0, 7, T - 1):
        ok, worst = oracle.within_tolerance(ys[t], olay.forward(xs[t]).y)
        assert ok, f"{name} token {t}: worst error/bound {worst:.3f}"
    tier.close()
    ref.close()


def test_tier_multi_token_call_and_full_cache(cuda_lib):
    """Calls of several tokens; with as many slots as experts every expert is copied once
    and later calls only hit."""
    fm = cuda_lib
    shape = synth.LayerShape(512, 128, 32, 4, 4, 1, 0)
    w, ref, tier, rb = _setup(fm, shape, 32, shape.n_experts, 4)
    from fmoe_synth.torch_layer import make_device_x
    x = make_device_x(32, 0, 32, shape.hidden)
    y_ref = ref.forward(x)
    y = torch.empty_like(x)
    for t0 in range(0, 32, 4):
        tier.forward(x[t0:t0 + 4], y=y[t0:t0 + 4])
    torch.cuda.synchronize()
    assert tier.error() == 0
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    st = tier.stats()
    assert st["misses"] <= shape.n_experts
    before = st["misses"]
    tier.forward(x[:4], y=y[:4])  # every expert of these tokens is cached by now
    torch.cuda.synchronize()
    assert tier.stats()["misses"] == before
    tier.close()
    ref.close()
