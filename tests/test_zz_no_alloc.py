"""fmoe_layer_forward_noalloc: the layer forward for callers that cannot allocate
device memory (code that runs where cudaMalloc is unavailable or forbidden, or a host
framework that owns all device memory), so cannot hand the library a workspace.  It
keeps its scratch in one fixed device array inside the library.

Its output must match fmoe_layer_forward (the workspace path) on two calls in a row,
within the same tolerance the other layer tests use.  This file is collected last so
that a run stopping at the first failure has run every other test before it.
"""
import numpy as np
import pytest
import torch

import fmoe_synth as synth
import oracle

pytestmark = pytest.mark.gpu


def _bf(t):
    return oracle.bf16_to_f64(t.view(torch.int16).cpu().numpy().view(np.uint16))


@pytest.mark.parametrize("name", ["tiny", "layer4096"])
def test_noalloc_forward_matches_workspace_forward(cuda_lib, name):
    from fmoe_synth.torch_layer import make_device_layer, make_device_x
    fm = cuda_lib
    shape = synth.CONFIGS[name]["shape"]
    w = make_device_layer(shape, 0, 0)
    cfg = fm.fmoe_config(shape.hidden, shape.inter, shape.n_experts, shape.top_k, shape.bits,
                         shape.has_shared, shape.router_bias)
    assert fm.fmoe_workspace_bytes(cfg) <= fm.NOALLOC_SCRATCH_BYTES
    ref_layer = fm.Layer.create(cfg, w.experts, w.router, w.router_bias, w.shared_gate)
    # a second handle on the same weights, never given a workspace
    bare = fm.fmoe_layer_create(cfg, w.experts, w.router, w.router_bias, w.shared_gate)
    try:
        T = 6
        x = make_device_x(3, 0, T, shape.hidden)
        y_ref = torch.empty_like(x)
        for t in range(T):
            fm.fmoe_layer_forward(ref_layer.handle, x[t:t + 1], x[t:t + 1], 1, y_ref[t:t + 1])
        torch.cuda.synchronize()
        assert ref_layer.error() == 0
        ref = _bf(y_ref)
        for call in range(2):  # two calls in a row on the shared scratch array
            y = torch.full_like(x, float("nan"))
            for t in range(T):
                fm.fmoe_layer_forward_noalloc(bare, x[t:t + 1], x[t:t + 1], 1, y[t:t + 1])
            torch.cuda.synchronize()
            got = _bf(y)
            for t in range(T):
                ok, worst = oracle.within_tolerance(got[t], ref[t])
                assert ok, f"call {call} token {t}: worst error/bound {worst:.3f}"
            assert np.array_equal(got, ref), f"call {call}: not bit-identical to the workspace path"
    finally:
        fm.fmoe_layer_destroy(bare)
        ref_layer.close()


def test_noalloc_rejects_layers_beyond_the_scratch_size(cuda_lib):
    fm = cuda_lib
    # hidden 4096, intermediate 1024, 512 experts, top-10: workspace above 128 KiB.
    # Rejected on the host before anything is enqueued, so small stand-in buffers do.
    cfg = fm.fmoe_config(4096, 1024, 512, 10, 4, 1, 0)
    assert fm.fmoe_workspace_bytes(cfg) > fm.NOALLOC_SCRATCH_BYTES
    experts = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    router = torch.zeros(1024, dtype=torch.float32, device="cuda")
    gs = torch.zeros(4096, dtype=torch.float32, device="cuda")
    h = fm.fmoe_layer_create(cfg, experts, router, None, gs)
    try:
        x = torch.zeros(1, 4096, dtype=torch.bfloat16, device="cuda")
        y = torch.zeros_like(x)
        with pytest.raises(fm.FmoeError) as e:
            fm.fmoe_layer_forward_noalloc(h, x, x, 1, y)
        assert e.value.status == 6
        torch.cuda.synchronize()
        assert int(y.view(torch.int16).abs().sum()) == 0
    finally:
        fm.fmoe_layer_destroy(h)
