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
    """A layer whose workspace exceeds the fixed array is refused before anything is
    enqueued.  The weight buffers have the sizes the config implies (zeros), so that
    even a launch that should not have happened would read only memory it owns."""
    fm = cuda_lib
    # hidden 64, intermediate 8192, 2 experts + shared, top-1: its h buffers alone take
    # 2 x 2 x 8192 x 4 bytes, more than the 128 KiB array
    H, I, E = 64, 8192, 2
    cfg = fm.fmoe_config(H, I, E, 1, 4, 1, 0)
    assert fm.fmoe_workspace_bytes(cfg) > fm.NOALLOC_SCRATCH_BYTES
    experts = torch.zeros(fm.fmoe_record_bytes(H, I, 4) * (E + 1), dtype=torch.uint8, device="cuda")
    router = torch.zeros(E, H, dtype=torch.float32, device="cuda")
    gs = torch.zeros(H, dtype=torch.float32, device="cuda")
    h = fm.fmoe_layer_create(cfg, experts, router, None, gs)
    try:
        x = torch.ones(1, H, dtype=torch.bfloat16, device="cuda")
        y = torch.zeros_like(x)
        with pytest.raises(fm.FmoeError) as e:
            fm.fmoe_layer_forward_noalloc(h, x, x, 1, y)
        assert e.value.status == 6
        torch.cuda.synchronize()
        assert int(y.view(torch.int16).abs().sum()) == 0
    finally:
        fm.fmoe_layer_destroy(h)


def test_noalloc_reports_device_errors(cuda_lib):
    """A device-side error of a no-allocation call (a bounded wait that runs out: one
    block is held back by the test hook, the others give up after 50 ms) is reported by
    fmoe_layer_get_error on the layer, which has no workspace, and cleared; the next
    call is correct again."""
    from fmoe_synth.torch_layer import make_device_layer, make_device_x
    fm = cuda_lib
    shape = synth.CONFIGS["tiny"]["shape"]
    w = make_device_layer(shape, 0, 0)
    cfg = fm.fmoe_config(shape.hidden, shape.inter, shape.n_experts, shape.top_k, shape.bits,
                         shape.has_shared, shape.router_bias)
    ref_layer = fm.Layer.create(cfg, w.experts, w.router, w.router_bias, w.shared_gate)
    bare = fm.fmoe_layer_create(cfg, w.experts, w.router, w.router_bias, w.shared_gate)
    try:
        x = make_device_x(4, 0, 1, shape.hidden)
        y_ref = ref_layer.forward(x)
        fm.fmoe_layer_set_wait_limit(bare, 50_000_000)
        fm.fmoe_layer_debug_hold_block(bare, 1)
        y = torch.zeros_like(x)
        fm.fmoe_layer_forward_noalloc(bare, x, x, 1, y)
        torch.cuda.synchronize()
        assert fm.fmoe_layer_get_error(bare) & fm.DEVERR_BARRIER_TIMEOUT
        assert fm.fmoe_layer_get_error(bare) == 0  # cleared
        fm.fmoe_layer_debug_hold_block(bare, -1)
        fm.fmoe_layer_forward_noalloc(bare, x, x, 1, y)
        torch.cuda.synchronize()
        assert fm.fmoe_layer_get_error(bare) == 0
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    finally:
        fm.fmoe_layer_destroy(bare)
        ref_layer.close()
