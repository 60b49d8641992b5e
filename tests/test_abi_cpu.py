"""The C-ABI library loads on a machine without a GPU and exports every symbol
include/fmoe.h declares; host-only entry points answer without a device."""
import ctypes
import os
import re

import pytest

import fmoe_synth as synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from bit_dequant_expert_softmax_b200 import build, fmoe
    build.build()
    return fmoe


def _declared():
    src = open(os.path.join(ROOT, "include", "fmoe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fmoe_[a-z_]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert len(names) == 36
    L = lib.lib()
    for n in names:
        assert hasattr(L, n), n
    assert sorted(lib.EXPORTS) == names


def test_record_bytes_matches_format(lib):
    for (H, I, b) in [(4096, 1024, 4), (4096, 1024, 2), (512, 128, 4), (64, 64, 2), (192, 320, 4)]:
        assert lib.fmoe_record_bytes(H, I, b) == synth.record_bytes(H, I, b)
    assert lib.fmoe_record_bytes(4096, 1000, 4) == 0
    assert lib.fmoe_record_bytes(4096, 1024, 3) == 0


def test_workspace_and_argument_checks(lib):
    cfg = lib.fmoe_config(4096, 1024, 512, 4, 4, 1, 0)
    assert lib.fmoe_workspace_bytes(cfg) > 0
    bad = lib.fmoe_config(4096, 1024, 512, 600, 4, 1, 0)
    assert lib.fmoe_workspace_bytes(bad) == 0
    L = lib.lib()
    h = ctypes.c_void_p()
    w = lib.fmoe_weights(None, None, None, None)
    assert L.fmoe_layer_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h)) == 1
    assert L.fmoe_layer_create(None, ctypes.byref(w), ctypes.byref(h)) == 1
    assert L.fmoe_route(None, None, 1, None, None, None, None) == 1
    assert L.fmoe_layer_forward(None, None, None, 1, None, None) == 1
    assert L.fmoe_rmsnorm(None, None, 1, 64, -1.0, None) == 1
    assert L.fmoe_status_string(4) == b"workspace missing or too small"


def test_stack_and_batch_argument_checks(lib):
    """Host-side checks of the stack, graph and batched entry points (no device work)."""
    L = lib.lib()
    cfg = lib.fmoe_config(4096, 1024, 512, 10, 4, 1, 1)
    b32 = lib.fmoe_batch_workspace_bytes(cfg, 32)
    assert b32 > lib.fmoe_batch_workspace_bytes(cfg, 1) > 0
    assert lib.fmoe_batch_workspace_bytes(cfg, 0) == 0
    assert lib.fmoe_batch_workspace_bytes(cfg, 65) == 0
    s = ctypes.c_void_p()
    assert L.fmoe_stack_create(None, 1, 1e-6, ctypes.byref(s)) == 1
    arr = (ctypes.c_void_p * 1)(None)
    assert L.fmoe_stack_create(arr, 1, 1e-6, ctypes.byref(s)) == 1
    assert L.fmoe_stack_create(arr, 0, 1e-6, ctypes.byref(s)) == 1
    assert L.fmoe_stack_forward(None, None, 1, 1, None) == 1
    assert L.fmoe_stack_graph_create(None, None, 1, 1, ctypes.byref(s)) == 1
    assert L.fmoe_graph_launch(None, None) == 1
    assert L.fmoe_graph_destroy(None) == 0
    assert L.fmoe_stack_destroy(None) == 0
    assert L.fmoe_block_forward(None, None, 1, 1e-6, None, None) == 1
    assert L.fmoe_layer_forward_batched(None, None, None, 1, None, None) == 1
    assert L.fmoe_block_forward_batched(None, None, 1, 1e-6, None, None) == 1
    assert L.fmoe_route_batched(None, None, 1, None, None, None, None) == 1


def _create(lib, cfg, experts=0x10000, router=0x20000, bias=0x30000, gate=0x40000):
    """fmoe_layer_create with fake (never dereferenced) weight addresses."""
    L = lib.lib()
    h = ctypes.c_void_p()
    w = lib.fmoe_weights(experts, router, bias, gate)
    return L.fmoe_layer_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h)), h


@pytest.mark.parametrize("fields", [
    (4000, 1024, 512, 4, 4, 1, 0),   # hidden not a multiple of 64
    (4096, 1000, 512, 4, 4, 1, 0),   # inter not a multiple of 64
    (4096, 1024, 512, 4, 3, 1, 0),   # bits other than 2 or 4
    (4096, 1024, 512, 0, 4, 1, 0),   # K = 0
    (4096, 1024, 4, 5, 4, 1, 0),     # K > E
    (4096, 1024, 0, 1, 4, 1, 0),     # no experts
    (4096, 1024, 512, 4, 4, 2, 0),   # has_shared not 0/1
    (4096, 1024, 512, 4, 4, 1, 7),   # has_router_bias not 0/1
    (-64, 1024, 512, 4, 4, 1, 0),    # negative size
])
def test_invalid_configs_are_rejected_on_the_host(lib, fields):
    cfg = lib.fmoe_config(*fields)
    assert lib.fmoe_workspace_bytes(cfg) == 0
    assert _create(lib, cfg)[0] == 1


def test_weight_pointer_checks(lib):
    cfg = lib.fmoe_config(4096, 1024, 512, 4, 4, 1, 1)
    assert _create(lib, cfg, experts=0x10000 + 128)[0] == 1      # records not 256-byte aligned
    assert _create(lib, cfg, router=0x20000 + 8)[0] == 1         # router not 16-byte aligned
    assert _create(lib, cfg, gate=0)[0] == 1                     # shared expert without its gate
    assert _create(lib, cfg, gate=0x40000 + 4)[0] == 1
    assert _create(lib, cfg, bias=0)[0] == 1                     # router bias declared, not given


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="checks the behaviour without a device")
def test_no_device_fails_loudly(lib):
    """Valid arguments but no CUDA device: the library refuses (FMOE_ERR_CUDA) instead of
    falling back to anything."""
    cfg = lib.fmoe_config(4096, 1024, 512, 4, 4, 1, 1)
    st, h = _create(lib, cfg)
    assert st == 3 and not h.value


def test_missing_library_raises(lib, monkeypatch, tmp_path):
    """Without the built library the binding raises; nothing else is tried."""
    monkeypatch.setattr(lib, "_lib", None)
    monkeypatch.setattr(lib, "SO", str(tmp_path / "libfmoe.so"))
    with pytest.raises(RuntimeError, match="missing"):
        lib.lib()
    with pytest.raises(RuntimeError):
        lib.fmoe_record_bytes(4096, 1024, 4)


def test_build_keeps_subnormals():
    """The library is built with -ftz=false and refuses flags that flush subnormals
    (the single-token dot products read codes as subnormal floats)."""
    from bit_dequant_expert_softmax_b200 import build as b
    assert "-ftz=false" in b.NVCC_FLAGS
    b.check_flags(b.NVCC_FLAGS)
    for bad in ("--use_fast_math", "-ftz=true"):
        with pytest.raises(ValueError):
            b.check_flags(b.NVCC_FLAGS + [bad])


def test_tier_buffer_bytes_and_host_checks(lib):
    """The host-memory tier's buffer size (cache of `slots` records, the shared record,
    two workspaces, routing buffers) and its argument checks, without a device."""
    cfg = lib.fmoe_config(512, 128, 32, 4, 4, 1, 0)
    rb = lib.fmoe_record_bytes(512, 128, 4)
    n8 = lib.fmoe_tier_buffer_bytes(cfg, 8, 1)
    n16 = lib.fmoe_tier_buffer_bytes(cfg, 16, 1)
    assert n8 > 9 * rb and 8 * rb <= n16 - n8 <= 8 * rb + 4096  # the cache layer's workspace grows a little
    assert lib.fmoe_tier_buffer_bytes(cfg, 0, 1) == 0
    assert lib.fmoe_tier_buffer_bytes(cfg, 33, 1) == 0   # more slots than experts
    assert lib.fmoe_tier_buffer_bytes(cfg, 8, 0) == 0
    L = lib.lib()
    h = ctypes.c_void_p()
    # NULL host records, NULL buffer: rejected before any device call
    assert L.fmoe_tier_create(ctypes.byref(cfg), None, None, None, None, None, None, n8, 8, 1, ctypes.byref(h)) == 1
    assert L.fmoe_tier_destroy(None) == 0


def test_batch_workspace_holds_tcgen05_tiles_only_on_request(lib, monkeypatch):
    """The tcgen05 kernels' activation tiles are sized into the batch workspace only
    when FMOE_GROUPED_TCGEN05=1 asks for them, and only for the shapes they take."""
    full = lib.fmoe_config(4096, 1024, 512, 10, 4, 1, 1)
    tiny = lib.fmoe_config(512, 128, 32, 4, 4, 1, 0)
    plain_full, plain_tiny = lib.fmoe_batch_workspace_bytes(full, 32), lib.fmoe_batch_workspace_bytes(tiny, 32)
    monkeypatch.setenv("FMOE_GROUPED_TCGEN05", "1")
    with_full, with_tiny = lib.fmoe_batch_workspace_bytes(full, 32), lib.fmoe_batch_workspace_bytes(tiny, 32)
    assert with_tiny == plain_tiny
    # 16-pair blocks of x (2 B per column + a sum per 64) and of h (hi + lo + sums)
    assert with_full - plain_full >= 22 * 16 * (2 * 4096 + 4096 // 16) + 22 * 16 * (4 * 1024 + 1024 // 16)
