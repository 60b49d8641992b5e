"""Thin ctypes binding of libfmoe.so (see include/fmoe.h for the contract).

Functions keep the C names; arguments are marshalled from torch CUDA tensors
(device memory and streams only: every step of the layer runs in the library's
kernels).  Loading fails loudly when the library is missing."""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(HERE, "libfmoe.so")

FMOE_OK = 0
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported configuration", 3: "CUDA error",
          4: "workspace missing or too small", 5: "device-side error", 6: "scratch limit of the no-allocation path"}
NOALLOC_SCRATCH_BYTES = 128 * 1024
DEVERR_BARRIER_TIMEOUT = 0x1
DEVERR_COPY_TIMEOUT = 0x2
DEVERR_BAD_EXPERT = 0x4
DEVERR_PLAN = 0x8
MAX_BATCH = 64

# every symbol include/fmoe.h declares
EXPORTS = ["fmoe_record_bytes", "fmoe_workspace_bytes", "fmoe_layer_create", "fmoe_layer_destroy",
           "fmoe_layer_set_workspace", "fmoe_route", "fmoe_expert_forward", "fmoe_layer_forward",
           "fmoe_rmsnorm", "fmoe_layer_get_error", "fmoe_layer_set_wait_limit",
           "fmoe_layer_debug_hold_block", "fmoe_layer_debug_timeline", "fmoe_layer_grid_size",
           "fmoe_layer_forward_noalloc", "fmoe_status_string", "fmoe_block_forward", "fmoe_stack_create",
           "fmoe_stack_destroy", "fmoe_stack_forward", "fmoe_stack_graph_create", "fmoe_graph_launch",
           "fmoe_graph_destroy", "fmoe_batch_workspace_bytes", "fmoe_layer_set_batch_workspace",
           "fmoe_layer_batched_kind",
           "fmoe_route_batched", "fmoe_layer_forward_batched", "fmoe_block_forward_batched",
           "fmoe_tier_buffer_bytes", "fmoe_tier_create", "fmoe_tier_forward", "fmoe_tier_stats",
           "fmoe_tier_get_error", "fmoe_tier_destroy", "fmoe_gdn_step"]


class FmoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, status)}")
        self.status = status


class fmoe_config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("inter", ctypes.c_int), ("n_experts", ctypes.c_int),
                ("top_k", ctypes.c_int), ("bits", ctypes.c_int), ("has_shared", ctypes.c_int),
                ("has_router_bias", ctypes.c_int)]


class fmoe_weights(ctypes.Structure):
    _fields_ = [("experts", ctypes.c_void_p), ("router", ctypes.c_void_p),
                ("router_bias", ctypes.c_void_p), ("shared_gate", ctypes.c_void_p)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(SO):
            raise RuntimeError(f"{SO} is missing: build it with bit_dequant_expert_softmax_b200.build.build()")
        L = ctypes.CDLL(SO)
        vp, i32, u64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64, ctypes.c_size_t
        L.fmoe_record_bytes.restype = sz
        L.fmoe_record_bytes.argtypes = [i32, i32, i32]
        L.fmoe_workspace_bytes.restype = sz
        L.fmoe_workspace_bytes.argtypes = [ctypes.POINTER(fmoe_config)]
        L.fmoe_layer_create.argtypes = [ctypes.POINTER(fmoe_config), ctypes.POINTER(fmoe_weights),
                                        ctypes.POINTER(vp)]
        L.fmoe_layer_destroy.argtypes = [vp]
        L.fmoe_layer_set_workspace.argtypes = [vp, vp, sz]
        L.fmoe_route.argtypes = [vp, vp, i32, vp, vp, vp, vp]
        L.fmoe_expert_forward.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, vp]
        L.fmoe_layer_forward.argtypes = [vp, vp, vp, i32, vp, vp]
        L.fmoe_rmsnorm.argtypes = [vp, vp, i32, i32, ctypes.c_double, vp]
        L.fmoe_block_forward.argtypes = [vp, vp, i32, ctypes.c_double, vp, vp]
        L.fmoe_stack_create.argtypes = [ctypes.POINTER(vp), i32, ctypes.c_double, ctypes.POINTER(vp)]
        L.fmoe_stack_destroy.argtypes = [vp]
        L.fmoe_stack_forward.argtypes = [vp, vp, i32, i32, vp]
        L.fmoe_stack_graph_create.argtypes = [vp, vp, i32, i32, ctypes.POINTER(vp)]
        L.fmoe_batch_workspace_bytes.restype = sz
        L.fmoe_batch_workspace_bytes.argtypes = [ctypes.POINTER(fmoe_config), i32]
        L.fmoe_layer_set_batch_workspace.argtypes = [vp, vp, sz, i32]
        L.fmoe_layer_batched_kind.argtypes = [vp]
        L.fmoe_layer_batched_kind.restype = i32
        L.fmoe_route_batched.argtypes = [vp, vp, i32, vp, vp, vp, vp]
        L.fmoe_layer_forward_batched.argtypes = [vp, vp, vp, i32, vp, vp]
        L.fmoe_block_forward_batched.argtypes = [vp, vp, i32, ctypes.c_double, vp, vp]
        L.fmoe_graph_launch.argtypes = [vp, vp]
        L.fmoe_graph_destroy.argtypes = [vp]
        L.fmoe_layer_forward_noalloc.argtypes = [vp, vp, vp, i32, vp, vp]
        L.fmoe_layer_get_error.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
        L.fmoe_layer_set_wait_limit.argtypes = [vp, u64]
        L.fmoe_layer_debug_hold_block.argtypes = [vp, i32]
        L.fmoe_layer_debug_timeline.argtypes = [vp, vp, i32]
        L.fmoe_layer_grid_size.argtypes = [vp]
        L.fmoe_layer_grid_size.restype = i32
        L.fmoe_tier_buffer_bytes.restype = sz
        L.fmoe_tier_buffer_bytes.argtypes = [ctypes.POINTER(fmoe_config), i32, i32]
        L.fmoe_tier_create.argtypes = [ctypes.POINTER(fmoe_config), vp, vp, vp, vp, vp, vp, sz, i32, i32,
                                       ctypes.POINTER(vp)]
        L.fmoe_tier_forward.argtypes = [vp, vp, vp, i32, vp, vp]
        L.fmoe_tier_stats.argtypes = [vp, ctypes.POINTER(u64), ctypes.POINTER(u64), ctypes.POINTER(u64)]
        L.fmoe_tier_get_error.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
        L.fmoe_tier_destroy.argtypes = [vp]
        L.fmoe_gdn_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, vp]
        L.fmoe_status_string.argtypes = [i32]
        L.fmoe_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(st: int, what: str):
    if st != FMOE_OK:
        raise FmoeError(st, what)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def fmoe_record_bytes(hidden: int, inter: int, bits: int) -> int:
    return lib().fmoe_record_bytes(hidden, inter, bits)


def fmoe_workspace_bytes(cfg: fmoe_config) -> int:
    return lib().fmoe_workspace_bytes(ctypes.byref(cfg))


def fmoe_layer_create(cfg: fmoe_config, experts, router, router_bias=None, shared_gate=None) -> int:
    w = fmoe_weights(_ptr(experts), _ptr(router), _ptr(router_bias), _ptr(shared_gate))
    h = ctypes.c_void_p()
    _check(lib().fmoe_layer_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h)), "fmoe_layer_create")
    return h.value


def fmoe_layer_destroy(handle: int):
    _check(lib().fmoe_layer_destroy(handle), "fmoe_layer_destroy")


def fmoe_layer_set_workspace(handle: int, ws):
    _check(lib().fmoe_layer_set_workspace(handle, ws.data_ptr(), ws.numel() * ws.element_size()),
           "fmoe_layer_set_workspace")


def fmoe_route(handle, x, T, idx, w, shared_sigma=None, stream=None):
    _check(lib().fmoe_route(handle, _ptr(x), T, _ptr(idx), _ptr(w), _ptr(shared_sigma), _stream(stream)),
           "fmoe_route")


def fmoe_expert_forward(handle, x, resid, T, idx, w, shared_sigma, y, stream=None):
    _check(lib().fmoe_expert_forward(handle, _ptr(x), _ptr(resid), T, _ptr(idx), _ptr(w), _ptr(shared_sigma),
                                     _ptr(y), _stream(stream)), "fmoe_expert_forward")


def fmoe_layer_forward(handle, x, resid, T, y, stream=None):
    _check(lib().fmoe_layer_forward(handle, _ptr(x), _ptr(resid), T, _ptr(y), _stream(stream)),
           "fmoe_layer_forward")


def fmoe_layer_forward_noalloc(handle, x, resid, T, y, stream=None):
    """fmoe_layer_forward on the library's fixed scratch array (no workspace, no
    allocation); see include/fmoe.h."""
    _check(lib().fmoe_layer_forward_noalloc(handle, _ptr(x), _ptr(resid), T, _ptr(y), _stream(stream)),
           "fmoe_layer_forward_noalloc")


def fmoe_gdn_step(state, q, k, v, alpha, beta, o, stream=None):
    """One GatedDeltaNet token step in place on state [heads, dv, dk] (fp32 CUDA tensors);
    o [heads, dv] gets the read-out (see include/fmoe.h)."""
    heads, dv, dk = state.shape
    _check(lib().fmoe_gdn_step(_ptr(state), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(o), heads, dk,
                               dv, _stream(stream)), "fmoe_gdn_step")


def fmoe_rmsnorm(h, out, T, H, eps=1e-6, stream=None):
    _check(lib().fmoe_rmsnorm(_ptr(h), _ptr(out), T, H, eps, _stream(stream)), "fmoe_rmsnorm")


def fmoe_block_forward(handle, h, T, eps, h_out, stream=None):
    _check(lib().fmoe_block_forward(handle, _ptr(h), T, eps, _ptr(h_out), _stream(stream)), "fmoe_block_forward")


def fmoe_stack_create(handles, eps=1e-6) -> int:
    arr = (ctypes.c_void_p * len(handles))(*handles)
    s = ctypes.c_void_p()
    _check(lib().fmoe_stack_create(arr, len(handles), eps, ctypes.byref(s)), "fmoe_stack_create")
    return s.value


def fmoe_stack_destroy(stack: int):
    _check(lib().fmoe_stack_destroy(stack), "fmoe_stack_destroy")


def fmoe_stack_forward(stack, h, T, batch=1, stream=None):
    _check(lib().fmoe_stack_forward(stack, _ptr(h), T, batch, _stream(stream)), "fmoe_stack_forward")


def fmoe_stack_graph_create(stack, h, T, batch=1) -> int:
    g = ctypes.c_void_p()
    _check(lib().fmoe_stack_graph_create(stack, _ptr(h), T, batch, ctypes.byref(g)), "fmoe_stack_graph_create")
    return g.value


def fmoe_batch_workspace_bytes(cfg: fmoe_config, max_tokens: int) -> int:
    return lib().fmoe_batch_workspace_bytes(ctypes.byref(cfg), max_tokens)


def fmoe_layer_set_batch_workspace(handle, ws, max_tokens: int):
    _check(lib().fmoe_layer_set_batch_workspace(handle, ws.data_ptr(), ws.numel() * ws.element_size(), max_tokens),
           "fmoe_layer_set_batch_workspace")


def fmoe_layer_batched_kind(handle) -> int:
    """2: tcgen05 grouped matvecs, 1: mma.sync ones, 0: no batch workspace."""
    return int(lib().fmoe_layer_batched_kind(handle))


def fmoe_route_batched(handle, x, T, idx, w, shared_sigma=None, stream=None):
    _check(lib().fmoe_route_batched(handle, _ptr(x), T, _ptr(idx), _ptr(w), _ptr(shared_sigma), _stream(stream)),
           "fmoe_route_batched")


def fmoe_layer_forward_batched(handle, x, resid, T, y, stream=None):
    _check(lib().fmoe_layer_forward_batched(handle, _ptr(x), _ptr(resid), T, _ptr(y), _stream(stream)),
           "fmoe_layer_forward_batched")


def fmoe_block_forward_batched(handle, h, T, eps, h_out, stream=None):
    _check(lib().fmoe_block_forward_batched(handle, _ptr(h), T, eps, _ptr(h_out), _stream(stream)),
           "fmoe_block_forward_batched")


def fmoe_graph_launch(graph, stream=None):
    _check(lib().fmoe_graph_launch(graph, _stream(stream)), "fmoe_graph_launch")


def fmoe_graph_destroy(graph):
    _check(lib().fmoe_graph_destroy(graph), "fmoe_graph_destroy")


def fmoe_layer_get_error(handle) -> int:
    e = ctypes.c_uint32(0)
    st = lib().fmoe_layer_get_error(handle, ctypes.byref(e))
    if st not in (0, 5):
        raise FmoeError(st, "fmoe_layer_get_error")
    return e.value


def fmoe_layer_set_wait_limit(handle, ns: int):
    _check(lib().fmoe_layer_set_wait_limit(handle, ns), "fmoe_layer_set_wait_limit")


def fmoe_layer_debug_hold_block(handle, cta: int):
    _check(lib().fmoe_layer_debug_hold_block(handle, cta), "fmoe_layer_debug_hold_block")


def fmoe_layer_debug_timeline(handle, buf, token: int = 0):
    _check(lib().fmoe_layer_debug_timeline(handle, _ptr(buf), token), "fmoe_layer_debug_timeline")


def fmoe_layer_grid_size(handle) -> int:
    return lib().fmoe_layer_grid_size(handle)


# ---------------------------------------------------------------------------
@dataclass
class Layer:
    """A layer handle plus the torch tensors it borrows (weights, workspace)."""
    handle: int
    cfg: fmoe_config
    experts: object
    router: object
    router_bias: object
    shared_gate: object
    workspace: object
    batch_workspace: object = None

    @staticmethod
    def create(cfg: fmoe_config, experts, router, router_bias=None, shared_gate=None) -> "Layer":
        import torch
        h = fmoe_layer_create(cfg, experts, router, router_bias, shared_gate)
        ws = torch.empty(fmoe_workspace_bytes(cfg), dtype=torch.uint8, device=experts.device)
        fmoe_layer_set_workspace(h, ws)
        return Layer(h, cfg, experts, router, router_bias, shared_gate, ws)

    def forward(self, x, resid=None, y=None, stream=None):
        import torch
        T = x.shape[0]
        resid = x if resid is None else resid
        y = torch.empty_like(x) if y is None else y
        fmoe_layer_forward(self.handle, x, resid, T, y, stream)
        return y

    def route(self, x, stream=None):
        import torch
        T = x.shape[0]
        K = self.cfg.top_k
        idx = torch.empty(T, K, dtype=torch.int32, device=x.device)
        w = torch.empty(T, K, dtype=torch.float32, device=x.device)
        sig = torch.empty(T, dtype=torch.float32, device=x.device)
        fmoe_route(self.handle, x, T, idx, w, sig, stream)
        return idx, w, sig

    def expert_forward(self, x, resid, idx, w, sig, y=None, stream=None):
        import torch
        y = torch.empty_like(x) if y is None else y
        fmoe_expert_forward(self.handle, x, resid, x.shape[0], idx, w, sig, y, stream)
        return y

    def block(self, h, h_out=None, eps=1e-6, stream=None):
        """Pre-norm block h + MoE(RMSNorm(h)); h_out may be h (in place)."""
        import torch
        h_out = torch.empty_like(h) if h_out is None else h_out
        fmoe_block_forward(self.handle, h, h.shape[0], eps, h_out, stream)
        return h_out

    def attach_batch(self, max_tokens: int):
        """Allocates and attaches the batched-path workspace for up to max_tokens tokens."""
        import torch
        n = fmoe_batch_workspace_bytes(self.cfg, max_tokens)
        if n == 0:
            raise FmoeError(1, "fmoe_batch_workspace_bytes")
        ws = torch.empty(n, dtype=torch.uint8, device=self.experts.device)
        fmoe_layer_set_batch_workspace(self.handle, ws, max_tokens)
        self.batch_workspace = ws
        return self

    def batched_kind(self) -> int:
        """2: the batched matvecs run on tcgen05, 1: on mma.sync, 0: no batch workspace."""
        return fmoe_layer_batched_kind(self.handle)

    def forward_batched(self, x, resid=None, y=None, stream=None):
        import torch
        resid = x if resid is None else resid
        y = torch.empty_like(x) if y is None else y
        fmoe_layer_forward_batched(self.handle, x, resid, x.shape[0], y, stream)
        return y

    def route_batched(self, x, stream=None):
        import torch
        T, K = x.shape[0], self.cfg.top_k
        idx = torch.empty(T, K, dtype=torch.int32, device=x.device)
        w = torch.empty(T, K, dtype=torch.float32, device=x.device)
        sig = torch.empty(T, dtype=torch.float32, device=x.device)
        fmoe_route_batched(self.handle, x, T, idx, w, sig, stream)
        return idx, w, sig

    def block_batched(self, h, h_out=None, eps=1e-6, stream=None):
        import torch
        h_out = torch.empty_like(h) if h_out is None else h_out
        fmoe_block_forward_batched(self.handle, h, h.shape[0], eps, h_out, stream)
        return h_out

    def error(self) -> int:
        return fmoe_layer_get_error(self.handle)

    def close(self):
        if self.handle:
            fmoe_layer_destroy(self.handle)
            self.handle = 0


def fmoe_tier_buffer_bytes(cfg: fmoe_config, slots: int, max_tokens: int) -> int:
    return lib().fmoe_tier_buffer_bytes(ctypes.byref(cfg), slots, max_tokens)


class Tier:
    """A layer whose routed experts live in host memory behind an HBM cache of `slots`
    records (see include/fmoe.h).  Keeps the host records, the device buffer and the
    router tensors alive."""

    def __init__(self, cfg: fmoe_config, host_experts, shared_record, router, router_bias, shared_gate,
                 slots: int, max_tokens: int = 1):
        import torch
        self.cfg = cfg
        self.keep = (host_experts, shared_record, router, router_bias, shared_gate)
        n = fmoe_tier_buffer_bytes(cfg, slots, max_tokens)
        if n == 0:
            raise FmoeError(1, "fmoe_tier_buffer_bytes")
        self.buf = torch.empty(n, dtype=torch.uint8, device=router.device)
        h = ctypes.c_void_p()
        _check(lib().fmoe_tier_create(ctypes.byref(cfg), _ptr(host_experts), _ptr(shared_record), _ptr(router),
                                      _ptr(router_bias), _ptr(shared_gate), self.buf.data_ptr(), n, slots,
                                      max_tokens, ctypes.byref(h)), "fmoe_tier_create")
        self.handle = h.value

    def forward(self, x, resid=None, y=None, stream=None):
        import torch
        resid = x if resid is None else resid
        y = torch.empty_like(x) if y is None else y
        _check(lib().fmoe_tier_forward(self.handle, _ptr(x), _ptr(resid), x.shape[0], _ptr(y), _stream(stream)),
               "fmoe_tier_forward")
        return y

    def stats(self):
        a, b, c = ctypes.c_uint64(), ctypes.c_uint64(), ctypes.c_uint64()
        _check(lib().fmoe_tier_stats(self.handle, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)),
               "fmoe_tier_stats")
        return {"hits": a.value, "misses": b.value, "bytes_h2d": c.value}

    def error(self) -> int:
        e = ctypes.c_uint32(0)
        st = lib().fmoe_tier_get_error(self.handle, ctypes.byref(e))
        if st not in (0, 5):
            raise FmoeError(st, "fmoe_tier_get_error")
        return e.value

    def close(self):
        if self.handle:
            lib().fmoe_tier_destroy(self.handle)
            self.handle = 0


class Stack:
    """Layers applied as pre-norm blocks; keeps the Layer objects alive."""

    def __init__(self, layers, eps=1e-6):
        self.layers = list(layers)
        self.eps = eps
        self.handle = fmoe_stack_create([L.handle for L in self.layers], eps)

    def forward(self, h, batch=1, stream=None):
        """Every token of h (bf16 [T, H]) through all layers, in place; batch > 1 runs
        steps of `batch` tokens on the batched path."""
        fmoe_stack_forward(self.handle, h, h.shape[0], batch, stream)
        return h

    def graph(self, h, batch=1) -> "Graph":
        return Graph(fmoe_stack_graph_create(self.handle, h, h.shape[0], batch), h)

    def close(self):
        if self.handle:
            fmoe_stack_destroy(self.handle)
            self.handle = 0


class Graph:
    """A captured stack decode over the buffer h (kept alive with the graph)."""

    def __init__(self, handle: int, h):
        self.handle = handle
        self.h = h

    def launch(self, stream=None):
        fmoe_graph_launch(self.handle, stream)

    def close(self):
        if self.handle:
            fmoe_graph_destroy(self.handle)
            self.handle = 0
