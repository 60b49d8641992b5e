"""ctypes access to the device-side generator ``_synth.so`` (fills torch CUDA
buffers with the same values the numpy generator produces)."""
import ctypes
import os

from .build import SO

_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(SO):
            raise RuntimeError(f"{SO} is missing: run fmoe_synth.build.build() first")
        L = ctypes.CDLL(SO)
        u64, i32, vp = ctypes.c_uint64, ctypes.c_int, ctypes.c_void_p
        L.fmoe_synth_record_bytes.restype = ctypes.c_size_t
        L.fmoe_synth_record_bytes.argtypes = [i32, i32, i32]
        L.fmoe_synth_fill_records.argtypes = [vp, i32, i32, i32, u64, i32, i32, i32, vp]
        L.fmoe_synth_fill_router.argtypes = [vp, u64, i32, i32, i32, vp]
        L.fmoe_synth_fill_shared_gate.argtypes = [vp, u64, i32, i32, vp]
        L.fmoe_synth_fill_router_bias.argtypes = [vp, u64, i32, i32, vp]
        L.fmoe_synth_fill_x.argtypes = [vp, u64, i32, i32, i32, vp]
        L.fmoe_synth_host_normals.argtypes = [vp, u64, u64, u64]
        L.fmoe_synth_host_normals.restype = None
        L.fmoe_synth_host_record.argtypes = [vp, i32, i32, i32, u64, i32, i32]
        L.fmoe_synth_host_record.restype = None
        _lib = L
    return _lib


def _stream():
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"{what} failed with CUDA error {rc}")


def fill_records(dst, H, I, bits, seed, layer, expert0, n_experts):
    """Fill ``n_experts`` consecutive packed records into the uint8 CUDA tensor ``dst``."""
    _check(lib().fmoe_synth_fill_records(ctypes.c_void_p(dst.data_ptr()), H, I, bits, seed, layer,
                                         expert0, n_experts, _stream()), "fill_records")


def fill_router(dst, seed, layer, E, H):
    _check(lib().fmoe_synth_fill_router(ctypes.c_void_p(dst.data_ptr()), seed, layer, E, H, _stream()),
           "fill_router")


def fill_shared_gate(dst, seed, layer, H):
    _check(lib().fmoe_synth_fill_shared_gate(ctypes.c_void_p(dst.data_ptr()), seed, layer, H, _stream()),
           "fill_shared_gate")


def fill_router_bias(dst, seed, layer, E):
    _check(lib().fmoe_synth_fill_router_bias(ctypes.c_void_p(dst.data_ptr()), seed, layer, E, _stream()),
           "fill_router_bias")


def fill_x(dst, seed, t0, T, H):
    """bf16 [T, H] token activations (dst: int16/bfloat16 CUDA tensor)."""
    _check(lib().fmoe_synth_fill_x(ctypes.c_void_p(dst.data_ptr()), seed, t0, T, H, _stream()), "fill_x")
