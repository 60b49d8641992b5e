"""Device-resident synthetic layers (torch CUDA tensors filled by the device-side
generator).  Inputs only: no arithmetic of the layer lives here."""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import LayerShape, record_bytes
from . import device as dev


@dataclass
class DeviceLayerWeights:
    shape: LayerShape
    seed: int
    layer: int
    experts: torch.Tensor      # uint8 [(E + shared) * record_bytes]
    router: torch.Tensor       # fp32 [E, H]
    router_bias: torch.Tensor  # fp32 [E] or None
    shared_gate: torch.Tensor  # fp32 [H] or None


def make_device_layer(shape: LayerShape, seed: int, layer: int, device="cuda",
                      chunk_experts: int = 64) -> DeviceLayerWeights:
    H, I, E = shape.hidden, shape.inter, shape.n_experts
    n = E + shape.has_shared
    rb = record_bytes(H, I, shape.bits)
    experts = torch.empty(n * rb, dtype=torch.uint8, device=device)
    for e0 in range(0, n, chunk_experts):
        m = min(chunk_experts, n - e0)
        dev.fill_records(experts[e0 * rb:(e0 + m) * rb], H, I, shape.bits, seed, layer, e0, m)
    router = torch.empty(E, H, dtype=torch.float32, device=device)
    dev.fill_router(router, seed, layer, E, H)
    rbias = None
    if shape.router_bias:
        rbias = torch.empty(E, dtype=torch.float32, device=device)
        dev.fill_router_bias(rbias, seed, layer, E)
    gs = None
    if shape.has_shared:
        gs = torch.empty(H, dtype=torch.float32, device=device)
        dev.fill_shared_gate(gs, seed, layer, H)
    return DeviceLayerWeights(shape, seed, layer, experts, router, rbias, gs)


def make_device_x(seed: int, t0: int, T: int, H: int, device="cuda") -> torch.Tensor:
    """bf16 [T, H] activations of tokens t0 .. t0+T-1 (as a torch.bfloat16 tensor)."""
    x = torch.empty(T, H, dtype=torch.int16, device=device)
    dev.fill_x(x, seed, t0, T, H)
    return x.view(torch.bfloat16)
