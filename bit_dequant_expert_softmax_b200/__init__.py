"""B200 (sm_100a) routed-expert MoE layer: the C-ABI library libfmoe.so and its
Python binding.  The layer: router matvec, softmax / top-K / renormalisation,
group-wise 4- or 2-bit dequantised SwiGLU experts and the combine with a
sigmoid-gated shared expert and the residual."""
from . import fmoe  # noqa: F401
