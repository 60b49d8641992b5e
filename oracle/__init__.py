"""fp64 CPU oracle for the routed-expert MoE layer — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The library under
``bit_dequant_expert_softmax_b200`` never imports it, and this package never
imports the library: the two share no code.  The only shared module is the
seeded input generator ``fmoe_synth``, which holds no arithmetic of the layer.

See ``oracle/fmoe_oracle.py`` for the definitions and their sources.
"""
from .fmoe_oracle import *  # noqa: F401,F403
