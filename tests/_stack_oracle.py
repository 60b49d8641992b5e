"""Oracle evaluations of synthetic layers (single tokens of a layer, single
pre-norm blocks), in a form a spawned process pool can run (only numpy, the oracle
and the input generator are imported here)."""
import numpy as np

import fmoe_synth as synth
import oracle


def block_case(args):
    """(seed, layer, shape fields, h as bf16 bits) -> (idx, w, sigma, y unrounded,
    logits)."""
    seed, layer, fields, h_bits = args
    shape = synth.LayerShape(*fields)
    lay = oracle.synthetic_layer(seed, layer, shape, lazy=True)
    h = oracle.bf16_to_f64(np.asarray(h_bits, dtype=np.uint16))
    r = oracle.block_forward(lay, h)
    return r.idx, r.w, r.sigma, r.y, r.logits


def shape_fields(shape):
    return (shape.hidden, shape.inter, shape.n_experts, shape.top_k, shape.bits, shape.has_shared,
            shape.router_bias)


def layer_tokens(args):
    """(seed, layer, shape fields, [x as bf16 bits, ...]) -> [(idx, w, sigma, y
    unrounded, logits), ...]: the single-layer forward of each token (resid = x).
    Decoded routed experts are dropped after each token (full-size experts take
    about 100 MB each as float64); the shared expert is kept."""
    seed, layer, fields, xs = args
    shape = synth.LayerShape(*fields)
    lay = oracle.synthetic_layer(seed, layer, shape, lazy=True)
    out = []
    for bits in xs:
        x = oracle.bf16_to_f64(np.asarray(bits, dtype=np.uint16))
        r = lay.forward(x)
        out.append((r.idx, r.w, r.sigma, r.y, r.logits))
        shared = lay._cache.get(shape.n_experts)
        lay._cache = {} if shared is None else {shape.n_experts: shared}
    return out
