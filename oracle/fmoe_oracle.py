"""Plain, slow, fp64 reference of the routed-expert MoE layer (test infrastructure).

Imported only by ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / reference leg.  Nothing in the CUDA library calls it, and it
calls nothing of the library.

Sources (the Flash-MoE pages):

* hotdry.top article "48GB内存运行397B模型", section "MoE稀疏架构": a layer has
  512 routed experts of which K are active per token, plus one shared expert.
* same article, section "量化策略", and the juejin.cn article section
  "Metal 着色器": expert weights are 4-bit (or 2-bit) codes dequantised as
  ``code * scale + bias`` before they meet the activation; the FMA rewrite
  ``fma(code, scale*x, bias*x)`` is the same sum reordered.
* same article, section "Metal GPU管线", and the juejin.cn list of shaders:
  fused SwiGLU ``silu(gate) * up``; fused combine of the expert outputs with the
  residual and a sigmoid-gated shared expert; two-pass RMS normalisation.
* tinai-dev README page, "Pipeline mỗi lớp": routing on the GPU, then
  softmax and top-K on the CPU.
* intelliparadigm.com page, section 2.1 (router snippet): softmax over all
  experts, then top-K on the probabilities.

Readings where the pages are silent, taken here:

* group size 64 along the input (reduction) dimension, one (scale, bias) pair
  per group and row; codes low-bits-first inside little-endian uint32 words;
* top-K ordered by probability descending, ties to the lower expert index;
  the K probabilities are renormalised to sum to one;
* shared expert gate ``sigma = 1 / (1 + exp(-g_s . x))`` with a vector g_s;
* single-layer output ``y = resid + sum_k w_k o_k + sigma o_s``;
* stacked layers are pre-norm blocks ``h <- h + MoE(RMSNorm(h))`` with gamma = 1,
  eps = 1e-6, the normalised vector rounded to bf16.

Everything is float64.  Dequantised weights ``scale * q + bias`` are exact in
float64 (a bf16 times a <= 4-bit integer needs <= 12 significand bits).
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional

import numpy as np

import fmoe_synth as synth

GROUP = 64


# ----------------------------------------------------------------------------
# storage decoding
# ----------------------------------------------------------------------------
def bf16_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns -> float64 (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(v) -> np.ndarray:
    """Round float64 values to bf16 (nearest, ties to even); returns bit patterns.

    Written from the definition: keep 8 significant bits of the binary
    significand, rounding the discarded part to nearest with ties to even.
    Normal-range values only (the layer's values never leave it)."""
    v = np.atleast_1d(np.asarray(v, dtype=np.float64))
    out = np.zeros(v.shape, dtype=np.uint16)
    for idx, x in np.ndenumerate(v):
        if x == 0.0:
            out[idx] = 0x8000 if math.copysign(1.0, x) < 0 else 0
            continue
        m, e = math.frexp(abs(x))          # |x| = m 2^e, m in [0.5, 1)
        scaled = m * 256.0                 # exact
        lo = math.floor(scaled)
        frac = scaled - lo
        if frac > 0.5 or (frac == 0.5 and lo % 2 == 1):
            lo += 1
        r = math.ldexp(lo, e - 8)
        if x < 0:
            r = -r
        out[idx] = np.float32(r).view(np.uint32) >> 16
    return out


def unpack_codes(words: np.ndarray, bits: int) -> np.ndarray:
    """uint32 words [..., W] -> integer codes [..., W * 32/bits], code k of a word
    taken from bits [bits*k, bits*k + bits) (lowest bits first).

    4-bit (or 2-bit) expert weights packed into 32-bit words: hotdry.top,
    "量化策略"; the order inside a word is a reading (the pages are silent)."""
    words = np.asarray(words, dtype=np.uint32)
    per = 32 // bits
    mask = (1 << bits) - 1
    codes = np.empty(words.shape + (per,), dtype=np.int64)
    for k in range(per):
        codes[..., k] = (words.astype(np.int64) >> (bits * k)) & mask
    return codes.reshape(words.shape[:-1] + (words.shape[-1] * per,))


def dequantise(codes: np.ndarray, sb: np.ndarray) -> np.ndarray:
    """Explicit dequantisation W[r, c] = scale[r, c//64] * q[r, c] + bias[r, c//64].

    ``sb`` holds one uint32 per (row, group): bf16 scale in the low half,
    bf16 bias in the high half.  The affine form ``code * scale + bias`` is that of
    hotdry.top, "量化策略", and of the juejin.cn shader section "Metal 着色器" (whose
    ``fma(code, scale*x, bias*x)`` is the same product reordered); the group of 64
    along the input dimension is the reading that fits the pages' 6.75 MB per
    expert."""
    sb = np.asarray(sb, dtype=np.uint32)
    scale = bf16_to_f64((sb & 0xFFFF).astype(np.uint16))
    bias = bf16_to_f64((sb >> 16).astype(np.uint16))
    rows, cols = codes.shape
    g = np.arange(cols) // GROUP
    return scale[:, g] * codes.astype(np.float64) + bias[:, g]


@dataclass
class DenseExpert:
    Wg: np.ndarray  # [I, H]
    Wu: np.ndarray  # [I, H]
    Wd: np.ndarray  # [H, I]


def record_regions(H: int, I: int, bits: int) -> dict:
    """Byte layout of one packed expert record (the library's weight format):
    four regions, each starting at a multiple of 256 bytes:
    gate/up code rows interleaved by row, gate/up (scale, bias) rows interleaved
    by row, down code rows, down (scale, bias) rows."""
    def al(n):
        return (n + 255) // 256 * 256
    qh, qi = H * bits // 8, I * bits // 8
    sh, si = H // GROUP * 4, I // GROUP * 4
    o0 = 0
    o1 = al(o0 + I * 2 * qh)
    o2 = al(o1 + I * 2 * sh)
    o3 = al(o2 + H * qi)
    size = al(o3 + H * si)
    return dict(gu_q=o0, gu_sb=o1, d_q=o2, d_sb=o3, size=size, qh=qh, qi=qi, sh=sh, si=si)


def decode_record(rec: np.ndarray, H: int, I: int, bits: int) -> DenseExpert:
    """Read one packed record and dequantise its three matrices to float64 (gate
    and up [I, H], down [H, I]: the expert FFN of hotdry.top, "Metal GPU管线")."""
    R = record_regions(H, I, bits)
    rec = np.asarray(rec, dtype=np.uint8)
    wh, wi = H * bits // 32, I * bits // 32
    gu_q = rec[R["gu_q"]:R["gu_q"] + I * 2 * R["qh"]].view(np.uint32).reshape(I, 2, wh)
    gu_sb = rec[R["gu_sb"]:R["gu_sb"] + I * 2 * R["sh"]].view(np.uint32).reshape(I, 2, H // GROUP)
    d_q = rec[R["d_q"]:R["d_q"] + H * R["qi"]].view(np.uint32).reshape(H, wi)
    d_sb = rec[R["d_sb"]:R["d_sb"] + H * R["si"]].view(np.uint32).reshape(H, I // GROUP)
    Wg = dequantise(unpack_codes(gu_q[:, 0, :], bits), gu_sb[:, 0, :])
    Wu = dequantise(unpack_codes(gu_q[:, 1, :], bits), gu_sb[:, 1, :])
    Wd = dequantise(unpack_codes(d_q, bits), d_sb)
    return DenseExpert(Wg, Wu, Wd)


# ----------------------------------------------------------------------------
# the layer, step by step
# ----------------------------------------------------------------------------
def router_logits(x: np.ndarray, Wr: np.ndarray, bias: Optional[np.ndarray] = None) -> np.ndarray:
    """l_e = sum_c Wr[e, c] x_c (+ b_e), float64 (router GEMV; routing runs on the
    GPU in tinai-dev README, "Pipeline mỗi lớp").  The bias is the batched
    workload's per-expert popularity skew."""
    l = Wr.astype(np.float64) @ np.asarray(x, dtype=np.float64)
    if bias is not None:
        l = l + np.asarray(bias, dtype=np.float64)
    return l


def softmax(l: np.ndarray) -> np.ndarray:
    """Softmax over all experts (intelliparadigm.com, section 2.1 router snippet),
    shifted by the maximum (the same value in exact arithmetic)."""
    m = np.max(l)
    e = np.exp(l - m)
    return e / np.sum(e)


def topk_renorm(l: np.ndarray, K: int):
    """Softmax over all experts, top-K by probability (descending, ties to the
    lower index), then the K probabilities renormalised to sum to one
    (intelliparadigm.com, section 2.1: softmax, then top-K on the probabilities;
    tinai-dev README, "Pipeline mỗi lớp": softmax + top-K routing).  The
    renormalisation and the tie rule are readings.

    The softmax is strictly increasing in the logit, so the K largest
    probabilities belong to the K largest logits, and two probabilities are equal
    exactly when their logits are.  The order is taken on the logits: in fp64 the
    probabilities of logits more than ~745 below the largest underflow to 0.0 and
    would tie, which the exact probabilities never do."""
    l = np.asarray(l, dtype=np.float64)
    p = softmax(l)
    order = sorted(range(len(l)), key=lambda e: (-l[e], e))
    idx = np.array(order[:K], dtype=np.int64)
    w = p[idx] / np.sum(p[idx])
    return idx, w


def silu(t: np.ndarray) -> np.ndarray:
    """silu(t) = t * sigmoid(t), the gate activation of the fused SwiGLU (hotdry.top,
    "Metal GPU管线")."""
    return t / (1.0 + np.exp(-t))


def expert_ffn(ex: DenseExpert, x: np.ndarray) -> np.ndarray:
    """o = W_d (silu(W_g x) * (W_u x)) in float64 (hotdry.top, "Metal GPU管线":
    fused SwiGLU, then the down projection)."""
    x = np.asarray(x, dtype=np.float64)
    g = ex.Wg @ x
    u = ex.Wu @ x
    h = silu(g) * u
    return ex.Wd @ h


def expert_hidden(ex: DenseExpert, x: np.ndarray) -> np.ndarray:
    """h = silu(W_g x) * (W_u x), the SwiGLU hidden vector alone."""
    x = np.asarray(x, dtype=np.float64)
    return silu(ex.Wg @ x) * (ex.Wu @ x)


def shared_sigma(gs: np.ndarray, x: np.ndarray) -> float:
    """sigma = 1 / (1 + exp(-g_s . x)), the sigmoid gate of the shared expert
    (hotdry.top, "Metal GPU管线"); a vector g_s is the reading.  For a negative
    argument the same value is written exp(s) / (1 + exp(s)), which does not
    overflow."""
    s = float(np.asarray(gs, dtype=np.float64) @ np.asarray(x, dtype=np.float64))
    if s >= 0.0:
        return 1.0 / (1.0 + math.exp(-s))
    e = math.exp(s)
    return e / (1.0 + e)


@dataclass
class LayerResult:
    y: np.ndarray        # float64 [H], unrounded
    idx: np.ndarray      # int64 [K]
    w: np.ndarray        # float64 [K]
    sigma: float
    logits: np.ndarray   # float64 [E]


class OracleLayer:
    """One MoE layer held as packed records (numpy uint8) plus router tensors.

    ``records`` may be a callable ``e -> record bytes`` so that full-size layers
    regenerate only the experts a token selects."""

    def __init__(self, H, I, E, K, bits, records, router, shared_gate=None,
                 router_bias=None, has_shared=True):
        self.H, self.I, self.E, self.K, self.bits = H, I, E, K, bits
        self._records = records
        self.router = np.asarray(router, dtype=np.float32)
        self.shared_gate = None if shared_gate is None else np.asarray(shared_gate, dtype=np.float32)
        self.router_bias = None if router_bias is None else np.asarray(router_bias, dtype=np.float32)
        self.has_shared = has_shared
        self._cache = {}

    def expert(self, e: int) -> DenseExpert:
        if e not in self._cache:
            if callable(self._records):
                rec = self._records(e)
            else:
                rb = record_regions(self.H, self.I, self.bits)["size"]
                rec = self._records[e * rb:(e + 1) * rb]
            self._cache[e] = decode_record(rec, self.H, self.I, self.bits)
        return self._cache[e]

    def route(self, x: np.ndarray):
        l = router_logits(x, self.router, self.router_bias)
        idx, w = topk_renorm(l, self.K)
        sig = shared_sigma(self.shared_gate, x) if self.has_shared else 0.0
        return idx, w, sig, l

    def forward(self, x: np.ndarray, resid: Optional[np.ndarray] = None) -> LayerResult:
        """y = resid + sum_k w_k o_k(x) + sigma o_s(x); resid defaults to x (the
        fused combine with the residual and the sigmoid-gated shared expert of
        hotdry.top, "Metal GPU管线")."""
        x = np.asarray(x, dtype=np.float64)
        r = x if resid is None else np.asarray(resid, dtype=np.float64)
        idx, w, sig, l = self.route(x)
        y = r.copy()
        for k in range(self.K):
            y = y + w[k] * expert_ffn(self.expert(int(idx[k])), x)
        if self.has_shared:
            y = y + sig * expert_ffn(self.expert(self.E), x)
        return LayerResult(y=y, idx=idx, w=w, sigma=sig, logits=l)

    def expert_forward(self, x, resid, idx, w, sig) -> np.ndarray:
        """Combine for given routing (the split entry point)."""
        x = np.asarray(x, dtype=np.float64)
        y = np.asarray(resid, dtype=np.float64).copy()
        for k in range(len(idx)):
            y = y + float(w[k]) * expert_ffn(self.expert(int(idx[k])), x)
        if self.has_shared:
            y = y + float(sig) * expert_ffn(self.expert(self.E), x)
        return y


def rmsnorm_bf16(h: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """n = bf16(h / sqrt(mean(h^2) + eps)), gamma = 1; returns bf16 bit patterns.

    Two passes, the sum of squares and then the scaling, as in hotdry.top,
    "Metal GPU管线"; gamma = 1 and eps = 1e-6 are readings."""
    h = np.asarray(h, dtype=np.float64)
    ss = 0.0
    for v in h:
        ss += v * v
    r = math.sqrt(ss / h.size + eps)
    return f64_to_bf16_bits(h / r)


def block_forward(layer: OracleLayer, h: np.ndarray, eps: float = 1e-6) -> LayerResult:
    """One pre-norm block of a stack: n = bf16(RMSNorm(h)); the layer runs on n with
    the block input h as its residual, y = h + sum_k w_k o_k(n) + sigma o_s(n)
    (hotdry.top "Metal GPU管线": normalisation, experts and the residual combine of
    one layer; the stacks here keep no attention, so the block is norm + MoE +
    residual).  y is returned unrounded; the stack stores it as bf16."""
    h = np.asarray(h, dtype=np.float64)
    n = bf16_to_f64(rmsnorm_bf16(h, eps))
    return layer.forward(n, resid=h)


# ----------------------------------------------------------------------------
# synthetic layers built from the shared generator
# ----------------------------------------------------------------------------
def synthetic_layer(seed: int, layer: int, shape: "synth.LayerShape", lazy: bool = False) -> OracleLayer:
    H, I, E = shape.hidden, shape.inter, shape.n_experts
    if lazy:
        def rec(e, _s=seed, _l=layer):
            return synth.gen_record(_s, _l, e, H, I, shape.bits)
        records = rec
    else:
        records = synth.gen_layer_records(seed, layer, shape)
    router = synth.gen_router(seed, layer, E, H)
    gs = synth.gen_shared_gate(seed, layer, H) if shape.has_shared else None
    rb = synth.gen_router_bias(seed, layer, E) if shape.router_bias else None
    return OracleLayer(H, I, E, shape.top_k, shape.bits, records, router, gs, rb,
                       has_shared=bool(shape.has_shared))


def bf16_half_ulp(v) -> np.ndarray:
    """Half a unit in the last place of bf16 (8 significant bits) at magnitude |v|:
    the largest error of round-to-nearest to bf16 for values of that binade."""
    v = np.abs(np.asarray(v, dtype=np.float64))
    _, e = np.frexp(np.where(v > 0, v, 1.0))
    return np.where(v > 0, np.ldexp(1.0, e - 9), 0.0)


def within_tolerance(gpu: np.ndarray, ref: np.ndarray, rel: float = 2e-3, out_bf16: bool = True):
    """Per-element bound |gpu - ref| <= rel * (|ref| + rms(ref)) on the value before
    the output's rounding to bf16: with ``out_bf16`` the bf16 half-ulp at the
    bound's edge is added, because a correctly rounded bf16 value can itself be
    2^-8 |ref| away from ref, more than rel * |ref| for rel = 2e-3.
    Returns (ok, worst ratio of error to bound)."""
    ref = np.asarray(ref, dtype=np.float64)
    gpu = np.asarray(gpu, dtype=np.float64)
    rms = math.sqrt(float(np.mean(ref * ref)))
    bound = rel * (np.abs(ref) + rms)
    if out_bf16:
        bound = bound + bf16_half_ulp(np.abs(ref) + bound)
    ratio = np.abs(gpu - ref) / np.maximum(bound, 1e-300)
    return bool(np.all(ratio <= 1.0)), float(np.max(ratio)) if ratio.size else 0.0


def bf16_agreement(gpu: np.ndarray, ref: np.ndarray, min_rel_rms: float = 0.0):
    """(fraction of elements equal to ref rounded to nearest-even bf16,
    largest distance in bf16 ulps of ref's binade), over the elements with
    |ref| >= min_rel_rms * rms(ref).  Near-zero outputs are left out with
    min_rel_rms > 0: an fp32 sum whose terms are of size rms has an absolute
    rounding error that can exceed the bf16 ulp of a result much smaller than rms."""
    ref = np.asarray(ref, dtype=np.float64)
    gpu = np.asarray(gpu, dtype=np.float64)
    keep = np.abs(ref) >= min_rel_rms * math.sqrt(float(np.mean(ref * ref)))
    ref, gpu = ref[keep], gpu[keep]
    if ref.size == 0:
        return 1.0, 0.0
    rb = bf16_to_f64(f64_to_bf16_bits(ref))
    ulp = 2.0 * bf16_half_ulp(ref)
    d = np.abs(gpu - rb) / np.where(ulp > 0, ulp, 1.0)
    return float(np.mean(gpu == rb)), float(np.max(d))


# ----------------------------------------------------------------------------
# GatedDeltaNet step (the linear-attention layers' state update)
# ----------------------------------------------------------------------------
def gdn_step(S: np.ndarray, q: np.ndarray, k: np.ndarray, v: np.ndarray, alpha: float, beta: float):
    """One token of a GatedDeltaNet head: the state S [dv, dk] is scaled by the gate
    alpha, read at the key k, moved towards the value v by a rank-1 update of strength
    beta, and read at the query q.  Returns (S_new, o), float64.

    The pages implement this step with BLAS on a 64-head x 128 x 128 state: a scaling,
    matrix-vector products and a rank-1 update (hotdry.top, "Metal GPU管线", the
    linear-attention paragraph: cblas_sscal, cblas_sgemv, cblas_sger).  The update they
    compose is the gated delta rule of GatedDeltaNet (Yang, Kautz, Hatamizadeh, "Gated
    Delta Networks", ICLR 2025), taken here in the pages' order:
      S <- alpha * S            (scale)
      u  = S k                  (matrix-vector)
      S <- S + beta (v - u) k^T (rank-1 update)
      o  = S q                  (matrix-vector)"""
    S = np.asarray(S, dtype=np.float64)
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    S = float(alpha) * S
    u = S @ k
    S = S + float(beta) * np.outer(v - u, k)
    o = S @ q
    return S, o
