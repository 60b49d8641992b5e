"""Seeded synthetic inputs for the routed-expert MoE layer (host side, numpy).

This module is the one place where test inputs come from. It is shared by the
fp64 CPU oracle (``oracle/``) and by the tests and benchmark that drive the CUDA
library, and it holds none of the layer's arithmetic: it only draws random
numbers, rounds them to the storage types and lays them out in the packed
expert-record format.

Workload recipe (the synthetic configurations of the routed-expert decode path
described on the Flash-MoE pages, "MoE稀疏架构" / "量化策略" sections of the
hotdry.top article and the results table of the tinai-dev README page):

* q codes: raw random bits, so every 4-bit nibble (2-bit crumb) is uniform.
* scale = bf16(|N(0,1)| * 0.02); bias = bf16(-c * scale + N(0, 1e-3)) with
  c = 8 for 4-bit and c = 2 for 2-bit, one (scale, bias) pair per 64-element
  group along the input dimension of every weight row.
* router weights fp32 N(0, 0.02); shared-expert gate vector fp32 N(0, 0.02);
  optional router bias fp32 N(0, 1).
* token activations x = bf16(z / sqrt(mean(z^2) + 1e-6)), z ~ N(0, 1).

``N(m, s)`` means mean m and standard deviation s throughout.

Generator definition (implemented identically, operation by operation, in
``fmoe_synth/csrc/synth.cu`` for device-side filling; the two agree bit for
bit because every floating-point step is a single IEEE-754 double operation
with round-to-nearest and no fused multiply-add):

* ``mix64`` is the SplitMix64 finaliser (Steele, Lea, Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014).
* a stream key is derived from (seed, layer, expert, tensor) by
  ``key = seed; for v in (layer, expert, tensor): key = mix64(key ^ mix64((v+1)*GAMMA))``.
* draw ``i`` of a stream is ``mix64(key + (i+1)*GAMMA)`` (mod 2^64): a
  counter-based generator, so any element can be produced independently.
* a uniform in (0, 1] is ``((r >> 11) + 1) * 2^-53``.
* normal number ``j`` of a stream uses draws ``2j`` and ``2j+1`` through the
  Box-Muller transform ``sqrt(-2 ln u1) * cos(2 pi u2)``, with ``ln`` and
  ``cos`` evaluated by the short series below (not libm), so that host and
  device produce the same bits.
* 32-bit q words: word ``i`` of a tensor is the low half of draw ``i // 2``
  when ``i`` is even and the high half when odd.
* bf16 rounding is round-to-nearest-even of the exact double value.

Packed expert record (the library's weight format; the byte layout is defined
in ``include/fmoe.h`` and repeated here so that this module stands alone):

    record = [GU_Q | GU_SB | D_Q | D_SB], each region 256-byte aligned
    GU_Q : for r in 0..I-1: gate q-row r (H*b/8 bytes), then up q-row r
    GU_SB: for r in 0..I-1: gate (scale,bias) row r (H/64 pairs), then up row r
    D_Q  : for j in 0..H-1: down q-row j (I*b/8 bytes)
    D_SB : for j in 0..H-1: down (scale,bias) row j (I/64 pairs)

A q-row holds 32/b codes per little-endian uint32, code k of a word at bits
[b*k, b*k+b).  A (scale, bias) pair is one uint32: scale's bf16 bits in the
low half, bias's in the high half.  A layer is ``E`` routed records followed by
one shared-expert record, each record starting at a 256-byte boundary.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
M1 = 0xBF58476D1CE4E5B9
M2 = 0x94D049BB133111EB

# tensor ids of the random streams
T_GATE_Q, T_UP_Q, T_DOWN_Q = 0, 1, 2
T_GATE_SB, T_UP_SB, T_DOWN_SB = 3, 4, 5
T_ROUTER, T_SHARED_GATE, T_ROUTER_BIAS, T_X = 6, 7, 8, 9

GROUP = 64
ALIGN = 256

_LN2 = 0.6931471805599453
_SQRT_HALF = 0.7071067811865476
_TWO_PI = 6.283185307179586


# ----------------------------------------------------------------------------
# integer hashing (scalar python ints and vectorised uint64 numpy)
# ----------------------------------------------------------------------------
def mix64_int(z: int) -> int:
    z &= MASK64
    z = ((z ^ (z >> 30)) * M1) & MASK64
    z = ((z ^ (z >> 27)) * M2) & MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, layer: int, expert: int, tensor: int) -> int:
    key = seed & MASK64
    for v in (layer, expert, tensor):
        key = mix64_int(key ^ mix64_int(((v + 1) * GAMMA) & MASK64))
    return key


def _mix64_np(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.uint64, copy=False)
    z = (z ^ (z >> np.uint64(30))) * np.uint64(M1)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(M2)
    return z ^ (z >> np.uint64(31))


def draws(key: int, start: int, count: int) -> np.ndarray:
    """Draws ``start .. start+count-1`` of the stream ``key`` (uint64)."""
    with np.errstate(over="ignore"):
        i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
        z = np.uint64(key) + i * np.uint64(GAMMA)
        return _mix64_np(z)


def q_words(key: int, start_word: int, count: int) -> np.ndarray:
    """32-bit words ``start_word .. start_word+count-1`` of a code stream."""
    d0 = start_word // 2
    d1 = (start_word + count + 1) // 2
    r = draws(key, d0, d1 - d0)
    w = np.empty(2 * r.size, dtype=np.uint32)
    w[0::2] = (r & np.uint64(0xFFFFFFFF)).astype(np.uint32)
    w[1::2] = (r >> np.uint64(32)).astype(np.uint32)
    off = start_word - 2 * d0
    return w[off:off + count]


def uniform(r: np.ndarray) -> np.ndarray:
    return ((r >> np.uint64(11)) + np.uint64(1)).astype(np.float64) * (2.0 ** -53)


# ----------------------------------------------------------------------------
# deterministic ln / cos (same operation order as the device code)
# ----------------------------------------------------------------------------
def _ln_unit(u: np.ndarray) -> np.ndarray:
    """ln(u) for u in (0, 1]: u = m 2^e, m in [sqrt(1/2), sqrt(2)),
    ln m = 2 atanh(t) with t = (m-1)/(m+1), atanh by its odd power series."""
    m, e = np.frexp(u)
    low = m < _SQRT_HALF
    m = np.where(low, m * 2.0, m)
    e = np.where(low, e - 1, e).astype(np.float64)
    t = (m - 1.0) / (m + 1.0)
    t2 = t * t
    s = 1.0 / 23.0
    for k in range(10, 0, -1):
        s = (1.0 / (2 * k + 1)) + t2 * s
    s = t2 * s
    tt = 2.0 * t
    lnm = tt + tt * s
    return e * _LN2 + lnm


_COS_C = [1.0 / math.factorial(2 * k) for k in range(0, 10)]
_SIN_C = [1.0 / math.factorial(2 * k + 1) for k in range(0, 10)]


def _cos_2pi(u: np.ndarray) -> np.ndarray:
    """cos(2 pi u) for u in (0, 1] by exact reflections to [0, 1/8] and the
    Taylor series of cos / sin there."""
    v = np.where(u < 0.5, u, u - 1.0)
    a = np.abs(v)
    neg = a > 0.25
    a = np.where(neg, 0.5 - a, a)
    use_sin = a > 0.125
    b = np.where(use_sin, 0.25 - a, a)
    th = _TWO_PI * b
    th2 = th * th
    c = _COS_C[9] * ((-1.0) ** 9)
    for k in range(8, -1, -1):
        c = (_COS_C[k] * ((-1.0) ** k)) + th2 * c
    s = _SIN_C[9] * ((-1.0) ** 9)
    for k in range(8, -1, -1):
        s = (_SIN_C[k] * ((-1.0) ** k)) + th2 * s
    s = th * s
    r = np.where(use_sin, s, c)
    return np.where(neg, -r, r)


def normals(key: int, start: int, count: int) -> np.ndarray:
    """Normals ``start .. start+count-1`` of the stream ``key`` (float64)."""
    r = draws(key, 2 * start, 2 * count)
    u1 = uniform(r[0::2])
    u2 = uniform(r[1::2])
    return np.sqrt(-2.0 * _ln_unit(u1)) * _cos_2pi(u2)


# ----------------------------------------------------------------------------
# bf16 rounding (round to nearest even from double)
# ----------------------------------------------------------------------------
def bf16_bits(v: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns of ``v`` rounded to nearest even (normal range)."""
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)
    q = np.rint(m * 256.0)
    r = np.ldexp(q, e - 8)
    f = r.astype(np.float32)
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------
# configurations and tensors
# ----------------------------------------------------------------------------
@dataclass(frozen=True)
class LayerShape:
    hidden: int
    inter: int
    n_experts: int
    top_k: int
    bits: int = 4
    has_shared: int = 1
    router_bias: int = 0

    @property
    def codes_per_word(self) -> int:
        return 32 // self.bits


def _al(n: int) -> int:
    return (n + ALIGN - 1) // ALIGN * ALIGN


def record_layout(H: int, I: int, bits: int) -> dict:
    """Byte offsets / sizes of the four regions of one expert record."""
    qrow_h = H * bits // 8
    qrow_i = I * bits // 8
    sbrow_h = (H // GROUP) * 4
    sbrow_i = (I // GROUP) * 4
    gu_q = I * 2 * qrow_h
    gu_sb = I * 2 * sbrow_h
    d_q = H * qrow_i
    d_sb = H * sbrow_i
    o_gu_q = 0
    o_gu_sb = _al(o_gu_q + gu_q)
    o_d_q = _al(o_gu_sb + gu_sb)
    o_d_sb = _al(o_d_q + d_q)
    size = _al(o_d_sb + d_sb)
    return dict(qrow_h=qrow_h, qrow_i=qrow_i, sbrow_h=sbrow_h, sbrow_i=sbrow_i,
                o_gu_q=o_gu_q, o_gu_sb=o_gu_sb, o_d_q=o_d_q, o_d_sb=o_d_sb,
                gu_q=gu_q, gu_sb=gu_sb, d_q=d_q, d_sb=d_sb, size=size)


def record_bytes(H: int, I: int, bits: int) -> int:
    return record_layout(H, I, bits)["size"]


def bias_center(bits: int) -> float:
    return 8.0 if bits == 4 else 2.0


@dataclass
class ExpertPlain:
    """One expert in plain form: per-tensor code words and (scale, bias) pairs."""
    gate_q: np.ndarray  # uint32 [I, H*b/32]
    up_q: np.ndarray    # uint32 [I, H*b/32]
    down_q: np.ndarray  # uint32 [H, I*b/32]
    gate_sb: np.ndarray  # uint32 [I, H/64]  (scale bits | bias bits << 16)
    up_sb: np.ndarray
    down_sb: np.ndarray


def _sb_pairs(seed: int, layer: int, expert: int, tensor: int, rows: int, groups: int,
              bits: int) -> np.ndarray:
    key = stream_key(seed, layer, expert, tensor)
    n = normals(key, 0, 2 * rows * groups)
    s = bf16_bits(np.abs(n[0::2]) * 0.02)
    b = bf16_bits(-bias_center(bits) * bf16_to_f64(s) + 1e-3 * n[1::2])
    pair = s.astype(np.uint32) | (b.astype(np.uint32) << np.uint32(16))
    return pair.reshape(rows, groups)


def _q_tensor(seed: int, layer: int, expert: int, tensor: int, rows: int, words: int) -> np.ndarray:
    key = stream_key(seed, layer, expert, tensor)
    return q_words(key, 0, rows * words).reshape(rows, words)


def gen_expert(seed: int, layer: int, expert: int, H: int, I: int, bits: int) -> ExpertPlain:
    wh = H * bits // 32
    wi = I * bits // 32
    return ExpertPlain(
        gate_q=_q_tensor(seed, layer, expert, T_GATE_Q, I, wh),
        up_q=_q_tensor(seed, layer, expert, T_UP_Q, I, wh),
        down_q=_q_tensor(seed, layer, expert, T_DOWN_Q, H, wi),
        gate_sb=_sb_pairs(seed, layer, expert, T_GATE_SB, I, H // GROUP, bits),
        up_sb=_sb_pairs(seed, layer, expert, T_UP_SB, I, H // GROUP, bits),
        down_sb=_sb_pairs(seed, layer, expert, T_DOWN_SB, H, I // GROUP, bits),
    )


def pack_record(p: ExpertPlain, H: int, I: int, bits: int) -> np.ndarray:
    """Lay one expert out as a packed record (uint8 array of record_bytes)."""
    L = record_layout(H, I, bits)
    out = np.zeros(L["size"], dtype=np.uint8)
    gu = np.stack([p.gate_q, p.up_q], axis=1)  # [I, 2, words]
    out[L["o_gu_q"]:L["o_gu_q"] + L["gu_q"]] = gu.reshape(-1).view(np.uint8)
    gsb = np.stack([p.gate_sb, p.up_sb], axis=1)
    out[L["o_gu_sb"]:L["o_gu_sb"] + L["gu_sb"]] = gsb.reshape(-1).astype(np.uint32).view(np.uint8)
    out[L["o_d_q"]:L["o_d_q"] + L["d_q"]] = p.down_q.reshape(-1).view(np.uint8)
    out[L["o_d_sb"]:L["o_d_sb"] + L["d_sb"]] = p.down_sb.reshape(-1).astype(np.uint32).view(np.uint8)
    return out


def gen_record(seed: int, layer: int, expert: int, H: int, I: int, bits: int) -> np.ndarray:
    return pack_record(gen_expert(seed, layer, expert, H, I, bits), H, I, bits)


def gen_layer_records(seed: int, layer: int, shape: LayerShape) -> np.ndarray:
    """All records of a layer (E routed + shared), concatenated (uint8)."""
    n = shape.n_experts + shape.has_shared
    rb = record_bytes(shape.hidden, shape.inter, shape.bits)
    out = np.empty(n * rb, dtype=np.uint8)
    for e in range(n):
        out[e * rb:(e + 1) * rb] = gen_record(seed, layer, e, shape.hidden, shape.inter, shape.bits)
    return out


def gen_router(seed: int, layer: int, E: int, H: int) -> np.ndarray:
    key = stream_key(seed, layer, 0, T_ROUTER)
    return (0.02 * normals(key, 0, E * H)).astype(np.float32).reshape(E, H)


def gen_shared_gate(seed: int, layer: int, H: int) -> np.ndarray:
    key = stream_key(seed, layer, 0, T_SHARED_GATE)
    return (0.02 * normals(key, 0, H)).astype(np.float32)


def gen_router_bias(seed: int, layer: int, E: int) -> np.ndarray:
    key = stream_key(seed, layer, 0, T_ROUTER_BIAS)
    return normals(key, 0, E).astype(np.float32)


def gen_x_token(seed: int, token: int, H: int) -> np.ndarray:
    """bf16 bits [H] of token ``token``: RMS-normalised N(0,1).  The mean of
    squares is a left-to-right sum in double."""
    key = stream_key(seed, 0, token, T_X)
    z = normals(key, 0, H)
    ss = np.add.accumulate(z * z)[-1]
    r = math.sqrt(ss / H + 1e-6)
    return bf16_bits(z / r)


def gen_x(seed: int, t0: int, T: int, H: int) -> np.ndarray:
    return np.stack([gen_x_token(seed, t, H) for t in range(t0, t0 + T)])


# ----------------------------------------------------------------------------
# named configurations (the five synthetic workloads)
# ----------------------------------------------------------------------------
CONFIGS = {
    "tiny": dict(shape=LayerShape(512, 128, 32, 4, 4, 1, 0), layers=1, tokens=1, batch=1),
    "layer4096": dict(shape=LayerShape(4096, 1024, 512, 4, 4, 1, 0), layers=1, tokens=1000, batch=1),
    "stack24_4bit": dict(shape=LayerShape(4096, 1024, 512, 4, 4, 1, 0), layers=24, tokens=256, batch=1),
    "stack60_2bit": dict(shape=LayerShape(4096, 1024, 512, 4, 2, 1, 0), layers=60, tokens=128, batch=1),
    "stack16_batched": dict(shape=LayerShape(4096, 1024, 512, 10, 4, 1, 1), layers=16, tokens=2048, batch=32),
    # one layer of the batched stack, one 32-token step (a profiling case of the batched path)
    "batched_layer_k10": dict(shape=LayerShape(4096, 1024, 512, 10, 4, 1, 1), layers=1, tokens=32, batch=32),
}
